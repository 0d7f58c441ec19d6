// Cache writers: bulk prefill of keys already in the PCA basis, and the
// per-step append that rotates the new key by P (AQUA page, decode-step
// equations (1)-(2): the current token's key and value join the cache before
// scoring; AQUA page, appendix on complexity, step 1: the key is projected
// with P). Both write the key row, the value row and the key's leading
// index dims into the low-rank key index.
#pragma once

#include "common.cuh"

namespace loki {

struct PrefillParams {
    void* k_cache;
    void* v_cache;
    void* k_index;
    const int32_t* block_table;
    const int32_t* seq_lens;
    const void* k_rot;
    const void* v;
    KvMap kv;
    int num_blocks, Hkv, max_blocks, max_seq_len, max_len, index_dims;
};

// grid (max_blocks, batch * Hkv); one CTA writes one 16-token block of one
// kv head with 16-byte vectors (16 / sizeof(T) dims, inside one index slab).
template <typename T, int D>
__global__ void __launch_bounds__(256) prefill_kernel(const PrefillParams p) {
    constexpr int VEC = 16 / sizeof(T);
    const int jb = blockIdx.x;
    const int pair = blockIdx.y;
    const int b = pair / p.Hkv, h = pair - b * p.Hkv;
    int L = p.seq_lens[b];
    if (L < 0 || L > p.max_seq_len) {
        if (threadIdx.x == 0 && jb == 0) flag_error(LOKI_DEVERR_SEQ_LEN);
        L = L < 0 ? 0 : p.max_seq_len;
    }
    if (jb * kBlockTokens >= L) return;
    int pb = p.block_table[(int64_t)b * p.max_blocks + jb];
    if (pb < 0 || pb >= p.num_blocks) {
        if (threadIdx.x == 0) flag_error(LOKI_DEVERR_BLOCK_ID);
        return;
    }
    const int64_t ipage = page_offset(pb, h, p.Hkv, p.index_dims);
    const int64_t src_row0 = (((int64_t)b * p.Hkv + h) * p.max_len + (int64_t)jb * kBlockTokens) * D;
    const T* ks = reinterpret_cast<const T*>(p.k_rot) + src_row0;
    const T* vs = reinterpret_cast<const T*>(p.v) + src_row0;
    T *kd, *vd;
    kv_rows(p.kv, p.k_cache, p.v_cache, pb, h, p.Hkv, D, kd, vd);
    if (!kd) return;
    T* xd = reinterpret_cast<T*>(p.k_index) + ipage;
    constexpr int per_tok = D / VEC;
    for (int i = threadIdx.x; i < kBlockTokens * per_tok; i += blockDim.x) {
        const int tok = i / per_tok;
        const int dim = (i - tok * per_tok) * VEC;
        if (jb * kBlockTokens + tok >= L) continue;
        const uint4 kv = *reinterpret_cast<const uint4*>(ks + tok * D + dim);
        const uint4 vv = *reinterpret_cast<const uint4*>(vs + tok * D + dim);
        *reinterpret_cast<uint4*>(kd + row_offset_in_page(tok, dim, D)) = kv;
        *reinterpret_cast<uint4*>(vd + row_offset_in_page(tok, dim, D)) = vv;
        if (dim < p.index_dims) {  // dim-major index: one element per dim
            const T* e = reinterpret_cast<const T*>(&kv);
#pragma unroll
            for (int i = 0; i < VEC; ++i) xd[index_offset_in_page(tok, dim + i)] = e[i];
        }
    }
}

struct AppendParams {
    void* k_cache;
    void* v_cache;
    void* k_index;
    const int32_t* block_table;
    const int32_t* seq_lens;
    const void* k_new;
    const void* v_new;
    const float* P;   // nullable
    const float* Ak;  // nullable: [Hkv][D][index_dims], the index row is k A_k
    KvMap kv;
    int num_blocks, Hkv, max_blocks, max_seq_len, index_dims;
};

// grid (batch * Hkv), 256 threads. k_tilde[c] = sum_i k[i] P[i][c] in fp32:
// thread (row group rg, column quad cq) sums its D/8 rows for 4 columns from
// one round of independent 16-byte loads of P; the 8 row groups' partial sums
// are added in shared memory; the result is rounded to nearest even.
template <typename T, int D>
__global__ void __launch_bounds__(256) append_kernel(const AppendParams p) {
    constexpr int NQ = D / 4;         // column quads
    constexpr int NRG = 256 / NQ;     // row groups (8 for D = 128, 16 for D = 64)
    constexpr int RPG = D / NRG;      // rows per group
    __shared__ float part[NRG][D];
    __shared__ float kin[D];
    const int pair = blockIdx.x;
    const int b = pair / p.Hkv, h = pair - b * p.Hkv;
    const int tid = threadIdx.x;
    // a decode launched as this kernel's programmatic dependent may start now:
    // it waits for this grid before it reads the token written here
    griddep_launch_dependents();
    int L = p.seq_lens[b];
    if (L < 0 || L > p.max_seq_len) {
        if (tid == 0) flag_error(LOKI_DEVERR_SEQ_LEN);
        return;
    }
    if (L == 0) return;
    const int pos = L - 1;
    int pb = p.block_table[(int64_t)b * p.max_blocks + pos / kBlockTokens];
    if (pb < 0 || pb >= p.num_blocks) {
        if (tid == 0) flag_error(LOKI_DEVERR_BLOCK_ID);
        return;
    }
    const int row = pos % kBlockTokens;
    const int64_t src = ((int64_t)b * p.Hkv + h) * D;
    const int cq = tid % NQ, rg = tid / NQ;
    float4 pv[RPG];
    if (p.P) {
        const float* Ph = p.P + (int64_t)h * D * D;
#pragma unroll
        for (int i = 0; i < RPG; ++i) pv[i] = *reinterpret_cast<const float4*>(Ph + (rg * RPG + i) * D + 4 * cq);
    }
    if (tid < D) kin[tid] = Elem<T>::to_f(reinterpret_cast<const T*>(p.k_new)[src + tid]);
    __syncthreads();
    if (p.P) {
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int i = 0; i < RPG; ++i) {
            const float x = kin[rg * RPG + i];
            a0 = fmaf(x, pv[i].x, a0);
            a1 = fmaf(x, pv[i].y, a1);
            a2 = fmaf(x, pv[i].z, a2);
            a3 = fmaf(x, pv[i].w, a3);
        }
        *reinterpret_cast<float4*>(&part[rg][4 * cq]) = make_float4(a0, a1, a2, a3);
    }
    __syncthreads();
    if (tid < D) {
        const int c = tid;
        float x;
        if (p.P) {
            x = 0.f;
#pragma unroll
            for (int g = 0; g < NRG; ++g) x += part[g][c];
        } else {
            x = kin[c];
        }
        const T kt = Elem<T>::from_f(x);
        T *kd, *vd;
        kv_rows(p.kv, p.k_cache, p.v_cache, pb, h, p.Hkv, D, kd, vd);
        if (kd) kd[row_offset_in_page(row, c, D)] = kt;
        if (c < p.index_dims) {
            T xv = kt;
            if (p.Ak) {  // key factor of an asymmetric score: (k A_k)[c], summed in row order
                const float* Ac = p.Ak + (int64_t)h * D * p.index_dims + c;
                float s = 0.f;
                for (int i = 0; i < D; ++i) s = fmaf(kin[i], Ac[(int64_t)i * p.index_dims], s);
                xv = Elem<T>::from_f(s);
            }
            reinterpret_cast<T*>(p.k_index)[page_offset(pb, h, p.Hkv, p.index_dims) + index_offset_in_page(row, c)] =
                xv;
        }
        if (vd) vd[row_offset_in_page(row, c, D)] = reinterpret_cast<const T*>(p.v_new)[src + c];
    }
}

// Key index of an asymmetric score factorisation for every cached token
// (SAKI page, abstract: the keys' own rank-r factor): index row
// round((k A_k)[c]) from keys k in the original basis, fp32 sums in row order
// (the same order as the append, so both write identical rows).
struct IndexParams {
    void* k_index;
    const int32_t* block_table;
    const int32_t* seq_lens;
    const void* k;     // [batch][Hkv][max_len][D], original basis
    const float* Ak;   // [Hkv][D][index_dims]
    int num_blocks, Hkv, max_blocks, max_seq_len, max_len, index_dims;
};

constexpr int kIndexTile = 64;  // tokens per CTA

template <int D>
constexpr int index_smem_bytes(int index_dims) {
    return D * index_dims * 4 + kIndexTile * (D + 1) * 4;
}

// grid (tiles of kIndexTile tokens, batch * Hkv), 256 threads. A_k[h] and the
// tile's keys (as fp32, rows padded to D + 1 words: conflict-free column
// reads) are staged in shared memory; each work item is 4 tokens x 4 columns.
template <typename T, int D>
__global__ void __launch_bounds__(256) index_keys_kernel(const IndexParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int I = p.index_dims;
    float* A = reinterpret_cast<float*>(smem);  // [D][I]
    float* kt = A + D * I;                      // [kIndexTile][D + 1]
    const int tile = blockIdx.x, pair = blockIdx.y;
    const int b = pair / p.Hkv, h = pair - b * p.Hkv;
    int L = p.seq_lens[b];
    if (L < 0 || L > p.max_seq_len) {
        if (threadIdx.x == 0 && tile == 0) flag_error(LOKI_DEVERR_SEQ_LEN);
        L = L < 0 ? 0 : p.max_seq_len;
    }
    const int t0 = tile * kIndexTile;
    if (t0 >= L) return;
    const int nt = min(kIndexTile, L - t0);
    const float4* Ah = reinterpret_cast<const float4*>(p.Ak + (int64_t)h * D * I);
    for (int e = threadIdx.x; e < D * I / 4; e += blockDim.x) reinterpret_cast<float4*>(A)[e] = Ah[e];
    const T* ks = reinterpret_cast<const T*>(p.k) + (((int64_t)b * p.Hkv + h) * p.max_len + t0) * D;
    for (int e = threadIdx.x; e < kIndexTile * D; e += blockDim.x) {
        const int t = e / D, a = e - t * D;
        kt[t * (D + 1) + a] = t < nt ? Elem<T>::to_f(ks[e]) : 0.f;
    }
    __syncthreads();
    const int nq = I / 4;
    for (int item = threadIdx.x; item < (kIndexTile / 4) * nq; item += blockDim.x) {
        const int tq = item / nq, cq = item - tq * nq;
        if (4 * tq >= nt) continue;
        float acc[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.f;
        for (int a = 0; a < D; ++a) {
            const float4 w = *reinterpret_cast<const float4*>(A + a * I + 4 * cq);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float x = kt[(4 * tq + u) * (D + 1) + a];
                acc[u][0] = fmaf(x, w.x, acc[u][0]);
                acc[u][1] = fmaf(x, w.y, acc[u][1]);
                acc[u][2] = fmaf(x, w.z, acc[u][2]);
                acc[u][3] = fmaf(x, w.w, acc[u][3]);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int t = t0 + 4 * tq + u;
            if (4 * tq + u >= nt) break;
            const int pb = p.block_table[(int64_t)b * p.max_blocks + t / kBlockTokens];
            if (pb < 0 || pb >= p.num_blocks) {
                flag_error(LOKI_DEVERR_BLOCK_ID);
                continue;
            }
            T* xd = reinterpret_cast<T*>(p.k_index) + page_offset(pb, h, p.Hkv, I);
#pragma unroll
            for (int v = 0; v < 4; ++v)
                xd[index_offset_in_page(t % kBlockTokens, 4 * cq + v)] = Elem<T>::from_f(acc[u][v]);
        }
    }
}

}  // namespace loki
