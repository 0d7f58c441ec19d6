// Dense decode attention, the full-attention comparison path (AQUA page,
// decode-step equations (3)-(5) over every cached token), as flash-decode
// split-K:
//   rotate_query_kernel  q_hat = q P[h] for every query head, into workspace
//   dense_split_kernel   one CTA per (split, sequence, kv head) runs AttnCore
//                        over a contiguous token range and writes its (o, m, l)
//                        partial to the workspace
//   merge_kernel         combines the splits of each query head
// The partials in global memory are the workspace (scratch) of this path.
#pragma once

#include "attn_core.cuh"

namespace loki {

constexpr int kDenseSplitTokens = 512;

struct DenseParams {
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_table;
    const int32_t* seq_lens;
    const void* q;
    const float* P;
    float* out;
    float* qhat;   // workspace [batch][Hq][D]
    float* parts;  // workspace [batch * Hkv][splits][G][D + 2]
    int num_blocks, Hkv, max_blocks, max_seq_len, splits;
    float scale_log2;
};

// grid (batch * Hkv), 256 threads: q_hat_j[c] = sum_i q_j[i] P[h][i][c].
template <typename T, int D, int G>
__global__ void __launch_bounds__(256) rotate_query_kernel(const DenseParams p) {
    __shared__ float qf[G * D];
    const int pair = blockIdx.x;
    const int b = pair / p.Hkv, h = pair - b * p.Hkv;
    const int Hq = p.Hkv * G;
    const T* qg = reinterpret_cast<const T*>(p.q) + ((int64_t)b * Hq + h * G) * D;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) qf[i] = Elem<T>::to_f(qg[i]);
    __syncthreads();
    const float* Ph = p.P + (int64_t)h * D * D;
    for (int o = threadIdx.x; o < G * D; o += blockDim.x) {
        const int j = o / D, c = o - j * D;
        float a = 0.f;
#pragma unroll 16
        for (int i = 0; i < D; ++i) a = fmaf(qf[j * D + i], Ph[i * D + c], a);
        p.qhat[((int64_t)b * Hq + h * G) * D + o] = a;
    }
}

// grid (splits, batch * Hkv), 256 threads.
template <typename T, int D, int G>
__global__ void __launch_bounds__(256) dense_split_kernel(const DenseParams p) {
    using Core = AttnCore<T, D, G>;
    constexpr int NCH = Core::NCH;
    constexpr int NW = 8;
    __shared__ float qs[G * D];
    __shared__ float wpart[NW * G * (D + 2)];
    const int split = blockIdx.x;
    const int pair = blockIdx.y;
    const int b = pair / p.Hkv, h = pair - b * p.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Hq = p.Hkv * G;
    int L = p.seq_lens[b];
    if (L < 0 || L > p.max_seq_len) {
        if (tid == 0 && split == 0) flag_error(LOKI_DEVERR_SEQ_LEN);
        L = L < 0 ? 0 : p.max_seq_len;
    }
    const int t_lo = split * kDenseSplitTokens;
    const int t_hi = min(L, t_lo + kDenseSplitTokens);
    const int n = max(0, t_hi - t_lo);
    for (int i = tid; i < G * D; i += blockDim.x) qs[i] = p.qhat[((int64_t)b * Hq + h * G) * D + i];
    __syncthreads();

    const T* kc = reinterpret_cast<const T*>(p.k_cache);
    const T* vc = reinterpret_cast<const T*>(p.v_cache);
    const int32_t* row_tbl = p.block_table + (int64_t)b * p.max_blocks;
    Core core;
    core.init(qs, p.scale_log2, lane);
    typename Core::raw_t kA[NCH], vA[NCH], kB[NCH], vB[NCH];
    uint32_t validA = 0, validB = 0;
    const int nchunks = (n + NCH - 1) / NCH;
    auto load = [&](typename Core::raw_t (&kr)[NCH], typename Core::raw_t (&vr)[NCH], uint32_t& valid, int ch) {
        valid = 0;
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int idx = ch * NCH + i;
            if (idx < n) {
                const int t = t_lo + idx;
                int pb = row_tbl[t >> 4];
                if (pb < 0 || pb >= p.num_blocks) {
                    flag_error(LOKI_DEVERR_BLOCK_ID);
                    pb = 0;
                }
                const int64_t page = page_offset(pb, h, p.Hkv, D);
                kr[i] = Core::V::load(Core::key_ptr(kc, page, t & 15, lane));
                vr[i] = Core::V::load(Core::val_ptr(vc, page, t & 15, lane));
                valid |= 1u << i;
            } else {
                kr[i] = Core::zero_raw();
                vr[i] = Core::zero_raw();
            }
        }
    };
    int ch = warp;
    if (ch < nchunks) load(kA, vA, validA, ch);
    for (; ch < nchunks; ch += 2 * NW) {
        if (ch + NW < nchunks) load(kB, vB, validB, ch + NW);
        core.consume(kA, vA, validA, lane);
        if (ch + NW >= nchunks) break;
        if (ch + 2 * NW < nchunks) load(kA, vA, validA, ch + 2 * NW);
        core.consume(kB, vB, validB, lane);
    }
    core.store_partial(wpart + warp * G * (D + 2), lane);
    __syncthreads();
    float* dst = p.parts + ((int64_t)pair * p.splits + split) * G * (D + 2);
    for (int o = tid; o < G * D; o += blockDim.x) {
        const int j = o / D, c = o - j * D;
        const Merged mg = merge_partials<D>(wpart, NW, G * (D + 2), j, c);
        dst[j * (D + 2) + c] = mg.o;
        if (c == 0) {
            dst[j * (D + 2) + D] = mg.m;
            dst[j * (D + 2) + D + 1] = mg.l;
        }
    }
}

// grid (batch * Hq), D threads.
template <int D, int G>
__global__ void __launch_bounds__(D) merge_kernel(const DenseParams p) {
    const int qh = blockIdx.x;
    const int Hq = p.Hkv * G;
    const int b = qh / Hq, jq = qh - b * Hq;
    const int h = jq / G, j = jq - h * G;
    const int pair = b * p.Hkv + h;
    const float* src = p.parts + (int64_t)pair * p.splits * G * (D + 2);
    const Merged mg = merge_partials<D>(src, p.splits, G * (D + 2), j, threadIdx.x);
    p.out[(int64_t)qh * D + threadIdx.x] = mg.l > 0.f ? mg.o / mg.l : 0.f;
}

}  // namespace loki
