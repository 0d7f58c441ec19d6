// Cache writers: bulk prefill of keys already in the PCA basis, and the
// per-step append that rotates the new key by P (AQUA page, decode-step
// equations (1)-(2): the current token's key and value join the cache before
// scoring; AQUA page, appendix step 1: the key is projected with P).
#pragma once

#include "common.cuh"

namespace loki {

struct PrefillParams {
    void* k_cache;
    void* v_cache;
    const int32_t* block_table;
    const int32_t* seq_lens;
    const void* k_rot;
    const void* v;
    int num_blocks, Hkv, max_blocks, max_seq_len, max_len;
};

// grid (max_blocks, batch * Hkv); one CTA writes one 16-token block of one
// kv head; 16-byte vectors of 16 / sizeof(T) dims, all inside one key slab.
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
    const int64_t page = page_offset(pb, h, p.Hkv, D);
    const int64_t src_row0 = (((int64_t)b * p.Hkv + h) * p.max_len + (int64_t)jb * kBlockTokens) * D;
    const T* ks = reinterpret_cast<const T*>(p.k_rot) + src_row0;
    const T* vs = reinterpret_cast<const T*>(p.v) + src_row0;
    T* kd = reinterpret_cast<T*>(p.k_cache) + page;
    T* vd = reinterpret_cast<T*>(p.v_cache) + page;
    constexpr int per_tok = D / VEC;
    for (int i = threadIdx.x; i < kBlockTokens * per_tok; i += blockDim.x) {
        const int tok = i / per_tok;
        const int dim = (i - tok * per_tok) * VEC;
        if (jb * kBlockTokens + tok >= L) continue;
        const uint4 kv = *reinterpret_cast<const uint4*>(ks + tok * D + dim);
        const uint4 vv = *reinterpret_cast<const uint4*>(vs + tok * D + dim);
        *reinterpret_cast<uint4*>(kd + key_offset_in_page(tok, dim)) = kv;
        *reinterpret_cast<uint4*>(vd + value_offset_in_page(tok, dim, D)) = vv;
    }
}

struct AppendParams {
    void* k_cache;
    void* v_cache;
    const int32_t* block_table;
    const int32_t* seq_lens;
    const void* k_new;
    const void* v_new;
    const float* P;  // nullable
    int num_blocks, Hkv, max_blocks, max_seq_len;
};

// grid (batch * Hkv), D threads. Thread c computes rotated dim c as an fp32
// chain over i = 0 .. D-1 of k[i] * P[i][c], then rounds to nearest even.
template <typename T, int D>
__global__ void __launch_bounds__(D) append_kernel(const AppendParams p) {
    __shared__ float kin[D];
    const int pair = blockIdx.x;
    const int b = pair / p.Hkv, h = pair - b * p.Hkv;
    const int c = threadIdx.x;
    int L = p.seq_lens[b];
    if (L < 0 || L > p.max_seq_len) {
        if (c == 0) flag_error(LOKI_DEVERR_SEQ_LEN);
        return;
    }
    if (L == 0) return;
    const int pos = L - 1;
    int pb = p.block_table[(int64_t)b * p.max_blocks + pos / kBlockTokens];
    if (pb < 0 || pb >= p.num_blocks) {
        if (c == 0) flag_error(LOKI_DEVERR_BLOCK_ID);
        return;
    }
    const int row = pos % kBlockTokens;
    const int64_t src = ((int64_t)b * p.Hkv + h) * D;
    kin[c] = Elem<T>::to_f(reinterpret_cast<const T*>(p.k_new)[src + c]);
    __syncthreads();
    float x;
    if (p.P) {
        const float* Ph = p.P + (int64_t)h * D * D;
        float a = 0.f;
#pragma unroll 16
        for (int i = 0; i < D; ++i) a = fmaf(kin[i], Ph[i * D + c], a);
        x = a;
    } else {
        x = kin[c];
    }
    const int64_t page = page_offset(pb, h, p.Hkv, D);
    reinterpret_cast<T*>(p.k_cache)[page + key_offset_in_page(row, c)] = Elem<T>::from_f(x);
    reinterpret_cast<T*>(p.v_cache)[page + value_offset_in_page(row, c, D)] =
        reinterpret_cast<const T*>(p.v_new)[src + c];
}

}  // namespace loki
