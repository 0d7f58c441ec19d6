// Warp-level exact attention over a stream of cached tokens (AQUA page,
// decode-step equations (3)-(5): logits q_hat . k over the full head
// dimension, scaled; softmax; weighted sum of values), for the G query heads
// that share one kv head. Online softmax in base 2 keeps one running maximum
// per head, so the tokens can arrive in any order and in several pieces whose
// partial results (max m, sum l, unnormalised output o) merge exactly.
//
// Work split inside a warp: lane l owns head dimensions [l*DPL, l*DPL + DPL)
// (DPL = D / 32) of every token's key row and value row, so a token costs one
// 8-byte (bf16, D = 128) read of its key piece and one of its value piece per
// lane (from global memory or from a shared-memory staging copy). A chunk of
// NCH tokens gives each lane NCH * G partial dot products, which one
// transpose-reduce sums across the warp.
#pragma once

#include "common.cuh"

namespace loki {

template <typename T, int D, int G, int NCH_ = ((G >= 8) ? 4 : 8)>
struct AttnCore {
    static constexpr int DPL = D / 32;
    static constexpr int NCH = NCH_;                   // tokens per chunk
    static constexpr int NV = NCH * G;                 // values per transpose-reduce
    static constexpr int LOG_NV = NV == 2 ? 1 : NV == 4 ? 2 : NV == 8 ? 3 : NV == 16 ? 4 : 5;
    static constexpr int LOG_G = G == 1 ? 0 : (G == 2 ? 1 : (G == 4 ? 2 : 3));
    static constexpr int SH = 5 - LOG_NV;              // lane >> SH = value index
    static_assert(NV >= 2 && NV <= 32 && (NV & (NV - 1)) == 0, "chunk geometry");
    using V = Vec<T, DPL>;
    using raw_t = typename V::raw_t;

    float q[G][DPL];     // rotated query, pre-multiplied by scale * log2(e)
    float acc[G][DPL];   // unnormalised output for this lane's dims
    float m;             // running max of base-2 logits for this lane's head
    float l;             // running sum of weights (replica 0 of each value only)

    __device__ __forceinline__ void init(const float* qhat, float scale_log2, int lane) {
#pragma unroll
        for (int j = 0; j < G; ++j)
#pragma unroll
            for (int i = 0; i < DPL; ++i) {
                q[j][i] = qhat[j * D + lane * DPL + i] * scale_log2;
                acc[j][i] = 0.f;
            }
        m = -INFINITY;
        l = 0.f;
    }

    // Address of this lane's key piece / value piece of `row` in a block.
    static __device__ __forceinline__ const T* key_ptr(const T* kc, int64_t page, int row, int lane) {
        return kc + page + row_offset_in_page(row, lane * DPL, D);
    }
    static __device__ __forceinline__ const T* val_ptr(const T* vc, int64_t page, int row, int lane) {
        return vc + page + row_offset_in_page(row, lane * DPL, D);
    }

    static __device__ __forceinline__ raw_t zero_raw() {
        raw_t r;
        memset(&r, 0, sizeof(r));
        return r;
    }

    // One chunk of NCH tokens; token n is present iff bit n of `valid`.
    __device__ __forceinline__ void consume(const raw_t (&kr)[NCH], const raw_t (&vr)[NCH], uint32_t valid,
                                            int lane) {
        float part[NV];
#pragma unroll
        for (int n = 0; n < NCH; ++n) {
            float kf[DPL];
            V::to_float(kr[n], kf);
#pragma unroll
            for (int j = 0; j < G; ++j) {
                float s = 0.f;
#pragma unroll
                for (int i = 0; i < DPL; ++i) s = fmaf(q[j][i], kf[i], s);
                part[n * G + j] = s;
            }
        }
        float z = transpose_reduce<NV>(part, lane);
        const int vi = lane >> SH;            // value index held by this lane
        const int n_own = vi >> LOG_G;        // its token within the chunk
        const bool ok = (valid >> n_own) & 1u;
        z = ok ? z : -INFINITY;
        // chunk maximum per head: reduce over the lane bits that encode the token
        const float cmax = warp_max_xor(z, SH + LOG_G, 5);
        const float m_new = fmaxf(m, cmax);
        const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m - m_new);
        const float pz = ok ? exp2f(z - m_new) : 0.f;
        m = m_new;
        const bool replica0 = (lane & ((1 << SH) - 1)) == 0;
        l = l * alpha + (replica0 ? pz : 0.f);
#pragma unroll
        for (int j = 0; j < G; ++j) {
            const float a = __shfl_sync(kFull, alpha, j << SH);
#pragma unroll
            for (int i = 0; i < DPL; ++i) acc[j][i] *= a;
        }
#pragma unroll
        for (int n = 0; n < NCH; ++n) {
            float vf[DPL];
            V::to_float(vr[n], vf);
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const float pj = __shfl_sync(kFull, pz, (n * G + j) << SH);
#pragma unroll
                for (int i = 0; i < DPL; ++i) acc[j][i] = fmaf(pj, vf[i], acc[j][i]);
            }
        }
    }

    // Writes this warp's partial (o[D], m, l per head) to dst[G][D + 2].
    __device__ __forceinline__ void store_partial(float* dst, int lane) {
        float lt = warp_sum_xor(l, 0, SH);
        lt = warp_sum_xor(lt, SH + LOG_G, 5);   // now: total of the lane's head
#pragma unroll
        for (int j = 0; j < G; ++j) {
#pragma unroll
            for (int i = 0; i < DPL; ++i) dst[j * (D + 2) + lane * DPL + i] = acc[j][i];
            if (lane == (j << SH)) {
                dst[j * (D + 2) + D] = m;
                dst[j * (D + 2) + D + 1] = lt;
            }
        }
    }
};

// Merge of n partials src[k * stride + ...] laid out as [G][D + 2] (o, m, l)
// for head j, dimension c: returns (sum_k w_k o_k[c], sum_k w_k l_k, M) with
// w_k = 2^(m_k - M), M = max_k m_k. Empty partials have m = -inf.
struct Merged {
    float o, l, m;
};
template <int D>
__device__ __forceinline__ Merged merge_partials(const float* src, int n, int stride, int j, int c) {
    float M = -INFINITY;
    for (int k = 0; k < n; ++k) M = fmaxf(M, src[k * stride + j * (D + 2) + D]);
    Merged r{0.f, 0.f, M};
    if (M == -INFINITY) return r;
    for (int k = 0; k < n; ++k) {
        const float* pk = src + k * stride + j * (D + 2);
        const float mk = pk[D];
        if (mk == -INFINITY) continue;
        const float w = exp2f(mk - M);
        r.o = fmaf(w, pk[c], r.o);
        r.l = fmaf(w, pk[D + 1], r.l);
    }
    return r;
}

}  // namespace loki
