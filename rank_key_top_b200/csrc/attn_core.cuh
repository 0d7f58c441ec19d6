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

namespace loki {

// ---------------------------------------------------------------------------
// Tensor-core variant for bf16 caches: the same exact attention (AQUA page,
// decode-step equations (3)-(5)) with the two contractions of a chunk of 8
// staged tokens on warp-level MMA (m16n8k16, bf16 inputs, fp32 accumulate):
//   logits  S[8 tok x 8 col] = K[8 tok x D] . Qt[D x 8 col]
//   output  Ot[D x 8 col]  += Vt[D x 8 tok] . Pt[8 tok x 8 col]
// Column n of Qt / Pt is head n/2, part n%2: each fp32 query value (and each
// softmax weight) is split into a bf16 high part and a bf16 remainder, so the
// products keep about 16 significant bits and the accumulation is fp32. With
// G = 8 a second group of 8 columns carries heads 4..7. Rows 8..15 of each
// m16 tile are unused (8 tokens per chunk).
//
// Lane l = 4g + t then owns, after the logits MMA, token g's logit for head
// t (and t + 4), and after the output MMA, head t's output for dims
// {16m + g, 16m + g + 8 : m < D/16}: the running max and the rescale of a
// lane's accumulators concern its own head only.
//
// Staging layout of one chunk (written by cp.async): 8 key rows then 8 value
// rows of D bf16 each; the 16-byte piece c of row r sits at piece c ^ (r & 7)
// so that every ldmatrix below is free of bank conflicts.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t& r0, uint32_t& r1, const void* row_ptr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(smem_u32(row_ptr)));
}
__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t& r0, uint32_t& r1, const void* row_ptr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(smem_u32(row_ptr)));
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            const void* row_ptr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(row_ptr)));
}
// bf16 pair {lo16 = a, hi16 = b}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(a));
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(b));
    return lo | (hi << 16);
}
// high (part 0) or remainder (part 1) of x in bf16
__device__ __forceinline__ float split_part(float x, int part) {
    const float h = __bfloat162float(__float2bfloat16_rn(x));
    return part ? x - h : h;
}

template <int D, int G>
struct MmaAttnCore {
    static constexpr int NCH = 8;              // tokens per chunk
    static constexpr int KS = D / 16;          // k-steps of the logits MMA, m-tiles of the output MMA
    static constexpr int NG = G > 4 ? 2 : 1;   // column groups of 8 (4 heads each)
    static constexpr int ROWB = D * 2;         // bytes of one staged row
    static constexpr int CHUNK_BYTES = 2 * NCH * ROWB;

    uint32_t qb[NG][KS][2];   // Qt fragments (scale * log2(e) folded in)
    float acc[NG][KS][4];     // Ot accumulators
    float m[NG];              // running max of this lane's head (per column group)
    float l[NG];              // this lane's running sum of weights (its token g)

    // byte offset of piece c of staged row r (key rows: kv = 0, value rows: kv = 1)
    static __device__ __forceinline__ int staged_offset(int kv, int r, int c) {
        return kv * NCH * ROWB + r * ROWB + ((c ^ (r & 7)) << 4);
    }

    __device__ __forceinline__ void init(const float* qhat, float scale_log2, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int ng = 0; ng < NG; ++ng) {
            const int head = ng * 4 + (g >> 1);
            const int part = g & 1;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                float v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int d = ks * 16 + 2 * t + (e & 1) + (e >> 1) * 8;
                    v[e] = head < G ? split_part(qhat[head * D + d] * scale_log2, part) : 0.f;
                }
                qb[ng][ks][0] = pack_bf16(v[0], v[1]);
                qb[ng][ks][1] = pack_bf16(v[2], v[3]);
            }
#pragma unroll
            for (int ks = 0; ks < KS; ++ks)
                acc[ng][ks][0] = acc[ng][ks][1] = acc[ng][ks][2] = acc[ng][ks][3] = 0.f;
            m[ng] = -INFINITY;
            l[ng] = 0.f;
        }
    }

    // One staged chunk; token n is present iff bit n of `valid` (absent rows
    // are zero-filled by the staging copy).
    __device__ __forceinline__ void consume(const unsigned char* chunk, uint32_t valid, int lane) {
        const int g = lane >> 2, t = lane & 3;
        // ldmatrix row addresses: lanes 0-7 rows 0-7 of piece 2s, lanes 8-15 of piece 2s+1
        const int lr = lane & 7, lh = (lane >> 3) & 1;
        float z[NG];
#pragma unroll
        for (int ng = 0; ng < NG; ++ng) {
            float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t a0, a2;
                ldmatrix_x2(a0, a2, chunk + staged_offset(0, lr, 2 * ks + lh));
                mma_16816_bf16(s, a0, 0u, a2, 0u, qb[ng][ks][0], qb[ng][ks][1]);
            }
            z[ng] = s[0] + s[1];  // token g, head 4 ng + t: high part + remainder
        }
        const bool ok = (valid >> g) & 1u;
        float p[NG], alpha[NG];
#pragma unroll
        for (int ng = 0; ng < NG; ++ng) {
            const float zz = ok ? z[ng] : -INFINITY;
            float cm = zz;
            cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 4));
            cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 8));
            cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 16));
            const float m_new = fmaxf(m[ng], cm);
            alpha[ng] = (m_new == -INFINITY) ? 1.f : exp2f(m[ng] - m_new);
            p[ng] = ok ? exp2f(zz - m_new) : 0.f;
            m[ng] = m_new;
            l[ng] = l[ng] * alpha[ng] + p[ng];
        }
        // Pt fragments: lane needs weights of tokens 2t, 2t+1 for column g
#pragma unroll
        for (int ng = 0; ng < NG; ++ng) {
            const int src = (g >> 1);
            const float pa = __shfl_sync(kFull, p[ng], 4 * (2 * t) + src);
            const float pb = __shfl_sync(kFull, p[ng], 4 * (2 * t + 1) + src);
            const uint32_t b0 = pack_bf16(split_part(pa, g & 1), split_part(pb, g & 1));
            const bool rescale = __any_sync(kFull, alpha[ng] != 1.f);
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                if (rescale) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[ng][mt][e] *= alpha[ng];
                }
                uint32_t a0, a1;
                ldmatrix_x2_trans(a0, a1, chunk + staged_offset(1, lr, 2 * mt + lh));
                mma_16816_bf16(acc[ng][mt], a0, a1, 0u, 0u, b0, 0u);
            }
        }
    }

    // This warp's partial (o[D], m, l per head) to dst[G][D + 2].
    __device__ __forceinline__ void store_partial(float* dst, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int ng = 0; ng < NG; ++ng) {
            const int head = ng * 4 + t;
            float lt = l[ng];
            lt += __shfl_xor_sync(kFull, lt, 4);
            lt += __shfl_xor_sync(kFull, lt, 8);
            lt += __shfl_xor_sync(kFull, lt, 16);
            if (head < G) {
#pragma unroll
                for (int mt = 0; mt < KS; ++mt) {
                    dst[head * (D + 2) + mt * 16 + g] = acc[ng][mt][0] + acc[ng][mt][1];
                    dst[head * (D + 2) + mt * 16 + g + 8] = acc[ng][mt][2] + acc[ng][mt][3];
                }
                if (g == 0) {
                    dst[head * (D + 2) + D] = m[ng];
                    dst[head * (D + 2) + D + 1] = lt;
                }
            }
        }
    }
};

}  // namespace loki
