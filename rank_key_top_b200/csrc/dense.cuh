// Dense decode attention, the full-attention comparison path (AQUA page,
// decode-step equations (3)-(5) over every cached token), as flash-decode
// split-K:
//   rotate_query_kernel  q_hat = q P[h] for every query head, into workspace
//   dense_split_kernel   one CTA per (split, sequence, kv head) stages the
//                        split's key and value rows with cp.async, runs the
//                        attention core over them and writes its (o, m, l)
//                        partial to the workspace; a split is 1024 tokens, or
//                        2048 when that still leaves several waves of CTAs
//   merge_kernel         combines the splits of each query head
// The partials in global memory are the workspace (scratch) of this path.
#pragma once

#include <type_traits>

#include "attn_core.cuh"

namespace loki {

constexpr int kDenseSplitTokens = 1024;  // the workspace is sized for splits of this many tokens

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
    KvMap kv;
    int num_blocks, Hkv, max_blocks, max_seq_len, splits;
    int split_tokens;  // kDenseSplitTokens or a multiple of it
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

// Geometry of dense_split_kernel: 16 warps; each warp stages chunks of NCH
// consecutive tokens (key rows then value rows) into GS shared-memory slots
// with cp.async and consumes them with the tensor-core core (bf16) or the
// CUDA-core core (fp32), as the sparse gather does.
constexpr int kDenseThreads = 512;
template <typename T, int D, int G>
struct DenseGeom {
    static constexpr bool MMA = std::is_same<T, __nv_bfloat16>::value;
    using Core = AttnCore<T, D, G, (8 * G > 32 ? 32 / G : 8)>;
    using MCore = MmaAttnCore<D, G>;
    static constexpr int NW = kDenseThreads / 32;
    static constexpr int NCH = MMA ? MCore::NCH : Core::NCH;  // divides 16: a chunk lies in one block
    static constexpr int TB = 2 * D * (int)sizeof(T);
    static constexpr int CHUNK_BYTES = NCH * TB;
    static constexpr int WPART_BYTES = NW * G * (D + 2) * 4;
    static constexpr int QS_BYTES = G * D * 4;
    static constexpr int GS_FIT = (200 * 1024 - WPART_BYTES - QS_BYTES) / (NW * CHUNK_BYTES);
    static constexpr int GS = GS_FIT < 1 ? 1 : (GS_FIT > 4 ? 4 : GS_FIT);
    static constexpr int STAGE_BYTES = NW * GS * CHUNK_BYTES;
    static constexpr int SMEM_BYTES = STAGE_BYTES + WPART_BYTES + QS_BYTES;
    static_assert(16 % NCH == 0, "a chunk must not straddle a block");
};

// grid (splits, batch * Hkv), kDenseThreads threads, DenseGeom::SMEM_BYTES of
// dynamic shared memory. The split's tokens [t_lo, t_hi) are read once, in
// 16-byte cp.async pieces of whole rows (the 8 rows of a chunk are contiguous
// in their block), and attended by all query heads of the group.
template <typename T, int D, int G>
__global__ void __launch_bounds__(kDenseThreads) dense_split_kernel(const DenseParams p) {
    using Geom = DenseGeom<T, D, G>;
    using Core = typename Geom::Core;
    constexpr int NW = Geom::NW, NCH = Geom::NCH, TB = Geom::TB, GS = Geom::GS;
    constexpr int ROWB = D * (int)sizeof(T);
    constexpr int PIECES = TB / 16;  // 16-byte pieces of one token (key row + value row)
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char* stage = smem;
    float* wpart = reinterpret_cast<float*>(smem + Geom::STAGE_BYTES);
    float* qs = reinterpret_cast<float*>(smem + Geom::STAGE_BYTES + Geom::WPART_BYTES);
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
    const int t_lo = split * p.split_tokens;
    const int n = max(0, min(L, t_lo + p.split_tokens) - t_lo);
    for (int i = tid; i < G * D; i += kDenseThreads) qs[i] = p.qhat[((int64_t)b * Hq + h * G) * D + i];

    const unsigned char* kbytes = reinterpret_cast<const unsigned char*>(p.k_cache);
    const unsigned char* vbytes = reinterpret_cast<const unsigned char*>(p.v_cache);
    const int32_t* row_tbl = p.block_table + (int64_t)b * p.max_blocks;
    unsigned char* wst = stage + warp * GS * Geom::CHUNK_BYTES;
    const int nchunks = (n + NCH - 1) / NCH;
    const int my_n = nchunks > warp ? (nchunks - warp + NW - 1) / NW : 0;
    // stage chunk m of this warp (tokens t_lo + ch*NCH .. + NCH) into slot m % GS
    auto fetch = [&](int m) {
        if (m < my_n) {
            unsigned char* dst = wst + (m % GS) * Geom::CHUNK_BYTES;
            const int ch = warp + m * NW;
            const int tc = t_lo + ch * NCH;  // first token of the chunk, < L
            int pb = row_tbl[tc >> 4];
            bool okp = true;
            if (pb < 0 || pb >= p.num_blocks) {
                flag_error(LOKI_DEVERR_BLOCK_ID);
                pb = 0;
                okp = false;
            }
            // the chunk lies in one block: one page, on the device or (offloaded) on the host
            KvPage loc{pb, false};
            if (p.kv.home) {
                okp = okp && kv_locate(p.kv, pb, loc);
                if (!okp) loc = KvPage{0, false};
            }
            if (!loc.host) {
                const int64_t at0 = page_offset(loc.page, h, p.Hkv, D) * (int64_t)sizeof(T) + (int64_t)(tc & 15) * ROWB;
#pragma unroll
                for (int i = 0; i < NCH * PIECES / 32; ++i) {
                    const int pc = lane + 32 * i;
                    const int r = pc / PIECES, w = pc - r * PIECES;
                    const int kv = w >= PIECES / 2, c = w - kv * (PIECES / 2);
                    const bool ok = okp && ch * NCH + r < n;
                    const unsigned char* src = ok ? (kv ? vbytes : kbytes) + at0 + (int64_t)r * ROWB + c * 16 : kbytes;
                    int off;
                    if constexpr (Geom::MMA) off = Geom::MCore::staged_offset(kv, r, c);
                    else off = r * TB + kv * ROWB + c * 16;
                    cp_async16(dst + off, src, ok);
                }
            } else {  // mapped host memory: plain loads, then the shared-memory stores
                const int64_t at0 = page_offset(loc.page, h, p.Hkv, D) * (int64_t)sizeof(T) + (int64_t)(tc & 15) * ROWB;
                for (int i = 0; i < NCH * PIECES / 32; ++i) {
                    const int pc = lane + 32 * i;
                    const int r = pc / PIECES, w = pc - r * PIECES;
                    const int kv = w >= PIECES / 2, c = w - kv * (PIECES / 2);
                    const bool ok = ch * NCH + r < n;
                    int off;
                    if constexpr (Geom::MMA) off = Geom::MCore::staged_offset(kv, r, c);
                    else off = r * TB + kv * ROWB + c * 16;
                    *reinterpret_cast<uint4*>(dst + off) =
                        ok ? *reinterpret_cast<const uint4*>((kv ? p.kv.host_v : p.kv.host_k) + at0 + (int64_t)r * ROWB + c * 16)
                           : make_uint4(0, 0, 0, 0);
                }
            }
        }
        cp_async_commit();
    };
    auto run = [&](auto& core) {
        for (int m = 0; m < GS - 1; ++m) fetch(m);
        for (int m = 0; m < my_n; ++m) {
            fetch(m + GS - 1);
            cp_async_wait<GS - 1>();
            __syncwarp();
            const unsigned char* src = wst + (m % GS) * Geom::CHUNK_BYTES;
            uint32_t valid = 0;
#pragma unroll
            for (int r = 0; r < NCH; ++r)
                if ((warp + m * NW) * NCH + r < n) valid |= 1u << r;
            if constexpr (Geom::MMA) {
                core.consume(src, valid, lane);
            } else {
                typename Core::raw_t kr[NCH], vr[NCH];
#pragma unroll
                for (int r = 0; r < NCH; ++r) {
                    kr[r] = Core::V::load(reinterpret_cast<const T*>(src + r * TB) + lane * Core::DPL);
                    vr[r] = Core::V::load(reinterpret_cast<const T*>(src + r * TB + ROWB) + lane * Core::DPL);
                }
                core.consume(kr, vr, valid, lane);
            }
            __syncwarp();
        }
        cp_async_wait<0>();
        core.store_partial(wpart + warp * G * (D + 2), lane);
    };
    __syncthreads();  // qs
    if constexpr (Geom::MMA) {
        typename Geom::MCore core;
        core.init(qs, p.scale_log2, lane);
        run(core);
    } else {
        Core core;
        core.init(qs, p.scale_log2, lane);
        run(core);
    }
    __syncthreads();
    float* dst = p.parts + ((int64_t)pair * p.splits + split) * G * (D + 2);
    for (int o = tid; o < G * D; o += kDenseThreads) {
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
