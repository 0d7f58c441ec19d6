// Fused Loki sparse decode step: one thread-block cluster of C CTAs per
// (sequence, kv head). The sequence's tokens are split into C contiguous
// ranges of whole 16-token blocks, one per CTA, and every phase stays on chip:
//
//  1. prologue: P[h] arrives in shared memory by one bulk async copy (TMA
//     engine); q_hat_j = q_j P[h] for the group's G query heads (AQUA page,
//     appendix step 1: project the query with P). The key stream of phase 2
//     is already in flight meanwhile.
//  2. rank-r scoring (AQUA page, related work on LoKi: slice the leading
//     dimensions after projection; Loki page, abstract: scores in the
//     low-dimensional space). Each warp owns a private ring of bulk-copy
//     slots; a slot receives the leading r/16 key slabs of one block, one
//     contiguous run of r*16 elements. Scores become order-preserving uint32
//     keys in shared memory; the histogram of their top 11 bits is built on
//     the fly.
//  3. top-k (Loki page, abstract: rank and select tokens): an exact radix
//     select with digits of 11, 11 and 10 bits. After each digit the CTAs
//     of the cluster sum their histograms through distributed shared memory,
//     so every CTA finds the same boundary digit. The result is the k-th
//     largest key tau and the number `need` of keys equal to tau to keep;
//     those go to the lowest token indices (ties to the lower index), CTA by
//     CTA in rank order. The recent window (aitopics page, LRQK abstract) is
//     appended. Kept tokens become an ascending list of local indices.
//  4. exact attention over the kept tokens (AQUA page, decode-step equations
//     (3)-(5)) by AttnCore, each warp on its share of the list, loads of the
//     next chunk in flight while the current one is consumed.
//  5. the warps' partials merge per CTA, then rank 0 merges the CTAs'
//     partials through distributed shared memory and writes the output.
#pragma once

#include <cooperative_groups.h>

#include "attn_core.cuh"

namespace loki {

namespace cg = cooperative_groups;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRingBytesPerWarp = 8192;
constexpr int kMaxSlots = 16;
constexpr int kHistBins = 2048;  // 11-bit digits (10 in the last pass)
constexpr int kCtaTokenCap = 16384;

struct SparseParams {
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_table;
    const int32_t* seq_lens;
    const int32_t* k_per_seq;
    const void* q;
    const float* P;
    float* out;
    int32_t* sel;
    int num_blocks, Hkv, max_blocks, max_seq_len;
    int r, k, W, group_max;
    float scale_log2;
    int C;           // CTAs per (sequence, kv head), = cluster size
    int cta_tokens;  // token capacity of one CTA, multiple of 16
    int slots;       // ring slots per warp
    int slot_bytes;  // bytes of one block's leading r dims
    // shared-memory layout, byte offsets
    int off_keys, off_ring, off_list, off_qf, off_qhat, off_qs, off_tbl, off_hist, off_bars, off_part,
        off_misc, smem_bytes;
};

// Exclusive suffix sum over the block: returns sum of v over threads > tid.
__device__ __forceinline__ uint32_t block_suffix_exclusive(uint32_t v, uint32_t* wsum, int lane, int warp) {
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_down_sync(kFull, x, o);
        if (lane + o < 32) x += y;
    }
    if (lane == 0) wsum[warp] = x;
    __syncthreads();
    uint32_t other = 0;
    for (int w = warp + 1; w < kWarps; ++w) other += wsum[w];
    __syncthreads();
    return x - v + other;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, 1) sparse_decode_kernel(const SparseParams p) {
    using Core = AttnCore<T, D, G>;
    constexpr int NCH = Core::NCH;
    extern __shared__ __align__(128) unsigned char smem[];
    cg::cluster_group cluster = cg::this_cluster();

    const int crank = (int)cluster.block_rank();
    const int pair = blockIdx.y;
    const int b = pair / p.Hkv;
    const int h = pair - b * p.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Hq = p.Hkv * G;

    uint32_t* keys = reinterpret_cast<uint32_t*>(smem + p.off_keys);
    float* Ps = reinterpret_cast<float*>(smem + p.off_keys);  // P[h] staging, before keys exist
    unsigned char* ring = smem + p.off_ring;
    float* wpart = reinterpret_cast<float*>(smem + p.off_ring);  // warp partials, after scoring
    uint16_t* list = reinterpret_cast<uint16_t*>(smem + p.off_list);
    float* qf = reinterpret_cast<float*>(smem + p.off_qf);
    float* qhat = reinterpret_cast<float*>(smem + p.off_qhat);
    float* qs = reinterpret_cast<float*>(smem + p.off_qs);
    int32_t* tbl = reinterpret_cast<int32_t*>(smem + p.off_tbl);
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + p.off_hist);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
    float* part = reinterpret_cast<float*>(smem + p.off_part);
    int32_t* misc = reinterpret_cast<int32_t*>(smem + p.off_misc);
    // misc: [0] boundary digit, [1] count above it, [8..15] warp sums,
    //       [16..23] warp gt counts, [24..31] warp eq counts, [32] list length

    // ---- sequence geometry (identical in every CTA of the cluster) ----
    int L = p.seq_lens[b];
    if (L < 0 || L > p.max_seq_len) {
        if (tid == 0 && crank == 0) flag_error(LOKI_DEVERR_SEQ_LEN);
        L = L < 0 ? 0 : p.max_seq_len;
    }
    const int Weff = p.W < L ? p.W : L;
    const int ncand = L - Weff;
    int kb = p.k;
    if (p.k_per_seq) {
        kb = p.k_per_seq[b];
        if (kb < 0 || kb > p.k) {
            if (tid == 0 && crank == 0) flag_error(LOKI_DEVERR_K);
            kb = kb < 0 ? 0 : p.k;
        }
    }
    const int keff = kb < ncand ? kb : ncand;
    const int nblk = (L + kBlockTokens - 1) / kBlockTokens;
    const int bpc = (nblk + p.C - 1) / p.C;
    const int blk0 = crank * bpc;
    const int t0 = blk0 * kBlockTokens;
    const int n_loc = max(0, min(L - t0, bpc * kBlockTokens));
    const int nblk_loc = (n_loc + kBlockTokens - 1) / kBlockTokens;
    const int n_cand_loc = max(0, min(ncand - t0, n_loc));
    const int nblk_score = (n_cand_loc + kBlockTokens - 1) / kBlockTokens;

    // ---- 1. prologue ----
    const int S = p.slots;
    uint64_t* pbar = bars + kWarps * kMaxSlots;
    if (tid == 0) {
        for (int i = 0; i < kWarps * kMaxSlots + 1; ++i) mbar_init(&bars[i], 1);
        fence_mbarrier_init();
    }
    for (int i = tid; i < 2 * kHistBins; i += kThreads) hist[i] = 0;
    for (int jb = tid; jb < nblk_loc; jb += kThreads) {
        int pb = p.block_table[(int64_t)b * p.max_blocks + blk0 + jb];
        if (pb < 0 || pb >= p.num_blocks) {
            flag_error(LOKI_DEVERR_BLOCK_ID);
            pb = 0;
        }
        tbl[jb] = pb;
    }
    const T* qg = reinterpret_cast<const T*>(p.q) + ((int64_t)b * Hq + h * G) * D;
    for (int i = tid; i < G * D; i += kThreads) qf[i] = Elem<T>::to_f(qg[i]);
    __syncthreads();

    if (tid == 0) {
        mbar_arrive_expect_tx(pbar, D * D * 4);
        bulk_copy_g2s(Ps, p.P + (int64_t)h * D * D, D * D * 4, pbar);
    }
    unsigned char* wring = ring + warp * kRingBytesPerWarp;
    uint64_t* wbar = bars + warp * kMaxSlots;
    const int my_blocks = nblk_score > warp ? (nblk_score - warp + kWarps - 1) / kWarps : 0;
    const unsigned char* kbytes = reinterpret_cast<const unsigned char*>(p.k_cache);
    auto issue = [&](int it) {
        const int jb = warp + it * kWarps;
        const int slot = it % S;
        const unsigned char* src = kbytes + page_offset(tbl[jb], h, p.Hkv, D) * (int64_t)sizeof(T);
        mbar_arrive_expect_tx(&wbar[slot], (uint32_t)p.slot_bytes);
        bulk_copy_g2s(wring + slot * p.slot_bytes, src, (uint32_t)p.slot_bytes, &wbar[slot]);
    };
    if (lane == 0) {
        const int first = my_blocks < S ? my_blocks : S;
        for (int it = 0; it < first; ++it) issue(it);
    }

    const bool okP = mbar_wait_bounded(pbar, 0);
    for (int o = tid; o < G * D; o += kThreads) {
        const int j = o / D, c = o - j * D;
        float a = 0.f;
#pragma unroll 8
        for (int i = 0; i < D; ++i) a = fmaf(qf[j * D + i], Ps[i * D + c], a);
        qhat[o] = okP ? a : 0.f;
    }
    __syncthreads();
    if (!p.group_max) {
        for (int c = tid; c < p.r; c += kThreads) {
            float s = 0.f;
            for (int j = 0; j < G; ++j) s += qhat[j * D + c];
            qs[c] = s;
        }
    }
    __syncthreads();

    // ---- 2. rank-r scoring ----
    {
        const int R16 = p.r / kSlabDims;
        const int tok = lane >> 1, half = lane & 1;
        bool failed = false;
        for (int it = 0; it < my_blocks; ++it) {
            const int slot = it % S;
            const uint32_t parity = (uint32_t)(it / S) & 1u;
            if (!failed) failed = __any_sync(kFull, !mbar_wait_bounded(&wbar[slot], parity));
            const T* sl = reinterpret_cast<const T*>(wring + slot * p.slot_bytes);
            float s;
            if (!p.group_max) {
                float a = 0.f;
                for (int sb = 0; sb < R16; ++sb) {
                    float kf[8];
                    Vec<T, 8>::to_float(Vec<T, 8>::load(sl + sb * 256 + tok * 16 + half * 8), kf);
                    const float* qq = qs + sb * 16 + half * 8;
#pragma unroll
                    for (int i = 0; i < 8; ++i) a = fmaf(qq[i], kf[i], a);
                }
                s = a + __shfl_xor_sync(kFull, a, 1);
            } else {
                float ag[G];
#pragma unroll
                for (int j = 0; j < G; ++j) ag[j] = 0.f;
                for (int sb = 0; sb < R16; ++sb) {
                    float kf[8];
                    Vec<T, 8>::to_float(Vec<T, 8>::load(sl + sb * 256 + tok * 16 + half * 8), kf);
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        const float* qq = qhat + j * D + sb * 16 + half * 8;
#pragma unroll
                        for (int i = 0; i < 8; ++i) ag[j] = fmaf(qq[i], kf[i], ag[j]);
                    }
                }
                s = -INFINITY;
#pragma unroll
                for (int j = 0; j < G; ++j) s = fmaxf(s, ag[j] + __shfl_xor_sync(kFull, ag[j], 1));
            }
            const int li = (warp + it * kWarps) * kBlockTokens + tok;
            if (half == 0 && li < n_cand_loc) {
                const uint32_t key = score_key(s);
                keys[li] = key;
                atomicAdd(&hist[key >> 21], 1u);
            }
            __syncwarp();
            if (lane == 0 && it + S < my_blocks) {
                fence_proxy_async_smem();
                issue(it + S);
            }
        }
    }
    __syncthreads();

    // ---- 3. top-k over the cluster ----
    // mode 0: keep every candidate, 1: keep none, 2: threshold tau / quota
    const int mode = keff >= ncand ? 0 : (keff == 0 ? 1 : 2);
    uint32_t tau = 0;
    int quota = 0;
    if (mode == 2) {
        uint32_t prefix = 0, pmask = 0;
        int krem = keff;
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
            const int nbins = pass == 2 ? 1024 : 2048;
            uint32_t* hcur = hist + (pass & 1) * kHistBins;
            if (pass > 0) {
                for (int i = tid; i < n_cand_loc; i += kThreads) {
                    const uint32_t key = keys[i];
                    if ((key & pmask) == prefix) atomicAdd(&hcur[(key >> shift) & (nbins - 1)], 1u);
                }
            }
            __syncthreads();
            cluster.sync();
            const int bpt = nbins / kThreads;  // 8 or 4 bins per thread
            uint32_t hv[8];
            uint32_t tsum = 0;
            for (int j = 0; j < bpt; ++j) {
                uint32_t s = 0;
                for (int c = 0; c < p.C; ++c) s += cluster.map_shared_rank(hcur, c)[tid * bpt + j];
                hv[j] = s;
                tsum += s;
            }
            uint32_t run = block_suffix_exclusive(tsum, reinterpret_cast<uint32_t*>(misc + 8), lane, warp);
            for (int j = bpt - 1; j >= 0; --j) {
                if (run < (uint32_t)krem && run + hv[j] >= (uint32_t)krem) {
                    misc[0] = tid * bpt + j;
                    misc[1] = (int)run;
                }
                run += hv[j];
            }
            __syncthreads();
            const int beta = misc[0];
            krem -= misc[1];
            prefix |= (uint32_t)beta << shift;
            pmask |= (uint32_t)(nbins - 1) << shift;
            if (pass < 2) {
                uint32_t* hnext = hist + ((pass + 1) & 1) * kHistBins;
                for (int i = tid; i < kHistBins; i += kThreads) hnext[i] = 0;
            }
            __syncthreads();
        }
        tau = prefix;
        // keys equal to tau: the last pass counted them per CTA in bin (tau & 1023)
        int eq_before = 0;
        for (int c = 0; c < crank; ++c) eq_before += (int)cluster.map_shared_rank(hist, c)[tau & 1023u];
        const int eq_mine = (int)hist[tau & 1023u];
        quota = min(max(krem - eq_before, 0), eq_mine);
    }

    // ---- compaction of the kept local tokens into `list`, ascending ----
    {
        const int chunk = (((n_cand_loc + kWarps - 1) / kWarps) + 31) & ~31;
        const int lo = warp * chunk;
        const int hi = min(lo + chunk, n_cand_loc);
        const unsigned lt_mask = (1u << lane) - 1u;
        int cnt_gt = 0, cnt_eq = 0;
        for (int base = lo; base < hi; base += 32) {
            const int i = base + lane;
            const bool in = i < hi;
            const uint32_t key = in ? keys[i] : 0u;
            const bool gt = in && (mode == 0 || (mode == 2 && key > tau));
            const bool eq = in && mode == 2 && key == tau;
            cnt_gt += __popc(__ballot_sync(kFull, gt));
            cnt_eq += __popc(__ballot_sync(kFull, eq));
        }
        if (lane == 0) {
            misc[16 + warp] = cnt_gt;
            misc[24 + warp] = cnt_eq;
        }
        __syncthreads();
        // warp w keeps all its keys above tau and the equal ones whose rank
        // among the CTA's equal keys (in index order) is below the quota
        int eq_base = 0, out_base = 0, total = 0, eb = 0;
        for (int w = 0; w < kWarps; ++w) {
            const int take = min(max(quota - eb, 0), misc[24 + w]);
            if (w < warp) {
                out_base += misc[16 + w] + take;
                eq_base += misc[24 + w];
            }
            total += misc[16 + w] + take;
            eb += misc[24 + w];
        }
        int run_eq = eq_base, run_out = out_base;
        for (int base = lo; base < hi; base += 32) {
            const int i = base + lane;
            const bool in = i < hi;
            const uint32_t key = in ? keys[i] : 0u;
            const bool gt = in && (mode == 0 || (mode == 2 && key > tau));
            const bool eq = in && mode == 2 && key == tau;
            const unsigned beq = __ballot_sync(kFull, eq);
            const bool take = gt || (eq && run_eq + __popc(beq & lt_mask) < quota);
            const unsigned bt = __ballot_sync(kFull, take);
            if (take) list[run_out + __popc(bt & lt_mask)] = (uint16_t)i;
            run_eq += __popc(beq);
            run_out += __popc(bt);
        }
        for (int i = tid; i < n_loc - n_cand_loc; i += kThreads) list[total + i] = (uint16_t)(n_cand_loc + i);
        if (tid == 0) misc[32] = total + (n_loc - n_cand_loc);
        __syncthreads();
    }
    const int n_list = misc[32];

    // ---- optional export of the kept set ----
    if (p.sel) {
        cluster.sync();
        int before = 0, all = 0;
        for (int c = 0; c < p.C; ++c) {
            const int nc = cluster.map_shared_rank(misc, c)[32];
            if (c < crank) before += nc;
            all += nc;
        }
        const int width = p.k + p.W;
        int32_t* dst = p.sel + (int64_t)pair * width;
        for (int i = tid; i < n_list; i += kThreads) dst[before + i] = t0 + (int)list[i];
        if (crank == p.C - 1)
            for (int i = all + tid; i < width; i += kThreads) dst[i] = -1;
    }

    // ---- 4. exact attention over the kept tokens ----
    {
        const T* kc = reinterpret_cast<const T*>(p.k_cache);
        const T* vc = reinterpret_cast<const T*>(p.v_cache);
        Core core;
        core.init(qhat, p.scale_log2, lane);
        typename Core::raw_t kA[NCH], vA[NCH], kB[NCH], vB[NCH];
        uint32_t validA = 0, validB = 0;
        const int nchunks = (n_list + NCH - 1) / NCH;
        auto load = [&](typename Core::raw_t (&kr)[NCH], typename Core::raw_t (&vr)[NCH], uint32_t& valid,
                        int ch) {
            valid = 0;
#pragma unroll
            for (int n = 0; n < NCH; ++n) {
                const int idx = ch * NCH + n;
                if (idx < n_list) {
                    const int li = list[idx];
                    const int64_t page = page_offset(tbl[li >> 4], h, p.Hkv, D);
                    kr[n] = Core::V::load(Core::key_ptr(kc, page, li & 15, lane));
                    vr[n] = Core::V::load(Core::val_ptr(vc, page, li & 15, lane));
                    valid |= 1u << n;
                } else {
                    kr[n] = Core::zero_raw();
                    vr[n] = Core::zero_raw();
                }
            }
        };
        int ch = warp;
        if (ch < nchunks) load(kA, vA, validA, ch);
        for (; ch < nchunks; ch += 2 * kWarps) {
            if (ch + kWarps < nchunks) load(kB, vB, validB, ch + kWarps);
            core.consume(kA, vA, validA, lane);
            if (ch + kWarps >= nchunks) break;
            if (ch + 2 * kWarps < nchunks) load(kA, vA, validA, ch + 2 * kWarps);
            core.consume(kB, vB, validB, lane);
        }
        core.store_partial(wpart + warp * G * (D + 2), lane);
    }
    __syncthreads();

    // ---- 5. merge: warps -> CTA partial -> cluster rank 0 -> out ----
    for (int o = tid; o < G * D; o += kThreads) {
        const int j = o / D, c = o - j * D;
        const Merged mg = merge_partials<D>(wpart, kWarps, G * (D + 2), j, c);
        part[j * (D + 2) + c] = mg.o;
        if (c == 0) {
            part[j * (D + 2) + D] = mg.m;
            part[j * (D + 2) + D + 1] = mg.l;
        }
    }
    cluster.sync();
    if (crank == 0) {
        for (int o = tid; o < G * D; o += kThreads) {
            const int j = o / D, c = o - j * D;
            float M = -INFINITY;
            for (int r = 0; r < p.C; ++r) M = fmaxf(M, cluster.map_shared_rank(part, r)[j * (D + 2) + D]);
            float num = 0.f, den = 0.f;
            if (M != -INFINITY) {
                for (int r = 0; r < p.C; ++r) {
                    const float* pr = cluster.map_shared_rank(part, r) + j * (D + 2);
                    const float mr = pr[D];
                    if (mr == -INFINITY) continue;
                    const float w = exp2f(mr - M);
                    num = fmaf(w, pr[c], num);
                    den = fmaf(w, pr[D + 1], den);
                }
            }
            p.out[((int64_t)b * Hq + h * G + j) * D + c] = den > 0.f ? num / den : 0.f;
        }
    }
    cluster.sync();
}

}  // namespace loki
