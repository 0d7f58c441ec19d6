// Fused Loki sparse decode step: one thread-block cluster of C CTAs per
// (sequence, kv head). CTA c owns the fixed token range [c * cta_tokens,
// (c + 1) * cta_tokens) of its sequence (whole 16-token blocks), and every
// phase stays on chip:
//
//  1. prologue: the key-index stream of phase 2 starts at once; meanwhile
//     q_hat_j = q_j P[h] for the group's G query heads (AQUA page, appendix on
//     complexity, step 1), register-blocked over (row group, column quad) of P.
//  2. rank-r scoring (AQUA page, related work on LoKi: slice the leading
//     dimensions after projection; Loki page, abstract: scores in the
//     low-dimensional space). Each warp owns a private ring of S slots; a
//     slot receives r index dims of one 16-token block (dim-major: one row
//     of 16 tokens per dim; the leading r dims are one contiguous run of
//     r*16 elements) as 16-byte cp.async pieces from all lanes; with r <= 32
//     a warp loads two blocks before scoring either.
//     Scores become order-preserving uint32 keys in shared memory; the
//     histogram of their top 11 bits is built on the fly with shared
//     atomics. Three other scorers share the kernel (template argument SC,
//     at the kernel's declaration): the single index dims of largest query
//     magnitude, the index slabs with the most query energy, and asymmetric
//     factors (q A_q against an index of k A_k).
//  3. top-k (Loki page, abstract: rank and select tokens): an exact radix
//     select with digits of 11, 11 and 10 bits. After each digit the CTAs of
//     the cluster sum their histograms through distributed shared memory, so
//     every CTA finds the same boundary digit. One pass after the first digit
//     sorts the keys into kept-for-sure and candidates; the later digits see
//     only the candidates. The result is the k-th largest key tau and the
//     number of keys equal to tau to keep; those go to the lowest token
//     indices (ties to the lower index), CTA by CTA in rank order. The recent
//     window (aitopics page, LRQK abstract) is appended. Kept tokens become
//     an ascending list of local indices.
//  4. exact attention over the kept tokens (AQUA page, decode-step equations
//     (3)-(5)): each warp stages chunks of key rows and value rows into
//     shared memory with cp.async (the next chunk in flight while the current
//     one is consumed) and runs MmaAttnCore (bf16, warp-level MMA) or
//     AttnCore (fp32, CUDA cores) on them.
//  5. the warps' partials merge per CTA into a slot of rank 0's shared
//     memory (distributed shared memory stores); after one cluster barrier
//     rank 0 combines the slots and writes the output.
#pragma once

#include <cooperative_groups.h>

#include <type_traits>

#include "attn_core.cuh"

namespace loki {

namespace cg = cooperative_groups;

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxSlots = 16;
constexpr int kHistBins = 2048;  // 11-bit digits (10 in the last pass)
constexpr int kCtaTokenCap = 16384;

struct SparseParams {
    const void* k_cache;
    const void* v_cache;
    const void* k_index;
    const int32_t* block_table;
    const int32_t* seq_lens;
    const int32_t* k_per_seq;
    const void* q;
    const float* P;
    const float* Aq;  // [Hkv][D][index_dims] query factor (asymmetric scorer only)
    float* out;
    int32_t* sel;
    KvMap kv;
    int num_blocks, Hkv, max_blocks, max_seq_len, index_dims;
    int batch;
    int longest_first;  // clusters take the sequences longest first (batch <= 64)
    int r, k, W, group_max;
    float scale_log2;
    int C;           // CTAs per (sequence, kv head), = cluster size
    int cta_tokens;  // token capacity of one CTA, multiple of 16
    int slots;       // ring slots per warp
    int slot_bytes;  // bytes of one block's leading r index dims
    int ring_bytes_per_warp;
    // shared-memory layout, byte offsets. keys and ring are adjacent: after the
    // scoring the ring region holds the candidate buffer (head) and the kept
    // list (tail), and the gather stages rows across keys + ring minus list.
    int off_keys, keys_bytes, off_ring, ring_bytes, off_list, off_qf, off_qhat, off_qs, off_tbl, off_hist,
        off_part, off_misc, smem_bytes;
};

#ifndef LOKI_GATHER_CHUNK
#define LOKI_GATHER_CHUNK 8
#endif
template <typename T, int D, int G>
struct SparseGeom {
    // bf16 caches: tensor-core attention on 8-token chunks; fp32: CUDA cores
    static constexpr bool MMA = std::is_same<T, __nv_bfloat16>::value;
    using Core = AttnCore<T, D, G, (LOKI_GATHER_CHUNK * G > 32 ? 32 / G : LOKI_GATHER_CHUNK)>;
    using MCore = MmaAttnCore<D, G>;
    static constexpr int NCH = MMA ? MCore::NCH : Core::NCH;
    static constexpr int TB = 2 * D * (int)sizeof(T);  // key row + value row bytes
    static constexpr int CHUNK_BYTES = NCH * TB;
    static constexpr int GS_FIT = (160 * 1024) / (kWarps * CHUNK_BYTES);
    static constexpr int GS = GS_FIT < 1 ? 1 : (GS_FIT > 8 ? 8 : GS_FIT);  // staged chunks per warp
    static constexpr int STAGE_BYTES = kWarps * GS * CHUNK_BYTES;
    static constexpr int WPART_BYTES = kWarps * G * (D + 2) * 4;
    static constexpr int QSCRATCH_BYTES = (2048 / D) * G * D * 4;  // row groups x G x D floats
};


// Exclusive prefix sum over the lanes of a warp.
__device__ __forceinline__ int warp_exclusive_scan(int v, int lane) {
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    return x - v;
}

// Exclusive suffix sum over the block: returns sum of v over threads > tid.
// wsum: kWarps words of shared scratch, free again once every thread of the
// block has passed the next block-wide barrier.
__device__ __forceinline__ uint32_t block_suffix_exclusive(uint32_t v, uint32_t* wsum, int lane, int warp) {
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(kFull, x, o);
        if (lane + o < 32) x += y;
    }
    if (lane == 0) wsum[warp] = x;  // warp total
    __syncthreads();
    // every warp forms the suffix over the warp totals itself (one barrier)
    const uint32_t t = lane < kWarps ? wsum[lane] : 0u;
    uint32_t s = t;
#pragma unroll
    for (int o = 1; o < kWarps; o <<= 1) {
        const uint32_t y = __shfl_down_sync(kFull, s, o);
        if (lane + o < kWarps) s += y;
    }
    return x - v + __shfl_sync(kFull, s - t, warp);  // totals of the warps after this one
}

// One digit of the cluster-wide radix select. Sums the cluster's histograms
// hcur[0 .. nbins) (nbins <= 4 * kThreads, a multiple of 4) through distributed
// shared memory and finds the digit where the count of keys from the top
// reaches krem. Returns (digit, count above it) in every thread. Called by all
// threads of every CTA of the cluster; not inlined, so the three digits share
// one copy of the code.
__device__ __noinline__ int2 radix_boundary(const uint32_t* hcur, int nbins, int krem, int32_t* misc, int C) {
    cg::cluster_group cluster = cg::this_cluster();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    cluster.sync();  // every thread of every CTA: the histograms are complete and visible
    uint32_t hv[4] = {0u, 0u, 0u, 0u};  // bins 4 tid .. 4 tid + 3
    if (4 * tid < nbins) {
#pragma unroll 4
        for (int c = 0; c < C; ++c) {  // unrolled: the ranks' loads are in flight together
            const uint4 v = reinterpret_cast<const uint4*>(cluster.map_shared_rank(hcur, c))[tid];
            hv[0] += v.x;
            hv[1] += v.y;
            hv[2] += v.z;
            hv[3] += v.w;
        }
    }
    const uint32_t tsum = hv[0] + hv[1] + hv[2] + hv[3];
    uint32_t run = block_suffix_exclusive(tsum, reinterpret_cast<uint32_t*>(misc + 8), lane, warp);
#pragma unroll
    for (int j = 3; j >= 0; --j) {
        if (run < (uint32_t)krem && run + hv[j] >= (uint32_t)krem) {
            misc[0] = 4 * tid + j;
            misc[1] = (int)run;
            misc[2] = (int)hv[j];  // the boundary bin's count over the cluster
        }
        run += hv[j];
    }
    __syncthreads();
    return make_int2(misc[0], misc[1]);
}

// Scorers (template argument SC):
//  kScoreLeading: q_hat_j against the leading r index dims (Loki).
//  kScoreMagnitude: per (sequence, kv head) and step, the r single index dims
//    of largest magnitude of the query that ranks the tokens (AQUA page,
//    Algorithm 1 in prose and appendix on complexity, steps 2-4): |sum_j
//    q_hat_j[c]| (SUM) or sum_j q_hat_j[c]^2 (MAX), ties to the lower dim. A
//    chosen dim of a block is one 16-element row of the dim-major index.
//  kScoreSlabs: the r / 16 index slabs (16 consecutive dims) that hold the
//    most energy of that query, ties to the lower slab (a coarser variant).
//  kScoreAsym: q_j A_q[h] against the leading r dims of an index that holds
//    k A_k (SAKI page, abstract: asymmetric query and key factors of the
//    score operator); the exact attention still uses q_hat = q P.
constexpr int kScoreLeading = 0, kScoreMagnitude = 1, kScoreSlabs = 2, kScoreAsym = 3;
constexpr int kSelDims = 128;  // misc words 128 .. 255: the chosen index dims in slot order

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                                  const void* row_ptr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(row_ptr)));
}

template <typename T, int D, int G, int SC>
__global__ void __launch_bounds__(kThreads, 1) sparse_decode_kernel(const SparseParams p) {
    constexpr bool MAG = SC == kScoreMagnitude || SC == kScoreSlabs;  // dims chosen per step
    constexpr bool ASYM = SC == kScoreAsym;
    using Geom = SparseGeom<T, D, G>;
    using Core = typename Geom::Core;
    constexpr int NCH = Geom::NCH;
    constexpr int TB = Geom::TB;
    constexpr int GS = Geom::GS;
    extern __shared__ __align__(128) unsigned char smem[];
    cg::cluster_group cluster = cg::this_cluster();

    const int crank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = (int)blockIdx.y % p.Hkv;
    const int Hq = p.Hkv * G;

    uint32_t* keys = reinterpret_cast<uint32_t*>(smem + p.off_keys);
    float* qscratch = reinterpret_cast<float*>(smem + p.off_keys);  // prologue only
    unsigned char* stage = smem + p.off_keys;                        // gather only (keys + ring)
    float* wpart = reinterpret_cast<float*>(smem + p.off_keys);     // after the gather
    unsigned char* ring = smem + p.off_ring;
    uint16_t* list = reinterpret_cast<uint16_t*>(smem + p.off_list);
    uint32_t* cand = reinterpret_cast<uint32_t*>(ring);             // select only (ring head)
    float* wts = reinterpret_cast<float*>(smem + p.off_qf);         // merge weights [G][kWarps]
    float* qhat = reinterpret_cast<float*>(smem + p.off_qhat);
    float* qs = reinterpret_cast<float*>(smem + p.off_qs);
    int32_t* tbl = reinterpret_cast<int32_t*>(smem + p.off_tbl);
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + p.off_hist);
    float* part = reinterpret_cast<float*>(smem + p.off_part);
    // the query the scoring uses, [G][D] rows: q_hat, or (asymmetric) q A_q
    // in `part`, whose first G x D floats only rank 0's own merge writes
    const float* qsc = ASYM ? part : qhat;
    int32_t* misc = reinterpret_cast<int32_t*>(smem + p.off_misc);
    // misc: [0] boundary digit, [1] count above it, [2] its bin count, [8..39] suffix-sum scratch,
    //       [40..55] warp kept counts, [56..71] warp equal counts, [72] list length,
    //       [73] the sequence (longest first), [104..111] slab energies (slab
    //       scorer), [128..255] chosen dims (MAG)

    // ---- which sequence ----
    // Over several waves of clusters the sequences go longest first (ties:
    // the lower index), so that the short ones fill the last wave: cluster
    // row j takes the sequence of rank j. Warp 0 ranks up to 64 lengths.
    int b = (int)blockIdx.y / p.Hkv;
    if (p.longest_first) {
        if (warp == 0) {
            const int l0 = lane < p.batch ? p.seq_lens[lane] : 0;
            const int l1 = lane + 32 < p.batch ? p.seq_lens[lane + 32] : 0;
            int r0 = 0, r1 = 0;
            for (int i = 0; i < p.batch; ++i) {
                const int li = __shfl_sync(kFull, i < 32 ? l0 : l1, i & 31);
                r0 += (li > l0 || (li == l0 && i < lane)) ? 1 : 0;
                r1 += (li > l1 || (li == l1 && i < lane + 32)) ? 1 : 0;
            }
            if (lane < p.batch && r0 == b) misc[73] = lane;
            if (lane + 32 < p.batch && r1 == b) misc[73] = lane + 32;
        }
        __syncthreads();
        b = misc[73];
    }
    const int pair = b * p.Hkv + h;

    // ---- sequence geometry ----
    // CTA crank owns the fixed token range [crank * cta_tokens, + cta_tokens)
    // of its sequence, so its block-table loads need not wait for the length.
    // In one wave of clusters the launch takes as long as the longest
    // sequence whatever the split of the shorter ones; over several waves a
    // CTA with a short or empty range ends early and frees its SM.
    const int cta_blocks = p.cta_tokens / kBlockTokens;
    const int blk0 = crank * cta_blocks;
    const int t0 = blk0 * kBlockTokens;
    // block-table entries of this warp's blocks jb = warp + it * kWarps:
    // lane l holds those of it = l and it = l + 32 (at most 64 per warp);
    // entries past the end of the sequence are loaded but never used
    const int32_t* trow = p.block_table + (int64_t)b * p.max_blocks + blk0;
    int tb0 = 0, tb1 = 0;
    const int j0 = warp + lane * kWarps, j1 = warp + (lane + 32) * kWarps;
    {
        const int lim = min(cta_blocks, p.max_blocks - blk0);
        if (j0 < lim) tb0 = trow[j0];
        if (j1 < lim) tb1 = trow[j1];
    }
    // the prologue's P and q loads do not depend on the length either
    constexpr int NQ = D / 4;             // q_hat: thread (row group rg, column quad cq)
    constexpr int NRG = kThreads / NQ;
    constexpr int RPG = D / NRG;
    const int cq = tid % NQ, rg = tid / NQ;
    float4 pv[RPG];
    {
        const float* Ph = p.P + (int64_t)h * D * D;
#pragma unroll
        for (int i = 0; i < RPG; ++i) pv[i] = *reinterpret_cast<const float4*>(Ph + (rg * RPG + i) * D + 4 * cq);
    }
    // the group's queries, G x D elements: 16-byte piece i read by thread i
    // (whole 128-byte requests, which matters when q is read in place from
    // host memory) and staged in the q_hat region until the first barrier
    const T* qg = reinterpret_cast<const T*>(p.q) + ((int64_t)b * Hq + h * G) * D;
    constexpr int QP = G * D * (int)sizeof(T) / 16;
    static_assert(QP <= kThreads && QP * 16 == G * D * (int)sizeof(T), "query pieces");
    uint4 qpiece = make_uint4(0u, 0u, 0u, 0u);
    if (tid < QP) qpiece = reinterpret_cast<const uint4*>(qg)[tid];
    typename Vec<T, RPG>::raw_t qraw[G];
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
    const int n_loc = max(0, min(L - t0, p.cta_tokens));
    const int nblk_loc = (n_loc + kBlockTokens - 1) / kBlockTokens;
    const int n_cand_loc = max(0, min(ncand - t0, n_loc));
    const int nblk_score = (n_cand_loc + kBlockTokens - 1) / kBlockTokens;

    // ---- 1. prologue: every global load is issued before the first barrier ----
    const int S = p.slots;

    // each warp starts its key-index stream as soon as its block-table
    // entries arrive, before any CTA-wide barrier
    unsigned char* wring = ring + warp * p.ring_bytes_per_warp;
    auto checked = [&](int pb) {
        if (pb < 0 || pb >= p.num_blocks) {
            flag_error(LOKI_DEVERR_BLOCK_ID);
            return 0;
        }
        return pb;
    };
    tb0 = j0 < nblk_loc ? checked(tb0) : 0;
    tb1 = j1 < nblk_loc ? checked(tb1) : 0;
    const int my_blocks = nblk_score > warp ? (nblk_score - warp + kWarps - 1) / kWarps : 0;
    const unsigned char* xbytes = reinterpret_cast<const unsigned char*>(p.k_index);
    auto entry = [&](int it) {  // all lanes: block of this warp's iteration it
        const int v0 = __shfl_sync(kFull, tb0, it & 31);
        const int v1 = __shfl_sync(kFull, tb1, it & 31);
        return it < 32 ? v0 : v1;
    };
    // Ring of S slots per warp (S a power of two dividing kMaxSlots): every
    // lane copies 16-byte pieces of a block with cp.async (pieces lane,
    // lane + 32, ...). Each refill commits kMaxSlots / S groups, the block's
    // and empty ones (all empty past the warp's last block), so that exactly
    // kMaxSlots - 1 groups are younger than the oldest block in flight and
    // waiting for it is always cp.async.wait_group kMaxSlots - 1: no run-time
    // count, no division in the loop.
    const int smask = S - 1;
    const int pad = kMaxSlots / S - 1;
    auto refill = [&](int it) {  // all lanes; slot it & smask is free
        if (it < my_blocks) {
            const int pb = entry(it);
            const unsigned char* src = xbytes + page_offset(pb, h, p.Hkv, p.index_dims) * (int64_t)sizeof(T);
            unsigned char* dst = wring + (it & smask) * p.slot_bytes;
            // dim row i of the slot <- index dim i (or the i-th chosen dim)
            // of the block's 16 tokens; bf16 rows swap their two 16-byte
            // halves on rows 4..7 mod 8, so that ldmatrix.trans is free of
            // bank conflicts
            if constexpr (!MAG) {
                // the leading r dims: one contiguous run of the page (bf16:
                // the half swap of rows 4..7 mod 8 is bit 4 of the byte
                // offset flipped where bit 7 is set). The scoring loop is
                // issue-bound; the per-piece row arithmetic of the general
                // form below cost about 2.5 us at 32k tokens.
                for (int o = lane * 16; o < p.slot_bytes; o += 32 * 16)
                    cp_async16(dst + (sizeof(T) == 2 ? (o ^ ((o >> 3) & 16)) : o), src + o, true);
            } else {
                constexpr int PPR = (int)sizeof(T);  // 16-byte pieces of one dim row
                for (int pc = lane; pc < p.r * PPR; pc += 32) {
                    const int row = pc / PPR, part = pc - row * PPR;
                    const int dim = misc[kSelDims + row];
                    const int dpart = sizeof(T) == 2 ? (part ^ ((row >> 2) & 1)) : part;
                    cp_async16(dst + row * 16 * (int)sizeof(T) + dpart * 16, src + dim * 16 * (int)sizeof(T) + part * 16,
                               true);
                }
            }
        }
        cp_async_commit();
        for (int i = 0; i < pad; ++i) cp_async_commit();
    };
    // Launched as the programmatic dependent of the step's append, the kernel
    // must not read the appended token (position L - 1) before that grid is
    // done. With a recent window the token is not a scoring candidate and is
    // first read by the gather; without one the key index may hold it.
    // (The scoring copies whole 16-token blocks: bytes of a token that is not
    // a candidate may be read while being written; they are never used.)
    // (the magnitude scorer knows which slabs to fetch only after q_hat)
    if constexpr (!MAG) {
        if (p.W == 0) griddep_wait();
        for (int it = 0; it < S; ++it) refill(it);
    }
    for (int i = tid; i < 2 * kHistBins; i += kThreads) hist[i] = 0;
    if (j0 < nblk_loc) tbl[j0] = tb0;
    if (j1 < nblk_loc) tbl[j1] = tb1;
    if (tid < QP) reinterpret_cast<uint4*>(qhat)[tid] = qpiece;
    __syncthreads();
    // this thread's RPG rows of each query (q_hat overwrites the staging only
    // after the next barrier)
#pragma unroll
    for (int j = 0; j < G; ++j) qraw[j] = Vec<T, RPG>::load(reinterpret_cast<const T*>(qhat) + j * D + rg * RPG);

    {   // q_hat = q P[h]: each thread sums its RPG rows for its 4 columns
        float qv[G][RPG];
#pragma unroll
        for (int j = 0; j < G; ++j) Vec<T, RPG>::to_float(qraw[j], qv[j]);
        float a[G][4];
#pragma unroll
        for (int j = 0; j < G; ++j) a[j][0] = a[j][1] = a[j][2] = a[j][3] = 0.f;
#pragma unroll
        for (int i = 0; i < RPG; ++i) {
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const float x = qv[j][i];
                a[j][0] = fmaf(x, pv[i].x, a[j][0]);
                a[j][1] = fmaf(x, pv[i].y, a[j][1]);
                a[j][2] = fmaf(x, pv[i].z, a[j][2]);
                a[j][3] = fmaf(x, pv[i].w, a[j][3]);
            }
        }
#pragma unroll
        for (int j = 0; j < G; ++j)
            *reinterpret_cast<float4*>(qscratch + (rg * G + j) * D + 4 * cq) =
                make_float4(a[j][0], a[j][1], a[j][2], a[j][3]);
        __syncthreads();
        for (int o = tid; o < G * D; o += kThreads) {
            float s = 0.f;
            for (int g = 0; g < NRG; ++g) s += qscratch[g * G * D + o];
            qhat[o] = s;
        }
        __syncthreads();
        if constexpr (ASYM) {
            // q A_q[h], first r columns, with q_hat's blocking: thread
            // (rg, cq) sums its RPG rows for its 4 columns, the row groups'
            // partial sums are added in the same order as for q_hat
            const int I = p.index_dims;
            float a[G][4];
#pragma unroll
            for (int j = 0; j < G; ++j) a[j][0] = a[j][1] = a[j][2] = a[j][3] = 0.f;
            if (4 * cq < p.r) {
                const float* Ah = p.Aq + (int64_t)h * D * I;
                float qv[G][RPG];
#pragma unroll
                for (int j = 0; j < G; ++j) Vec<T, RPG>::to_float(qraw[j], qv[j]);
#pragma unroll
                for (int i = 0; i < RPG; ++i) {
                    const float4 av = *reinterpret_cast<const float4*>(Ah + (int64_t)(rg * RPG + i) * I + 4 * cq);
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        const float x = qv[j][i];
                        a[j][0] = fmaf(x, av.x, a[j][0]);
                        a[j][1] = fmaf(x, av.y, a[j][1]);
                        a[j][2] = fmaf(x, av.z, a[j][2]);
                        a[j][3] = fmaf(x, av.w, a[j][3]);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < G; ++j)
                *reinterpret_cast<float4*>(qscratch + (rg * G + j) * D + 4 * cq) =
                    make_float4(a[j][0], a[j][1], a[j][2], a[j][3]);
            __syncthreads();
            for (int o = tid; o < G * D; o += kThreads) {
                if (o % D >= p.r) continue;
                float s = 0.f;
                for (int g = 0; g < NRG; ++g) s += qscratch[g * G * D + o];
                part[o] = s;
            }
            __syncthreads();
        }
        if (!p.group_max) {
            for (int c = tid; c < (MAG ? p.index_dims : p.r); c += kThreads) {
                float s = 0.f;
                for (int j = 0; j < G; ++j) s += qsc[j * D + c];
                qs[c] = s;
            }
        }
        __syncthreads();
        if constexpr (SC == kScoreMagnitude) {
            // the r dims of largest magnitude among the first index_dims:
            // |summed query| (SUM) or the heads' summed squares (MAX), ties to
            // the lower dim, listed in ascending order
            float* w = reinterpret_cast<float*>(smem + p.off_keys);  // the keys region is free until scoring
            const int I = p.index_dims;
            if (tid < I) {
                float x = 0.f;
                if (!p.group_max) {
                    x = fabsf(qs[tid]);
                } else {
                    for (int j = 0; j < G; ++j) x = fmaf(qhat[j * D + tid], qhat[j * D + tid], x);
                }
                w[tid] = x;
            }
            __syncthreads();
            bool chosen = false;
            if (tid < I) {
                const float x = w[tid];
                int rank = 0;
                for (int o = 0; o < I; ++o) rank += w[o] > x || (w[o] == x && o < tid);
                chosen = rank < p.r;
            }
            const unsigned bal = __ballot_sync(kFull, chosen);
            if (lane == 0 && warp < 4) misc[112 + warp] = __popc(bal);
            __syncthreads();
            if (chosen) {
                int pos = __popc(bal & ((1u << lane) - 1u));
                for (int v = 0; v < warp; ++v) pos += misc[112 + v];
                misc[kSelDims + pos] = tid;
            }
            __syncthreads();
            if (p.W == 0) griddep_wait();
            for (int it = 0; it < S; ++it) refill(it);
        } else if constexpr (SC == kScoreSlabs) {
            // slab energy: squared norm of the summed query over the slab (SUM),
            // or summed over the group's heads (MAX); the r / 16 largest, ties
            // to the lower slab, listed in ascending slab order
            const int nsl = p.index_dims / kSlabDims, R16 = p.r / kSlabDims;
            float* en = reinterpret_cast<float*>(misc + 104);
            if (tid < nsl) {
                float w = 0.f;
                for (int c = tid * kSlabDims; c < (tid + 1) * kSlabDims; ++c) {
                    if (!p.group_max) {
                        w = fmaf(qs[c], qs[c], w);
                    } else {
                        for (int j = 0; j < G; ++j) w = fmaf(qhat[j * D + c], qhat[j * D + c], w);
                    }
                }
                en[tid] = w;
            }
            __syncthreads();
            if (tid == 0) {
                int n = 0;
                for (int sl = 0; sl < nsl; ++sl) {
                    int rank = 0;
                    for (int o = 0; o < nsl; ++o) rank += en[o] > en[sl] || (en[o] == en[sl] && o < sl);
                    if (rank < R16) {
                        for (int c = 0; c < kSlabDims; ++c) misc[kSelDims + n * kSlabDims + c] = sl * kSlabDims + c;
                        ++n;
                    }
                }
            }
            __syncthreads();
            if (p.W == 0) griddep_wait();
            for (int it = 0; it < S; ++it) refill(it);
        }
    }

    // ---- 2. rank-r scoring ----
    // A warp takes one block per iteration: its slot is read into registers and
    // refilled with the block S iterations ahead before the arithmetic. bf16 index:
    // the 16 x 16 tile of each slab (16 tokens x 16 dims) times a fragment whose
    // columns hold the score vector split into bf16 high part and remainder
    // (SUM: the summed query in columns 0, 1; MAX: q_hat_j in columns 2j, 2j+1,
    // a second column group for heads 4..7), on warp-level MMA with fp32
    // accumulation. fp32 index: CUDA-core dot products.
    {
        auto wait_slot = [&]() {  // all lanes: the oldest slot in flight has landed
            cp_async_wait<kMaxSlots - 1>();
            __syncwarp();
        };
        auto mma_body = [&](auto rmax_tag) {
            constexpr int RMAX = decltype(rmax_tag)::value;
            constexpr int SG = G > 4 ? 2 : 1;
            const int R16 = p.r / kSlabDims;
            const int g = lane >> 2, t = lane & 3;
            const int ngroups = p.group_max ? SG : 1;
            uint32_t qb[SG][RMAX][2];
#pragma unroll
            for (int ng = 0; ng < SG; ++ng)
#pragma unroll
                for (int sb = 0; sb < RMAX; ++sb) {
                    float v[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float x = 0.f;
                        if (sb < R16) {
                            const int i = sb * 16 + 2 * t + (e & 1) + (e >> 1) * 8;  // slot row
                            const int d = MAG ? misc[kSelDims + i] : i;
                            if (!p.group_max) {
                                x = (ng == 0 && g < 2) ? split_part(qs[d], g & 1) : 0.f;
                            } else {
                                const int head = ng * 4 + (g >> 1);
                                x = head < G ? split_part(qsc[head * D + d], g & 1) : 0.f;
                            }
                        }
                        v[e] = x;
                    }
                    qb[ng][sb][0] = pack_bf16(v[0], v[1]);
                    qb[ng][sb][1] = pack_bf16(v[2], v[3]);
                }
            // ldmatrix.trans row address of this lane: matrix m = lane / 8 holds
            // tokens 8 (m & 1) .. + 7 of dims 8 (m >> 1) + (lane & 7) of the k-step
            const int mrow = (lane & 7) + 8 * (lane >> 4), mhalf = (lane >> 3) & 1;
            // byte offset of that row in slab 0 (slab sb adds 512: 16 rows of 32 bytes,
            // and row + 16 sb swaps its halves exactly when row does)
            const int loff = mrow * 32 + ((mhalf ^ ((mrow >> 2) & 1)) << 4);
            // block it's slot into fragments, then the slot's refill
            auto load_block = [&](int it, uint32_t (&a)[RMAX][4]) {
                wait_slot();
                const unsigned char* sl = wring + (it & smask) * p.slot_bytes;
#pragma unroll
                for (int sb = 0; sb < RMAX; ++sb)
                    if (sb < R16) ldmatrix_x4_trans(a[sb][0], a[sb][1], a[sb][2], a[sb][3], sl + sb * 512 + loff);
                __syncwarp();
                refill(it + S);
            };
            // block it's scores, keys and digit-0 histogram counts
            auto score_block = [&](int it, const uint32_t (&a)[RMAX][4]) {
                float sc0 = -INFINITY, sc1 = -INFINITY;  // tokens g and g + 8
#pragma unroll
                for (int ng = 0; ng < SG; ++ng) {
                    if (ng < ngroups) {
                        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int sb = 0; sb < RMAX; ++sb)
                            if (sb < R16) mma_16816_bf16(c, a[sb][0], a[sb][1], a[sb][2], a[sb][3], qb[ng][sb][0], qb[ng][sb][1]);
                        float h0 = c[0] + c[1], h1 = c[2] + c[3];  // column pair t: head 4 ng + t (MAX) / qs (SUM, t = 0)
                        if (p.group_max) {
                            if (ng * 4 + t >= G) h0 = h1 = -INFINITY;
                            h0 = fmaxf(h0, __shfl_xor_sync(kFull, h0, 1));
                            h0 = fmaxf(h0, __shfl_xor_sync(kFull, h0, 2));
                            h1 = fmaxf(h1, __shfl_xor_sync(kFull, h1, 1));
                            h1 = fmaxf(h1, __shfl_xor_sync(kFull, h1, 2));
                        }
                        sc0 = fmaxf(sc0, h0);
                        sc1 = fmaxf(sc1, h1);
                    }
                }
                if (t == 0) {
                    const int base = (warp + it * kWarps) * kBlockTokens;
                    if (base + g < n_cand_loc) {
                        const uint32_t key = score_key(sc0);
                        keys[base + g] = key;
                        atomicAdd(&hist[key >> 21], 1u);
                    }
                    if (base + g + 8 < n_cand_loc) {
                        const uint32_t key = score_key(sc1);
                        keys[base + g + 8] = key;
                        atomicAdd(&hist[key >> 21], 1u);
                    }
                }
            };
            // U blocks per iteration (two when the fragments are small): both
            // are loaded before either is scored, so their MMA chains overlap.
            // A second block past the warp's last one reads a stale slot and
            // stores nothing (its tokens are past n_cand_loc); its refill
            // commits empty groups only.
            constexpr int U = RMAX <= 2 ? 2 : 1;
            for (int it = 0; it < my_blocks; it += U) {
                uint32_t a[U][RMAX][4];
#pragma unroll
                for (int u = 0; u < U; ++u) load_block(it + u, a[u]);
#pragma unroll
                for (int u = 0; u < U; ++u) score_block(it + u, a[u]);
            }
        };
        // CUDA cores: lane (token = lane % 16, half = lane / 16) sums its half
        // of the slot's dim rows in fp32; the halves are added
        auto body = [&](auto rmax_tag) {
            constexpr int RMAX = decltype(rmax_tag)::value;
            const int tok = lane & 15, hf = lane >> 4;
            const int rh = p.r / 2;
            for (int it = 0; it < my_blocks; ++it) {
                wait_slot();
                const T* sl = reinterpret_cast<const T*>(wring + (it & smask) * p.slot_bytes);
                float x[RMAX * 8];
#pragma unroll
                for (int i = 0; i < RMAX * 8; ++i) x[i] = i < rh ? Elem<T>::to_f(sl[(hf * rh + i) * 16 + tok]) : 0.f;
                __syncwarp();
                refill(it + S);
                float sc;
                if (!p.group_max) {
                    float a = 0.f;
#pragma unroll
                    for (int i = 0; i < RMAX * 8; ++i)
                        if (i < rh) {
                            const int row = hf * rh + i;
                            a = fmaf(qs[MAG ? misc[kSelDims + row] : row], x[i], a);
                        }
                    sc = a + __shfl_xor_sync(kFull, a, 16);
                } else {
                    float m = -INFINITY;
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        float a = 0.f;
#pragma unroll
                        for (int i = 0; i < RMAX * 8; ++i)
                            if (i < rh) {
                                const int row = hf * rh + i;
                                a = fmaf(qsc[j * D + (MAG ? misc[kSelDims + row] : row)], x[i], a);
                            }
                        m = fmaxf(m, a + __shfl_xor_sync(kFull, a, 16));
                    }
                    sc = m;
                }
                const int li = (warp + it * kWarps) * kBlockTokens + tok;
                if (hf == 0 && li < n_cand_loc) {
                    const uint32_t key = score_key(sc);
                    keys[li] = key;
                    atomicAdd(&hist[key >> 21], 1u);
                }
            }
        };
        if constexpr (Geom::MMA) {
            if (p.r <= 2 * kSlabDims)
                mma_body(std::integral_constant<int, 2>{});
            else
                mma_body(std::integral_constant<int, D / kSlabDims>{});
        } else {
            if (p.r <= 2 * kSlabDims)
                body(std::integral_constant<int, 2>{});
            else
                body(std::integral_constant<int, D / kSlabDims>{});
        }
    }
    cp_async_wait<0>();  // the empty trailing groups
    __syncthreads();

    // ---- 3. top-k over the cluster ----
    // mode 0: keep every candidate, 1: keep none, 2: threshold tau / quota.
    // Thread t owns row t of the keys (keys 32 t .. 32 t + 31, bit b of its
    // masks = key 32 t + b); rows in thread order, bits in order, are token
    // order. A full pass over the keys costs about a microsecond, so there is
    // one: after digit 0 it marks the keys above the
    // boundary bin (kept whatever tau is) and the keys inside it (the
    // candidates, a few percent); digits 1 and 2 and the final comparison with
    // tau look at the candidates only. The three digits share one copy of the
    // boundary search (radix_boundary). Digit 2 is skipped when digit 1's
    // boundary bin is kept whole (its count over the cluster is what is still
    // needed): then every candidate at or above the bin's 22-bit prefix is kept.
    const int mode = keff >= ncand ? 0 : (keff == 0 ? 1 : 2);
    const int row0 = 32 * tid;
    const int nv = n_cand_loc - row0;  // valid keys in this row (may exceed 32)
    const uint32_t vmask = nv >= 32 ? kFull : (nv > 0 ? (1u << nv) - 1u : 0u);
    uint32_t rowgt = mode == 0 ? vmask : 0u, roweq = 0u;
    int quota = 0;
    if (mode == 2) {
        // digit 0 (top 11 bits): its histogram was built while scoring
        const int2 d0 = radix_boundary(hist, 2048, keff, misc, p.C);
        const uint32_t beta0 = (uint32_t)d0.x;
        int krem = keff - d0.y;
        uint32_t rowcand = 0u;
        if (nv > 0) {  // the keys region is a multiple of 32 keys
            const uint4* kv = reinterpret_cast<const uint4*>(keys + row0);
            uint4 v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = kv[j ^ (lane & 7)];  // XOR-rotated: conflict-free
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c = j ^ (lane & 7);
                const uint32_t x[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
                uint32_t g = 0u, e = 0u;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    g |= (uint32_t)((x[u] >> 21) > beta0) << u;
                    e |= (uint32_t)((x[u] >> 21) == beta0) << u;
                }
                rowgt |= g << (4 * c);
                rowcand |= e << (4 * c);
            }
            rowgt &= vmask;
            rowcand &= vmask;
        }
        // Each warp copies its candidates into its own segment of `cand` (lane
        // offsets from a warp scan) and histograms that dense list: predicated
        // shared atomics over all keys would be slow, since almost every
        // warp-wide atomic would have a lane or two active.
        uint32_t* wcand = cand + 1024 * warp;  // warp w's rows: keys [1024 w, 1024 w + 1024)
        int nw;                                 // entries in wcand
        {
            const int cnt = __popc(rowcand);
            int off = warp_exclusive_scan(cnt, lane);
            nw = __shfl_sync(kFull, off + cnt, 31);
            for (uint32_t t = rowcand; t; t &= t - 1u) wcand[off++] = keys[row0 + __ffs(t) - 1];
            __syncwarp();
        }
        // digit 1 (next 11 bits)
        uint32_t* h1 = hist + kHistBins;
        for (int i = lane; i < nw; i += 32) atomicAdd(&h1[(wcand[i] >> 10) & 2047u], 1u);
        const int2 d1 = radix_boundary(h1, 2048, krem, misc, p.C);
        const int bin1 = misc[2];  // read before the next search overwrites it
        krem -= d1.y;
        const uint32_t pre22 = (beta0 << 21) | ((uint32_t)d1.x << 10);
        if (bin1 == krem && pre22 != 0u) {
            // every key of the boundary bin is kept (the same decision in every
            // CTA of the cluster): the kept keys are those >= pre22, no ties to split
            const uint32_t tau = pre22 - 1u;
            for (uint32_t t = rowcand; t; t &= t - 1u) {
                const int bit = __ffs(t) - 1;
                rowgt |= (uint32_t)(keys[row0 + bit] > tau) << bit;
            }
        } else {
            // digit 2 (last 10 bits) into buffer 0: every CTA of the cluster has
            // read it, the cluster barrier of the previous search orders that
            for (int i = tid; i < kHistBins; i += kThreads) hist[i] = 0;
            __syncthreads();
            for (int i = lane; i < nw; i += 32) {
                const uint32_t x = wcand[i];
                if ((x & 0xFFFFFC00u) == pre22) atomicAdd(&hist[x & 1023u], 1u);
            }
            const int2 d2 = radix_boundary(hist, 1024, krem, misc, p.C);
            const uint32_t tau = pre22 | (uint32_t)d2.x;
            krem -= d2.y;
            // keys equal to tau: the last histogram counted them per CTA in bin (tau & 1023)
            int eq_before = 0;
            for (int c = 0; c < crank; ++c) eq_before += (int)cluster.map_shared_rank(hist, c)[tau & 1023u];
            const int eq_mine = (int)hist[tau & 1023u];
            quota = min(max(krem - eq_before, 0), eq_mine);
            // the candidates against tau
            for (uint32_t t = rowcand; t; t &= t - 1u) {
                const int bit = __ffs(t) - 1;
                const uint32_t x = keys[row0 + bit];
                rowgt |= (uint32_t)(x > tau) << bit;
                roweq |= (uint32_t)(x == tau) << bit;
            }
        }
    }

    // ---- compaction of the kept local tokens into `list`, ascending ----
    {
        const int ngt = __reduce_add_sync(kFull, __popc(rowgt));
        const int neq = __reduce_add_sync(kFull, __popc(roweq));
        if (lane == 0) {
            misc[40 + warp] = ngt;
            misc[56 + warp] = neq;
        }
        __syncthreads();
        // warp w keeps all its keys above tau and the equal ones whose rank
        // among the CTA's equal keys (in index order) is below the quota
        int eq_base = 0, out_base = 0, total = 0, eb = 0;
        for (int w = 0; w < kWarps; ++w) {
            const int take = min(max(quota - eb, 0), misc[56 + w]);
            if (w < warp) {
                out_base += misc[40 + w] + take;
                eq_base += misc[56 + w];
            }
            total += misc[40 + w] + take;
            eb += misc[56 + w];
        }
        uint32_t rowtake = rowgt;
        {
            int r = eq_base + warp_exclusive_scan(__popc(roweq), lane);
            for (uint32_t e = roweq; e; e &= e - 1u, ++r)
                if (r < quota) rowtake |= e & (0u - e);
        }
        int pos = out_base + warp_exclusive_scan(__popc(rowtake), lane);
        for (uint32_t t = rowtake; t; t &= t - 1u) list[pos++] = (uint16_t)(row0 + (__ffs(t) - 1));
        for (int i = tid; i < n_loc - n_cand_loc; i += kThreads) list[total + i] = (uint16_t)(n_cand_loc + i);
        if (tid == 0) misc[72] = total + (n_loc - n_cand_loc);
        __syncthreads();
    }
    const int n_list = misc[72];
    if (p.kv.touch)  // per block: the kept rows this call gathers from it
        for (int i = tid; i < n_list; i += kThreads) atomicAdd(p.kv.touch + tbl[list[i] >> 4], 1u);

    // ---- optional export of the kept set ----
    if (p.sel) {
        cluster.sync();
        int before = 0, all = 0;
        for (int c = 0; c < p.C; ++c) {
            const int nc = cluster.map_shared_rank(misc, c)[72];
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
    griddep_wait();  // the appended token's key and value rows (no-op when already waited)
    {
        const unsigned char* kbytes = reinterpret_cast<const unsigned char*>(p.k_cache);
        const unsigned char* vbytes = reinterpret_cast<const unsigned char*>(p.v_cache);
        constexpr int ROWB = D * (int)sizeof(T);
        constexpr int PIECES = TB / 16;  // 16-byte pieces of one token (key row + value row)
        unsigned char* wst = stage + warp * GS * Geom::CHUNK_BYTES;
        const int nchunks = (n_list + NCH - 1) / NCH;
        const int my_n = nchunks > warp ? (nchunks - warp + kWarps - 1) / kWarps : 0;
        // stage chunk m of this warp (tokens list[ch*NCH .. ch*NCH+NCH)) into
        // slot m % GS. The bf16 path runs one of two copies of the gather loop,
        // chosen once per launch: with the home-map branch taken per chunk the
        // all-device gather measured about 1.3 us slower at 32k tokens.
        auto fetch_dev = [&](int m) {
            if (m < my_n) {
                unsigned char* dst = wst + (m % GS) * Geom::CHUNK_BYTES;
                const int ch = warp + m * kWarps;
                for (int pc = lane; pc < NCH * PIECES; pc += 32) {
                    const int n = pc / PIECES, w = pc - n * PIECES;
                    const int kv = w >= PIECES / 2, c = w - kv * (PIECES / 2);
                    const int idx = ch * NCH + n;
                    const bool ok = idx < n_list;
                    const unsigned char* src = kbytes;
                    if (ok) {
                        const int li = list[idx];
                        const int64_t at = page_offset(tbl[li >> 4], h, p.Hkv, D) * (int64_t)sizeof(T) +
                                           (int64_t)(li & 15) * ROWB + c * 16;
                        src = (kv ? vbytes : kbytes) + at;
                    }
                    int off;
                    if constexpr (Geom::MMA) off = Geom::MCore::staged_offset(kv, n, c);
                    else off = n * TB + kv * ROWB + c * 16;
                    cp_async16(dst + off, src, ok);
                }
            }
            cp_async_commit();
        };
        // rows of offloaded blocks come over the host link by plain loads of
        // their mapped pages: only the kept rows cross it
        auto fetch_map = [&](int m) {
            if (m < my_n) {
                unsigned char* dst = wst + (m % GS) * Geom::CHUNK_BYTES;
                const int ch = warp + m * kWarps;
                for (int pc = lane; pc < NCH * PIECES; pc += 32) {
                    const int n = pc / PIECES, w = pc - n * PIECES;
                    const int kv = w >= PIECES / 2, c = w - kv * (PIECES / 2);
                    const int idx = ch * NCH + n;
                    bool ok = idx < n_list, host = false;
                    const unsigned char* src = kbytes;
                    if (ok) {
                        const int li = list[idx];
                        KvPage loc;
                        ok = kv_locate(p.kv, tbl[li >> 4], loc);
                        if (ok) {
                            host = loc.host;
                            const int64_t at = page_offset(loc.page, h, p.Hkv, D) * (int64_t)sizeof(T) +
                                               (int64_t)(li & 15) * ROWB + c * 16;
                            src = (host ? (kv ? p.kv.host_v : p.kv.host_k) : (kv ? vbytes : kbytes)) + at;
                        }
                    }
                    int off;
                    if constexpr (Geom::MMA) off = Geom::MCore::staged_offset(kv, n, c);
                    else off = n * TB + kv * ROWB + c * 16;
                    if (host) *reinterpret_cast<uint4*>(dst + off) = *reinterpret_cast<const uint4*>(src);
                    else cp_async16(dst + off, src, ok);
                }
            }
            cp_async_commit();
        };
        auto run = [&](auto& core, auto&& fetch) {
            for (int m = 0; m < GS - 1; ++m) fetch(m);
            for (int m = 0; m < my_n; ++m) {
                fetch(m + GS - 1);
                cp_async_wait<GS - 1>();
                __syncwarp();
                const unsigned char* src = wst + (m % GS) * Geom::CHUNK_BYTES;
                uint32_t valid = 0;
#pragma unroll
                for (int n = 0; n < NCH; ++n)
                    if ((warp + m * kWarps) * NCH + n < n_list) valid |= 1u << n;
                if constexpr (Geom::MMA) {
                    core.consume(src, valid, lane);
                } else {
                    typename Core::raw_t kr[NCH], vr[NCH];
#pragma unroll
                    for (int n = 0; n < NCH; ++n) {
                        kr[n] = Core::V::load(reinterpret_cast<const T*>(src + n * TB) + lane * Core::DPL);
                        vr[n] = Core::V::load(reinterpret_cast<const T*>(src + n * TB + ROWB) + lane * Core::DPL);
                    }
                    core.consume(kr, vr, valid, lane);
                }
                __syncwarp();
            }
            cp_async_wait<0>();
            __syncthreads();  // every warp is done with the staging area
            core.store_partial(wpart + warp * G * (D + 2), lane);
        };
        if constexpr (Geom::MMA) {
            typename Geom::MCore core;
            core.init(qhat, p.scale_log2, lane);
            if (!p.kv.home) run(core, fetch_dev);
            else run(core, fetch_map);
        } else {
            // (the fp32 path keeps one loop with the branch per chunk: two
            // copies of it measured about 1.8 us slower on the single-head
            // d64 L1024 workload)
            Core core;
            core.init(qhat, p.scale_log2, lane);
            run(core, [&](int m) {
                if (!p.kv.home) fetch_dev(m);
                else fetch_map(m);
            });
        }
    }
    __syncthreads();

    // ---- 5. merge: warps -> CTA partial in rank 0's shared memory -> out ----
    // Every CTA writes its partial (per head: G x D numerators, running max,
    // denominator) into slot crank of rank 0's `part`; one cluster barrier
    // publishes them, and rank 0 combines the slots and writes the output.
    // No CTA reads another's shared memory after that barrier, so the others
    // may exit at once.
    {
        float* dst = cluster.map_shared_rank(part, 0) + crank * G * (D + 2);
        if (warp < G) {  // warp j: head j's max and denominator over the CTA's warps
            const int j = warp;
            const float* wp = wpart + lane * G * (D + 2) + j * (D + 2);
            const float mw = lane < kWarps ? wp[D] : -INFINITY;
            const float M = warp_max_xor(mw, 0, 5);
            const float wt = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
            const float l = warp_sum_xor(lane < kWarps ? wt * wp[D + 1] : 0.f, 0, 5);
            if (lane < kWarps) wts[j * kWarps + lane] = wt;
            if (lane == 0) {
                dst[j * (D + 2) + D] = M;
                dst[j * (D + 2) + D + 1] = l;
            }
        }
        __syncthreads();
        for (int o = tid; o < G * D; o += kThreads) {
            const int j = o / D, c = o - j * D;
            float a = 0.f;
#pragma unroll 4
            for (int w = 0; w < kWarps; ++w) a = fmaf(wts[j * kWarps + w], wpart[w * G * (D + 2) + j * (D + 2) + c], a);
            dst[j * (D + 2) + c] = a;
        }
    }
    cluster.sync();
    if (crank == 0) {
        for (int o = tid; o < G * D; o += kThreads) {
            const int j = o / D, c = o - j * D;
            float M = -INFINITY;
            for (int r = 0; r < p.C; ++r) M = fmaxf(M, part[(r * G + j) * (D + 2) + D]);
            float num = 0.f, den = 0.f;
            if (M != -INFINITY) {
                for (int r = 0; r < p.C; ++r) {
                    const float* pr = part + (r * G + j) * (D + 2);
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
}

}  // namespace loki
