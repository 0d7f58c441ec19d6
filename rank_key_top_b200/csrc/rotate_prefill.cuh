// Prefill with the rotation done on the GPU: K~ = K P for every prompt token
// (AQUA page, appendix on complexity, step 1: keys are projected with P; the
// information-retention paragraph: row vectors, k~ = k P), written into the
// paged cache with the value rows and the key index, as loki_prefill_cache
// lays them out.
//
// bf16 caches: a real GEMM per kv head, [tokens x D] x [D x D], on the 5th
// generation tensor cores, as a warp-specialised pipeline. Each CTA takes a
// contiguous range of the batch's 128-token tiles (pair-major; P_h is reloaded
// where the range crosses into the next (sequence, kv head)). P_h sits in
// shared memory as two bf16 terms (P = P_hi + P_lo, the second holding the
// remainder of the first), K-major with the 128-byte swizzle. Roles:
//   warp 0     streams key tiles with tensor-map copies (cp.async.bulk.tensor,
//              the 128-byte swizzle the MMA operand wants) into a ring of
//              STAGES tiles, one mbarrier per stage for "landed" and one for
//              "free";
//   warp 1     allocates two D-column fp32 accumulators in tensor memory and,
//              from one lane, issues tcgen05.mma (M = 128 tokens, N = D,
//              K = D, once per term) into accumulator (tile & 1); its commits
//              free the key stage and announce the accumulator;
//   warps 2-3  copy the value rows of the range's 16-token blocks: bulk
//              copies (one per block) into kRotVSlots shared-memory slots per
//              warp, then 16-byte stores into the block's cache page;
//   warps 4-11 read an accumulator with tcgen05.ld (warp w reads lanes
//              32 (w % 4) .. + 31, i.e. tokens, and one half of the columns),
//              hand it back to the MMA warp, round to bf16 and stage the key
//              rows (128-byte swizzle, conflict-free) and index pages in
//              shared memory; then one lane per 16-token block stores them
//              (whole blocks of device pages by tensor-map store and bulk
//              copy, partial blocks and host pages by plain stores).
// So tile i's epilogue overlaps tile i + 1's MMAs and the copies of tiles
// i + 2 .. i + STAGES. The products of bf16 keys with each term of P are exact
// and accumulate in fp32, so the result carries about 16 significant bits of P
// before it is rounded to bf16. Every wait is bounded (2 s of the global
// timer); a timeout sets LOKI_DEVERR_TIMEOUT and stops the CTA's work, which
// still waits for its copies and MMAs in flight before it frees the tensor
// memory.
// fp32 caches: CUDA cores, fp32 products and sums, as the step's append.
#pragma once

#include <cuda.h>  // CUtensorMap (the type only; the library calls the driver through the runtime)

#include "common.cuh"

namespace loki {

struct RotateParams {
    void* k_cache;
    void* v_cache;
    void* k_index;
    const int32_t* block_table;
    const int32_t* seq_lens;
    const void* k;  // [batch][Hkv][max_len][D], unrotated
    const void* v;  // [batch][Hkv][max_len][D]
    const float* P;
    KvMap kv;
    int num_blocks, Hkv, max_blocks, max_seq_len, max_len, index_dims;
    int tiles_per_pair;  // ceil(max_seq_len / 128)
    int64_t total_tiles; // pairs * tiles_per_pair
};

constexpr int kRotTile = 128;  // tokens per MMA tile (the M of the instruction)
constexpr int kRotVWarp0 = 2, kRotVWarps = 2, kRotEpiWarp0 = 4, kRotEpiWarps = 8;
constexpr int kRotThreads = (kRotEpiWarp0 + kRotEpiWarps) * 32;
constexpr int kRotVSlots = 4;  // value blocks in flight per value warp

// Shared memory of rotate_prefill_tc_kernel<D>: B_hi, B_lo, the key ring, the
// value-block slots, the mbarriers (full[S], empty[S], acc_full[2],
// acc_free[2], fin, one per value slot), the tensor memory address and the
// abort flag; 1024 bytes of alignment slack.
// the epilogue warps' own barrier (named barrier 1)
__device__ __forceinline__ void epi_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kRotEpiWarps * 32) : "memory");
}
// bulk copies between shared and global memory (the copy engine; no registers)
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
                 "r"(bytes)
                 : "memory");
}
// tiled 2-D tensor store shared -> global at element coordinates (x, y) >= 0
__device__ __forceinline__ void tma_store_2d(const void* tmap, int x, int y, const void* src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tmap), "r"(x),
                 "r"(y), "r"(smem_u32(src))
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

template <int D>
struct RotGeom {
    static constexpr int STAGES = 2;
    static constexpr int A_BYTES = kRotTile * D * 2;
    static constexpr int B_BYTES = D * D * 2;
    static constexpr int V_BYTES = kBlockTokens * D * 2;  // one 16-token block of value rows
    static constexpr int XI_BYTES = kBlockTokens * D * 2; // one block's index page, at most D dims
    static constexpr int OFF_A = 2 * B_BYTES;
    static constexpr int OFF_V = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_K = OFF_V + kRotVWarps * kRotVSlots * V_BYTES;  // the tile's rotated key rows
    static constexpr int OFF_X = OFF_K + kRotTile * D * 2;                    // and its index pages
    static constexpr int OFF_BAR = OFF_X + (kRotTile / kBlockTokens) * XI_BYTES;
    static constexpr int NBAR = 2 * STAGES + 5 + kRotVWarps * kRotVSlots;
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
    static constexpr uint32_t TMEM_COLS = 2 * D;  // two D-column fp32 accumulators
};

// ---------------------------------------------------------------------------
// tcgen05 / tensor-memory wrappers (cta_group::1)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {  // one whole warp
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // one whole warp
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] x B[smem desc], kind::f16 (bf16 inputs, fp32 accumulator)
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}
// the mbarrier receives one arrival when every earlier tcgen05.mma of this thread has completed
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// 32 consecutive fp32 columns of this thread's accumulator lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major operand with the 128-byte
// swizzle: rows of 128 bytes (64 bf16 of K), 8-row groups 1024 bytes apart;
// `addr` is the first byte the instruction reads (the 1024-byte aligned atom
// plus 32 bytes per 16-element K step).
__device__ __forceinline__ uint64_t umma_desc_k128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);   // start address, bits [0, 14)
    d |= (uint64_t)1u << 16;                  // leading byte offset (unused for this layout), bits [16, 30)
    d |= (uint64_t)(1024u >> 4) << 32;        // stride byte offset: 8 rows x 128 bytes, bits [32, 46)
    d |= (uint64_t)1u << 46;                  // descriptor version of this architecture, bits [46, 48)
    d |= (uint64_t)2u << 61;                  // layout: 128-byte swizzle, bits [61, 64)
    return d;
}
// Instruction descriptor: fp32 accumulator, bf16 A and B, both K-major, N x M.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
    return (1u << 4)                       // accumulator format F32
           | (1u << 7)                     // A format BF16
           | (1u << 10)                    // B format BF16
           | ((uint32_t)(N >> 3) << 17)    // N / 8
           | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// Byte offset of 16-byte chunk c (0 .. D/8 - 1) of row r in a K-major
// operand of R rows stored as D/64 swizzle atoms of R x 128 bytes each.
__host__ __device__ __forceinline__ int sw128_offset(int R, int r, int c) {
    return (c >> 3) * (R * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// grid (CTAs), kRotThreads threads, RotGeom<D>::SMEM bytes of dynamic shared
// memory. CTA c takes tiles [c T / G, (c + 1) T / G) of the T = pairs x
// tiles_per_pair tiles (pair-major); tiles past a sequence's end are skipped.
// tmap: the keys [batch * Hkv * max_len rows][D] bf16, box 64 x 128, 128-byte
// swizzle. kmap: the key cache's device pages as [pages * Hkv * 16 rows][D]
// bf16, box 64 x 16, 128-byte swizzle (the store side).
template <int D>
__global__ void __launch_bounds__(kRotThreads, 1)
    rotate_prefill_tc_kernel(const __grid_constant__ RotateParams p, const __grid_constant__ CUtensorMap tmap,
                             const __grid_constant__ CUtensorMap kmap) {
    using RG = RotGeom<D>;
    constexpr int STAGES = RG::STAGES;
    constexpr int KSTEPS = D / 16;  // MMA K steps per term
    constexpr uint32_t IDESC = umma_idesc_bf16(kRotTile, D);
    extern __shared__ unsigned char smem_raw[];
    // operand atoms need 1024-byte alignment
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* sBhi = smem;
    unsigned char* sBlo = smem + RG::B_BYTES;
    unsigned char* sA = smem + RG::OFF_A;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + RG::OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;
    uint64_t* acc_free = acc_full + 2;
    uint64_t* fin = acc_free + 2;
    uint64_t* vbar = fin + 1;  // [kRotVWarps][kRotVSlots]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(vbar + kRotVWarps * kRotVSlots);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t f_begin = p.total_tiles * blockIdx.x / gridDim.x;
    const int64_t f_end = p.total_tiles * (blockIdx.x + 1) / gridDim.x;
    if (f_begin >= f_end) return;  // uniform per CTA: nothing allocated yet

    if (tid == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_free[i], kRotEpiWarps);
        }
        mbar_init(fin, 1);
        for (int i = 0; i < kRotVWarps * kRotVSlots; ++i) mbar_init(&vbar[i], 1);
        *abort_flag = 0;
    }
    if (warp == 1) tmem_alloc(tmem_slot, RG::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    uint32_t gi = 0;          // tiles of earlier segments (every role counts alike)
    uint32_t issued = 0;      // producer: tiles whose copies were issued
    uint32_t vdone = 0;       // value warp: blocks of earlier segments it copied
    int64_t f = f_begin;
    while (f < f_end) {
        // one segment: this CTA's tiles of one (sequence, kv head)
        const int pair = (int)(f / p.tiles_per_pair);
        const int64_t seg_end = min(f_end, (int64_t)(pair + 1) * p.tiles_per_pair);
        const int b = pair / p.Hkv, h = pair - b * p.Hkv;
        int L = p.seq_lens[b];
        if (L < 0 || L > p.max_seq_len) {
            if (tid == 0 && f == (int64_t)pair * p.tiles_per_pair) flag_error(LOKI_DEVERR_SEQ_LEN);
            L = L < 0 ? 0 : p.max_seq_len;
        }
        const int ti0 = (int)(f - (int64_t)pair * p.tiles_per_pair);
        const int ti1 = min((int)(seg_end - (int64_t)pair * p.tiles_per_pair), (L + kRotTile - 1) / kRotTile);
        f = seg_end;
        const int n = ti1 - ti0;
        if (n <= 0) continue;  // uniform: every thread skips the segment

        // B operands: B[n][k] = P[k][n] split into bf16 terms, one 16-byte
        // chunk (8 consecutive k) per item. The previous segment's MMAs are
        // complete (its epilogue waited for every accumulator).
        const float* Ph = p.P + (int64_t)h * D * D;
        for (int it = tid; it < D * (D / 8); it += kRotThreads) {
            const int nn = it / (D / 8), c = it - nn * (D / 8);
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float x0 = Ph[(c * 8 + 2 * j) * D + nn], x1 = Ph[(c * 8 + 2 * j + 1) * D + nn];
                const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
                const __nv_bfloat16 l0 = __float2bfloat16_rn(x0 - __bfloat162float(h0));
                const __nv_bfloat16 l1 = __float2bfloat16_rn(x1 - __bfloat162float(h1));
                hi[j] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
                lo[j] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
            }
            const int off = sw128_offset(D, nn, c);
            *reinterpret_cast<uint4*>(sBhi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(sBlo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        fence_async_smem();  // the generic-proxy writes become visible to the tensor cores
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        const int32_t* trow = p.block_table + (int64_t)b * p.max_blocks;
        if (warp == 0) {
            // ---- key tiles: tensor-map copies into the ring ----
            if (lane == 0) {
                const int row0 = pair * p.max_len;
                for (int i = 0; i < n && !*abort_flag; ++i) {
                    const uint32_t g = gi + i, s = g % STAGES, u = g / STAGES;
                    if (u >= 1 && !mbar_wait_timed(&empty[s], (u - 1) & 1u)) {
                        *abort_flag = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], RG::A_BYTES);
#pragma unroll
                    for (int box = 0; box < D / 64; ++box)
                        tma_load_2d(sA + s * RG::A_BYTES + box * (kRotTile * 128), &tmap, box * 64,
                                    row0 + (ti0 + i) * kRotTile, &full[s]);
                    issued = g + 1;
                }
            }
        } else if (warp == 1) {
            // ---- MMAs: two terms of P into accumulator (tile & 1) ----
            if (lane == 0) {
                for (int i = 0; i < n && !*abort_flag; ++i) {
                    const uint32_t g = gi + i, s = g % STAGES, u = g / STAGES, a = g & 1u, v = g >> 1;
                    if (!mbar_wait_timed(&full[s], u & 1u) || (v >= 1 && !mbar_wait_timed(&acc_free[a], (v - 1) & 1u))) {
                        *abort_flag = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + s * RG::A_BYTES), bh0 = smem_u32(sBhi), bl0 = smem_u32(sBlo);
                    const uint32_t acc = tmem + a * D;
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks) {
                        const uint32_t koff = (uint32_t)(ks & 3) * 32u;  // 16 bf16 of K inside the 128-byte row
                        const uint32_t aa = a0 + (uint32_t)(ks >> 2) * (kRotTile * 128) + koff;
                        const uint32_t bh = bh0 + (uint32_t)(ks >> 2) * (D * 128) + koff;
                        umma_bf16(acc, umma_desc_k128(aa), umma_desc_k128(bh), IDESC, ks > 0);
                    }
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks) {
                        const uint32_t koff = (uint32_t)(ks & 3) * 32u;
                        const uint32_t aa = a0 + (uint32_t)(ks >> 2) * (kRotTile * 128) + koff;
                        const uint32_t bl = bl0 + (uint32_t)(ks >> 2) * (D * 128) + koff;
                        umma_bf16(acc, umma_desc_k128(aa), umma_desc_k128(bl), IDESC, true);
                    }
                    umma_commit(&empty[s]);     // the key stage is free once these MMAs complete
                    umma_commit(&acc_full[a]);  // and the accumulator is ready
                }
            }
        } else if (warp < kRotEpiWarp0) {
            // ---- value rows: bulk copy of each block into a slot, then out to its page ----
            const int vw = warp - kRotVWarp0;
            unsigned char* slots = smem + RG::OFF_V + vw * kRotVSlots * RG::V_BYTES;
            uint64_t* bars = vbar + vw * kRotVSlots;
            const unsigned char* vsrc = reinterpret_cast<const unsigned char*>(p.v) +
                                        ((int64_t)b * p.Hkv + h) * p.max_len * (int64_t)(D * 2);
            const int jb0 = ti0 * (kRotTile / kBlockTokens) + vw;
            const int jb1 = (min(ti1 * kRotTile, L) + kBlockTokens - 1) / kBlockTokens;
            const int nb = jb1 > jb0 ? (jb1 - jb0 + kRotVWarps - 1) / kRotVWarps : 0;  // this warp's blocks
            auto bytes_of = [&](int m) { return min(kBlockTokens, L - (jb0 + m * kRotVWarps) * kBlockTokens) * (D * 2); };
            auto issue = [&](int m) {  // lane 0: block m of this warp into slot (vdone + m) % kRotVSlots
                const uint32_t slot = (vdone + m) % kRotVSlots;
                const int j = jb0 + m * kRotVWarps;
                const uint32_t nbytes = (uint32_t)bytes_of(m);
                mbar_arrive_expect_tx(&bars[slot], nbytes);
                bulk_load(slots + slot * RG::V_BYTES, vsrc + (int64_t)j * kBlockTokens * (D * 2), nbytes, &bars[slot]);
            };
            if (lane == 0)
                for (int m = 0; m < kRotVSlots && m < nb; ++m) issue(m);
            bool vok = true;
            for (int m = 0; m < nb; ++m) {
                const uint32_t c = vdone + m, slot = c % kRotVSlots;
                vok = mbar_wait_timed(&bars[slot], (c / kRotVSlots) & 1u) && vok;
                const int j = jb0 + m * kRotVWarps;
                const int pb = trow[j];
                KvPage loc;
                bool dst_ok = false;
                if (pb < 0 || pb >= p.num_blocks) {
                    if (lane == 0) flag_error(LOKI_DEVERR_BLOCK_ID);
                } else {
                    dst_ok = kv_locate(p.kv, pb, loc);
                }
                const int nbytes = bytes_of(m);
                unsigned char* src = slots + slot * RG::V_BYTES;
                if (dst_ok && vok) {
                    const int64_t off = page_offset(loc.page, h, p.Hkv, D) * 2;
                    if (!loc.host) {  // device page: a bulk store straight from the slot
                        if (lane == 0) {
                            bulk_store(reinterpret_cast<unsigned char*>(p.v_cache) + off, src, nbytes);
                            bulk_commit();
                        }
                    } else {  // host page: 16-byte stores through its mapping
                        unsigned char* dst = p.kv.host_v + off;
                        for (int o = lane * 16; o < nbytes; o += 32 * 16)
                            *reinterpret_cast<uint4*>(dst + o) = *reinterpret_cast<const uint4*>(src + o);
                    }
                }
                __syncwarp();
                if (lane == 0 && m + kRotVSlots < nb) {
                    bulk_wait_read_all();  // the store out of this slot has read it
                    fence_async_smem();    // and the lanes' reads come before the copy's writes
                    issue(m + kRotVSlots);
                }
            }
            if (lane == 0) bulk_wait_all();
            if (!vok && lane == 0) *abort_flag = 1;
            vdone += nb;
        } else {
            // ---- epilogue: accumulator -> bf16 key rows and index dims ----
            // The tile's rows are staged in shared memory as D/64 column atoms of
            // [128 rows][128 bytes] with the 128-byte swizzle (conflict-free) and
            // its index pages as [block][I dims][16 tokens]; then one lane per
            // block stores them: full blocks of device pages by tensor-map store
            // (rows) and bulk copy (index), the rest by plain stores.
            const int e = warp - kRotEpiWarp0;
            const int quarter = warp & 3, half = e >> 2;
            unsigned char* sK = smem + RG::OFF_K;
            unsigned char* sX = smem + RG::OFF_X;
            const int I = p.index_dims;
            // Every epilogue warp passes both named barriers of every tile, also
            // after an abort (a barrier missed by one warp would never open): an
            // aborted warp only skips the waits and the work.
            for (int i = 0; i < n; ++i) {
                const uint32_t g = gi + i, a = g & 1u, v = g >> 1;
                bool live = __shfl_sync(kFull, *abort_flag, 0) == 0;
                if (live) {
                    const bool ok = mbar_wait_timed(&acc_full[a], v & 1u);
                    if (!__all_sync(kFull, ok)) {
                        if (lane == 0) *abort_flag = 1;
                        live = false;
                    }
                }
                const int r = 32 * quarter + lane;  // the thread's row (token) of the tile
                uint32_t w[D / 64][16];  // this token's columns of the half, rounded to bf16 pairs
                if (live) {
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < D / 64; ++cc) {
                    uint32_t acc[32];
                    tmem_ld32(tmem + ((uint32_t)(32 * quarter) << 16) + a * D + (uint32_t)(half * (D / 2) + 32 * cc),
                              acc);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const __nv_bfloat16 e0 = __float2bfloat16_rn(__uint_as_float(acc[2 * j]));
                        const __nv_bfloat16 e1 = __float2bfloat16_rn(__uint_as_float(acc[2 * j + 1]));
                        w[cc][j] = (uint32_t)__bfloat16_as_ushort(e0) | ((uint32_t)__bfloat16_as_ushort(e1) << 16);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_free[a]);  // the MMAs may refill it
                }
                // the staging area is free once the last tile's stores have read it
                if (e == 0 && lane < kRotTile / kBlockTokens) bulk_wait_read_all();
                epi_sync();
                if (live) {
#pragma unroll
                for (int cc = 0; cc < D / 64; ++cc) {
                    const int c0 = half * (D / 2) + 32 * cc;  // first column of this 32-column piece
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int col = c0 + 8 * q;
                        const int atom = col >> 6, chunk = (col & 63) >> 3;
                        *reinterpret_cast<uint4*>(sK + atom * (kRotTile * 128) + r * 128 + ((chunk ^ (r & 7)) << 4)) =
                            make_uint4(w[cc][4 * q], w[cc][4 * q + 1], w[cc][4 * q + 2], w[cc][4 * q + 3]);
                        if (col < I) {  // dim-major index: one element per dim
#pragma unroll
                            for (int u = 0; u < 8; ++u)
                                reinterpret_cast<unsigned short*>(sX + (r >> 4) * RG::XI_BYTES)[(col + u) * 16 + (r & 15)] =
                                    (unsigned short)(w[cc][4 * q + u / 2] >> (16 * (u & 1)));
                        }
                    }
                }
                fence_async_smem();  // the staged rows become visible to the copy engine
                }
                epi_sync();
                // one lane per 16-token block of the tile stores it
                const int t0 = (ti0 + i) * kRotTile;
                for (int bi = lane; bi < kRotTile / kBlockTokens; bi += 32) {
                    if (e != 0 || !live) break;
                    const int tb = t0 + bi * kBlockTokens;
                    if (tb >= L) break;
                    const int rows = min(kBlockTokens, L - tb);
                    const int pb = trow[tb >> 4];
                    if (pb < 0 || pb >= p.num_blocks) {
                        flag_error(LOKI_DEVERR_BLOCK_ID);
                        continue;
                    }
                    KvPage loc;
                    if (!kv_locate(p.kv, pb, loc)) continue;
                    unsigned char* xpage = reinterpret_cast<unsigned char*>(p.k_index) + page_offset(pb, h, p.Hkv, I) * 2;
                    const unsigned char* xs = sX + bi * RG::XI_BYTES;
                    if (rows == kBlockTokens && !loc.host) {
                        const int y = (int)((loc.page * p.Hkv + h) * kBlockTokens);
#pragma unroll
                        for (int atom = 0; atom < D / 64; ++atom)
                            tma_store_2d(&kmap, atom * 64, y, sK + atom * (kRotTile * 128) + bi * kBlockTokens * 128);
                        bulk_store(xpage, xs, I * kBlockTokens * 2);
                        bulk_commit();
                    } else {
                        unsigned char* kpage = (loc.host ? p.kv.host_k : reinterpret_cast<unsigned char*>(p.k_cache)) +
                                               page_offset(loc.page, h, p.Hkv, D) * 2;
                        for (int rr = 0; rr < rows; ++rr) {
                            const int row = bi * kBlockTokens + rr;
                            for (int ch = 0; ch < D / 8; ++ch)
                                *reinterpret_cast<uint4*>(kpage + rr * (D * 2) + ch * 16) = *reinterpret_cast<const uint4*>(
                                    sK + (ch >> 3) * (kRotTile * 128) + row * 128 + (((ch & 7) ^ (row & 7)) << 4));
                            for (int d = 0; d < I; ++d)
                                reinterpret_cast<unsigned short*>(xpage)[d * 16 + rr] =
                                    reinterpret_cast<const unsigned short*>(xs)[d * 16 + rr];
                        }
                    }
                }
            }
            if (e == 0 && lane < kRotTile / kBlockTokens) bulk_wait_all();
        }
        __syncthreads();  // every role is done with the segment
        gi += n;
    }

    // teardown: every MMA and every tensor-map copy this CTA issued has
    // completed before the tensor memory is freed and the CTA exits
    if (warp == 1 && lane == 0) {
        umma_commit(fin);
        mbar_wait_timed(fin, 0);
    }
    if (warp == 0 && lane == 0 && *abort_flag) {
        for (uint32_t g = issued > STAGES ? issued - STAGES : 0; g < issued; ++g)
            mbar_wait_timed(&full[g % STAGES], (g / STAGES) & 1u);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, RG::TMEM_COLS);
}

template <int D>
constexpr int rotate_smem_bytes() {
    return RotGeom<D>::SMEM;
}

// fp32 caches: grid (ceil(max_seq_len / 16), batch * Hkv), 256 threads; one
// 16-token block per CTA, each token as the step's append computes it.
template <int D>
__global__ void __launch_bounds__(256) rotate_prefill_f32_kernel(const RotateParams p) {
    constexpr int NQ = D / 4;
    constexpr int NRG = 256 / NQ;
    constexpr int RPG = D / NRG;
    __shared__ float part[NRG][D];
    __shared__ float kin[D];
    const int jb = blockIdx.x;
    const int pair = blockIdx.y;
    const int b = pair / p.Hkv, h = pair - b * p.Hkv;
    const int tid = threadIdx.x;
    int L = p.seq_lens[b];
    if (L < 0 || L > p.max_seq_len) {
        if (tid == 0 && jb == 0) flag_error(LOKI_DEVERR_SEQ_LEN);
        L = L < 0 ? 0 : p.max_seq_len;
    }
    if (jb * kBlockTokens >= L) return;
    const int pb = p.block_table[(int64_t)b * p.max_blocks + jb];
    if (pb < 0 || pb >= p.num_blocks) {
        if (tid == 0) flag_error(LOKI_DEVERR_BLOCK_ID);
        return;
    }
    const int cq = tid % NQ, rg = tid / NQ;
    float4 pv[RPG];
    const float* Ph = p.P + (int64_t)h * D * D;
#pragma unroll
    for (int i = 0; i < RPG; ++i) pv[i] = *reinterpret_cast<const float4*>(Ph + (rg * RPG + i) * D + 4 * cq);
    const int64_t src0 = (((int64_t)b * p.Hkv + h) * p.max_len) * D;
    float *kc, *vc;
    kv_rows(p.kv, p.k_cache, p.v_cache, pb, h, p.Hkv, D, kc, vc);
    if (!kc) return;
    float* xc = reinterpret_cast<float*>(p.k_index) + page_offset(pb, h, p.Hkv, p.index_dims);
    const float* ks = reinterpret_cast<const float*>(p.k) + src0;
    const float* vs = reinterpret_cast<const float*>(p.v) + src0;
    for (int r = 0; r < kBlockTokens && jb * kBlockTokens + r < L; ++r) {
        const int t = jb * kBlockTokens + r;
        if (tid < D) kin[tid] = ks[(int64_t)t * D + tid];
        __syncthreads();
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
        __syncthreads();
        if (tid < D) {
            float x = 0.f;
#pragma unroll
            for (int g = 0; g < NRG; ++g) x += part[g][tid];
            kc[row_offset_in_page(r, tid, D)] = x;
            if (tid < p.index_dims) xc[index_offset_in_page(r, tid)] = x;
            vc[row_offset_in_page(r, tid, D)] = vs[(int64_t)t * D + tid];
        }
        __syncthreads();
    }
}

}  // namespace loki
