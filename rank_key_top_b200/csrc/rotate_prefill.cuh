// Prefill with the rotation done on the GPU: K~ = K P for every prompt token
// (AQUA page, appendix on complexity, step 1: keys are projected with P; the
// information-retention paragraph: row vectors, k~ = k P), written into the
// paged cache with the value rows and the key index, as loki_prefill_cache
// lays them out.
//
// bf16 caches: a real GEMM per kv head, [tokens x D] x [D x D], on the 5th
// generation tensor cores. One CTA (8 warps) keeps P_h in shared memory as
// two bf16 terms (P = P_hi + P_lo, the second term holding the remainder of
// the first), streams 128-token tiles of K in with cp.async, and issues
// tcgen05.mma (M = 128 tokens, N = D, K = D, both operands K-major with the
// 128-byte swizzle) into a 128-lane x D-column fp32 accumulator in tensor
// memory (lane = token, column = output dim; warps w and w + 4 read the two
// column halves of the same 32 lanes): the
// products of bf16 keys with each term are exact and the sum is accumulated
// in fp32, so the result carries about 16 significant bits of P before it is
// rounded to bf16. The epilogue reads the accumulator with tcgen05.ld (warps w
// and w + 4 own lanes 32 (w % 4) .. + 31, i.e. tokens, and split the columns),
// rounds to nearest even and writes key rows and index dims; the value rows
// are copied, one 16-token block per warp.
// fp32 caches: CUDA cores, fp32 products and sums, as the step's append.
#pragma once

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
    int tiles_per_cta;
};

constexpr int kRotTile = 128;     // tokens per MMA tile (the M of the instruction)
constexpr int kRotThreads = 256;  // 8 warps: warps w and w + 4 read accumulator lanes 32 (w % 4) .. + 31

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

// grid (ceil(tiles / tiles_per_cta), batch * Hkv), kRotThreads threads,
// dynamic shared memory rotate_smem_bytes<D>() (+ 1 KB for alignment).
template <int D>
__global__ void __launch_bounds__(kRotThreads) rotate_prefill_tc_kernel(const RotateParams p) {
    constexpr int KSTEPS = D / 16;         // MMA K steps per term
    constexpr int A_BYTES = kRotTile * D * 2;
    constexpr int B_BYTES = D * D * 2;
    constexpr uint32_t TMEM_COLS = D;      // fp32 accumulator: one column per output dim (D = 64 or 128)
    constexpr uint32_t IDESC = umma_idesc_bf16(kRotTile, D);
    extern __shared__ unsigned char smem_raw[];
    // operand atoms need 1024-byte alignment
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* sA = smem;
    unsigned char* sBhi = smem + A_BYTES;
    unsigned char* sBlo = sBhi + B_BYTES;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sBlo + B_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);

    const int pair = blockIdx.y;
    const int b = pair / p.Hkv, h = pair - b * p.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int L = p.seq_lens[b];
    if (L < 0 || L > p.max_seq_len) {
        if (tid == 0 && blockIdx.x == 0) flag_error(LOKI_DEVERR_SEQ_LEN);
        L = L < 0 ? 0 : p.max_seq_len;
    }
    const int tile0 = blockIdx.x * p.tiles_per_cta;
    const int ntiles = min(p.tiles_per_cta, (L + kRotTile - 1) / kRotTile - tile0);
    if (ntiles <= 0) return;  // uniform per CTA: nothing allocated yet

    // B operands: B[n][k] = P[k][n] split into bf16 terms, one 16-byte chunk
    // (8 consecutive k) per item
    const float* Ph = p.P + (int64_t)h * D * D;
    for (int it = tid; it < D * (D / 8); it += kRotThreads) {
        const int n = it / (D / 8), c = it - n * (D / 8);
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float x0 = Ph[(c * 8 + 2 * j) * D + n], x1 = Ph[(c * 8 + 2 * j + 1) * D + n];
            const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
            const __nv_bfloat16 l0 = __float2bfloat16_rn(x0 - __bfloat162float(h0));
            const __nv_bfloat16 l1 = __float2bfloat16_rn(x1 - __bfloat162float(h1));
            hi[j] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
            lo[j] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
        }
        const int off = sw128_offset(D, n, c);
        *reinterpret_cast<uint4*>(sBhi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(sBlo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    if (tid == 0) mbar_init(bar, 1);
    if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const unsigned char* ksrc =
        reinterpret_cast<const unsigned char*>(p.k) + ((int64_t)b * p.Hkv + h) * p.max_len * (int64_t)(D * 2);
    const unsigned char* vsrc =
        reinterpret_cast<const unsigned char*>(p.v) + ((int64_t)b * p.Hkv + h) * p.max_len * (int64_t)(D * 2);
    const int32_t* trow = p.block_table + (int64_t)b * p.max_blocks;
    __nv_bfloat16* xc = reinterpret_cast<__nv_bfloat16*>(p.k_index);
    bool ok_all = true;

    // A: the key rows of tile ti, zero past the sequence (one commit group)
    auto load_a = [&](int ti) {
        const int t_base = (tile0 + ti) * kRotTile;
        for (int it = tid; it < kRotTile * (D / 8); it += kRotThreads) {
            const int r = it / (D / 8), c = it - r * (D / 8);
            const bool ok = t_base + r < L;
            const unsigned char* src = ok ? ksrc + (int64_t)(t_base + r) * (D * 2) + c * 16 : ksrc;
            cp_async16(sA + sw128_offset(kRotTile, r, c), src, ok);
        }
        cp_async_commit();
    };
    load_a(0);
    // Per tile: the MMAs read A, then (A free again) the next tile's keys
    // stream in while this tile's values are copied and its accumulator is
    // written out.
    for (int ti = 0; ti < ntiles; ++ti) {
        const int t_base = (tile0 + ti) * kRotTile;
        cp_async_wait<0>();
        fence_async_smem();  // the generic-proxy writes become visible to the tensor cores
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            const uint32_t a0 = smem_u32(sA), bh0 = smem_u32(sBhi), bl0 = smem_u32(sBlo);
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                const uint32_t koff = (uint32_t)(ks & 3) * 32u;  // 16 bf16 of K inside the 128-byte row
                const uint32_t a = a0 + (uint32_t)(ks >> 2) * (kRotTile * 128) + koff;
                const uint32_t bh = bh0 + (uint32_t)(ks >> 2) * (D * 128) + koff;
                umma_bf16(tmem, umma_desc_k128(a), umma_desc_k128(bh), IDESC, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                const uint32_t koff = (uint32_t)(ks & 3) * 32u;
                const uint32_t a = a0 + (uint32_t)(ks >> 2) * (kRotTile * 128) + koff;
                const uint32_t bl = bl0 + (uint32_t)(ks >> 2) * (D * 128) + koff;
                umma_bf16(tmem, umma_desc_k128(a), umma_desc_k128(bl), IDESC, true);
            }
            umma_commit(bar);
        }
        // the tile's value rows: warp w copies block w of the tile (16 rows,
        // contiguous in the source and in its cache page); the loads are issued
        // before the wait for the MMAs, the stores after it
        constexpr int PPL = D / 16;  // 16-byte pieces per lane of one block (16 rows x D bf16)
        constexpr int BPW = kRotTile / kBlockTokens / (kRotThreads / 32);  // blocks per warp
        static_assert(BPW >= 1 && BPW * kBlockTokens * (kRotThreads / 32) == kRotTile, "blocks per warp");
        uint4 val[BPW][PPL];
        unsigned char* vdst[BPW];
        int vbytes[BPW];
#pragma unroll
        for (int bi = 0; bi < BPW; ++bi) {
            vdst[bi] = nullptr;
            vbytes[bi] = 0;
            const int tb = t_base + (BPW * warp + bi) * kBlockTokens;
            if (tb >= L) continue;
            const int pb = trow[tb >> 4];
            if (pb < 0 || pb >= p.num_blocks) {
                if (lane == 0) flag_error(LOKI_DEVERR_BLOCK_ID);
                continue;
            }
            __nv_bfloat16 *kd, *vd;
            kv_rows(p.kv, p.k_cache, p.v_cache, pb, h, p.Hkv, D, kd, vd);
            if (!vd) continue;
            vbytes[bi] = min(kBlockTokens, L - tb) * (D * 2);
            vdst[bi] = reinterpret_cast<unsigned char*>(vd);
            const unsigned char* src = vsrc + (int64_t)tb * (D * 2);
#pragma unroll
            for (int j = 0; j < PPL; ++j) {
                const int o = (lane + 32 * j) * 16;
                if (o < vbytes[bi]) val[bi][j] = *reinterpret_cast<const uint4*>(src + o);
            }
        }
        // this thread's token for the epilogue, and its block
        const int r = 32 * (warp & 3) + lane;
        const int t = t_base + r;
        int pb = -1;
        __nv_bfloat16* kpage = nullptr;  // this token's key page
        if (t < L) {
            pb = trow[t >> 4];
            if (pb < 0 || pb >= p.num_blocks) {
                flag_error(LOKI_DEVERR_BLOCK_ID);
                pb = -1;
            } else {
                __nv_bfloat16* vd;
                kv_rows(p.kv, p.k_cache, p.v_cache, pb, h, p.Hkv, D, kpage, vd);
                if (!kpage) pb = -1;
            }
        }
        const bool ok = mbar_wait_bounded(bar, (uint32_t)ti & 1u);
        ok_all = ok_all && ok;
        tc_fence_after();
        if (ti + 1 < ntiles && ok) load_a(ti + 1);  // the MMAs are done with A
#pragma unroll
        for (int bi = 0; bi < BPW; ++bi) {
#pragma unroll
            for (int j = 0; j < PPL; ++j) {
                const int o = (lane + 32 * j) * 16;
                if (o < vbytes[bi]) *reinterpret_cast<uint4*>(vdst[bi] + o) = val[bi][j];
            }
        }
        // epilogue: thread (warp w, lane l) holds token t_base + 32 (w % 4) + l,
        // columns [w / 4 * D / 2, + D / 2)
#pragma unroll
        for (int cc = 0; cc < D / 2; cc += 32) {
            const int c0 = (warp >> 2) * (D / 2) + cc;
            uint32_t acc[32];
            tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)c0, acc);
            tmem_ld_wait();
            if (ok && pb >= 0) {
                uint32_t w[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const __nv_bfloat16 e0 = __float2bfloat16_rn(__uint_as_float(acc[2 * j]));
                    const __nv_bfloat16 e1 = __float2bfloat16_rn(__uint_as_float(acc[2 * j + 1]));
                    w[j] = (uint32_t)__bfloat16_as_ushort(e0) | ((uint32_t)__bfloat16_as_ushort(e1) << 16);
                }
                __nv_bfloat16* krow = kpage + row_offset_in_page(t & 15, c0, D);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4*>(krow + 8 * q) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                if (c0 < p.index_dims) {  // index_dims is a multiple of 16: whole slabs
                    __nv_bfloat16* xpage = xc + page_offset(pb, h, p.Hkv, p.index_dims);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int dim = c0 + 8 * q;
                        if (dim < p.index_dims) {  // dim-major index: one element per dim
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                xpage[index_offset_in_page(t & 15, dim + e)] =
                                    __ushort_as_bfloat16((unsigned short)(w[4 * q + e / 2] >> (16 * (e & 1))));
                        }
                    }
                }
            }
        }
        // every thread's accumulator reads are done before the next tile's MMAs overwrite it
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (!ok_all) {
        // a wait gave up (flagged): give the tensor cores time to finish with the
        // accumulator before it is freed
        mbar_wait_bounded(bar, (uint32_t)(ntiles - 1) & 1u);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

template <int D>
constexpr int rotate_smem_bytes() {
    return kRotTile * D * 2 + 2 * D * D * 2 + 16 + 1024;  // A, B_hi, B_lo, barrier + slot, alignment slack
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
