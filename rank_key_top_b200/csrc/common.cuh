// Device-side helpers shared by the libloki kernels: cache layout, typed
// loads, order-preserving score keys, warp helpers and the device error
// word. Included once, by loki.cu, so that every kernel and the error word
// live in one translation unit.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "loki.h"

namespace loki {

constexpr int kBlockTokens = LOKI_BLOCK_TOKENS;  // tokens per paged block
constexpr int kSlabDims = 16;                    // dims per key slab

// Sticky device error word (LOKI_DEVERR_* bits), one per device.
__device__ uint32_t g_device_error;

__device__ __forceinline__ void flag_error(uint32_t bits) { atomicOr(&g_device_error, bits); }

// ---------------------------------------------------------------------------
// Paged cache layout. Block p of kv head h starts at element
// (p * Hkv + h) * 16 * D in the key and value caches, and at
// (p * Hkv + h) * 16 * I in the key index (I = index dims).
//   keys, values: [16 tokens][D]     (one contiguous row per token)
//   key index:    [I dims][16 tokens] (dim-major: one dim of the block's 16
//                 tokens is one contiguous run of 16 elements, and the
//                 leading r dims are one contiguous run of r*16 elements)
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int64_t page_offset(int64_t block, int h, int Hkv, int D) {
    return (block * Hkv + h) * (int64_t)(kBlockTokens * D);
}
__host__ __device__ __forceinline__ int row_offset_in_page(int token, int dim, int D) {
    return token * D + dim;
}
__host__ __device__ __forceinline__ int index_offset_in_page(int token, int dim) {
    return dim * kBlockTokens + token;
}

// ---------------------------------------------------------------------------
// Where the key and value rows of a physical block live (LRQK page, abstract:
// a mixed GPU-CPU cache; the low-rank key index always stays on the device).
// Without a home map, block p's rows are device page p. With one, home[p] >= 0
// names a device page and home[p] < 0 the pinned host page -(home[p] + 1),
// read and written through its device mapping.
// ---------------------------------------------------------------------------
struct KvMap {
    const int32_t* home;  // [num_blocks] or nullptr
    unsigned char* host_k;
    unsigned char* host_v;
    uint32_t* touch;      // [num_blocks] or nullptr: kept rows gathered per block
    int dev_pages, host_pages;
};

// The page holding block pb's rows and which pool it is in; false (and the
// block-id error bit) for a home entry outside its pool.
struct KvPage {
    int64_t page;
    bool host;
};
__device__ __forceinline__ bool kv_locate(const KvMap& m, int pb, KvPage& loc) {
    if (!m.home) {
        loc.page = pb;
        loc.host = false;
        return true;
    }
    const int e = m.home[pb];
    loc.host = e < 0;
    loc.page = loc.host ? -(int64_t)e - 1 : e;
    if (loc.page >= (loc.host ? m.host_pages : m.dev_pages)) {
        flag_error(LOKI_DEVERR_BLOCK_ID);
        return false;
    }
    return true;
}
// Element pointers of head h's key and value rows of block pb (nullptr when
// the home entry is invalid).
template <typename T>
__device__ __forceinline__ void kv_rows(const KvMap& m, void* k_cache, void* v_cache, int pb, int h, int Hkv,
                                        int D, T*& k, T*& v) {
    KvPage loc;
    if (!kv_locate(m, pb, loc)) {
        k = v = nullptr;
        return;
    }
    const int64_t off = page_offset(loc.page, h, Hkv, D);
    k = reinterpret_cast<T*>(loc.host ? m.host_k : reinterpret_cast<unsigned char*>(k_cache)) + off;
    v = reinterpret_cast<T*>(loc.host ? m.host_v : reinterpret_cast<unsigned char*>(v_cache)) + off;
}

// ---------------------------------------------------------------------------
// Typed element access.
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float to_f(float x) { return x; }
    static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// N consecutive elements (N * sizeof(T) in {4, 8, 16, 32} bytes, naturally
// aligned) loaded with the widest vector load and converted to fp32.
template <typename T, int N> struct Vec;

template <int N> struct Vec<__nv_bfloat16, N> {
    static_assert(N == 2 || N == 4 || N == 8, "bf16 vector width");
    using raw_t = typename std::conditional<N == 2, uint32_t,
                  typename std::conditional<N == 4, uint2, uint4>::type>::type;
    static __device__ __forceinline__ raw_t load(const __nv_bfloat16* p) {
        return *reinterpret_cast<const raw_t*>(p);
    }
    static __device__ __forceinline__ void unpack_word(uint32_t w, float* f) {
        f[0] = __uint_as_float(w << 16);
        f[1] = __uint_as_float(w & 0xffff0000u);
    }
    static __device__ __forceinline__ void to_float(const raw_t& r, float* f) {
        if constexpr (N == 2) {
            unpack_word(r, f);
        } else if constexpr (N == 4) {
            unpack_word(r.x, f);
            unpack_word(r.y, f + 2);
        } else {
            unpack_word(r.x, f);
            unpack_word(r.y, f + 2);
            unpack_word(r.z, f + 4);
            unpack_word(r.w, f + 6);
        }
    }
};

template <int N> struct Vec<float, N> {
    static_assert(N == 2 || N == 4 || N == 8, "f32 vector width");
    struct raw8 { float4 a, b; };
    using raw_t = typename std::conditional<N == 2, float2,
                  typename std::conditional<N == 4, float4, raw8>::type>::type;
    static __device__ __forceinline__ raw_t load(const float* p) {
        if constexpr (N == 8) {
            raw8 r;
            r.a = *reinterpret_cast<const float4*>(p);
            r.b = *reinterpret_cast<const float4*>(p + 4);
            return r;
        } else {
            return *reinterpret_cast<const raw_t*>(p);
        }
    }
    static __device__ __forceinline__ void to_float(const raw_t& r, float* f) {
        if constexpr (N == 2) {
            f[0] = r.x; f[1] = r.y;
        } else if constexpr (N == 4) {
            f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w;
        } else {
            f[0] = r.a.x; f[1] = r.a.y; f[2] = r.a.z; f[3] = r.a.w;
            f[4] = r.b.x; f[5] = r.b.y; f[6] = r.b.z; f[7] = r.b.w;
        }
    }
};

// ---------------------------------------------------------------------------
// Order-preserving map of an fp32 score to a uint32 key: a > b (as floats,
// with -0 == +0) iff key(a) > key(b). -0 is canonicalised to +0 first.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s + 0.0f);  // -0 + 0 = +0 under round-to-nearest
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------------------
// Shared-memory addresses.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous copy global -> shared (cp.async, L2 only), and its
// commit groups. With valid false nothing is read and the 16 bytes are zeroed.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, bool valid) {
    const int n = valid ? 16 : 0;  // 0: nothing is read, the 16 bytes are zero-filled
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------------------
// mbarriers in shared memory: init, and a bounded wait for a phase.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Waits for phase `parity` of `bar`, polling at most kWaitLimit times; on
// giving up it sets LOKI_DEVERR_TIMEOUT and returns false.
constexpr uint32_t kWaitLimit = 1u << 24;
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    flag_error(LOKI_DEVERR_TIMEOUT);
    return false;
}
// Waits for phase `parity` of `bar` for at most limit_ns of the global timer;
// on giving up it sets LOKI_DEVERR_TIMEOUT and returns false.
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s
__device__ __forceinline__ bool mbar_wait_timed(uint64_t* bar, uint32_t parity) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try(bar, parity)) return true;
        if ((i & 255u) == 0 && global_ns() - t0 > kWaitNs) break;
    }
    flag_error(LOKI_DEVERR_TIMEOUT);
    return false;
}
// One arrival that also announces tx_bytes of asynchronous copies to come.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t tx_bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(tx_bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Tiled 2-D tensor copy global -> shared (no multicast), completing on `bar`:
// the box at element coordinates (x, y) of the tensor map; x times the
// element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// One arrival on `bar` once every cp.async this thread issued before has
// landed (the arrival counts toward the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch. A kernel launched as a programmatic
// dependent may start while the kernel before it in the stream still runs;
// griddep_wait() returns once that kernel has completed and its writes are
// visible (at once when there is no such dependency). griddep_launch_dependents()
// lets the dependent of this kernel start launching.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Warp helpers.
// ---------------------------------------------------------------------------
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_max_xor(float v, int lo_bit, int hi_bit) {
    for (int b = lo_bit; b < hi_bit; ++b) v = fmaxf(v, __shfl_xor_sync(kFull, v, 1 << b));
    return v;
}
__device__ __forceinline__ float warp_sum_xor(float v, int lo_bit, int hi_bit) {
    for (int b = lo_bit; b < hi_bit; ++b) v += __shfl_xor_sync(kFull, v, 1 << b);
    return v;
}

// Transpose-reduce: every lane holds NV partial values; afterwards the values
// are summed over all 32 lanes and lane l holds the total of value index
// (l >> (5 - log2(NV))). Uses NV - 1 + (5 - log2 NV) shuffles instead of
// 5 * NV.
template <int NV>
__device__ __forceinline__ float transpose_reduce(float (&v)[NV], int lane) {
    static_assert(NV >= 1 && NV <= 32 && (NV & (NV - 1)) == 0, "NV power of two <= 32");
    int n = NV;
    int mask = 16;
#pragma unroll
    for (int level = 0; level < 5; ++level) {
        if (n > 1) {
            const int half = n >> 1;
            const bool upper = (lane & mask) != 0;
#pragma unroll
            for (int i = 0; i < NV / 2; ++i) {
                if (i < half) {
                    float send = upper ? v[i] : v[i + half];
                    float keep = upper ? v[i + half] : v[i];
                    v[i] = keep + __shfl_xor_sync(kFull, send, mask);
                }
            }
            n = half;
        } else {
            v[0] += __shfl_xor_sync(kFull, v[0], mask);
        }
        mask >>= 1;
    }
    return v[0];
}

}  // namespace loki
