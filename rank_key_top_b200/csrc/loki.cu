// libloki: host entry points of the C ABI declared in include/loki.h.
// Every kernel is included here so that the device error word and all
// kernels share one translation unit.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>
#include <vector>

#include "cache_kernels.cuh"
#include "dense.cuh"
#include "pca.cuh"
#include "rotate_prefill.cuh"
#include "sparse_decode.cuh"
#include "sparse_launch.cuh"

using namespace loki;

namespace {

constexpr double kLog2e = 1.4426950408889634;

// An NVTX range around one entry point's host work (its checks and
// launches), so that a timeline tool shows which call issued which kernels.
// Without a tool attached the calls do nothing.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

size_t elem_size(loki_dtype dt) { return dt == LOKI_BF16 ? 2 : 4; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by every call that reads a cache.
loki_status check_cache(const loki_cache* c) {
    if (!c) return LOKI_ERR_INVALID_ARG;
    if (c->dtype != LOKI_F32 && c->dtype != LOKI_BF16) return LOKI_ERR_INVALID_ARG;
    if (c->num_blocks < 0 || c->num_kv_heads < 1 || c->head_dim < 1) return LOKI_ERR_INVALID_ARG;
    if (c->head_dim != 64 && c->head_dim != 128) return LOKI_ERR_UNSUPPORTED;
    if (c->index_dims < kSlabDims || c->index_dims > c->head_dim || c->index_dims % kSlabDims != 0)
        return LOKI_ERR_INVALID_ARG;
    if (c->num_blocks > 0 && (!c->k_cache || !c->v_cache || !c->k_index)) return LOKI_ERR_INVALID_ARG;
    if (!aligned16(c->k_cache) || !aligned16(c->v_cache) || !aligned16(c->k_index)) return LOKI_ERR_INVALID_ARG;
    if (c->kv_home) {
        if (c->num_device_pages < 0 || c->num_host_pages < 0) return LOKI_ERR_INVALID_ARG;
        if (c->num_host_pages > 0 && (!c->k_host || !c->v_host)) return LOKI_ERR_INVALID_ARG;
        if (!aligned16(c->k_host) || !aligned16(c->v_host)) return LOKI_ERR_INVALID_ARG;
    }
    return LOKI_OK;
}

// The kernels' view of where key and value rows live.
KvMap kv_map_of(const loki_cache* c) {
    KvMap m;
    m.home = c->kv_home;
    m.host_k = c->kv_home ? reinterpret_cast<unsigned char*>(c->k_host) : nullptr;
    m.host_v = c->kv_home ? reinterpret_cast<unsigned char*>(c->v_host) : nullptr;
    m.touch = c->kv_touch;
    m.dev_pages = c->kv_home ? c->num_device_pages : c->num_blocks;
    m.host_pages = c->kv_home ? c->num_host_pages : 0;
    return m;
}

loki_status check_batch(const loki_batch* bt) {
    if (!bt) return LOKI_ERR_INVALID_ARG;
    if (bt->batch < 0 || bt->max_blocks_per_seq < 0 || bt->max_seq_len < 0) return LOKI_ERR_INVALID_ARG;
    if (bt->batch == 0) return LOKI_OK;
    if (!bt->block_table || !bt->seq_lens) return LOKI_ERR_INVALID_ARG;
    if ((int64_t)bt->max_seq_len > (int64_t)bt->max_blocks_per_seq * kBlockTokens) return LOKI_ERR_INVALID_ARG;
    return LOKI_OK;
}

// Launch errors of this call only: a pending error left by earlier, unrelated
// work is cleared when a call starts (clear_pending_error), and the error of
// a failed launch is read and cleared (launch_status), so that it is reported
// once, by the call that caused it.
void clear_pending_error() { cudaGetLastError(); }

loki_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? LOKI_OK : LOKI_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Dispatch over element type, head dim and group size.
// ---------------------------------------------------------------------------
template <template <typename, int, int> class F, typename... A>
loki_status dispatch_tdg(loki_dtype dt, int D, int G, A&&... a) {
#define LOKI_CASE(T_, D_, G_) \
    if (D == D_ && G == G_) return F<T_, D_, G_>::run(std::forward<A>(a)...);
#define LOKI_CASES_D(T_, D_) LOKI_CASE(T_, D_, 1) LOKI_CASE(T_, D_, 2) LOKI_CASE(T_, D_, 4) LOKI_CASE(T_, D_, 8)
    if (dt == LOKI_BF16) {
        LOKI_CASES_D(__nv_bfloat16, 64)
        LOKI_CASES_D(__nv_bfloat16, 128)
    } else {
        LOKI_CASES_D(float, 64)
        LOKI_CASES_D(float, 128)
    }
#undef LOKI_CASES_D
#undef LOKI_CASE
    return LOKI_ERR_UNSUPPORTED;
}

// Argument checks and launches shared by the entry points (the checks run on
// the host before anything is launched).
loki_status check_append(const loki_cache* cache, const loki_batch* batch, const void* k_new, const void* v_new,
                         const float* P) {
    loki_status st = check_cache(cache);
    if (st != LOKI_OK) return st;
    if ((st = check_batch(batch)) != LOKI_OK) return st;
    if (batch->batch == 0) return LOKI_OK;
    if (!k_new || !v_new) return LOKI_ERR_INVALID_ARG;
    if (P && !aligned16(P)) return LOKI_ERR_INVALID_ARG;
    if ((int64_t)batch->batch * cache->num_kv_heads > INT32_MAX / 2) return LOKI_ERR_UNSUPPORTED;
    return LOKI_OK;
}

loki_status launch_append(const loki_cache* cache, const loki_batch* batch, const void* k_new, const void* v_new,
                          const float* P, cudaStream_t s, const float* Ak = nullptr) {
    AppendParams p;
    p.Ak = Ak;
    p.k_cache = cache->k_cache;
    p.v_cache = cache->v_cache;
    p.kv = kv_map_of(cache);
    p.k_index = cache->k_index;
    p.index_dims = cache->index_dims;
    p.block_table = batch->block_table;
    p.seq_lens = batch->seq_lens;
    p.k_new = k_new;
    p.v_new = v_new;
    p.P = P;
    p.num_blocks = cache->num_blocks;
    p.Hkv = cache->num_kv_heads;
    p.max_blocks = batch->max_blocks_per_seq;
    p.max_seq_len = batch->max_seq_len;
    const int grid = batch->batch * cache->num_kv_heads;
    const int D = cache->head_dim;
    clear_pending_error();
    if (cache->dtype == LOKI_BF16) {
        if (D == 64) append_kernel<__nv_bfloat16, 64><<<grid, 256, 0, s>>>(p);
        else append_kernel<__nv_bfloat16, 128><<<grid, 256, 0, s>>>(p);
    } else {
        if (D == 64) append_kernel<float, 64><<<grid, 256, 0, s>>>(p);
        else append_kernel<float, 128><<<grid, 256, 0, s>>>(p);
    }
    return launch_status();
}

loki_status check_decode(const loki_cache* cache, const loki_batch* batch, const void* q, int32_t num_q_heads,
                         const float* P, int32_t r, int32_t k, int32_t recent_window,
                         loki_group_reduce group_reduce, float scale, const float* out) {
    loki_status st = check_cache(cache);
    if (st != LOKI_OK) return st;
    if ((st = check_batch(batch)) != LOKI_OK) return st;
    const int Hkv = cache->num_kv_heads, D = cache->head_dim;
    if (num_q_heads < 1 || num_q_heads % Hkv != 0) return LOKI_ERR_INVALID_ARG;
    if (k < 0 || recent_window < 0 || (k == 0 && recent_window == 0)) return LOKI_ERR_INVALID_ARG;
    if (r < 1 || r > D) return LOKI_ERR_INVALID_ARG;
    if (group_reduce != LOKI_GROUP_SUM && group_reduce != LOKI_GROUP_MAX) return LOKI_ERR_INVALID_ARG;
    if (!(scale >= 0.f) || std::isinf(scale)) return LOKI_ERR_INVALID_ARG;
    if ((int64_t)k + recent_window > INT32_MAX / 2) return LOKI_ERR_INVALID_ARG;
    if (batch->batch == 0) return LOKI_OK;
    if (!q || !P || !out) return LOKI_ERR_INVALID_ARG;
    if (!aligned16(P) || !aligned16(q)) return LOKI_ERR_INVALID_ARG;
    const int G = num_q_heads / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return LOKI_ERR_UNSUPPORTED;
    if (r % kSlabDims != 0) return LOKI_ERR_UNSUPPORTED;
    if (r > cache->index_dims) return LOKI_ERR_INVALID_ARG;
    if ((int64_t)batch->batch * Hkv > 65535) return LOKI_ERR_UNSUPPORTED;
    if (batch->max_seq_len > loki_decode_max_seq_len(D, cache->dtype)) return LOKI_ERR_UNSUPPORTED;
    return LOKI_OK;
}

// Long sequences with large groups can exceed the shared memory of any
// cluster size: checked after the arguments, before anything is launched.
loki_status check_decode_fits(const loki_cache* cache, const loki_batch* batch, int32_t num_q_heads, int32_t r) {
    const int Hkv = cache->num_kv_heads;
    return dispatch_tdg<SparseFits>(cache->dtype, cache->head_dim, num_q_heads / Hkv, (int)r,
                                    (int)(batch->batch * Hkv), (int)batch->max_seq_len, device_info());
}

loki_status launch_decode(const loki_cache* cache, const loki_batch* batch, const void* q, int32_t num_q_heads,
                          const float* P, int32_t r, int32_t k, const int32_t* k_per_seq, int32_t recent_window,
                          loki_group_reduce group_reduce, float scale, float* out, int32_t* selected_idx,
                          cudaStream_t s, bool programmatic, int scorer = kScoreLeading,
                          const float* Aq = nullptr) {
    const int Hkv = cache->num_kv_heads, D = cache->head_dim;
    const int G = num_q_heads / Hkv;
    const int pairs = batch->batch * Hkv;
    const DeviceInfo di = device_info();
    clear_pending_error();
    SparseParams p;
    p.k_cache = cache->k_cache;
    p.v_cache = cache->v_cache;
    p.kv = kv_map_of(cache);
    p.k_index = cache->k_index;
    p.block_table = batch->block_table;
    p.seq_lens = batch->seq_lens;
    p.k_per_seq = k_per_seq;
    p.q = q;
    p.P = P;
    p.Aq = Aq;
    p.out = out;
    p.sel = selected_idx;
    p.num_blocks = cache->num_blocks;
    p.Hkv = Hkv;
    p.max_blocks = batch->max_blocks_per_seq;
    p.max_seq_len = batch->max_seq_len;
    p.index_dims = cache->index_dims;
    p.batch = batch->batch;
    p.longest_first = 0;
    p.r = r;
    p.k = k;
    p.W = recent_window;
    p.group_max = group_reduce == LOKI_GROUP_MAX ? 1 : 0;
    const double sc = scale == 0.f ? 1.0 / std::sqrt((double)D) : (double)scale;
    p.scale_log2 = (float)(sc * kLog2e);
    return dispatch_tdg<SparseLaunch>(cache->dtype, D, G, p, pairs, (int)batch->max_seq_len, di, s, programmatic,
                                      scorer);
}

// The driver's tensor-map encoder, looked up once through the runtime (the
// library links only the runtime).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

// Tensor map of key rows [rows][D] bf16 (row stride D * 2 bytes) with a
// 64-column x box_rows box and the 128-byte swizzle of the MMA operand; rows
// past the end read as zero.
bool encode_key_map(CUtensorMap* map, const void* keys, int64_t rows, int D, int box_rows) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(keys), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

size_t loki_cache_bytes(int32_t num_blocks, int32_t num_kv_heads, int32_t head_dim, loki_dtype dtype) {
    if (num_blocks < 0 || num_kv_heads < 1 || (head_dim != 64 && head_dim != 128)) return 0;
    if (dtype != LOKI_F32 && dtype != LOKI_BF16) return 0;
    return (size_t)num_blocks * num_kv_heads * kBlockTokens * head_dim * elem_size(dtype);
}

size_t loki_index_bytes(int32_t num_blocks, int32_t num_kv_heads, int32_t index_dims, loki_dtype dtype) {
    if (num_blocks < 0 || num_kv_heads < 1 || index_dims < kSlabDims || index_dims > 128 ||
        index_dims % kSlabDims != 0)
        return 0;
    if (dtype != LOKI_F32 && dtype != LOKI_BF16) return 0;
    return (size_t)num_blocks * num_kv_heads * kBlockTokens * index_dims * elem_size(dtype);
}

int32_t loki_abi_version(void) { return LOKI_ABI_VERSION; }

const char* loki_status_string(loki_status s) {
    switch (s) {
        case LOKI_OK: return "ok";
        case LOKI_ERR_INVALID_ARG: return "invalid argument";
        case LOKI_ERR_UNSUPPORTED: return "unsupported shape or option";
        case LOKI_ERR_WORKSPACE: return "workspace missing or too small";
        case LOKI_ERR_CUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

loki_status loki_device_error(int32_t clear, uint32_t* bits) {
    if (!bits) return LOKI_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return LOKI_ERR_CUDA;
    if (cudaMemcpyFromSymbol(bits, g_device_error, sizeof(uint32_t)) != cudaSuccess) return LOKI_ERR_CUDA;
    if (clear) {
        const uint32_t zero = 0;
        if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(uint32_t)) != cudaSuccess) return LOKI_ERR_CUDA;
    }
    return LOKI_OK;
}

loki_status loki_prefill_cache(const loki_cache* cache, const loki_batch* batch, const void* k_rot,
                               const void* v, int32_t max_len, loki_stream_t stream) {
    NvtxRange nvtx_range("loki_prefill_cache");
    loki_status st = check_cache(cache);
    if (st != LOKI_OK) return st;
    if ((st = check_batch(batch)) != LOKI_OK) return st;
    if (batch->batch == 0 || batch->max_blocks_per_seq == 0) return LOKI_OK;
    if (!k_rot || !v || max_len < batch->max_seq_len) return LOKI_ERR_INVALID_ARG;
    if (!aligned16(k_rot) || !aligned16(v)) return LOKI_ERR_INVALID_ARG;
    if ((int64_t)batch->batch * cache->num_kv_heads > 65535) return LOKI_ERR_UNSUPPORTED;
    PrefillParams p;
    p.k_cache = cache->k_cache;
    p.v_cache = cache->v_cache;
    p.kv = kv_map_of(cache);
    p.k_index = cache->k_index;
    p.index_dims = cache->index_dims;
    p.block_table = batch->block_table;
    p.seq_lens = batch->seq_lens;
    p.k_rot = k_rot;
    p.v = v;
    p.num_blocks = cache->num_blocks;
    p.Hkv = cache->num_kv_heads;
    p.max_blocks = batch->max_blocks_per_seq;
    p.max_seq_len = batch->max_seq_len;
    p.max_len = max_len;
    const int nblk = (batch->max_seq_len + kBlockTokens - 1) / kBlockTokens;
    if (nblk == 0) return LOKI_OK;
    dim3 grid(nblk, batch->batch * cache->num_kv_heads);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int D = cache->head_dim;
    clear_pending_error();
    if (cache->dtype == LOKI_BF16) {
        if (D == 64) prefill_kernel<__nv_bfloat16, 64><<<grid, 256, 0, s>>>(p);
        else prefill_kernel<__nv_bfloat16, 128><<<grid, 256, 0, s>>>(p);
    } else {
        if (D == 64) prefill_kernel<float, 64><<<grid, 256, 0, s>>>(p);
        else prefill_kernel<float, 128><<<grid, 256, 0, s>>>(p);
    }
    return launch_status();
}

loki_status loki_prefill_rotate(const loki_cache* cache, const loki_batch* batch, const void* k, const void* v,
                                const float* P, int32_t max_len, loki_stream_t stream) {
    NvtxRange nvtx_range("loki_prefill_rotate");
    loki_status st = check_cache(cache);
    if (st != LOKI_OK) return st;
    if ((st = check_batch(batch)) != LOKI_OK) return st;
    if (batch->batch == 0 || batch->max_seq_len == 0) return LOKI_OK;
    if (!k || !v || !P) return LOKI_ERR_INVALID_ARG;
    if (max_len < batch->max_seq_len) return LOKI_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(P)) return LOKI_ERR_INVALID_ARG;
    if ((int64_t)batch->batch * cache->num_kv_heads > 65535) return LOKI_ERR_UNSUPPORTED;
    RotateParams p;
    p.k_cache = cache->k_cache;
    p.v_cache = cache->v_cache;
    p.kv = kv_map_of(cache);
    p.k_index = cache->k_index;
    p.block_table = batch->block_table;
    p.seq_lens = batch->seq_lens;
    p.k = k;
    p.v = v;
    p.P = P;
    p.num_blocks = cache->num_blocks;
    p.Hkv = cache->num_kv_heads;
    p.max_blocks = batch->max_blocks_per_seq;
    p.max_seq_len = batch->max_seq_len;
    p.max_len = max_len;
    p.index_dims = cache->index_dims;
    const int pairs = batch->batch * cache->num_kv_heads;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int D = cache->head_dim;
    if (cache->dtype == LOKI_BF16) {
        // the keys as a 2-D tensor [batch * Hkv * max_len rows][D], box 64 x 128, 128-byte swizzle
        const int64_t rows = (int64_t)pairs * max_len;
        if (rows + kRotTile > INT32_MAX) return LOKI_ERR_UNSUPPORTED;
        CUtensorMap tmap, kmap;
        if (!encode_key_map(&tmap, k, rows, D, kRotTile)) return LOKI_ERR_CUDA;
        // the key cache's device pages as [pages * Hkv * 16 rows][D], the store side
        const int64_t dev_pages = cache->kv_home ? cache->num_device_pages : cache->num_blocks;
        const int64_t krows = std::max<int64_t>(1, dev_pages) * cache->num_kv_heads * kBlockTokens;
        if (krows > INT32_MAX) return LOKI_ERR_UNSUPPORTED;
        if (!encode_key_map(&kmap, cache->k_cache, krows, D, kBlockTokens)) return LOKI_ERR_CUDA;
        p.tiles_per_pair = (batch->max_seq_len + kRotTile - 1) / kRotTile;
        p.total_tiles = (int64_t)pairs * p.tiles_per_pair;
        auto launch = [&](auto kern, int smem) {
            if (ensure_smem_attr((const void*)kern, smem) != cudaSuccess) return LOKI_ERR_CUDA;
            int per_sm = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRotThreads, smem) != cudaSuccess ||
                per_sm < 1) {
                cudaGetLastError();
                return LOKI_ERR_CUDA;
            }
            const int64_t ctas = std::min<int64_t>(p.total_tiles, (int64_t)per_sm * std::max(1, device_info().sms));
            clear_pending_error();
            kern<<<(unsigned)ctas, kRotThreads, smem, s>>>(p, tmap, kmap);
            return launch_status();
        };
        if (D == 64) return launch(rotate_prefill_tc_kernel<64>, rotate_smem_bytes<64>());
        return launch(rotate_prefill_tc_kernel<128>, rotate_smem_bytes<128>());
    }
    const dim3 grid((batch->max_seq_len + kBlockTokens - 1) / kBlockTokens, pairs);
    clear_pending_error();
    if (D == 64) rotate_prefill_f32_kernel<64><<<grid, 256, 0, s>>>(p);
    else rotate_prefill_f32_kernel<128><<<grid, 256, 0, s>>>(p);
    return launch_status();
}

loki_status loki_pca_basis(const void* keys, int32_t num_heads, int64_t n, int32_t head_dim, loki_dtype dtype,
                           float* P, float* eigvals, loki_stream_t stream) {
    NvtxRange nvtx_range("loki_pca_basis");
    if (num_heads < 0 || n < 0) return LOKI_ERR_INVALID_ARG;
    if (dtype != LOKI_F32 && dtype != LOKI_BF16) return LOKI_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return LOKI_ERR_UNSUPPORTED;
    if (num_heads == 0) return LOKI_OK;
    if (n < 2) return LOKI_ERR_INVALID_ARG;
    if (!keys || !P) return LOKI_ERR_INVALID_ARG;
    if (num_heads > 65535) return LOKI_ERR_UNSUPPORTED;
    PcaParams p;
    p.keys = keys;
    p.P = P;
    p.eigvals = eigvals;
    p.n = n;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    auto launch = [&](auto kern, int smem) {
        if (ensure_smem_attr((const void*)kern, smem) != cudaSuccess) return LOKI_ERR_CUDA;
        clear_pending_error();
        kern<<<num_heads, kPcaThreads, smem, s>>>(p);
        return launch_status();
    };
    if (dtype == LOKI_BF16) {
        if (head_dim == 64) return launch(pca_kernel<__nv_bfloat16, 64>, pca_smem_bytes<64>());
        return launch(pca_kernel<__nv_bfloat16, 128>, pca_smem_bytes<128>());
    }
    if (head_dim == 64) return launch(pca_kernel<float, 64>, pca_smem_bytes<64>());
    return launch(pca_kernel<float, 128>, pca_smem_bytes<128>());
}

loki_status loki_append_keys(const loki_cache* cache, const loki_batch* batch, const void* k_new,
                             const void* v_new, const float* P, loki_stream_t stream) {
    NvtxRange nvtx_range("loki_append_keys");
    const loki_status st = check_append(cache, batch, k_new, v_new, P);
    if (st != LOKI_OK || batch->batch == 0) return st;
    return launch_append(cache, batch, k_new, v_new, P, reinterpret_cast<cudaStream_t>(stream));
}

loki_status loki_append_keys_asym(const loki_cache* cache, const loki_batch* batch, const void* k_new,
                                  const void* v_new, const float* P, const float* A_k, loki_stream_t stream) {
    NvtxRange nvtx_range("loki_append_keys_asym");
    const loki_status st = check_append(cache, batch, k_new, v_new, P);
    if (st != LOKI_OK || batch->batch == 0) return st;
    if (!A_k || !aligned16(A_k)) return LOKI_ERR_INVALID_ARG;
    return launch_append(cache, batch, k_new, v_new, P, reinterpret_cast<cudaStream_t>(stream), A_k);
}

loki_status loki_index_keys(const loki_cache* cache, const loki_batch* batch, const void* k, const float* A_k,
                            int32_t max_len, loki_stream_t stream) {
    NvtxRange nvtx_range("loki_index_keys");
    loki_status st = check_cache(cache);
    if (st != LOKI_OK) return st;
    if ((st = check_batch(batch)) != LOKI_OK) return st;
    if (batch->batch == 0 || batch->max_seq_len == 0) return LOKI_OK;
    if (!k || !A_k || max_len < batch->max_seq_len) return LOKI_ERR_INVALID_ARG;
    if (!aligned16(A_k)) return LOKI_ERR_INVALID_ARG;
    if ((int64_t)batch->batch * cache->num_kv_heads > 65535) return LOKI_ERR_UNSUPPORTED;
    IndexParams p;
    p.k_index = cache->k_index;
    p.block_table = batch->block_table;
    p.seq_lens = batch->seq_lens;
    p.k = k;
    p.Ak = A_k;
    p.num_blocks = cache->num_blocks;
    p.Hkv = cache->num_kv_heads;
    p.max_blocks = batch->max_blocks_per_seq;
    p.max_seq_len = batch->max_seq_len;
    p.max_len = max_len;
    p.index_dims = cache->index_dims;
    const dim3 grid((batch->max_seq_len + kIndexTile - 1) / kIndexTile, batch->batch * cache->num_kv_heads);
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int D = cache->head_dim;
    auto launch = [&](auto kern, int smem) {
        if (ensure_smem_attr((const void*)kern, smem) != cudaSuccess) return LOKI_ERR_CUDA;
        clear_pending_error();
        kern<<<grid, 256, smem, s>>>(p);
        return launch_status();
    };
    if (cache->dtype == LOKI_BF16) {
        if (D == 64) return launch(index_keys_kernel<__nv_bfloat16, 64>, index_smem_bytes<64>(p.index_dims));
        return launch(index_keys_kernel<__nv_bfloat16, 128>, index_smem_bytes<128>(p.index_dims));
    }
    if (D == 64) return launch(index_keys_kernel<float, 64>, index_smem_bytes<64>(p.index_dims));
    return launch(index_keys_kernel<float, 128>, index_smem_bytes<128>(p.index_dims));
}

int32_t loki_decode_max_seq_len(int32_t head_dim, loki_dtype dtype) {
    (void)dtype;
    if (head_dim != 64 && head_dim != 128) return 0;
    return 16 * kCtaTokenCap;
}

size_t loki_decode_workspace_bytes(const loki_cache* cache, const loki_batch* batch, int32_t num_q_heads,
                                   int32_t k, int32_t recent_window) {
    (void)cache;
    (void)batch;
    (void)num_q_heads;
    (void)k;
    (void)recent_window;
    return 0;  // the fused kernel keeps every intermediate on chip
}

loki_status loki_decode_attention(const loki_cache* cache, const loki_batch* batch, const void* q,
                                  int32_t num_q_heads, const float* P, int32_t r, int32_t k,
                                  const int32_t* k_per_seq, int32_t recent_window,
                                  loki_group_reduce group_reduce, float scale, float* out,
                                  int32_t* selected_idx, void* workspace, size_t workspace_bytes,
                                  loki_stream_t stream) {
    NvtxRange nvtx_range("loki_decode_attention");
    (void)workspace;
    (void)workspace_bytes;
    loki_status st = check_decode(cache, batch, q, num_q_heads, P, r, k, recent_window, group_reduce, scale, out);
    if (st != LOKI_OK || batch->batch == 0) return st;
    if ((st = check_decode_fits(cache, batch, num_q_heads, r)) != LOKI_OK) return st;
    return launch_decode(cache, batch, q, num_q_heads, P, r, k, k_per_seq, recent_window, group_reduce, scale, out,
                         selected_idx, reinterpret_cast<cudaStream_t>(stream), false);
}

loki_status loki_decode_attention_scored(const loki_cache* cache, const loki_batch* batch, const void* q,
                                         int32_t num_q_heads, const float* P, int32_t r, int32_t k,
                                         const int32_t* k_per_seq, int32_t recent_window,
                                         loki_group_reduce group_reduce, float scale, loki_scorer scorer,
                                         float* out, int32_t* selected_idx, void* workspace,
                                         size_t workspace_bytes, loki_stream_t stream) {
    NvtxRange nvtx_range("loki_decode_attention_scored");
    (void)workspace;
    (void)workspace_bytes;
    int sc;
    switch (scorer) {
        case LOKI_SCORER_LEADING: sc = kScoreLeading; break;
        case LOKI_SCORER_MAGNITUDE: sc = kScoreMagnitude; break;
        case LOKI_SCORER_MAGNITUDE_SLABS: sc = kScoreSlabs; break;
        default: return LOKI_ERR_INVALID_ARG;
    }
    loki_status st = check_decode(cache, batch, q, num_q_heads, P, r, k, recent_window, group_reduce, scale, out);
    if (st != LOKI_OK || batch->batch == 0) return st;
    if ((st = check_decode_fits(cache, batch, num_q_heads, r)) != LOKI_OK) return st;
    return launch_decode(cache, batch, q, num_q_heads, P, r, k, k_per_seq, recent_window, group_reduce, scale, out,
                         selected_idx, reinterpret_cast<cudaStream_t>(stream), false, sc);
}

loki_status loki_decode_attention_asym(const loki_cache* cache, const loki_batch* batch, const void* q,
                                       int32_t num_q_heads, const float* P, const float* A_q, int32_t r, int32_t k,
                                       const int32_t* k_per_seq, int32_t recent_window,
                                       loki_group_reduce group_reduce, float scale, float* out,
                                       int32_t* selected_idx, void* workspace, size_t workspace_bytes,
                                       loki_stream_t stream) {
    NvtxRange nvtx_range("loki_decode_attention_asym");
    (void)workspace;
    (void)workspace_bytes;
    loki_status st = check_decode(cache, batch, q, num_q_heads, P, r, k, recent_window, group_reduce, scale, out);
    if (st != LOKI_OK || batch->batch == 0) return st;
    if (!A_q || !aligned16(A_q)) return LOKI_ERR_INVALID_ARG;
    if ((st = check_decode_fits(cache, batch, num_q_heads, r)) != LOKI_OK) return st;
    return launch_decode(cache, batch, q, num_q_heads, P, r, k, k_per_seq, recent_window, group_reduce, scale, out,
                         selected_idx, reinterpret_cast<cudaStream_t>(stream), false, kScoreAsym, A_q);
}

// Regions of loki_decode_step_host's staging buffer: k_new, v_new, q, out.
struct StepStaging {
    size_t k_off, v_off, q_off, o_off, k_bytes, q_bytes, o_bytes, total;
};
static bool step_staging(const loki_cache* cache, const loki_batch* batch, int32_t num_q_heads, StepStaging* st) {
    if (check_cache(cache) != LOKI_OK || check_batch(batch) != LOKI_OK || num_q_heads < 1) return false;
    const size_t es = elem_size(cache->dtype), D = (size_t)cache->head_dim, B = (size_t)batch->batch;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    st->k_bytes = B * cache->num_kv_heads * D * es;
    st->q_bytes = B * (size_t)num_q_heads * D * es;
    st->o_bytes = B * (size_t)num_q_heads * D * 4;
    st->k_off = 0;
    st->v_off = up(st->k_bytes);
    st->q_off = st->v_off + up(st->k_bytes);
    st->o_off = st->q_off + up(st->q_bytes);
    st->total = st->o_off + up(st->o_bytes);
    return true;
}

// The address under which the current device reads and writes a host buffer
// in place, if it can: page-locked memory mapped into the device's address
// space (cudaHostAlloc / cudaMallocHost memory, and cudaHostRegister'ed
// memory, under unified addressing, where that address is the host address
// itself). nullptr for pageable memory or any other answer.
static void* mapped_host_address(const void* host) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, host) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (a.type != cudaMemoryTypeHost || a.devicePointer != host) return nullptr;
    return a.devicePointer;
}

size_t loki_decode_step_host_bytes(const loki_cache* cache, const loki_batch* batch, int32_t num_q_heads) {
    StepStaging st;
    return step_staging(cache, batch, num_q_heads, &st) ? st.total : 0;
}

loki_status loki_decode_step_host(const loki_cache* cache, const loki_batch* batch, const void* k_new_host,
                                  const void* v_new_host, const void* q_host, int32_t num_q_heads, const float* P,
                                  int32_t r, int32_t k, const int32_t* k_per_seq, int32_t recent_window,
                                  loki_group_reduce group_reduce, float scale, float* out_host, void* staging,
                                  size_t staging_bytes, loki_stream_t stream) {
    NvtxRange nvtx_range("loki_decode_step_host");
    StepStaging st;
    if (!step_staging(cache, batch, num_q_heads, &st)) {
        loki_status e = check_cache(cache);
        if (e == LOKI_OK) e = check_batch(batch);
        return e == LOKI_OK ? LOKI_ERR_INVALID_ARG : e;
    }
    if (batch->batch == 0) return LOKI_OK;
    if (!k_new_host || !v_new_host || !q_host || !out_host) return LOKI_ERR_INVALID_ARG;
    if (!staging || staging_bytes < st.total) return LOKI_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(staging) & 255u) != 0) return LOKI_ERR_INVALID_ARG;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // Mapped page-locked buffers are read and written in place by the kernels
    // (the append reads k_new and v_new, the decode's prologue reads q and its
    // merge writes out, all with plain loads and stores over the host link):
    // no copy engine on the step's path. Otherwise the buffers go through
    // `staging`, one cudaMemcpyAsync each.
    {
        void* mk = mapped_host_address(k_new_host);
        void* mv = mapped_host_address(v_new_host);
        void* mq = mapped_host_address(q_host);
        void* mo = mapped_host_address(out_host);
        const uintptr_t es = elem_size(cache->dtype);  // the append reads single elements
        if (mk && mv && mq && mo && reinterpret_cast<uintptr_t>(mk) % es == 0 &&
            reinterpret_cast<uintptr_t>(mv) % es == 0 && (reinterpret_cast<uintptr_t>(mo) & 3u) == 0) {
            float* out_mapped = reinterpret_cast<float*>(mo);
            loki_status e = check_append(cache, batch, mk, mv, P);
            if (e == LOKI_OK) e = check_decode(cache, batch, mq, num_q_heads, P, r, k, recent_window, group_reduce,
                                               scale, out_mapped);
            if (e == LOKI_OK) {
                if ((e = check_decode_fits(cache, batch, num_q_heads, r)) != LOKI_OK) return e;
                clear_pending_error();
                if ((e = launch_append(cache, batch, mk, mv, P, s)) != LOKI_OK) return e;
                return launch_decode(cache, batch, mq, num_q_heads, P, r, k, k_per_seq, recent_window, group_reduce,
                                     scale, out_mapped, nullptr, s, true);
            }
            // (an unaligned q falls through to the staged copies, as do
            // inputs off their element alignment and an unaligned out)
        }
    }
    char* dev = reinterpret_cast<char*>(staging);
    void* dk = dev + st.k_off;
    void* dv = dev + st.v_off;
    void* dq = dev + st.q_off;
    float* dout = reinterpret_cast<float*>(dev + st.o_off);
    // every argument of the step, checked before the first copy
    loki_status e = check_append(cache, batch, dk, dv, P);
    if (e != LOKI_OK) return e;
    e = check_decode(cache, batch, dq, num_q_heads, P, r, k, recent_window, group_reduce, scale, dout);
    if (e != LOKI_OK) return e;
    if ((e = check_decode_fits(cache, batch, num_q_heads, r)) != LOKI_OK) return e;
    clear_pending_error();
    if (cudaMemcpyAsync(dk, k_new_host, st.k_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dv, v_new_host, st.k_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dq, q_host, st.q_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
        cudaGetLastError();
        return LOKI_ERR_CUDA;
    }
    if ((e = launch_append(cache, batch, dk, dv, P, s)) != LOKI_OK) return e;
    if ((e = launch_decode(cache, batch, dq, num_q_heads, P, r, k, k_per_seq, recent_window, group_reduce, scale, dout,
                           nullptr, s, true)) != LOKI_OK)
        return e;
    if (cudaMemcpyAsync(out_host, dout, st.o_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) {
        cudaGetLastError();
        return LOKI_ERR_CUDA;
    }
    return LOKI_OK;
}

loki_status loki_decode_step(const loki_cache* cache, const loki_batch* batch, const void* k_new, const void* v_new,
                             const void* q, int32_t num_q_heads, const float* P, int32_t r, int32_t k,
                             const int32_t* k_per_seq, int32_t recent_window, loki_group_reduce group_reduce,
                             float scale, float* out, int32_t* selected_idx, void* workspace,
                             size_t workspace_bytes, loki_stream_t stream) {
    NvtxRange nvtx_range("loki_decode_step");
    (void)workspace;
    (void)workspace_bytes;
    loki_status st = check_append(cache, batch, k_new, v_new, P);
    if (st != LOKI_OK) return st;
    st = check_decode(cache, batch, q, num_q_heads, P, r, k, recent_window, group_reduce, scale, out);
    if (st != LOKI_OK || batch->batch == 0) return st;
    if ((st = check_decode_fits(cache, batch, num_q_heads, r)) != LOKI_OK) return st;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = launch_append(cache, batch, k_new, v_new, P, s)) != LOKI_OK) return st;
    return launch_decode(cache, batch, q, num_q_heads, P, r, k, k_per_seq, recent_window, group_reduce, scale, out,
                         selected_idx, s, true);
}

}  // extern "C"

namespace {

int dense_splits(int max_seq_len, int split_tokens = kDenseSplitTokens) {
    return std::max(1, (max_seq_len + split_tokens - 1) / split_tokens);
}

// Tokens per split of the dense path: twice the base split when that still
// gives at least four waves of CTAs (one CTA per SM), which halves the CTAs'
// fixed costs (pipeline fill and drain, launch, partial write): measured on
// B200 0.232 -> 0.204 ms at batch 8 x 8 kv heads x L 32768 and 0.531 -> 0.454 ms
// for 512 pairs of 4k-16k tokens, while 32 pairs of 4096 tokens (one partial
// wave) went from 38 to 46 us and keep the base split.
int dense_split_tokens(int64_t pairs, int max_seq_len, int sms) {
    const int64_t ctas = pairs * dense_splits(max_seq_len, 2 * kDenseSplitTokens);
    return ctas >= 4 * (int64_t)std::max(1, sms) ? 2 * kDenseSplitTokens : kDenseSplitTokens;
}

template <typename T, int D, int G>
struct DenseLaunch {
    static loki_status run(DenseParams p, int batch, cudaStream_t s) {
        using Geom = DenseGeom<T, D, G>;
        auto split_kern = dense_split_kernel<T, D, G>;
        if (ensure_smem_attr((const void*)split_kern, Geom::SMEM_BYTES) != cudaSuccess) return LOKI_ERR_CUDA;
        clear_pending_error();
        const int pairs = batch * p.Hkv;
        rotate_query_kernel<T, D, G><<<pairs, 256, 0, s>>>(p);
        split_kern<<<dim3(p.splits, pairs), kDenseThreads, Geom::SMEM_BYTES, s>>>(p);
        merge_kernel<D, G><<<batch * p.Hkv * G, D, 0, s>>>(p);
        return launch_status();
    }
};

}  // namespace

extern "C" {

size_t loki_dense_workspace_bytes(const loki_cache* cache, const loki_batch* batch, int32_t num_q_heads) {
    if (check_cache(cache) != LOKI_OK || check_batch(batch) != LOKI_OK || num_q_heads < 1) return 0;
    const size_t D = cache->head_dim;
    const size_t G = (size_t)num_q_heads / cache->num_kv_heads;
    const size_t qhat = (size_t)batch->batch * num_q_heads * D * 4;
    const size_t parts = (size_t)batch->batch * cache->num_kv_heads * dense_splits(batch->max_seq_len) * G *
                         (D + 2) * 4;
    return ((qhat + 255) & ~(size_t)255) + parts;
}

loki_status loki_dense_attention(const loki_cache* cache, const loki_batch* batch, const void* q,
                                 int32_t num_q_heads, const float* P, float scale, float* out,
                                 void* workspace, size_t workspace_bytes, loki_stream_t stream) {
    NvtxRange nvtx_range("loki_dense_attention");
    loki_status st = check_cache(cache);
    if (st != LOKI_OK) return st;
    if ((st = check_batch(batch)) != LOKI_OK) return st;
    const int Hkv = cache->num_kv_heads, D = cache->head_dim;
    if (num_q_heads < 1 || num_q_heads % Hkv != 0) return LOKI_ERR_INVALID_ARG;
    if (!(scale >= 0.f) || std::isinf(scale)) return LOKI_ERR_INVALID_ARG;
    if (batch->batch == 0) return LOKI_OK;
    if (!q || !P || !out) return LOKI_ERR_INVALID_ARG;
    const int G = num_q_heads / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return LOKI_ERR_UNSUPPORTED;
    const int splits = dense_splits(batch->max_seq_len);
    if ((int64_t)batch->batch * Hkv > 65535 || splits > INT32_MAX / 4) return LOKI_ERR_UNSUPPORTED;
    const size_t need = loki_dense_workspace_bytes(cache, batch, num_q_heads);
    if (!workspace || workspace_bytes < need) return LOKI_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LOKI_ERR_INVALID_ARG;
    DenseParams p;
    p.k_cache = cache->k_cache;
    p.v_cache = cache->v_cache;
    p.kv = kv_map_of(cache);
    p.block_table = batch->block_table;
    p.seq_lens = batch->seq_lens;
    p.q = q;
    p.P = P;
    p.out = out;
    const size_t qhat_bytes = ((size_t)batch->batch * num_q_heads * D * 4 + 255) & ~(size_t)255;
    p.qhat = reinterpret_cast<float*>(workspace);
    p.parts = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + qhat_bytes);
    p.num_blocks = cache->num_blocks;
    p.Hkv = Hkv;
    p.max_blocks = batch->max_blocks_per_seq;
    p.max_seq_len = batch->max_seq_len;
    // fewer, longer splits than the workspace is sized for when they fill the GPU
    p.split_tokens = dense_split_tokens((int64_t)batch->batch * Hkv, batch->max_seq_len, device_info().sms);
    p.splits = dense_splits(batch->max_seq_len, p.split_tokens);
    const double sc = scale == 0.f ? 1.0 / std::sqrt((double)D) : (double)scale;
    p.scale_log2 = (float)(sc * kLog2e);
    return dispatch_tdg<DenseLaunch>(cache->dtype, D, G, p, batch->batch, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Dense decode attention with the library's own scratch, for callers that
// cannot allocate device memory. The scratch is a file-scope device array, so
// every GPU that loads the library holds LOKI_DENSE_STATIC_SCRATCH_BYTES of
// it until the process exits; all calls on a device share it.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_dense_static_scratch[LOKI_DENSE_STATIC_SCRATCH_BYTES];

namespace {

// Device address of the static scratch on the current device. In host code
// the array's name is only a host-side stand-in, so the address is taken
// once per device with cudaGetSymbolAddress (with that device current).
loki_status static_scratch_address(void** out) {
    static std::mutex mu;
    static std::map<int, void*> addr;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOKI_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    auto it = addr.find(dev);
    if (it == addr.end()) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_dense_static_scratch) != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return LOKI_ERR_CUDA;
        }
        it = addr.emplace(dev, ptr).first;
    }
    *out = it->second;
    return LOKI_OK;
}

}  // namespace

extern "C" loki_status loki_dense_attention_static(const loki_cache* cache, const loki_batch* batch, const void* q,
                                                   int32_t num_q_heads, const float* P, float scale, float* out,
                                                   loki_stream_t stream) {
    NvtxRange nvtx_range("loki_dense_attention_static");
    void* scratch = nullptr;
    loki_status st = static_scratch_address(&scratch);
    if (st != LOKI_OK) return st;
    if (check_cache(cache) == LOKI_OK && check_batch(batch) == LOKI_OK && num_q_heads >= 1 &&
        loki_dense_workspace_bytes(cache, batch, num_q_heads) > (size_t)LOKI_DENSE_STATIC_SCRATCH_BYTES)
        return LOKI_ERR_WORKSPACE;  // these sizes need more scratch than the built-in array holds
    return loki_dense_attention(cache, batch, q, num_q_heads, P, scale, out, scratch,
                                (size_t)LOKI_DENSE_STATIC_SCRATCH_BYTES, stream);
}

// ---------------------------------------------------------------------------
// Host offload of key and value pages (LRQK page, abstract: only the kept
// rows of offloaded blocks cross the host link; the blocks the selection
// keeps hitting are brought to the device between steps).
// ---------------------------------------------------------------------------
namespace {

size_t block_page_bytes(const loki_cache* c) {
    return (size_t)c->num_kv_heads * kBlockTokens * (size_t)c->head_dim * elem_size(c->dtype);
}

}  // namespace

extern "C" {

int32_t loki_offload_plan(int32_t num_blocks, int32_t* kv_home, int32_t* spare_page, const uint32_t* touch,
                          int32_t max_moves, loki_page_move* moves) {
    if (num_blocks < 0 || max_moves < 0 || !spare_page || *spare_page < 0) return -1;
    if (num_blocks > 0 && (!kv_home || !touch)) return -1;
    if (max_moves > 0 && !moves) return -1;
    std::vector<int32_t> on_host, on_dev;
    for (int32_t b = 0; b < num_blocks; ++b) {
        if (kv_home[b] == *spare_page) return -1;
        (kv_home[b] < 0 ? on_host : on_dev).push_back(b);
    }
    const size_t n = std::min({(size_t)max_moves, on_host.size(), on_dev.size()});
    // hottest offloaded blocks first, coldest device blocks first; ties to the lower id
    std::partial_sort(on_host.begin(), on_host.begin() + n, on_host.end(), [&](int32_t a, int32_t b) {
        return touch[a] != touch[b] ? touch[a] > touch[b] : a < b;
    });
    std::partial_sort(on_dev.begin(), on_dev.begin() + n, on_dev.end(), [&](int32_t a, int32_t b) {
        return touch[a] != touch[b] ? touch[a] < touch[b] : a < b;
    });
    int32_t done = 0;
    for (size_t i = 0; i < n; ++i) {
        const int32_t in = on_host[i], out = on_dev[i];
        if (touch[in] <= touch[out]) break;
        loki_page_move m;
        m.block_in = in;
        m.block_out = out;
        m.host_page = -(kv_home[in] + 1);
        m.device_page = *spare_page;
        m.freed_page = kv_home[out];
        kv_home[in] = m.device_page;
        kv_home[out] = -(m.host_page + 1);
        *spare_page = m.freed_page;
        moves[done++] = m;
    }
    return done;
}

loki_status loki_offload_apply(const loki_cache* cache, const loki_page_move* moves, int32_t num_moves,
                               const int32_t* kv_home_host, loki_stream_t stream) {
    NvtxRange nvtx_range("loki_offload_apply");
    loki_status st = check_cache(cache);
    if (st != LOKI_OK) return st;
    if (!cache->kv_home || num_moves < 0 || (num_moves > 0 && !moves)) return LOKI_ERR_INVALID_ARG;
    if (cache->num_blocks > 0 && !kv_home_host) return LOKI_ERR_INVALID_ARG;
    for (int32_t i = 0; i < num_moves; ++i) {
        const loki_page_move& m = moves[i];
        if (m.block_in < 0 || m.block_in >= cache->num_blocks || m.block_out < 0 ||
            m.block_out >= cache->num_blocks || m.host_page < 0 || m.host_page >= cache->num_host_pages ||
            m.device_page < 0 || m.device_page >= cache->num_device_pages || m.freed_page < 0 ||
            m.freed_page >= cache->num_device_pages)
            return LOKI_ERR_INVALID_ARG;
    }
    const size_t pb = block_page_bytes(cache);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* dk = reinterpret_cast<char*>(cache->k_cache);
    char* dv = reinterpret_cast<char*>(cache->v_cache);
    char* hk = reinterpret_cast<char*>(cache->k_host);
    char* hv = reinterpret_cast<char*>(cache->v_host);
    clear_pending_error();
    bool ok = true;
    for (int32_t i = 0; i < num_moves && ok; ++i) {
        const loki_page_move& m = moves[i];
        // promote block_in into the free page, then demote block_out into the
        // host page block_in has just left (stream order keeps them apart)
        ok = cudaMemcpyAsync(dk + m.device_page * pb, hk + m.host_page * pb, pb, cudaMemcpyDefault, s) == cudaSuccess &&
             cudaMemcpyAsync(dv + m.device_page * pb, hv + m.host_page * pb, pb, cudaMemcpyDefault, s) == cudaSuccess &&
             cudaMemcpyAsync(hk + m.host_page * pb, dk + m.freed_page * pb, pb, cudaMemcpyDefault, s) == cudaSuccess &&
             cudaMemcpyAsync(hv + m.host_page * pb, dv + m.freed_page * pb, pb, cudaMemcpyDefault, s) == cudaSuccess;
    }
    if (ok && cache->num_blocks > 0)
        ok = cudaMemcpyAsync(const_cast<int32_t*>(cache->kv_home), kv_home_host, (size_t)cache->num_blocks * 4,
                             cudaMemcpyHostToDevice, s) == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        return LOKI_ERR_CUDA;
    }
    return LOKI_OK;
}

loki_status loki_host_device_pointer(void* host, void** device) {
    if (!host || !device) return LOKI_ERR_INVALID_ARG;
    void* d = nullptr;
    if (cudaHostGetDevicePointer(&d, host, 0) != cudaSuccess || !d) {
        cudaGetLastError();
        return LOKI_ERR_CUDA;
    }
    *device = d;
    return LOKI_OK;
}

}  // extern "C"
