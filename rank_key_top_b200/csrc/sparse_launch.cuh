// Launch geometry of sparse_decode_kernel: the device's SM count and shared
// memory, the cluster size, the shared-memory layout of a CTA (key ring depth,
// regions) and the launch itself. Host code; kept beside the kernel because
// together they fix what the kernel does on the device.
#pragma once

#include <cuda_runtime.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "sparse_decode.cuh"

namespace loki {

struct DeviceInfo {
    int sms = 0;
    int max_smem_optin = 0;
};

inline DeviceInfo device_info() {
    static std::mutex mu;
    static std::map<int, DeviceInfo> cache;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(dev);
    if (it != cache.end()) return it->second;
    DeviceInfo di;
    cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&di.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaGetLastError();  // no device: the attributes stay 0 and every shape is unsupported
    cache[dev] = di;
    return di;
}

// Allows `kern` up to `bytes` of dynamic shared memory on the current device:
// the attribute belongs to the function on that device, and it is raised
// (never lowered) as larger launches come, so every size up to the largest
// requested so far stays launchable.
inline cudaError_t ensure_smem_attr(const void* kern, int bytes) {
    static std::mutex mu;
    static std::map<std::pair<int, const void*>, int> allowed;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(dev, kern);
    auto it = allowed.find(key);
    if (it != allowed.end() && it->second >= bytes) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return e;
    }
    allowed[key] = bytes;
    return cudaSuccess;
}

// Shared-memory layout of one CTA for C CTAs per (sequence, kv head), with a
// key-index ring of ring_per_warp bytes per warp.
template <typename T, int D, int G>
void sparse_layout(SparseParams& p, int max_seq_len, int ring_per_warp) {
    using Geom = SparseGeom<T, D, G>;
    auto align = [](int x) { return (x + 127) & ~127; };
    const int nblk = (max_seq_len + kBlockTokens - 1) / kBlockTokens;
    p.cta_tokens = std::max(1, (nblk + p.C - 1) / p.C) * kBlockTokens;
    p.slot_bytes = p.r * kBlockTokens * (int)sizeof(T);
    // a power of two (the kernel's ring arithmetic relies on it)
    p.slots = 1;
    while (2 * p.slots <= kMaxSlots && 2 * p.slots * p.slot_bytes <= ring_per_warp) p.slots *= 2;
    p.ring_bytes_per_warp = p.slots * p.slot_bytes;
    const int list_bytes = align(p.cta_tokens * 2);
    int ring_bytes = align(kWarps * p.ring_bytes_per_warp);
    // after the scoring the ring region holds the select's candidate
    // segments (head, up to one key per token) and the kept list (tail)
    const int cand_bytes = align(p.cta_tokens * 4);
    if (ring_bytes < list_bytes + cand_bytes) ring_bytes = list_bytes + cand_bytes;
    int keys_bytes = align(std::max(p.cta_tokens * 4, Geom::QSCRATCH_BYTES));
    // the gather stages rows in keys + ring minus the list; the warp partials
    // of the merge go to keys + ring
    const int staged = std::max(Geom::STAGE_BYTES + list_bytes, Geom::WPART_BYTES);
    if (keys_bytes + ring_bytes < staged) keys_bytes = align(staged - ring_bytes);
    int off = 0;
    p.off_keys = off;
    p.keys_bytes = keys_bytes;
    off += keys_bytes;
    p.off_ring = off;
    p.ring_bytes = ring_bytes;
    off += ring_bytes;
    p.off_list = p.off_ring + ring_bytes - list_bytes;
    p.off_qf = off;  // merge weights
    off = align(off + G * kWarps * 4);
    p.off_qhat = off;
    off = align(off + G * D * 4);
    p.off_qs = off;
    off = align(off + D * 4);
    p.off_tbl = off;
    off = align(off + (p.cta_tokens / kBlockTokens) * 4);
    p.off_hist = off;
    off = align(off + 2 * kHistBins * 4);
    p.off_part = off;  // one partial slot per CTA of the cluster (used in rank 0)
    off = align(off + p.C * G * (D + 2) * 4);
    p.off_misc = off;
    off = align(off + 256 * 4);
    p.smem_bytes = off;
}

// The layout with the deepest key-index ring that fits in shared memory.
template <typename T, int D, int G>
bool sparse_layout_fit(SparseParams& p, int max_seq_len, int smem_optin) {
    for (int ring_per_warp : {8192, 6144, 4096, 2048}) {
        sparse_layout<T, D, G>(p, max_seq_len, ring_per_warp);
        if (p.smem_bytes <= smem_optin) return true;
    }
    return false;
}

// A CTA's fixed cost (launch share, prologue, select, merge) in units of the
// time it takes to stream one 16-token block; measured on B200 at about
// 20 us against 50 ns per block for rank 32.
constexpr int kCtaFixedBlocks = 400;

// Cluster size. The smallest size C0 whose CTAs hold at most kCtaTokenCap
// tokens each and whose layout fits in shared memory; then, among C0 and the
// larger sizes whose layout fits and that keep at least 512 tokens per CTA,
// the one with the least modelled time
//   waves(C) * (kCtaFixedBlocks + blocks per CTA(C)),
// waves(C) = ceil(pairs / resident(C)), where resident(C) is how many
// clusters of C CTAs the GPU holds at once (ties: the smaller C).
// resident(C, smem) returns that count from the device (0: the cluster never
// fits), or -1 when unknown, in which case sms / C stands in for it. Returns
// -1 when no size up to 16 fits.
template <typename T, int D, int G, typename R>
int choose_cluster(SparseParams& p, int max_seq_len, int pairs, int sms, int smem_optin, R&& resident) {
    const int nblk = (max_seq_len + kBlockTokens - 1) / kBlockTokens;
    const int cap_blocks = kCtaTokenCap / kBlockTokens;
    int C0 = std::max(1, (nblk + cap_blocks - 1) / cap_blocks);
    for (;; ++C0) {
        if (C0 > 16) return -1;
        p.C = C0;
        if (sparse_layout_fit<T, D, G>(p, max_seq_len, smem_optin)) break;
    }
    int best = -1;
    int64_t best_cost = 0;
    for (int cand = C0; cand <= 16; ++cand) {
        if (cand > C0 && nblk / cand < 32) break;
        p.C = cand;
        if (!sparse_layout_fit<T, D, G>(p, max_seq_len, smem_optin)) continue;
        int res = resident(cand, p.smem_bytes);
        if (res < 0) res = sms / cand;
        if (res < 1) continue;
        const int64_t waves = (pairs + res - 1) / res;
        const int64_t cost = waves * (kCtaFixedBlocks + (nblk + cand - 1) / cand);
        if (best < 0 || cost < best_cost) {
            best = cand;
            best_cost = cost;
        }
    }
    if (best < 0) return -1;
    p.C = best;
    sparse_layout_fit<T, D, G>(p, max_seq_len, smem_optin);
    return best;
}

template <typename T, int D, int G>
int choose_cluster(SparseParams& p, int max_seq_len, int pairs, int sms, int smem_optin) {
    return choose_cluster<T, D, G>(p, max_seq_len, pairs, sms, smem_optin, [](int, int) { return -1; });
}

// Clusters of `cluster` CTAs of this kernel with `smem` bytes of shared
// memory each that the current device holds at once, cached per device,
// cluster size and shared-memory size (0 when none fits or the query fails).
template <typename K>
int resident_clusters(K kern, int cluster, int smem, std::map<std::tuple<int, int, int>, int>& known,
                      std::mutex& mu) {
    int dev = 0;
    cudaGetDevice(&dev);
    const std::tuple<int, int, int> key(dev, cluster, smem);
    std::lock_guard<std::mutex> lock(mu);
    auto it = known.find(key);
    if (it != known.end()) return it->second;
    cudaLaunchConfig_t probe = {};
    probe.gridDim = dim3(cluster, 1, 1);
    probe.blockDim = dim3(kThreads, 1, 1);
    probe.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = cluster;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    probe.attrs = &attr;
    probe.numAttrs = 1;
    int n = 0;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, kern, &probe);
    if (e != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    known[key] = n;
    return n;
}

// Whether the decode kernel has a cluster size and layout for this shape
// (checked before anything of a call is launched).
template <typename T, int D, int G>
struct SparseFits {
    static loki_status run(int r, int pairs, int max_seq_len, const DeviceInfo& di) {
        SparseParams p = {};
        p.r = r;
        return choose_cluster<T, D, G>(p, max_seq_len, pairs, di.sms, di.max_smem_optin) < 1 ? LOKI_ERR_UNSUPPORTED
                                                                                           : LOKI_OK;
    }
};

template <typename T, int D, int G>
struct SparseLaunch {
    // scorer: kScoreLeading, kScoreMagnitude, kScoreSlabs or kScoreAsym
    static loki_status run(SparseParams p, int pairs, int max_seq_len, const DeviceInfo& di,
                           cudaStream_t stream, bool programmatic, int scorer) {
        switch (scorer) {
            case kScoreMagnitude: return run_kernel<kScoreMagnitude>(p, pairs, max_seq_len, di, stream, programmatic);
            case kScoreSlabs: return run_kernel<kScoreSlabs>(p, pairs, max_seq_len, di, stream, programmatic);
            case kScoreAsym: return run_kernel<kScoreAsym>(p, pairs, max_seq_len, di, stream, programmatic);
            default: return run_kernel<kScoreLeading>(p, pairs, max_seq_len, di, stream, programmatic);
        }
    }

    template <int SC>
    static loki_status run_kernel(SparseParams p, int pairs, int max_seq_len, const DeviceInfo& di,
                                  cudaStream_t stream, bool programmatic) {
        auto kern = sparse_decode_kernel<T, D, G, SC>;
        // per device: the shared-memory opt-in and non-portable cluster sizes
        // (both before the residency queries of the cluster choice)
        if (ensure_smem_attr((const void*)kern, di.max_smem_optin) != cudaSuccess) return LOKI_ERR_CUDA;
        {
            static std::mutex mu;
            static std::map<int, cudaError_t> cluster_attr;
            int dev = 0;
            cudaGetDevice(&dev);
            std::lock_guard<std::mutex> lock(mu);
            auto it = cluster_attr.find(dev);
            if (it == cluster_attr.end()) {
                cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
                if (e != cudaSuccess) cudaGetLastError();
                it = cluster_attr.emplace(dev, e).first;
            }
            if (it->second != cudaSuccess) return LOKI_ERR_CUDA;
        }
        static std::map<std::tuple<int, int, int>, int> resident;
        static std::mutex resident_mu;
        auto res = [&](int c, int smem) { return resident_clusters(kern, c, smem, resident, resident_mu); };
        if (choose_cluster<T, D, G>(p, max_seq_len, pairs, di.sms, di.max_smem_optin, res) < 1)
            return LOKI_ERR_UNSUPPORTED;
        // several waves of clusters: longest sequences first
        p.longest_first = p.batch > 1 && p.batch <= 64 && pairs > res(p.C, p.smem_bytes) ? 1 : 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(p.C, pairs, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = p.smem_bytes;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = p.C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        // programmatic dependent of the previous kernel in the stream (the
        // step's append): the kernel calls griddep_wait() before it reads
        // anything that kernel writes
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = programmatic ? 2 : 1;
        // a cluster that can never be resident is reported, not launched
        if (res(p.C, p.smem_bytes) < 1) return LOKI_ERR_UNSUPPORTED;
        if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) {
            cudaGetLastError();  // reported here, not by a later call
            return LOKI_ERR_CUDA;
        }
        return LOKI_OK;
    }
};

}  // namespace loki
