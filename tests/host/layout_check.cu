// Host-side check of the decode kernel's launch geometry (no GPU needed):
// for every cache type, head dim, group size, rank, sequence length and pair
// count, the cluster size and shared-memory layout chosen by choose_cluster /
// sparse_layout must satisfy the invariants the kernel relies on, or the shape
// must be reported unsupported (choose_cluster < 1; the library then returns
// LOKI_ERR_UNSUPPORTED before launching anything). Every sequence of up to
// kCtaTokenCap tokens must be supported. Prints one line per violation, the
// shortest unsupported length per (type, head dim, group), and
// "layout ok <cases>" at the end; exits 1 on any violation.
#include <cstdio>
#include <cstdlib>

#include "cache_kernels.cuh"
#include "dense.cuh"
#include "pca.cuh"
#include "rotate_prefill.cuh"
#include "sparse_launch.cuh"

using namespace loki;

static int failures = 0;
static long cases = 0;

#define CHECK(cond)                                                                                          \
    do {                                                                                                     \
        if (!(cond)) {                                                                                       \
            if (failures < 50)                                                                               \
                std::printf("FAIL %s: T=%s D=%d G=%d L=%d pairs=%d C=%d\n", #cond, tname, D, G, L, pairs, \
                            p.C);                                                                            \
            ++failures;                                                                                      \
        }                                                                                                    \
    } while (0)

template <typename T, int D, int G>
void check(const char* tname, int sms, int optin) {
    using Geom = SparseGeom<T, D, G>;
    const int lens[] = {1, 15, 16, 17, 300, 1000, 4096, 16384, 16385, 32768, 65536, 100000, 131072, 262144};
    const int pair_counts[] = {1, 2, 8, 64, 74, 148, 1000, 65535};
    int shortest_unsupported = 1 << 30;
    for (int L : lens)
        for (int pairs : pair_counts)
            for (int r = 16; r <= D; r += 16) {
                ++cases;
                SparseParams p = {};
                p.r = r;
                const int C = choose_cluster<T, D, G>(p, L, pairs, sms, optin);
                if (C < 1) {
                    CHECK(L > kCtaTokenCap);
                    if (L < shortest_unsupported) shortest_unsupported = L;
                    continue;
                }
                CHECK(C <= 16);
                CHECK(p.C == C);
                // token ranges: whole blocks, every token covered, no CTA wholly past the end
                CHECK(p.cta_tokens % kBlockTokens == 0);
                CHECK((long)p.C * p.cta_tokens >= L);
                CHECK((long)(p.C - 1) * p.cta_tokens < ((L + kBlockTokens - 1) / kBlockTokens) * kBlockTokens);
                CHECK(p.cta_tokens <= kCtaTokenCap);
                // the ring: a power of two of whole slots
                CHECK(p.slots >= 1 && p.slots <= kMaxSlots && (p.slots & (p.slots - 1)) == 0);
                CHECK(kMaxSlots % p.slots == 0);
                CHECK(p.slot_bytes == r * kBlockTokens * (int)sizeof(T));
                CHECK(p.ring_bytes_per_warp == p.slots * p.slot_bytes);
                CHECK(p.ring_bytes >= kWarps * p.ring_bytes_per_warp);
                // regions in order, 128-byte aligned, inside the dynamic shared memory
                const int offs[] = {p.off_keys, p.off_ring, p.off_qf, p.off_qhat, p.off_qs,
                                    p.off_tbl, p.off_hist, p.off_part, p.off_misc, p.smem_bytes};
                for (int i = 0; i + 1 < 10; ++i) CHECK(offs[i] < offs[i + 1]);
                for (int i = 0; i < 10; ++i) CHECK(offs[i] % 128 == 0);
                CHECK(p.off_keys == 0 && p.off_ring == p.off_keys + p.keys_bytes);
                CHECK(p.smem_bytes <= optin);
                // sizes of the regions the kernel indexes
                const int list_bytes = p.off_ring + p.ring_bytes - p.off_list;
                CHECK(list_bytes >= p.cta_tokens * 2);
                CHECK(p.off_list % 16 == 0);
                CHECK(p.off_ring + p.ring_bytes - list_bytes - p.off_ring >= p.cta_tokens * 4);  // candidates
                CHECK(p.keys_bytes >= p.cta_tokens * 4);                                            // keys
                CHECK(p.keys_bytes >= Geom::QSCRATCH_BYTES);                                        // q scratch
                CHECK(p.off_list - p.off_keys >= Geom::STAGE_BYTES);                                // gather staging
                CHECK(p.keys_bytes + p.ring_bytes >= Geom::WPART_BYTES);                            // warp partials
                CHECK(p.off_qhat - p.off_qf >= G * kWarps * 4);
                CHECK(p.off_qs - p.off_qhat >= G * D * 4);
                CHECK(p.off_tbl - p.off_qs >= D * 4);
                CHECK(p.off_hist - p.off_tbl >= (p.cta_tokens / kBlockTokens) * 4);
                CHECK(p.off_part - p.off_hist >= 2 * kHistBins * 4);
                CHECK(p.off_misc - p.off_part >= p.C * G * (D + 2) * 4);
                CHECK(p.off_misc - p.off_part >= G * D * 4);  // the asymmetric scorer's query
                CHECK(p.smem_bytes - p.off_misc >= 256 * 4);  // misc words, then the chosen dims
                CHECK(kSelDims + D <= 256);
                // spread: a cluster larger than needed only where it shortens the
                // modelled time (waves of resident clusters, sms / C of them, times
                // the blocks of one CTA) and keeps 512 tokens per CTA
                SparseParams q = {};
                q.r = r;
                const int cap_blocks = kCtaTokenCap / kBlockTokens;
                const int nblk = (L + kBlockTokens - 1) / kBlockTokens;
                int cmin = std::max(1, (nblk + cap_blocks - 1) / cap_blocks);
                for (; cmin <= 16; ++cmin) {
                    q.C = cmin;
                    if (sparse_layout_fit<T, D, G>(q, L, optin)) break;
                }
                CHECK(C >= cmin);
                if (C > cmin) {
                    auto cost = [&](int c) {
                        const long res = sms / c;
                        return res < 1 ? (1L << 62)
                                       : ((pairs + res - 1) / res) * (long)(kCtaFixedBlocks + (nblk + c - 1) / c);
                    };
                    CHECK(cost(C) < cost(cmin));
                    CHECK(nblk / C >= 32);
                }
            }
    if (shortest_unsupported < (1 << 30))
        std::printf("unsupported from L=%d: T=%s D=%d G=%d\n", shortest_unsupported, tname, D, G);
}

template <typename T, int D>
void check_groups(const char* tname, int sms, int optin) {
    check<T, D, 1>(tname, sms, optin);
    check<T, D, 2>(tname, sms, optin);
    check<T, D, 4>(tname, sms, optin);
    check<T, D, 8>(tname, sms, optin);
}

// The other kernels' fixed shared-memory sizes against the opt-in limit.
template <typename T, int D, int G>
void check_dense(const char* tname, int optin) {
    using Geom = DenseGeom<T, D, G>;
    ++cases;
    if (!(Geom::SMEM_BYTES <= optin && Geom::GS >= 1)) {
        std::printf("FAIL dense T=%s D=%d G=%d smem=%d\n", tname, D, G, Geom::SMEM_BYTES);
        ++failures;
    }
}

template <int D>
void check_fixed(int optin) {
    const int pca_static = 4 * (D / 2) * 4;  // the Jacobi round's rotation table
    const int sizes[] = {rotate_smem_bytes<D>(), pca_smem_bytes<D>() + pca_static};
    const char* names[] = {"rotate_prefill", "pca"};
    for (int i = 0; i < 2; ++i) {
        ++cases;
        if (sizes[i] > optin) {
            std::printf("FAIL %s D=%d smem=%d\n", names[i], D, sizes[i]);
            ++failures;
        }
    }
    for (int I = 16; I <= D; I += 16) {
        ++cases;
        if (index_smem_bytes<D>(I) > optin) {
            std::printf("FAIL index_keys D=%d I=%d smem=%d\n", D, I, index_smem_bytes<D>(I));
            ++failures;
        }
    }
}

int main() {
    const int sms = 148, optin = 227 * 1024;  // B200: SMs, opt-in shared memory per block
    check_dense<__nv_bfloat16, 64, 1>("bf16", optin);
    check_dense<__nv_bfloat16, 64, 2>("bf16", optin);
    check_dense<__nv_bfloat16, 64, 4>("bf16", optin);
    check_dense<__nv_bfloat16, 64, 8>("bf16", optin);
    check_dense<__nv_bfloat16, 128, 1>("bf16", optin);
    check_dense<__nv_bfloat16, 128, 2>("bf16", optin);
    check_dense<__nv_bfloat16, 128, 4>("bf16", optin);
    check_dense<__nv_bfloat16, 128, 8>("bf16", optin);
    check_dense<float, 64, 1>("f32", optin);
    check_dense<float, 64, 2>("f32", optin);
    check_dense<float, 64, 4>("f32", optin);
    check_dense<float, 64, 8>("f32", optin);
    check_dense<float, 128, 1>("f32", optin);
    check_dense<float, 128, 2>("f32", optin);
    check_dense<float, 128, 4>("f32", optin);
    check_dense<float, 128, 8>("f32", optin);
    check_fixed<64>(optin);
    check_fixed<128>(optin);
    check_groups<__nv_bfloat16, 64>("bf16", sms, optin);
    check_groups<__nv_bfloat16, 128>("bf16", sms, optin);
    check_groups<float, 64>("f32", sms, optin);
    check_groups<float, 128>("f32", sms, optin);
    if (failures) {
        std::printf("layout FAILED: %d violations in %ld cases\n", failures, cases);
        return 1;
    }
    std::printf("layout ok %ld\n", cases);
    return 0;
}
