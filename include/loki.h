/*
 * loki.h - C ABI of libloki.so: Loki-style low-rank-key sparse decode
 * attention on NVIDIA B200 (sm_100a).
 *
 * The method (Loki page, "Loki: Low-rank Keys for Efficient Sparse Attention",
 * abstract; AQUA page, related work on LoKi): keys are kept in the cache in a
 * PCA basis, K~ = K P. At a decode step the query is rotated into the same
 * basis, every cached token is scored with only the leading r rotated
 * dimensions, the k best tokens are kept (plus a fixed window of the most
 * recent tokens, as in the LRQK abstract on the aitopics page "low rank
 * approximation"), and exact softmax attention over the full head dimension
 * runs on just those tokens (AQUA page, decode-step equations (3)-(5)).
 *
 * Conventions for every call:
 *  - Ownership: the caller owns every buffer. The library never allocates
 *    device memory and never synchronises a stream inside these calls
 *    (loki_device_error is the one synchronous call).
 *  - Pointers: every data pointer is a DEVICE pointer on the current CUDA
 *    device (cudaMalloc, or the allocator of a framework). The loki_cache and
 *    loki_batch structs themselves are host structs that the call reads
 *    before it returns.
 *  - Execution: launches are asynchronous and ordered on `stream` (a
 *    cudaStream_t passed as void*; NULL is the legacy default stream).
 *  - Errors: arguments are validated on the host before any launch; a failed
 *    check returns a status and launches nothing. A launch failure returns
 *    LOKI_ERR_CUDA. Values that only the device can see (sequence lengths,
 *    block ids, per-sequence k) are checked by the kernels: an out-of-range
 *    value is clamped into range, so memory accesses stay in bounds, and a
 *    bit is set in the device error word that loki_device_error reads.
 *  - Row-vector convention throughout: x_hat = x P, P row-major [d][d].
 *  - Thread safety: calls on different streams may run concurrently.
 */
#ifndef LOKI_H
#define LOKI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LOKI_API __attribute__((visibility("default")))
#else
#define LOKI_API
#endif

#define LOKI_ABI_VERSION 5
#define LOKI_BLOCK_TOKENS 16 /* tokens per paged-cache block */

typedef void* loki_stream_t; /* a cudaStream_t */

typedef enum loki_status {
    LOKI_OK = 0,
    LOKI_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent sizes */
    LOKI_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels implement */
    LOKI_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
    LOKI_ERR_CUDA = 4         /* a CUDA runtime call or launch failed */
} loki_status;

typedef enum loki_dtype {
    LOKI_F32 = 0, /* binary32 cache, queries and new keys */
    LOKI_BF16 = 1 /* bfloat16 cache, queries and new keys */
} loki_dtype;

/* How the g query heads that share a kv head combine their approximate
 * scores into the one score that ranks a token for that kv head. The pages
 * are silent on grouped-query attention; SUM is the default reading (it
 * equals scoring with the sum of the group's rotated queries), MAX the
 * alternative. For g = 1 both are the same. */
typedef enum loki_group_reduce {
    LOKI_GROUP_SUM = 0,
    LOKI_GROUP_MAX = 1
} loki_group_reduce;

/* Which r index dims the approximate score uses (loki_decode_attention_scored).
 * LEADING: the leading r dims, a static slice after the projection (Loki page,
 * abstract; AQUA page, related work on LoKi).
 * MAGNITUDE: per (sequence, kv head) and step, the r single index dims of
 * largest magnitude of the query that ranks the tokens (AQUA page, Algorithm 1
 * in prose and appendix on complexity, steps 2-4: the top dims of |q_hat|, the
 * key cache sliced to those columns). Each chosen dim of a 16-token block is
 * one 16-element run of the dim-major key index.
 * MAGNITUDE_SLABS: a coarser variant that picks the r/16 slabs of 16
 * consecutive index dims with the most energy of that query (whole 16-dim
 * runs; not the pages' algorithm, kept for comparison). */
typedef enum loki_scorer {
    LOKI_SCORER_LEADING = 0,
    LOKI_SCORER_MAGNITUDE = 1,
    LOKI_SCORER_MAGNITUDE_SLABS = 2
} loki_scorer;

/* Device error word bits (loki_device_error). */
#define LOKI_DEVERR_SEQ_LEN 0x1u  /* a seq_lens entry outside [0, max_seq_len] */
#define LOKI_DEVERR_BLOCK_ID 0x2u /* a block-table entry outside [0, num_blocks) */
#define LOKI_DEVERR_K 0x4u        /* a k_per_seq entry outside [0, k] */
#define LOKI_DEVERR_TIMEOUT 0x8u  /* a bounded wait (tensor-core completion) gave up */

/* Paged KV cache in the library's own layout (LOKI_BLOCK_TOKENS tokens per
 * block), plus a low-rank key index. Physical block p of kv head h holds:
 *   keys (PCA basis)  [16 tokens][head_dim]  at element (p*Hkv + h)*16*head_dim
 *   values            [16 tokens][head_dim]  at element (p*Hkv + h)*16*head_dim
 *   key index         [index_dims][16 tokens]  at element (p*Hkv + h)*16*index_dims
 * The key index repeats the leading index_dims rotated dims of every key,
 * dim-major: element (c, t) of a block is at c*16 + t. The leading r <=
 * index_dims dims of a block are one contiguous run of r*16 elements, which is
 * what rank-r scoring streams, and any single dim of a block is one run of 16
 * elements (32 bytes in bf16), which is what the magnitude scorer reads; the
 * key rows stay whole (one contiguous row per token) for the exact attention
 * over the kept tokens. The index costs index_dims/head_dim of the key cache
 * (12.5% of keys + values for index_dims = 32, head_dim = 128). */
typedef struct loki_cache {
    void* k_cache;         /* device, loki_cache_bytes(), 16-byte aligned; not */
    void* v_cache;         /* NULL, even when every block is offloaded        */
    void* k_index;         /* device, loki_index_bytes(), 16-byte aligned */
    int32_t num_blocks;    /* physical blocks in each cache */
    int32_t num_kv_heads;  /* >= 1 */
    int32_t head_dim;      /* 64 or 128 */
    int32_t index_dims;    /* multiple of 16 in [16, head_dim]; the largest usable r */
    loki_dtype dtype;
    /* Optional offload of key and value rows to host memory (LRQK page,
     * abstract: a mixed GPU-CPU cache in which only the missing full-precision
     * rows of the kept tokens cross to the GPU). With kv_home NULL the fields
     * below except kv_touch are ignored, and block p's key and value rows are
     * device page p (k_cache and v_cache hold num_blocks pages). With kv_home
     * set, block p's rows are
     *   kv_home[p] >= 0: device page kv_home[p]; k_cache and v_cache hold
     *                    num_device_pages pages (loki_cache_bytes(
     *                    num_device_pages, ...) bytes each);
     *   kv_home[p] < 0:  host page -(kv_home[p] + 1) of k_host and v_host,
     *                    num_host_pages pages each in the same page layout.
     * A page holds one block's rows of every kv head (the layout above with p
     * the page number). The key index stays on the device whatever kv_home
     * says. Every call reads and writes offloaded rows in place through the
     * host pools' device mapping; a sparse decode reads only the kept rows of
     * offloaded blocks. An entry outside its pool sets LOKI_DEVERR_BLOCK_ID and
     * its rows read as zero and are not written. */
    const int32_t* kv_home;    /* device [num_blocks], or NULL */
    void* k_host;              /* device address (loki_host_device_pointer) of  */
    void* v_host;              /* pinned host memory, 16-byte aligned           */
    int32_t num_device_pages;  /* with kv_home: pages in k_cache and v_cache, >= 0 */
    int32_t num_host_pages;    /* with kv_home: pages in k_host and v_host, >= 0 */
    uint32_t* kv_touch;        /* nullable, device [num_blocks]: every sparse
                                  decode adds to entry p the number of kept rows
                                  it gathered from block p (over all kv heads);
                                  the offload planner's hit counts */
} loki_cache;

/* Per-sequence addressing of one decode batch. */
typedef struct loki_batch {
    const int32_t* block_table; /* device [batch][max_blocks_per_seq]: physical block
                                   of each 16-token logical block */
    const int32_t* seq_lens;    /* device [batch]: tokens in the cache per sequence,
                                   including the current token once appended */
    int32_t batch;              /* >= 0; 0 makes every call a no-op */
    int32_t max_blocks_per_seq; /* row length of block_table */
    int32_t max_seq_len;        /* host-known bound on every seq_lens entry;
                                   <= 16 * max_blocks_per_seq */
} loki_batch;

/* Bytes of EACH of k_cache and v_cache for the given shape; 0 for an invalid
 * shape. */
LOKI_API size_t loki_cache_bytes(int32_t num_blocks, int32_t num_kv_heads, int32_t head_dim,
                                 loki_dtype dtype);

/* Bytes of k_index for the given shape; 0 for an invalid shape. */
LOKI_API size_t loki_index_bytes(int32_t num_blocks, int32_t num_kv_heads, int32_t index_dims,
                                 loki_dtype dtype);

/* Prefill: write tokens [0, seq_lens[b]) of every sequence into the cache
 * (key rows, value rows and the key index).
 *
 * k_rot, v: device [batch][num_kv_heads][max_len][head_dim] in the cache type,
 * row-major, 16-byte aligned; max_len >= max_seq_len. The keys must already be
 * in the PCA basis (for example because P was folded into the key projection
 * weights); this call only lays rows out, it does no arithmetic. Tokens past
 * seq_lens[b] are not read. */
LOKI_API loki_status loki_prefill_cache(const loki_cache* cache, const loki_batch* batch,
                               const void* k_rot, const void* v, int32_t max_len,
                               loki_stream_t stream);

/* Prefill with the rotation on the GPU (AQUA page, appendix on complexity,
 * step 1, and the information-retention paragraph: keys are projected with P
 * as row vectors): for every sequence b, kv head h and token t < seq_lens[b],
 *   K~[b, h, t, :] = round(k[b, h, t, :] P[h]),  V[b, h, t, :] = v[b, h, t, :]
 * written as loki_prefill_cache lays rows out (key rows, value rows, key
 * index).
 *
 * k, v: device [batch][num_kv_heads][max_len][head_dim] in the cache type,
 * unrotated keys and values, 16-byte aligned; max_len >= max_seq_len.
 * P: device fp32 [num_kv_heads][head_dim][head_dim], row-major, 16-byte
 * aligned.
 * Precision: fp32 caches sum fp32 products in fp32, as loki_append_keys does.
 * bf16 caches run the product on the tensor cores with P split into two bf16
 * terms (P = P_hi + P_lo) and fp32 accumulation, i.e. about 16 significant
 * bits of P, then round to nearest even: the stored key equals the exactly
 * rounded product except where that product lies within about 2^-15 of its
 * magnitude from a rounding midpoint, where it may be the other neighbour.
 * Tokens past seq_lens[b] are not read. The key index gets the leading
 * index_dims of every rotated key. */
LOKI_API loki_status loki_prefill_rotate(const loki_cache* cache, const loki_batch* batch,
                                const void* k, const void* v, const float* P, int32_t max_len,
                                loki_stream_t stream);

/* Offline calibration of P (AQUA page, appendix on SVD: the leading columns
 * of the basis carry the most variance; Fig. 2: P calibrated once on
 * calibration keys): for every head h, the eigenvectors of the centred
 * covariance C = (1/n) sum_t (x_t - mu)^T (x_t - mu) of its n calibration
 * keys, as the columns of P[h] in descending eigenvalue order (ties to the
 * lower index), each column's sign chosen so that its entry of largest
 * magnitude is positive.
 *
 * keys: device [num_heads][n][head_dim] in `dtype`, original basis.
 * P: device fp32 [num_heads][head_dim][head_dim], row-major (written).
 * eigvals: nullable device fp32 [num_heads][head_dim] (written, descending).
 * Arithmetic: fp32 (covariance sums, cyclic Jacobi rotations until every
 * off-diagonal entry is below 2^-22 of the largest diagonal one); directions
 * of clustered eigenvalues are defined only up to rotations within the
 * cluster. n >= 2. No counterpart call in the pages: it is their offline
 * calibration step done on the device. */
/* Key index of an asymmetric score factorisation (SAKI page, abstract: the
 * score q k^T approximated as (q A_q)(k A_k)^T with rank-r factors from the
 * SVD of the covariance-weighted query-key operator), for every cached
 * token: index[b, h, t, c] = round(sum_i k[b, h, t, i] A_k[h][i][c]) for
 * c < index_dims (fp32 sums in row order i = 0, 1, ..., round to nearest
 * even to the cache type). The key and value rows are not touched.
 *
 * k: device [batch][num_kv_heads][max_len][head_dim] in the cache type, keys
 *    in the original basis (row t of sequence b, head h at
 *    ((b * num_kv_heads + h) * max_len + t) * head_dim).
 * A_k: device fp32 [num_kv_heads][head_dim][index_dims], row-major, 16-byte
 *    aligned. Computing A_k (and A_q) from calibration samples is the
 *    caller's offline step. max_len >= max_seq_len. */
LOKI_API loki_status loki_index_keys(const loki_cache* cache, const loki_batch* batch, const void* k,
                            const float* A_k, int32_t max_len, loki_stream_t stream);

LOKI_API loki_status loki_pca_basis(const void* keys, int32_t num_heads, int64_t n, int32_t head_dim,
                           loki_dtype dtype, float* P, float* eigvals, loki_stream_t stream);

/* Cache update of one decode step (AQUA page, decode-step equations (1)-(2),
 * for keys kept in the PCA basis): for every sequence b and kv head h,
 *   K~[b, h, seq_lens[b]-1, :] = round(k_new[b, h, :] P[h])   (fp32 accumulation,
 *                                round-to-nearest-even to the cache type),
 *                                its leading index_dims also into the key index
 *   V [b, h, seq_lens[b]-1, :] = v_new[b, h, :]
 * so seq_lens must already count the new token. Sequences with seq_lens[b] = 0
 * are skipped.
 *
 * k_new, v_new: device [batch][num_kv_heads][head_dim] in the cache type.
 * P: device fp32 [num_kv_heads][head_dim][head_dim], row-major, 16-byte
 * aligned; NULL means the keys are already in the PCA basis (copied as is). */
LOKI_API loki_status loki_append_keys(const loki_cache* cache, const loki_batch* batch,
                             const void* k_new, const void* v_new, const float* P,
                             loki_stream_t stream);

/* loki_append_keys for a cache whose key index holds k A_k (see
 * loki_index_keys): the key and value rows as loki_append_keys writes them,
 * the index row round(k_new A_k[h]) with the sums of loki_index_keys, so the
 * two give identical rows for the same key. A_k: device fp32
 * [num_kv_heads][head_dim][index_dims], 16-byte aligned (NULL is
 * LOKI_ERR_INVALID_ARG). */
LOKI_API loki_status loki_append_keys_asym(const loki_cache* cache, const loki_batch* batch,
                                  const void* k_new, const void* v_new, const float* P,
                                  const float* A_k, loki_stream_t stream);

/* Workspace bytes loki_decode_attention needs for these sizes (may be 0). */
LOKI_API size_t loki_decode_workspace_bytes(const loki_cache* cache, const loki_batch* batch,
                                   int32_t num_q_heads, int32_t k, int32_t recent_window);

/* One Loki sparse decode step for every sequence b and query head j, with
 * kv head h = j / g (g = num_q_heads / num_kv_heads, contiguous groups) and
 * L = seq_lens[b]:
 *   1. q_hat_j = q_j P[h]                                (fp32)
 *   2. candidates t in [0, L - W'), W' = min(recent_window, L); approximate
 *      score s_t = reduce_{j in group(h)} q_hat_j[:r] . K~[t, :r]
 *      (AQUA page, related work on LoKi: slicing after projection; Loki
 *      abstract: scores in the low-dimensional space; reduce = SUM or MAX)
 *   3. keep the min(k_b, candidates) largest s_t, ties to the lower t, plus
 *      the W' most recent tokens (aitopics page, LRQK abstract)
 *   4. out_j = softmax over the kept set of (q_hat_j . K~[t, :] * scale) times V
 *      (AQUA page, decode-step equations (3)-(5)), fp32.
 *
 * q: device [batch][num_q_heads][head_dim] in the cache type, unrotated,
 *    16-byte aligned.
 * P: device fp32 [num_kv_heads][head_dim][head_dim], 16-byte aligned.
 * r: leading dimensions used for scoring; a multiple of 16 in [16, index_dims]
 *    (r > index_dims is LOKI_ERR_INVALID_ARG).
 * k: tokens kept by score (the per-sequence maximum when k_per_seq is given).
 * k_per_seq: nullable device int32 [batch]; entries clamped to [0, k].
 * recent_window: W >= 0; k = 0 together with W = 0 is invalid.
 * scale: exact-logit scale; 0 means 1/sqrt(head_dim).
 * out: device fp32 [batch][num_q_heads][head_dim].
 * selected_idx: nullable device int32 [batch][num_kv_heads][k + recent_window]:
 *   the kept token indices of each (sequence, kv head) in ascending order,
 *   then -1 padding.
 * workspace: device, >= loki_decode_workspace_bytes(); may be NULL if that is 0.
 *
 * Unsupported (LOKI_ERR_UNSUPPORTED): head_dim other than 64/128, group size
 * other than 1, 2, 4, 8, r not a multiple of 16, max_seq_len above
 * loki_decode_max_seq_len(), or a long sequence whose per-CTA state does not
 * fit in shared memory for any cluster size (only above 16384 tokens, for
 * some combinations of group size, cache type and head_dim; group size 8 is
 * the most limited). All of these are found before anything is launched. */
LOKI_API loki_status loki_decode_attention(const loki_cache* cache, const loki_batch* batch,
                                  const void* q, int32_t num_q_heads, const float* P,
                                  int32_t r, int32_t k, const int32_t* k_per_seq,
                                  int32_t recent_window, loki_group_reduce group_reduce,
                                  float scale, float* out, int32_t* selected_idx,
                                  void* workspace, size_t workspace_bytes,
                                  loki_stream_t stream);

/* loki_decode_attention with a choice of scorer; LOKI_SCORER_LEADING gives
 * the same results as loki_decode_attention. Otherwise step 2 scores with a
 * set S of r index dims chosen per (sequence, kv head) and step among the
 * first index_dims (fp32, with u = sum_{j in group(h)} q_hat_j):
 *   LOKI_SCORER_MAGNITUDE (AQUA page, Algorithm 1 in prose; appendix on
 *     complexity, steps 2-4): the r dims c of largest |u[c]| (SUM) or of
 *     largest sum_j q_hat_j[c]^2 (MAX), ties to the lower dim;
 *   LOKI_SCORER_MAGNITUDE_SLABS: the r/16 slabs s (16 consecutive dims) of
 *     largest sum_{c in s} u[c]^2 (SUM) or sum_j sum_{c in s} q_hat_j[c]^2
 *     (MAX), ties to the lower slab;
 * and s_t = reduce_j sum_{c in S, ascending} q_hat_j[c] K~[t, c]. Steps 1, 3
 * and 4 are unchanged. The bytes read per candidate token are the same r
 * index elements as the leading scorer's; the index must hold the dims to
 * choose from. Arguments as for loki_decode_attention; an unknown scorer is
 * LOKI_ERR_INVALID_ARG. */
LOKI_API loki_status loki_decode_attention_scored(const loki_cache* cache, const loki_batch* batch,
                                         const void* q, int32_t num_q_heads, const float* P,
                                         int32_t r, int32_t k, const int32_t* k_per_seq,
                                         int32_t recent_window, loki_group_reduce group_reduce,
                                         float scale, loki_scorer scorer, float* out,
                                         int32_t* selected_idx, void* workspace,
                                         size_t workspace_bytes, loki_stream_t stream);

/* loki_decode_attention for a key index that holds k A_k (loki_index_keys,
 * loki_append_keys_asym): step 2 scores with the query factor instead,
 *   s_t = reduce_{j in group(h)} (q_j A_q[h])[:r] . index[t, :r]   (fp32),
 * where q_j A_q[h] is summed in the same order as q_hat (SAKI page, abstract:
 * asymmetric query and key factors of the score operator). Steps 1, 3 and 4
 * are unchanged: the exact attention uses q_hat = q P against the full keys.
 * A_q: device fp32 [num_kv_heads][head_dim][index_dims], 16-byte aligned;
 * its first r columns are used. Other arguments as for
 * loki_decode_attention. */
LOKI_API loki_status loki_decode_attention_asym(const loki_cache* cache, const loki_batch* batch,
                                       const void* q, int32_t num_q_heads, const float* P,
                                       const float* A_q, int32_t r, int32_t k,
                                       const int32_t* k_per_seq, int32_t recent_window,
                                       loki_group_reduce group_reduce, float scale, float* out,
                                       int32_t* selected_idx, void* workspace,
                                       size_t workspace_bytes, loki_stream_t stream);

/* One whole decode step: loki_append_keys(k_new, v_new, P) followed by
 * loki_decode_attention(...) on the same stream, with the same arguments and
 * the same results as those two calls (seq_lens already counts the new
 * token). The attention kernel is launched as a programmatic dependent of the
 * append kernel: it starts while the append runs and waits for it only
 * before it first reads the appended token (before the exact attention when
 * recent_window >= 1, before the scoring otherwise). Every argument is checked
 * before anything is launched; an error launches nothing. This entry point has
 * no counterpart in the pages: it packages their per-step cache update and
 * attention as one call. */
LOKI_API loki_status loki_decode_step(const loki_cache* cache, const loki_batch* batch,
                             const void* k_new, const void* v_new,
                             const void* q, int32_t num_q_heads, const float* P,
                             int32_t r, int32_t k, const int32_t* k_per_seq,
                             int32_t recent_window, loki_group_reduce group_reduce,
                             float scale, float* out, int32_t* selected_idx,
                             void* workspace, size_t workspace_bytes,
                             loki_stream_t stream);

/* Bytes of the device staging buffer loki_decode_step_host needs for these
 * sizes: the step's k_new, v_new and q (cache dtype) and its output (fp32),
 * each region 256-byte aligned; 0 for invalid arguments. */
LOKI_API size_t loki_decode_step_host_bytes(const loki_cache* cache, const loki_batch* batch,
                                            int32_t num_q_heads);

/* loki_decode_step for a caller that holds the step's inputs and output in
 * host memory: k_new_host, v_new_host ([batch][num_kv_heads][head_dim]) and
 * q_host ([batch][num_q_heads][head_dim]), all in the cache dtype, and
 * out_host ([batch][num_q_heads][head_dim] fp32). The step runs as
 * loki_decode_step with the same remaining arguments (no kept-index export),
 * all on `stream`, in one of two ways:
 *  - all four buffers page-locked and mapped into the device's address space
 *    (cudaHostAlloc / cudaMallocHost memory, or cudaHostRegister'ed memory,
 *    under unified addressing; out_host 4-byte and q_host 16-byte aligned):
 *    the kernels read the inputs and write the output in place over the host
 *    link, and `staging` is not touched;
 *  - otherwise the inputs are copied into `staging` (device,
 *    loki_decode_step_host_bytes bytes, 256-byte aligned) and the output back
 *    from it, one cudaMemcpyAsync per buffer; pageable memory makes those
 *    copies synchronous with the host.
 * `staging` is required either way. With page-locked memory the call is
 * asynchronous: the host buffers must stay untouched, and out_host unread,
 * until the stream has passed the step. Every argument is checked before
 * anything is issued; an error issues nothing. The caller owns every buffer;
 * the library allocates nothing. */
LOKI_API loki_status loki_decode_step_host(const loki_cache* cache, const loki_batch* batch,
                                           const void* k_new_host, const void* v_new_host,
                                           const void* q_host, int32_t num_q_heads, const float* P,
                                           int32_t r, int32_t k, const int32_t* k_per_seq,
                                           int32_t recent_window, loki_group_reduce group_reduce,
                                           float scale, float* out_host, void* staging,
                                           size_t staging_bytes, loki_stream_t stream);

/* Largest max_seq_len loki_decode_attention accepts for this cache shape
 * (262144 tokens). Some group sizes fit less in a CTA's shared memory: for
 * those, longer sequences are rejected with LOKI_ERR_UNSUPPORTED before any
 * launch (bf16: from 131072 tokens at head_dim 64 with group size 8; fp32:
 * from 65536 tokens at head_dim 128 with group size 8; every combination
 * accepts at least 16384 tokens). */
LOKI_API int32_t loki_decode_max_seq_len(int32_t head_dim, loki_dtype dtype);

/* Workspace bytes loki_dense_attention needs for these sizes. */
LOKI_API size_t loki_dense_workspace_bytes(const loki_cache* cache, const loki_batch* batch,
                                  int32_t num_q_heads);

/* Dense decode attention, the full-attention comparison path (AQUA page,
 * decode-step equations (3)-(5) over every cached token):
 *   out_j = softmax over t in [0, L) of (q_hat_j . K~[t, :] * scale) times V
 * with q_hat_j = q_j P[h]; by the rotation invariance of the AQUA page's
 * appendix this equals attention with the unrotated keys.
 * Arguments as for loki_decode_attention. Runs as flash-decode split-K: each
 * split writes (max, sum, unnormalised output) partials to the workspace and a
 * second kernel merges them. */
LOKI_API loki_status loki_dense_attention(const loki_cache* cache, const loki_batch* batch,
                                 const void* q, int32_t num_q_heads, const float* P,
                                 float scale, float* out, void* workspace,
                                 size_t workspace_bytes, loki_stream_t stream);

/* Size of the scratch array built into the library for
 * loki_dense_attention_static (16 MiB). */
#define LOKI_DENSE_STATIC_SCRATCH_BYTES (16u << 20)

/* loki_dense_attention for callers that cannot allocate device memory: a
 * serving engine that hands all device memory to its own arena at start-up,
 * a plugin host that exposes no allocator, or code that must not call
 * cudaMalloc because it can synchronise the device. This is an addition of
 * the library, not a step of the method, so no page has a counterpart.
 *
 * Same arguments and result as loki_dense_attention, without the workspace:
 * the split partials go to a scratch array inside the library
 * (LOKI_DENSE_STATIC_SCRATCH_BYTES; every GPU that loads the library holds it
 * until the process exits). The call allocates nothing.
 *  - Sizes whose loki_dense_workspace_bytes exceeds the array are rejected
 *    with LOKI_ERR_WORKSPACE before anything is launched.
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current); make that first call before any
 *    stream capture on the device.
 *  - All calls on a device share the one array, which keeps the last call's
 *    contents (every value a call reads it writes first, so nothing needs
 *    clearing). Calls whose executions overlap on the GPU (different streams
 *    without ordering) race on the array and must not be issued that way. */
LOKI_API loki_status loki_dense_attention_static(const loki_cache* cache, const loki_batch* batch,
                                                 const void* q, int32_t num_q_heads, const float* P,
                                                 float scale, float* out, loki_stream_t stream);

/* ------------------------------------------------------------------------
 * Host offload of key and value pages (LRQK page, abstract: the hit-and-miss
 * mechanism of a mixed GPU-CPU cache). Blocks whose rows the decodes keep
 * selecting are promoted to device pages and the least selected device blocks
 * take their place on the host, between decode steps.
 * ------------------------------------------------------------------------ */

/* One swap: block_in (offloaded, in host page host_page) moves to the free
 * device page device_page; block_out (on the device, in device page
 * freed_page) moves to host_page; freed_page is then the free device page. */
typedef struct loki_page_move {
    int32_t block_in;
    int32_t block_out;
    int32_t host_page;
    int32_t device_page;
    int32_t freed_page;
} loki_page_move;

/* Host-only planning of swaps (no CUDA call). kv_home is a host copy of the
 * cache's map [num_blocks] and spare_page the one device page no block uses;
 * touch is a host copy of kv_touch. Offloaded blocks in order of decreasing
 * touch count (ties: lower block id) are paired with device blocks in order of
 * increasing touch count (ties: lower block id); a pair is swapped while the
 * offloaded block's count is strictly the larger, at most max_moves swaps.
 * Writes the swaps to moves, updates kv_home and spare_page to the state after
 * them and returns their number, or -1 for invalid arguments (a NULL pointer,
 * num_blocks < 0, max_moves < 0, spare_page < 0 or used by a block). */
LOKI_API int32_t loki_offload_plan(int32_t num_blocks, int32_t* kv_home, int32_t* spare_page,
                                   const uint32_t* touch, int32_t max_moves, loki_page_move* moves);

/* Issues the swaps on the stream, in order: per move, block_in's key page and
 * value page host -> device_page, then block_out's key and value pages
 * freed_page -> host_page (one cudaMemcpyAsync per page); then the updated map
 * kv_home_host [num_blocks] -> cache->kv_home. Stream-ordered with the calls
 * before and after it on the stream. A pinned kv_home_host must stay unchanged
 * until the stream has passed the copy; a pageable one may change once the
 * call returns. Page and block numbers outside their pools give
 * LOKI_ERR_INVALID_ARG before anything is issued. */
LOKI_API loki_status loki_offload_apply(const loki_cache* cache, const loki_page_move* moves, int32_t num_moves,
                                        const int32_t* kv_home_host, loki_stream_t stream);

/* The device address of pinned host memory (cudaHostAlloc'd or registered
 * mapped); LOKI_ERR_CUDA if the memory is not mapped for the device. */
LOKI_API loki_status loki_host_device_pointer(void* host, void** device);

/* Reads (and with clear != 0 resets) the device error word of the current
 * device: an OR of LOKI_DEVERR_* bits set by kernels since the last clear.
 * Synchronises the device. */
LOKI_API loki_status loki_device_error(int32_t clear, uint32_t* bits);

/* Static description of a status code. */
LOKI_API const char* loki_status_string(loki_status status);

/* LOKI_ABI_VERSION of the loaded library. */
LOKI_API int32_t loki_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LOKI_H */
