/*
 * csa2.h -- C ABI of the CSA2 global-attention decode path over an FP4 KV cache
 * (libcsa2.so, sm_100a).
 *
 * The method: DeepSeek V4.1 Flash's CSA2 attention as described in
 *   "DeepSeek V4.1 Flash: architecture study notes" (macin.top), sections 1-4, and
 *   "DeepSeek V4.1 Flash goes online" (myzaker), sections "CSA2 attention" and
 *   "cache precision and tiering".
 * Every layer is statically Full, Reindex or Reuse.  A Full layer scans all
 * visible global entries, builds a shared candidate pool of at most 2048 blocks
 * of 8 positions and picks at most 512 entries; a Reindex layer re-scores only
 * inside that pool with its own index query; a Reuse layer takes the most recent
 * selection as is.  Each layer then attends, with its own query, over the
 * selected FP4 entries together with its own 128-token FP8 SWA window.
 *
 * Conventions (all entry points):
 *  - Every pointer is DEVICE memory owned by the caller unless stated otherwise.
 *    The library allocates nothing, keeps no state between calls (apart from
 *    the csa2_debug_set_waits test setting) and is re-entrant; calls on one
 *    stream execute in order.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  The returned status reports host-side validation
 *    (null pointers, sizes, capacities) and launch errors (CSA2_ERR_CUDA).
 *  - Bounds the host cannot see (device-resident positions, indices) are checked
 *    in the kernels: a violating row / index is skipped (a row outside a RoPE
 *    table is stored unrotated) and a CSA2_DEVERR_* bit is OR-ed into `*dev_err`
 *    (an int32 in device memory, may be NULL).  Read it
 *    with csa2_read_device_error().  Kernels never trap; their internal waits
 *    are bounded (0.5 s of wall time) and report CSA2_DEVERR_TIMEOUT.
 *  - Kernels are launched with programmatic dependent launch: each may be
 *    scheduled while the previous kernel of the stream finishes, but waits for it
 *    (completion and memory visibility) before its first global memory access, so
 *    results are stream-ordered exactly as with ordinary launches.  One exception:
 *    the sparse attention calls read the caller's q, q_pos and new SWA row before
 *    that wait (no kernel of this library writes them).  Those three must not be
 *    written by the immediately preceding kernel of the stream if that kernel
 *    itself triggers programmatic launch completion before its writes; ordinary
 *    kernels and copies (which trigger only at completion) are fine.
 *  - bf16 inputs are row-major and contiguous; "B" is the request count, "Tq"
 *    the number of query tokens per request (1 = decode, >1 = prefill chunk).
 *  - Numbers are finite: NaN/Inf inputs are outside the contract.
 */
#ifndef CSA2_H_
#define CSA2_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSA2_API __attribute__((visibility("default")))
#else
#define CSA2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *csa2_stream_t; /* same handle as cudaStream_t */

typedef enum csa2_status {
    CSA2_OK = 0,
    CSA2_ERR_INVALID_ARG = 1,   /* null pointer, bad size or shape */
    CSA2_ERR_CAPACITY = 2,      /* a cache or ring too small for the request */
    CSA2_ERR_WORKSPACE = 3,     /* workspace pointer null or smaller than required */
    CSA2_ERR_UNSUPPORTED = 4,   /* shape outside what the kernels implement */
    CSA2_ERR_CUDA = 5,          /* a CUDA launch or runtime call failed */
    CSA2_ERR_DEVICE_BOUNDS = 6  /* csa2_read_device_error found a device-side bit */
} csa2_status;

/* Device-side error bits OR-ed into *dev_err. */
#define CSA2_DEVERR_SLOT 0x1      /* append slot >= cap */
#define CSA2_DEVERR_INDEX 0x2     /* a Top-K or pool id outside the visible range */
#define CSA2_DEVERR_NMAX 0x4      /* a query sees more entries than n_max */
#define CSA2_DEVERR_RANGE 0x8     /* a dequantised SWA value beyond the fp16 range */
#define CSA2_DEVERR_TIMEOUT 0x10  /* a kernel's bounded wait gave up (internal error, or
                                     the csa2_debug_set_waits test hook) */
#define CSA2_DEVERR_ROPE 0x20     /* a row's position lies outside the RoPE table */
#define CSA2_DEVERR_PAGE 0x40     /* a block table entry names a page outside the pool */

/* Limits of the kernels. */
#define CSA2_KV_DIM 512           /* shared K=V latent width (MQA) */
#define CSA2_GROUP 16             /* channels per E4M3 scale */
#define CSA2_TOPK_MAX 512         /* at most 512 selected entries per query */
#define CSA2_BLOCK 8              /* positions per pool block */
#define CSA2_POOL_MAX 2048        /* at most 2048 pool blocks = 16384 positions */

/*
 * One global-KV group (shared by the Full layer and its Reindex / Reuse layers).
 * Main KV (FP4, study notes section 4: 4-bit E2M1 values, one 8-bit E4M3 scale
 * per 16 channels, 4 + 8/16 = 4.5 bits per value, no second-level scale):
 *   codes   uint8 [batch][cap][256]  two E2M1 codes per byte, even channel in
 *                                    the low nibble
 *   scales  uint8 [batch][cap][32]   E4M3, scale j covers channels 16j..16j+15
 * Indexer K (FP8 E4M3, one fp32 scale per entry; projected from the main KV
 * entry, myzaker "CSA2 attention"):
 *   idx_codes uint8 [batch][cap][d_idx],  idx_scale float [batch][cap]
 * Entry e covers tokens [ratio*e, ratio*e + ratio) (ratio 1 decoder, 2 encoder
 * groups, study notes section 3); the token at position t sees entries
 * 0 .. (t+1)/ratio - 1.
 */
typedef struct csa2_global_kv {
    uint8_t *codes;
    uint8_t *scales;
    uint8_t *idx_codes;
    float *idx_scale;
    int32_t batch;
    int32_t cap;
    int32_t d_idx;   /* 64 or 128 */
    int32_t ratio;   /* 1 or 2 */
} csa2_global_kv;

/*
 * One layer's SWA window (FP8 E4M3 with one fp32 scale per token; study notes
 * sections 1 and 4: a 128-token local window per layer, kept in FP8).
 * Token position p lives in ring slot p % window_cap.
 *   codes uint8 [batch][window_cap][512],  scale float [batch][window_cap]
 */
typedef struct csa2_swa {
    uint8_t *codes;
    float *scale;
    int32_t batch;
    int32_t window_cap;
} csa2_swa;

/*
 * RoPE applied inside the append (the _rope calls below).  The quantisation point
 * is after RoPE (myzaker "cache precision and tiering"), so a caller holding
 * pre-RoPE rows can rotate and quantise in one pass.  The pages give neither the
 * rotated channels nor the frequencies, so both are inputs:
 *   cos_sin  float [n_pos][pairs][2]: (cos, sin) of the angle of pair i at token
 *            position p, 8-byte aligned;
 *   start    first rotated channel of the 512-channel latent (even);
 *   pairs    rotated channel pairs (2i, 2i+1) = start + 2i, start + 2i + 1, with
 *            start + 2 * pairs <= 512.
 * A pair (x0, x1) at position p becomes, in fp32,
 *   y0 = fma(x0, c, -(x1 * s)),  y1 = fma(x0, s, x1 * c)   (products rounded first)
 * and each of y0, y1 is rounded to bf16 (nearest, ties to even), so the stored
 * codes equal those of the plain call given the rotated bf16 rows.  Channels
 * outside the range pass unchanged.  The position of an SWA row is its token
 * position; that of a main entry in slot e is ratio * e + ratio - 1 (its last
 * token).  Indexer-K rows are taken as given (not rotated).  A row whose
 * position is outside [0, n_pos) is stored unrotated and flags CSA2_DEVERR_ROPE.
 */
typedef struct csa2_rope {
    const float *cos_sin;
    int32_t n_pos;
    int32_t start;
    int32_t pairs;
} csa2_rope;

/*
 * a1/a2 quantise-append.  Main KV entries are quantised to FP4 after RoPE
 * (myzaker "cache precision": the quantisation point is after RoPE, so the
 * inputs here are post-RoPE): per 16 channels, scale = E4M3(amax / 6) and
 * code = E2M1(x / scale), both round-to-nearest-even with saturation.  The
 * indexer-K and SWA rows are quantised to E4M3 with sigma = amax / 448.
 *
 *   kv, kv_bf16 [B][T_kv][512], idxk_bf16 [B][T_kv][d_idx], kv_start [B]:
 *       entry i of request b goes to slot kv_start[b] + i.  kv may be NULL
 *       (then T_kv must be 0); kv_bf16 / idxk_bf16 may each be NULL to skip
 *       that plane.
 *   swa, swa_bf16 [B][T_swa][512], swa_start [B]:
 *       token i of request b is token position swa_start[b] + i, stored in
 *       ring slot (swa_start[b] + i) % window_cap.  swa may be NULL (T_swa 0).
 * Errors: CSA2_ERR_INVALID_ARG for bad pointers/sizes; slots >= cap are
 * skipped with CSA2_DEVERR_SLOT.
 */
CSA2_API csa2_status csa2_quantize_append(const csa2_global_kv *kv, const void *kv_bf16,
                                 const void *idxk_bf16, int32_t T_kv, const int32_t *kv_start,
                                 const csa2_swa *swa, const void *swa_bf16, int32_t T_swa,
                                 const int32_t *swa_start, int32_t *dev_err,
                                 csa2_stream_t stream);

/* csa2_quantize_append with RoPE applied to the main-KV and SWA rows first (see
 * csa2_rope; rope NULL = csa2_quantize_append).  Invalid rope fields (NULL table,
 * n_pos < 1, odd or negative start, pairs < 1, start + 2 * pairs > 512, a table
 * not 8-byte aligned) return CSA2_ERR_INVALID_ARG. */
CSA2_API csa2_status csa2_quantize_append_rope(const csa2_global_kv *kv, const void *kv_bf16,
                                               const void *idxk_bf16, int32_t T_kv,
                                               const int32_t *kv_start, const csa2_swa *swa,
                                               const void *swa_bf16, int32_t T_swa,
                                               const int32_t *swa_start, const csa2_rope *rope,
                                               int32_t *dev_err, csa2_stream_t stream);

/* Operation ids for csa2_workspace_size. */
#define CSA2_OP_INDEX_FULL 1
#define CSA2_OP_INDEX_REINDEX 2
#define CSA2_OP_SPARSE_ATTN 3

/* Bytes of workspace an operation needs (0 if none).  n_max: the largest number
 * of visible entries of any query of the call; H: attention heads; pool_blocks
 * as passed to the call.  Returns 0 for an unknown op. */
CSA2_API size_t csa2_workspace_size(int32_t op, int32_t B, int32_t Tq, int32_t n_max, int32_t H,
                           int32_t top_k, int32_t pool_blocks);

/*
 * a3-a5 Full layer: for every query, score every visible entry s with
 *   score(s) = sum_h w_h * relu(q_h . k_s)          (k_s: dequantised FP8 indexer K)
 * in the fixed fp32 order: per head an fma chain over even channels and one over
 * odd channels, added; then an fma chain over heads of (w_h, relu(a_h)); then
 * times the entry's scale.  Then
 *   pool_blocks > 0 (hierarchical, decoder): pool = the min(pool_blocks,
 *       ceil(N/8)) blocks of 8 positions with the largest block score (max over
 *       the block's visible positions), ascending ids, -1 padded; and Top-K =
 *       the top_k highest-scoring visible positions (taken inside the pool,
 *       which holds them all because pool_blocks >= top_k);
 *   pool_blocks == 0 (flat, encoder groups): Top-K over all visible entries.
 * Order: score descending, ties to the lower index.  Outputs ascending, -1 padded.
 *   q_idx_bf16 [B][Tq][H_I][d_idx], w [B][Tq][H_I] fp32, q_pos [B][Tq] token
 *   positions, n_max >= the visible count of every query, H_I in 1..16,
 *   top_k in 1..512, pool_blocks 0 or top_k..2048.
 *   pool_out [B][Tq][pool_blocks] (may be NULL when pool_blocks == 0),
 *   topk_out [B][Tq][top_k], topk_count [B][Tq].
 * Workspace: csa2_workspace_size(CSA2_OP_INDEX_FULL, B, Tq, n_max, 0, top_k,
 * pool_blocks) bytes, 256-byte aligned.
 */
CSA2_API csa2_status csa2_index_full(const csa2_global_kv *kv, const void *q_idx_bf16, const float *w,
                            const int32_t *q_pos, int32_t Tq, int32_t H_I, int32_t n_max,
                            int32_t pool_blocks, int32_t top_k, int32_t *pool_out,
                            int32_t *topk_out, int32_t *topk_count, void *workspace,
                            size_t ws_bytes, int32_t *dev_err, csa2_stream_t stream);

/*
 * a3-a5 Full layer with the scan on the tensor cores, for prefill chunks (Tq in
 * the hundreds or thousands), where the scan is Tq * N * H_I * d_idx
 * multiply-adds (DeepSeek V4.1 Flash study notes, section 2; myzaker "CSA2
 * attention": the same score as csa2_index_full).  The products q_h . k_s run
 * as bf16 tensor-core MMAs with fp32 accumulation: the E4M3 codes are exact in
 * bf16 and every product is exact in fp32, but the order of the fp32 sums over
 * channels and heads is the hardware's, not csa2_index_full's fixed order.  So
 * each score equals the exactly rounded one to within a few fp32 ulps of
 * sum_h w_h * |q_h| . |k_s| and the Top-K can differ from csa2_index_full's
 * only between positions whose scores lie within that bound of each other.
 * Arguments, outputs, workspace and errors are those of csa2_index_full, plus:
 * q_idx_bf16 must be 16-byte aligned (else CSA2_ERR_INVALID_ARG).  An MMA
 * tile is 128 entries against 256 / H_I query tokens of one request, so Tq = 1
 * works but wastes most of it: decode should call csa2_index_full.
 */
CSA2_API csa2_status csa2_index_full_tc(const csa2_global_kv *kv, const void *q_idx_bf16,
                                        const float *w, const int32_t *q_pos, int32_t Tq,
                                        int32_t H_I, int32_t n_max, int32_t pool_blocks,
                                        int32_t top_k, int32_t *pool_out, int32_t *topk_out,
                                        int32_t *topk_count, void *workspace, size_t ws_bytes,
                                        int32_t *dev_err, csa2_stream_t stream);

/*
 * csa2_index_full without a workspace argument, for callers that cannot allocate
 * device memory -- for example a backend plugin that runs inside a host
 * framework's execute callback where the framework owns all device memory, or a
 * latency-critical loop that cannot take cudaMalloc's device-wide sync.  The
 * pages have no counterpart: this is an interface convenience, not part of the
 * method.
 * Same arguments, results and errors as csa2_index_full; the scores and block
 * maxima live in a fixed array of CSA2_NOALLOC_SCRATCH_BYTES inside the library,
 * allocated on every GPU that loads the library and held until the process
 * exits.  A call that would need more than that (see csa2_workspace_size with
 * CSA2_OP_INDEX_FULL) returns CSA2_ERR_WORKSPACE and launches nothing.
 * The first call on a device looks up the array's device address (one-time
 * set-up, guarded by a mutex); make that first call before any stream capture.
 * Every call on a device shares the one array: calls that can overlap on the GPU
 * (different streams without ordering, or several host threads) race on it, so
 * order them.  Nothing in the array has to start at zero: each call writes all
 * the scratch it reads.
 */
#define CSA2_NOALLOC_SCRATCH_BYTES (16u << 20)
CSA2_API csa2_status csa2_index_full_noalloc(const csa2_global_kv *kv, const void *q_idx_bf16,
                                             const float *w, const int32_t *q_pos, int32_t Tq,
                                             int32_t H_I, int32_t n_max, int32_t pool_blocks,
                                             int32_t top_k, int32_t *pool_out,
                                             int32_t *topk_out, int32_t *topk_count,
                                             int32_t *dev_err, csa2_stream_t stream);

/*
 * Context parallel: a single request too long for one GPU is split by entry range
 * across shards (DeepSeek V4.1 Flash study notes, section 2 with report Figure 5: the
 * Full-layer scan is the only per-query cost that grows with the context).  Each
 * shard holds entries [entry_lo, entry_lo + cap) of every request in an ordinary
 * csa2_global_kv.  The steps, in order:
 *   1. csa2_index_full_slice on every shard: the Full scan of its slice and its local
 *      pool and Top-K, written as candidate keys;
 *   2. an all-gather of those lists (the caller's collective, e.g. NCCL), shard-major;
 *   3. csa2_index_merge: the exact global pool / Top-K (every item of the global
 *      selection is in its own shard's local selection, so the merge is exact), and
 *      each shard's own part of it as slice-local ids;
 *   4. csa2_sparse_attn_decode on every shard over its part (the shard holding the
 *      query's window passes swa_len, the others 0), then an all-gather of the
 *      partial outputs and lse, and csa2_attn_combine.
 * The pages define no API for this; these calls restate the same score, selection
 * order and softmax over a split cache.
 *
 * csa2_index_full_slice: csa2_index_full on a slice.  entry_lo >= 0, a multiple of 64
 * (so that blocks of 8 and 64 positions fall inside one slice); the query at token
 * position t sees the local entries e with entry_lo + e < (t + 1) / ratio; n_max >= the
 * local visible count of every query (<= cap).  Outputs, ascending in id:
 *   pool_keys_out [B][Tq][pool_blocks] (pool_blocks > 0): the slice's best blocks,
 *   topk_keys_out [B][Tq][top_k]: the slice's best entries,
 * each as the candidate key (order key << 32) | (0xFFFFFFFF - global id), where the
 * order key is larger for a larger score (equal scores equal keys) and 0 marks an
 * empty slot.  Block ids are global entry ids / 8.  Workspace and errors as for
 * csa2_index_full (with the local n_max); both outputs 8-byte aligned.
 */
CSA2_API csa2_status csa2_index_full_slice(const csa2_global_kv *kv, int64_t entry_lo,
                                           const void *q_idx_bf16, const float *w,
                                           const int32_t *q_pos, int32_t Tq, int32_t H_I,
                                           int32_t n_max, int32_t pool_blocks, int32_t top_k,
                                           uint64_t *pool_keys_out, uint64_t *topk_keys_out,
                                           void *workspace, size_t ws_bytes, int32_t *dev_err,
                                           csa2_stream_t stream);

/*
 * csa2_index_merge: the best k candidates by (score desc, id asc) of each query from
 * n_lists lists of candidate keys, lists [n_lists][BT][list_len] (shard-major, as an
 * all-gather lays them out), given in ascending slice order, each ascending in id
 * (as csa2_index_full_slice writes them).  n_lists * list_len <= 16384, k <= 2048.
 *   ids_out [BT][k] (or NULL): the global ids, ascending, -1 padded;
 *   count_out [BT] (or NULL): how many;
 *   local_out [BT][k] (or NULL): the same ids minus local_lo where local_lo <= id <
 *       local_hi, else -1 (a shard's own part, as ids of its slice).
 * For a pool, ids are block ids and local_lo / local_hi are block bounds.
 */
CSA2_API csa2_status csa2_index_merge(const uint64_t *lists, int32_t BT, int32_t n_lists,
                                      int32_t list_len, int32_t k, int64_t local_lo,
                                      int64_t local_hi, int32_t *ids_out, int32_t *count_out,
                                      int32_t *local_out, csa2_stream_t stream);

/*
 * csa2_attn_combine: one softmax over the union of the shards' keys from their
 * normalised partial results.  o_parts [n_parts][rows][512] fp32 (16-byte aligned),
 * lse_parts [n_parts][rows] (natural log, -inf = no key):
 *   lse = log sum_p exp(lse_p),  out = sum_p exp(lse_p - lse) o_p
 * (out 0 and lse -inf when every part is -inf).  rows = B * Tq * H.
 */
CSA2_API csa2_status csa2_attn_combine(const float *o_parts, const float *lse_parts, int32_t n_parts,
                                       int64_t rows, float *out, float *lse_out,
                                       csa2_stream_t stream);

/*
 * a6 Reindex layer: the same score with this layer's own q_idx / w, over the
 * visible positions of the pool's blocks only, then Top-K (same order, same
 * output form).  pool [B][Tq][pool_blocks] as written by csa2_index_full
 * (-1 = unused slot; the used slots ascending).  Workspace:
 * csa2_workspace_size(CSA2_OP_INDEX_REINDEX, B, Tq, 0, 0, top_k, pool_blocks)
 * bytes, 256-byte aligned (the candidates' scores and each slot's maximum).
 */
CSA2_API csa2_status csa2_index_reindex(const csa2_global_kv *kv, const void *q_idx_bf16, const float *w,
                               const int32_t *q_pos, int32_t Tq, int32_t H_I,
                               const int32_t *pool, int32_t pool_blocks, int32_t top_k,
                               int32_t *topk_out, int32_t *topk_count, void *workspace,
                               size_t ws_bytes, int32_t *dev_err, csa2_stream_t stream);

/*
 * csa2_index_reindex whose loads overlap the previous launch on the stream (same
 * arguments, workspace and results, bit for bit).  Precondition (the caller's), as for
 * csa2_sparse_attn_decode_reuse: no input (kv, q_idx_bf16, w, q_pos, pool) is written,
 * and the workspace not read, by the most recent ordinary launch of the library on
 * `stream` or by any launch since (a Reindex layer: its pool comes from the Full layer,
 * whose attention, at least, came in between).  The scoring kernel resolves the pool
 * and stages its rows without waiting for the previous launch, and waits for it before
 * it scores; the selection waits for the scoring as usual.
 */
CSA2_API csa2_status csa2_index_reindex_settled(const csa2_global_kv *kv, const void *q_idx_bf16,
                                                const float *w, const int32_t *q_pos, int32_t Tq,
                                                int32_t H_I, const int32_t *pool,
                                                int32_t pool_blocks, int32_t top_k,
                                                int32_t *topk_out, int32_t *topk_count,
                                                void *workspace, size_t ws_bytes,
                                                int32_t *dev_err, csa2_stream_t stream);

/*
 * a8 sparse attention.  For each query (request b, token position t = q_pos)
 * and head h:
 *   o_h = sum_j softmax_j(softmax_scale * q_h . v_j) v_j,  K = V = the entry,
 * over j in {topk entries (FP4, dequantised)} U {SWA tokens max(0,t-swa_len+1)..t
 * (FP8, dequantised)}, one softmax, no de-duplication.  A Reuse layer passes the
 * topk buffer of the layer it reuses.
 *   q_bf16 [B][Tq][H][512], topk [B][Tq][top_k] entry ids (-1 skipped; ids
 *   must be visible to the query, else skipped with CSA2_DEVERR_INDEX),
 *   swa_len in 0..window_cap-Tq+1, H a multiple of 16, top_k in 0..512.
 *   out [B][Tq][H][512] fp32, lse [B][Tq][H] fp32 (natural log; a query with
 *   no key gets o = 0 and lse = -inf).
 * Precondition: dequantised SWA values lie within +-65504 (else
 * CSA2_DEVERR_RANGE).  Workspace: csa2_workspace_size(CSA2_OP_SPARSE_ATTN, ...).
 */
CSA2_API csa2_status csa2_sparse_attn_decode(const csa2_global_kv *kv, const csa2_swa *swa,
                                    const void *q_bf16, const int32_t *q_pos, int32_t Tq,
                                    int32_t H, const int32_t *topk, int32_t top_k,
                                    int32_t swa_len, float softmax_scale, float *out,
                                    float *lse, void *workspace, size_t ws_bytes,
                                    int32_t *dev_err, csa2_stream_t stream);

/*
 * a2 + a8 fused for decode (Tq = 1): the SWA append of the query token followed by
 * the sparse attention, in one launch.  Equivalent to
 *   csa2_quantize_append(NULL, ..., swa, swa_bf16, 1, q_pos, ...)   (the ring row of
 *       token t = q_pos[b] at slot t % window_cap, FP8 with sigma = amax / 448)
 *   csa2_sparse_attn_decode(kv, swa, q_bf16, q_pos, 1, ...)
 * with the same ring bytes and the same outputs bit for bit (the kernel quantises the
 * row with the same routine and uses it directly as the window's newest key).  The
 * SWA row is the layer's own (DeepSeek V4.1 Flash study notes, section 1: each
 * layer keeps its own 128-token window); the pages define no fused form.
 *   swa_bf16 [B][512] bf16 (16-byte aligned), Tq must be 1 (else
 *   CSA2_ERR_UNSUPPORTED), swa_len >= 1 and swa non-NULL (else CSA2_ERR_INVALID_ARG);
 *   every other argument as for csa2_sparse_attn_decode.
 */
CSA2_API csa2_status csa2_sparse_attn_decode_append(const csa2_global_kv *kv, const csa2_swa *swa,
                                           const void *swa_bf16, const void *q_bf16,
                                           const int32_t *q_pos, int32_t Tq, int32_t H,
                                           const int32_t *topk, int32_t top_k, int32_t swa_len,
                                           float softmax_scale, float *out, float *lse,
                                           void *workspace, size_t ws_bytes, int32_t *dev_err,
                                           csa2_stream_t stream);

/* csa2_sparse_attn_decode_append with RoPE applied to the new SWA row (at its
 * token position q_pos) before it is quantised; rope NULL = the plain call.  Same
 * rope checks as csa2_quantize_append_rope. */
CSA2_API csa2_status csa2_sparse_attn_decode_append_rope(
    const csa2_global_kv *kv, const csa2_swa *swa, const void *swa_bf16, const void *q_bf16,
    const int32_t *q_pos, int32_t Tq, int32_t H, const int32_t *topk, int32_t top_k,
    int32_t swa_len, float softmax_scale, const csa2_rope *rope, float *out, float *lse,
    void *workspace, size_t ws_bytes, int32_t *dev_err, csa2_stream_t stream);

/*
 * The sparse attention of a Reuse layer (study notes section 2: a Reuse layer attends
 * over the selection of an earlier layer), launched so that it overlaps the previous
 * launch on the stream.  swa_bf16 non-NULL = the fused decode append of
 * csa2_sparse_attn_decode_append (Tq = 1), rope non-NULL (with swa_bf16) = its RoPE
 * form; both NULL = csa2_sparse_attn_decode.  Same arguments, checks and results, bit
 * for bit.
 *   Precondition (the caller's): no input of the call (kv, swa, q_bf16, q_pos, topk,
 *   swa_bf16, rope) is written, and no output (out, lse, the layer's ring row) read, by
 *   the most recent ordinary launch of the library on `stream` (any launch but this call
 *   and csa2_index_reindex_settled) or by any launch since (a Reuse layer: its topk comes
 *   from a Full or Reindex selection, and that layer's own attention, an ordinary
 *   launch, came in between).  The kernel lets the next launch start at once and reads
 *   its inputs, compacts the selection, and gathers and dequantises its first keys
 *   without waiting for the previous launch (an ordinary launch waits for its
 *   predecessor before it lets the next one start, so whatever was written before it is
 *   complete); its first score MMA waits for the previous launch to complete, so that
 *   the layers' compute stays in stream order.  A kernel outside the library that lets
 *   its dependents start early (programmatic dependent launch) must not write the
 *   inputs.
 */
CSA2_API csa2_status csa2_sparse_attn_decode_reuse(const csa2_global_kv *kv, const csa2_swa *swa,
                                                   const void *swa_bf16, const void *q_bf16,
                                                   const int32_t *q_pos, int32_t Tq, int32_t H,
                                                   const int32_t *topk, int32_t top_k,
                                                   int32_t swa_len, float softmax_scale,
                                                   const csa2_rope *rope, float *out, float *lse,
                                                   int32_t *dev_err, csa2_stream_t stream);

/*
 * Paged global KV (serving: requests of different lengths share one pool of pages;
 * the pages' cache is the one global KV of study notes section 5 / myzaker "cache
 * precision and tiering", here laid out in fixed-size pages).  The planes hold
 * n_pages pages of page_size entries each, in the same per-entry formats as
 * csa2_global_kv:
 *   codes [n_pages * page_size][256], scales [n_pages * page_size][32],
 *   idx_codes [n_pages * page_size][d_idx], idx_scale [n_pages * page_size];
 * entry e of request b lives in row
 *   block_table[b][e / page_size] * page_size + e % page_size
 * (block_table int32 [batch][max_pages], device).  The logical capacity of a request
 * is max_pages * page_size entries; its length is set by its query positions, as for
 * csa2_global_kv.  page_size is a power of two >= 256 (so that a scan tile, a pool
 * block and a 64-position block never straddle a page; else CSA2_ERR_UNSUPPORTED).
 * A table entry outside [0, n_pages) met by a kernel is skipped and flags
 * CSA2_DEVERR_PAGE (results are then undefined).  The pages define no paging: this is
 * the serving layout of the same cache.
 */
typedef struct csa2_paged_kv {
    uint8_t *codes;
    uint8_t *scales;
    uint8_t *idx_codes;
    float *idx_scale;
    const int32_t *block_table;
    int32_t batch;
    int32_t max_pages;
    int32_t page_size;
    int32_t n_pages;
    int32_t d_idx;   /* 64 or 128 */
    int32_t ratio;   /* 1 or 2 */
} csa2_paged_kv;

/* csa2_quantize_append(_rope) on a paged cache (rope NULL = no rotation). */
CSA2_API csa2_status csa2_quantize_append_paged(const csa2_paged_kv *kv, const void *kv_bf16,
                                                const void *idxk_bf16, int32_t T_kv,
                                                const int32_t *kv_start, const csa2_swa *swa,
                                                const void *swa_bf16, int32_t T_swa,
                                                const int32_t *swa_start, const csa2_rope *rope,
                                                int32_t *dev_err, csa2_stream_t stream);

/* csa2_index_full on a paged cache (same arguments, workspace and results). */
CSA2_API csa2_status csa2_index_full_paged(const csa2_paged_kv *kv, const void *q_idx_bf16,
                                           const float *w, const int32_t *q_pos, int32_t Tq,
                                           int32_t H_I, int32_t n_max, int32_t pool_blocks,
                                           int32_t top_k, int32_t *pool_out, int32_t *topk_out,
                                           int32_t *topk_count, void *workspace, size_t ws_bytes,
                                           int32_t *dev_err, csa2_stream_t stream);

/* csa2_index_reindex on a paged cache (same workspace). */
CSA2_API csa2_status csa2_index_reindex_paged(const csa2_paged_kv *kv, const void *q_idx_bf16,
                                              const float *w, const int32_t *q_pos, int32_t Tq,
                                              int32_t H_I, const int32_t *pool,
                                              int32_t pool_blocks, int32_t top_k,
                                              int32_t *topk_out, int32_t *topk_count,
                                              void *workspace, size_t ws_bytes,
                                              int32_t *dev_err, csa2_stream_t stream);

/* csa2_sparse_attn_decode on a paged cache.  swa_bf16 non-NULL = the fused decode
 * append of csa2_sparse_attn_decode_append (Tq = 1), rope non-NULL (with swa_bf16) =
 * its RoPE form; both NULL = the plain call. */
CSA2_API csa2_status csa2_sparse_attn_decode_paged(const csa2_paged_kv *kv, const csa2_swa *swa,
                                                   const void *swa_bf16, const void *q_bf16,
                                                   const int32_t *q_pos, int32_t Tq, int32_t H,
                                                   const int32_t *topk, int32_t top_k,
                                                   int32_t swa_len, float softmax_scale,
                                                   const csa2_rope *rope, float *out, float *lse,
                                                   int32_t *dev_err, csa2_stream_t stream);

/* The overlapping launches of the Reindex and Reuse layers on a paged cache: as
 * csa2_index_reindex_settled and csa2_sparse_attn_decode_reuse (same arguments as the
 * two calls above, the same preconditions, and results bit for bit equal to those
 * calls; the block table counts among the inputs that the previous launch must not
 * write). */
CSA2_API csa2_status csa2_index_reindex_paged_settled(const csa2_paged_kv *kv, const void *q_idx_bf16,
                                                      const float *w, const int32_t *q_pos, int32_t Tq,
                                                      int32_t H_I, const int32_t *pool,
                                                      int32_t pool_blocks, int32_t top_k,
                                                      int32_t *topk_out, int32_t *topk_count,
                                                      void *workspace, size_t ws_bytes,
                                                      int32_t *dev_err, csa2_stream_t stream);
CSA2_API csa2_status csa2_sparse_attn_decode_paged_reuse(const csa2_paged_kv *kv, const csa2_swa *swa,
                                                         const void *swa_bf16, const void *q_bf16,
                                                         const int32_t *q_pos, int32_t Tq, int32_t H,
                                                         const int32_t *topk, int32_t top_k,
                                                         int32_t swa_len, float softmax_scale,
                                                         const csa2_rope *rope, float *out, float *lse,
                                                         int32_t *dev_err, csa2_stream_t stream);

/* Synchronise `stream`, read *dev_err (device int32) into *bits_out (host),
 * reset it to 0, and return CSA2_ERR_DEVICE_BOUNDS if any bit was set. */
CSA2_API csa2_status csa2_read_device_error(int32_t *dev_err, int32_t *bits_out, csa2_stream_t stream);

/* Static description of a status code (never NULL). */
CSA2_API const char *csa2_status_string(csa2_status status);

/* ABI version: 100 * major + minor. */
CSA2_API int32_t csa2_abi_version(void);

/*
 * Test hook for the kernels' bounded waits; the pages have no counterpart (it is
 * not part of the method).  Every spin of a kernel on an mbarrier gives up after
 * limit_ns of wall time: the kernel then sets CSA2_DEVERR_TIMEOUT in *dev_err,
 * waits (bounded) for its own tensor-core work and copies in flight, frees its
 * tensor memory and returns, so that the CUDA context stays usable.
 * stuck_wait != 0 makes the first wait of every CTA of the tensor-core kernels
 * (the scan of csa2_index_full_tc and the sparse attention) wait on a barrier that
 * nothing signals, so that it always runs out: a test can drive the timeout path
 * without faulting or hanging a GPU.  The setting is process-wide and read by each
 * call when it launches; defaults: limit_ns = 500000000 (0.5 s), stuck_wait = 0.
 * Results of calls made with stuck_wait set are undefined (only the error bit is).
 */
CSA2_API void csa2_debug_set_waits(uint64_t limit_ns, int32_t stuck_wait);

#ifdef __cplusplus
}
#endif

#endif /* CSA2_H_ */
