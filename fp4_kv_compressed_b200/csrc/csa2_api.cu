// csa2_api.cu -- the extern "C" entry points of libcsa2: host-side validation,
// workspace layout and kernel launches.  No allocation, no state, no exceptions.
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "csa2.h"
#include "csa2_internal.h"

using namespace csa2;

namespace csa2 {

// The process-wide wait settings of csa2_debug_set_waits.
static std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitLimitNs};
static std::atomic<int32_t> g_stuck_wait{0};

WaitCfg current_wait_cfg() {
    WaitCfg w;
    w.limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
    w.stuck = g_stuck_wait.load(std::memory_order_relaxed);
    return w;
}

}  // namespace csa2

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Workspace layout of csa2_index_full: scores [BT][score_stride] fp32, then block
// maxima of 8 positions [BT][bmax_stride] (hierarchical rows, and flat rows longer than
// kFlatDirect), then maxima of 64 positions [BT][bmax64_stride] (flat rows longer than
// kFlatDirect; hierarchical rows of more than kPoolDirect blocks).  The selection of a
// long row goes through the block maxima; the select stages up to kPoolDirect block
// maxima directly.
constexpr int64_t kFlatDirect = 16384;
constexpr int64_t kPoolDirect = 16384;

struct FullLayout {
    int64_t score_stride, bmax_stride, bmax64_stride;
    size_t bmax_off, bmax64_off, total;
    bool bmax, bmax64;
};

FullLayout full_layout(int64_t BT, int64_t n_max, int32_t pool_blocks) {
    FullLayout L;
    L.score_stride = (int64_t)align_up((size_t)(n_max > 0 ? n_max : 1), 64);
    L.bmax_stride = (int64_t)align_up((size_t)((n_max + 7) / 8 > 0 ? (n_max + 7) / 8 : 1), 64);
    L.bmax64_stride = (int64_t)align_up((size_t)((n_max + 63) / 64 > 0 ? (n_max + 63) / 64 : 1), 64);
    L.bmax = pool_blocks > 0 || n_max > kFlatDirect;
    L.bmax64 = pool_blocks > 0 ? (n_max + 7) / 8 > kPoolDirect : n_max > kFlatDirect;
    L.bmax_off = align_up((size_t)BT * L.score_stride * sizeof(float), kAlign);
    L.bmax64_off = L.bmax_off + (L.bmax ? align_up((size_t)BT * L.bmax_stride * sizeof(float), kAlign) : 0);
    L.total = L.bmax64_off + (L.bmax64 ? align_up((size_t)BT * L.bmax64_stride * sizeof(float), kAlign) : 0);
    return L;
}

// A global-KV group as the kernels see it: the planes, the logical shape and the page
// map (contiguous for csa2_global_kv, a block table for csa2_paged_kv).
struct KvView {
    uint8_t *codes, *scales, *idx_codes;
    float *idx_scale;
    int32_t batch, cap, d_idx, ratio;
    PageMap pm;
};

const KvView *view_of(const csa2_global_kv *kv, KvView *v) {
    if (!kv) return nullptr;
    *v = KvView{kv->codes, kv->scales, kv->idx_codes, kv->idx_scale, kv->batch, kv->cap, kv->d_idx,
                kv->ratio, PageMap{nullptr, 0, 0, 0}};
    return v;
}

// Paged view: pages of page_size entries (a power of two >= 256, so that scan tiles, pool
// blocks and 64-position blocks never straddle a page), block table [batch][max_pages].
csa2_status paged_view(const csa2_paged_kv *kv, KvView *v, const KvView **out) {
    *out = nullptr;
    if (!kv) return CSA2_OK;
    if (!kv->block_table || !aligned(kv->block_table, 4)) return CSA2_ERR_INVALID_ARG;
    if (kv->page_size < 256 || kv->page_size > (1 << 20) || (kv->page_size & (kv->page_size - 1)))
        return CSA2_ERR_UNSUPPORTED;
    if (kv->max_pages < 1 || kv->n_pages < 1 || kv->batch < 1) return CSA2_ERR_INVALID_ARG;
    const int64_t cap = (int64_t)kv->max_pages * kv->page_size;
    if (cap > INT32_MAX || (int64_t)kv->n_pages * kv->page_size > ((int64_t)1 << 40)) return CSA2_ERR_UNSUPPORTED;
    int shift = 0;
    while ((1 << shift) < kv->page_size) ++shift;
    *v = KvView{kv->codes, kv->scales, kv->idx_codes, kv->idx_scale, kv->batch, (int32_t)cap, kv->d_idx,
                kv->ratio, PageMap{kv->block_table, shift, kv->max_pages, kv->n_pages}};
    *out = v;
    return CSA2_OK;
}

// Workspace of csa2_index_reindex: scores [BT][8 pool_blocks] fp32, then the maximum of
// each pool slot [BT][pool_blocks] fp32.
struct ReindexLayout {
    size_t bmax_off, total;
};
ReindexLayout reindex_layout(int64_t BT, int32_t pool_blocks) {
    ReindexLayout L;
    L.bmax_off = align_up((size_t)BT * pool_blocks * 8 * sizeof(float), kAlign);
    L.total = L.bmax_off + align_up((size_t)BT * pool_blocks * sizeof(float), kAlign);
    return L;
}

csa2_status check_kv(const KvView *kv, bool need_index) {
    if (!kv || !kv->codes || !kv->scales) return CSA2_ERR_INVALID_ARG;
    if (kv->batch <= 0 || kv->cap <= 0 || kv->ratio < 1 || kv->ratio > 64) return CSA2_ERR_INVALID_ARG;
    if (!aligned(kv->codes, 16) || !aligned(kv->scales, 16)) return CSA2_ERR_INVALID_ARG;
    if (need_index) {
        if (!kv->idx_codes || !kv->idx_scale) return CSA2_ERR_INVALID_ARG;
        if (kv->d_idx != 64 && kv->d_idx != 128) return CSA2_ERR_UNSUPPORTED;
        if (!aligned(kv->idx_codes, 16) || !aligned(kv->idx_scale, 4)) return CSA2_ERR_INVALID_ARG;
    }
    return CSA2_OK;
}

csa2_status launched(cudaError_t e) {
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return CSA2_ERR_CUDA;
    }
    return CSA2_OK;
}

bool hi_supported(int32_t H_I) {
    return H_I == 1 || H_I == 2 || H_I == 4 || H_I == 8 || H_I == 16;
}

}  // namespace

extern "C" {

int32_t csa2_abi_version(void) { return 106; }

void csa2_debug_set_waits(uint64_t limit_ns, int32_t stuck_wait) {
    g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
    g_stuck_wait.store(stuck_wait ? 1 : 0, std::memory_order_relaxed);
}

const char *csa2_status_string(csa2_status st) {
    switch (st) {
        case CSA2_OK: return "ok";
        case CSA2_ERR_INVALID_ARG: return "invalid argument";
        case CSA2_ERR_CAPACITY: return "cache or window capacity too small";
        case CSA2_ERR_WORKSPACE: return "workspace missing or too small";
        case CSA2_ERR_UNSUPPORTED: return "shape not supported by the kernels";
        case CSA2_ERR_CUDA: return "CUDA launch or runtime error";
        case CSA2_ERR_DEVICE_BOUNDS: return "device-side bounds check failed";
    }
    return "unknown status";
}

size_t csa2_workspace_size(int32_t op, int32_t B, int32_t Tq, int32_t n_max, int32_t H,
                           int32_t top_k, int32_t pool_blocks) {
    (void)H;
    (void)top_k;
    if (B <= 0 || Tq <= 0) return 0;
    const int64_t BT = (int64_t)B * Tq;
    switch (op) {
        case CSA2_OP_INDEX_FULL:
            return n_max > 0 ? full_layout(BT, n_max, pool_blocks).total : 0;
        case CSA2_OP_INDEX_REINDEX:
            return pool_blocks > 0 ? reindex_layout(BT, pool_blocks).total : 0;
        case CSA2_OP_SPARSE_ATTN:
            return 0;
        default:
            return 0;
    }
}

// RoPE descriptor -> kernel arguments (nullptr: no rotation).
static csa2_status rope_args(const csa2_rope *rope, RopeArgs *out) {
    memset(out, 0, sizeof(*out));
    if (!rope) return CSA2_OK;
    if (!rope->cos_sin || !aligned(rope->cos_sin, 8) || rope->n_pos < 1) return CSA2_ERR_INVALID_ARG;
    if (rope->start < 0 || rope->start % 2 != 0 || rope->pairs < 1 ||
        (int64_t)rope->start + 2 * (int64_t)rope->pairs > CSA2_KV_DIM)
        return CSA2_ERR_INVALID_ARG;
    out->cs = reinterpret_cast<const float2 *>(rope->cos_sin);
    out->n_pos = rope->n_pos;
    out->start = rope->start;
    out->pairs = rope->pairs;
    return CSA2_OK;
}

static csa2_status quantize_append(const KvView *kv, const void *kv_bf16,
                                   const void *idxk_bf16, int32_t T_kv, const int32_t *kv_start,
                                   const csa2_swa *swa, const void *swa_bf16, int32_t T_swa,
                                   const int32_t *swa_start, const csa2_rope *rope,
                                   int32_t *dev_err, csa2_stream_t stream) {
    QuantArgs a;
    memset(&a, 0, sizeof(a));
    a.dev_err = dev_err;
    csa2_status rs = rope_args(rope, &a.rope);
    if (rs != CSA2_OK) return rs;
    if (T_kv < 0 || T_swa < 0) return CSA2_ERR_INVALID_ARG;
    int32_t B = -1;
    if (T_kv > 0 && (kv_bf16 || idxk_bf16)) {
        csa2_status st = check_kv(kv, idxk_bf16 != nullptr);
        if (st != CSA2_OK) return st;
        if (!kv_start) return CSA2_ERR_INVALID_ARG;
        if (kv_bf16 && !aligned(kv_bf16, 16)) return CSA2_ERR_INVALID_ARG;
        if (idxk_bf16 && !aligned(idxk_bf16, 8)) return CSA2_ERR_INVALID_ARG;
        if (T_kv > kv->cap) return CSA2_ERR_CAPACITY;
        B = kv->batch;
        a.codes = kv->codes;
        a.scales = kv->scales;
        a.idx_codes = kv->idx_codes;
        a.idx_scale = kv->idx_scale;
        a.cap = kv->cap;
        a.d_idx = kv->d_idx;
        a.ratio = kv->ratio;
        a.pm = kv->pm;
        a.kv_bf16 = (const uint16_t *)kv_bf16;
        a.idxk_bf16 = (const uint16_t *)idxk_bf16;
        a.T_kv = T_kv;
        a.kv_start = kv_start;
        a.n_main = kv_bf16 ? (int64_t)B * T_kv : 0;
        a.n_idx = idxk_bf16 ? (int64_t)B * T_kv : 0;
    }
    if (T_swa > 0 && swa_bf16) {
        if (!swa || !swa->codes || !swa->scale || !swa_start) return CSA2_ERR_INVALID_ARG;
        if (swa->batch <= 0 || swa->window_cap <= 0) return CSA2_ERR_INVALID_ARG;
        if (B >= 0 && swa->batch != B) return CSA2_ERR_INVALID_ARG;
        if (!aligned(swa->codes, 16) || !aligned(swa->scale, 4) || !aligned(swa_bf16, 16))
            return CSA2_ERR_INVALID_ARG;
        if (T_swa > swa->window_cap) return CSA2_ERR_CAPACITY;
        a.swa_codes = swa->codes;
        a.swa_scale = swa->scale;
        a.wcap = swa->window_cap;
        a.swa_bf16 = (const uint16_t *)swa_bf16;
        a.T_swa = T_swa;
        a.swa_start = swa_start;
        a.n_swa = (int64_t)swa->batch * T_swa;
    }
    return launched(launch_quantize_append(a, (cudaStream_t)stream));
}

csa2_status csa2_quantize_append(const csa2_global_kv *kv, const void *kv_bf16,
                                 const void *idxk_bf16, int32_t T_kv, const int32_t *kv_start,
                                 const csa2_swa *swa, const void *swa_bf16, int32_t T_swa,
                                 const int32_t *swa_start, int32_t *dev_err,
                                 csa2_stream_t stream) {
    KvView v;
    return quantize_append(view_of(kv, &v), kv_bf16, idxk_bf16, T_kv, kv_start, swa, swa_bf16, T_swa,
                           swa_start, nullptr, dev_err, stream);
}

csa2_status csa2_quantize_append_rope(const csa2_global_kv *kv, const void *kv_bf16,
                                      const void *idxk_bf16, int32_t T_kv,
                                      const int32_t *kv_start, const csa2_swa *swa,
                                      const void *swa_bf16, int32_t T_swa,
                                      const int32_t *swa_start, const csa2_rope *rope,
                                      int32_t *dev_err, csa2_stream_t stream) {
    KvView v;
    return quantize_append(view_of(kv, &v), kv_bf16, idxk_bf16, T_kv, kv_start, swa, swa_bf16, T_swa,
                           swa_start, rope, dev_err, stream);
}

// Full layer: scan (exact CUDA-core order, or tensor cores) then pool / Top-K.
static csa2_status index_full(const KvView *kv, const void *q_idx_bf16, const float *w,
                              const int32_t *q_pos, int32_t Tq, int32_t H_I, int32_t n_max,
                              int32_t pool_blocks, int32_t top_k, int32_t *pool_out,
                              int32_t *topk_out, int32_t *topk_count, void *workspace,
                              size_t ws_bytes, int32_t *dev_err, csa2_stream_t stream, bool tc,
                              int64_t entry_lo = 0, uint64_t *pool_keys_out = nullptr,
                              uint64_t *topk_keys_out = nullptr) {
    csa2_status st = check_kv(kv, true);
    if (st != CSA2_OK) return st;
    if (!q_idx_bf16 || !w || !q_pos) return CSA2_ERR_INVALID_ARG;
    if (topk_keys_out == nullptr && (!topk_out || !topk_count)) return CSA2_ERR_INVALID_ARG;
    if (!aligned(q_idx_bf16, tc ? 16 : 4) || !aligned(w, 4)) return CSA2_ERR_INVALID_ARG;
    if (Tq <= 0 || n_max < 0) return CSA2_ERR_INVALID_ARG;
    if (!hi_supported(H_I)) return CSA2_ERR_UNSUPPORTED;
    if (top_k < 1 || top_k > CSA2_TOPK_MAX) return CSA2_ERR_UNSUPPORTED;
    if (pool_blocks != 0 && (pool_blocks < top_k || pool_blocks > CSA2_POOL_MAX))
        return CSA2_ERR_UNSUPPORTED;
    const int64_t BT = (int64_t)kv->batch * Tq;
    if (BT > 65535) return CSA2_ERR_UNSUPPORTED;   // grid.y limit
    const FullLayout L = full_layout(BT, n_max, pool_blocks);
    if (n_max > 0 && (!workspace || ws_bytes < L.total || !aligned(workspace, kAlign)))
        return CSA2_ERR_WORKSPACE;

    IndexArgs a;
    memset(&a, 0, sizeof(a));
    a.idx_codes = kv->idx_codes;
    a.idx_scale = kv->idx_scale;
    a.cap = kv->cap;
    a.d_idx = kv->d_idx;
    a.ratio = kv->ratio;
    a.q_idx = (const uint16_t *)q_idx_bf16;
    a.w = w;
    a.q_pos = q_pos;
    a.Tq = Tq;
    a.H_I = H_I;
    a.n_max = n_max;
    a.scores = (float *)workspace;
    a.score_stride = L.score_stride;
    // the tensor-core scan writes 8-position maxima for the pool only; the exact scan
    // writes both kinds whenever the layout has them
    a.bmax = workspace && (tc ? pool_blocks > 0 : L.bmax) ? (float *)((uint8_t *)workspace + L.bmax_off) : nullptr;
    a.bmax_stride = L.bmax_stride;
    a.bmax64 = workspace && !tc && L.bmax64 ? (float *)((uint8_t *)workspace + L.bmax64_off) : nullptr;
    a.bmax64_stride = L.bmax64_stride;
    a.pool_blocks = pool_blocks;
    a.pool_out = pool_out;
    a.top_k = top_k;
    a.topk_out = topk_out;
    a.topk_count = topk_count;
    a.dev_err = dev_err;
    a.wait = current_wait_cfg();
    a.entry_lo = entry_lo;
    a.pm = kv->pm;
    a.pool_keys_out = pool_keys_out;
    a.topk_keys_out = topk_keys_out;
    cudaStream_t s = (cudaStream_t)stream;
    st = launched(tc ? launch_index_scan_tc(a, (int)kv->batch, s) : launch_index_scan(a, (int)BT, s));
    if (st != CSA2_OK) return st;
    return launched(launch_select_full(a, (int)BT, s));
}

csa2_status csa2_index_full(const csa2_global_kv *kv, const void *q_idx_bf16, const float *w,
                            const int32_t *q_pos, int32_t Tq, int32_t H_I, int32_t n_max,
                            int32_t pool_blocks, int32_t top_k, int32_t *pool_out,
                            int32_t *topk_out, int32_t *topk_count, void *workspace,
                            size_t ws_bytes, int32_t *dev_err, csa2_stream_t stream) {
    KvView v;
    return index_full(view_of(kv, &v), q_idx_bf16, w, q_pos, Tq, H_I, n_max, pool_blocks, top_k, pool_out,
                      topk_out, topk_count, workspace, ws_bytes, dev_err, stream, false);
}

csa2_status csa2_index_full_tc(const csa2_global_kv *kv, const void *q_idx_bf16, const float *w,
                               const int32_t *q_pos, int32_t Tq, int32_t H_I, int32_t n_max,
                               int32_t pool_blocks, int32_t top_k, int32_t *pool_out,
                               int32_t *topk_out, int32_t *topk_count, void *workspace,
                               size_t ws_bytes, int32_t *dev_err, csa2_stream_t stream) {
    KvView v;
    return index_full(view_of(kv, &v), q_idx_bf16, w, q_pos, Tq, H_I, n_max, pool_blocks, top_k, pool_out,
                      topk_out, topk_count, workspace, ws_bytes, dev_err, stream, true);
}

csa2_status csa2_index_full_slice(const csa2_global_kv *kv, int64_t entry_lo,
                                  const void *q_idx_bf16, const float *w, const int32_t *q_pos,
                                  int32_t Tq, int32_t H_I, int32_t n_max, int32_t pool_blocks,
                                  int32_t top_k, uint64_t *pool_keys_out, uint64_t *topk_keys_out,
                                  void *workspace, size_t ws_bytes, int32_t *dev_err,
                                  csa2_stream_t stream) {
    if (entry_lo < 0 || entry_lo % 64 != 0 || !topk_keys_out) return CSA2_ERR_INVALID_ARG;
    if (pool_blocks > 0 && !pool_keys_out) return CSA2_ERR_INVALID_ARG;
    if (!aligned(topk_keys_out, 8) || (pool_keys_out && !aligned(pool_keys_out, 8))) return CSA2_ERR_INVALID_ARG;
    if (kv && entry_lo / 8 + (int64_t)kv->cap / 8 + 1 > INT32_MAX / 2) return CSA2_ERR_UNSUPPORTED;
    KvView v;
    return index_full(view_of(kv, &v), q_idx_bf16, w, q_pos, Tq, H_I, n_max, pool_blocks, top_k, nullptr,
                      nullptr, nullptr, workspace, ws_bytes, dev_err, stream, false, entry_lo,
                      pool_blocks > 0 ? pool_keys_out : nullptr, topk_keys_out);
}

csa2_status csa2_index_merge(const uint64_t *lists, int32_t BT, int32_t n_lists, int32_t list_len,
                             int32_t k, int64_t local_lo, int64_t local_hi, int32_t *ids_out,
                             int32_t *count_out, int32_t *local_out, csa2_stream_t stream) {
    if (!lists || BT <= 0 || n_lists <= 0 || list_len <= 0 || k <= 0) return CSA2_ERR_INVALID_ARG;
    if (!aligned(lists, 8)) return CSA2_ERR_INVALID_ARG;
    if (!ids_out && !local_out) return CSA2_ERR_INVALID_ARG;
    if (k > CSA2_POOL_MAX || (int64_t)n_lists * list_len > 16384) return CSA2_ERR_UNSUPPORTED;
    if (BT > 65535 * 32) return CSA2_ERR_UNSUPPORTED;
    return launched(launch_index_merge(lists, BT, n_lists, list_len, k, local_lo, local_hi, ids_out,
                                       count_out, local_out, (cudaStream_t)stream));
}

csa2_status csa2_attn_combine(const float *o_parts, const float *lse_parts, int32_t n_parts, int64_t rows,
                              float *out, float *lse_out, csa2_stream_t stream) {
    if (!o_parts || !lse_parts || !out || !lse_out || n_parts <= 0 || rows < 0) return CSA2_ERR_INVALID_ARG;
    if (!aligned(o_parts, 16) || !aligned(out, 16)) return CSA2_ERR_INVALID_ARG;
    return launched(launch_attn_combine(o_parts, lse_parts, n_parts, rows, out, lse_out,
                                        (cudaStream_t)stream));
}

static csa2_status index_reindex(const KvView *kv, const void *q_idx_bf16, const float *w,
                                 const int32_t *q_pos, int32_t Tq, int32_t H_I,
                                 const int32_t *pool, int32_t pool_blocks, int32_t top_k,
                                 int32_t *topk_out, int32_t *topk_count, void *workspace,
                                 size_t ws_bytes, int32_t *dev_err, csa2_stream_t stream,
                                 bool settled = false) {
    csa2_status st = check_kv(kv, true);
    if (st != CSA2_OK) return st;
    if (!q_idx_bf16 || !w || !q_pos || !pool || !topk_out || !topk_count) return CSA2_ERR_INVALID_ARG;
    if (!aligned(q_idx_bf16, 4) || !aligned(w, 4)) return CSA2_ERR_INVALID_ARG;
    if (Tq <= 0) return CSA2_ERR_INVALID_ARG;
    if (!hi_supported(H_I)) return CSA2_ERR_UNSUPPORTED;
    if (top_k < 1 || top_k > CSA2_TOPK_MAX) return CSA2_ERR_UNSUPPORTED;
    if (pool_blocks < 1 || pool_blocks > CSA2_POOL_MAX) return CSA2_ERR_UNSUPPORTED;
    const int64_t BT = (int64_t)kv->batch * Tq;
    if (BT > 65535) return CSA2_ERR_UNSUPPORTED;   // grid.y limit
    const ReindexLayout L = reindex_layout(BT, pool_blocks);
    if (!workspace || ws_bytes < L.total || !aligned(workspace, kAlign)) return CSA2_ERR_WORKSPACE;

    IndexArgs a;
    memset(&a, 0, sizeof(a));
    a.idx_codes = kv->idx_codes;
    a.idx_scale = kv->idx_scale;
    a.cap = kv->cap;
    a.d_idx = kv->d_idx;
    a.ratio = kv->ratio;
    a.q_idx = (const uint16_t *)q_idx_bf16;
    a.w = w;
    a.q_pos = q_pos;
    a.Tq = Tq;
    a.H_I = H_I;
    a.scores = (float *)workspace;
    a.score_stride = (int64_t)pool_blocks * 8;
    a.bmax = (float *)((uint8_t *)workspace + L.bmax_off);
    a.bmax_stride = pool_blocks;
    a.pool = pool;
    a.pool_blocks = pool_blocks;
    a.top_k = top_k;
    a.topk_out = topk_out;
    a.topk_count = topk_count;
    a.dev_err = dev_err;
    a.wait = current_wait_cfg();
    a.pm = kv->pm;
    a.settled = settled ? 1 : 0;
    cudaStream_t s = (cudaStream_t)stream;
    st = launched(launch_reindex_score(a, (int)BT, s));
    if (st != CSA2_OK) return st;
    return launched(launch_select_reindex(a, (int)BT, s));
}

csa2_status csa2_index_reindex(const csa2_global_kv *kv, const void *q_idx_bf16, const float *w,
                               const int32_t *q_pos, int32_t Tq, int32_t H_I,
                               const int32_t *pool, int32_t pool_blocks, int32_t top_k,
                               int32_t *topk_out, int32_t *topk_count, void *workspace,
                               size_t ws_bytes, int32_t *dev_err, csa2_stream_t stream) {
    KvView v;
    return index_reindex(view_of(kv, &v), q_idx_bf16, w, q_pos, Tq, H_I, pool, pool_blocks, top_k,
                         topk_out, topk_count, workspace, ws_bytes, dev_err, stream);
}

csa2_status csa2_index_reindex_settled(const csa2_global_kv *kv, const void *q_idx_bf16,
                                       const float *w, const int32_t *q_pos, int32_t Tq,
                                       int32_t H_I, const int32_t *pool, int32_t pool_blocks,
                                       int32_t top_k, int32_t *topk_out, int32_t *topk_count,
                                       void *workspace, size_t ws_bytes, int32_t *dev_err,
                                       csa2_stream_t stream) {
    KvView v;
    return index_reindex(view_of(kv, &v), q_idx_bf16, w, q_pos, Tq, H_I, pool, pool_blocks, top_k,
                         topk_out, topk_count, workspace, ws_bytes, dev_err, stream, true);
}

static csa2_status sparse_attn(const KvView *kv, const csa2_swa *swa, const void *swa_new_bf16,
                               const void *q_bf16, const int32_t *q_pos, int32_t Tq, int32_t H,
                               const int32_t *topk, int32_t top_k, int32_t swa_len,
                               float softmax_scale, const csa2_rope *rope, float *out,
                               float *lse, int32_t *dev_err, csa2_stream_t stream,
                               bool settled = false) {
    csa2_status st = check_kv(kv, false);
    if (st != CSA2_OK) return st;
    if (!q_bf16 || !q_pos || !out || !lse) return CSA2_ERR_INVALID_ARG;
    if (!aligned(q_bf16, 4) || !aligned(out, 8)) return CSA2_ERR_INVALID_ARG;
    if (Tq <= 0 || H < 16 || H % 16 != 0) return CSA2_ERR_UNSUPPORTED;
    if (top_k < 0 || top_k > CSA2_TOPK_MAX) return CSA2_ERR_UNSUPPORTED;
    if (top_k > 0 && !topk) return CSA2_ERR_INVALID_ARG;
    if (swa_len < 0) return CSA2_ERR_INVALID_ARG;
    if (swa_len > 0) {
        if (!swa || !swa->codes || !swa->scale || swa->window_cap <= 0) return CSA2_ERR_INVALID_ARG;
        if (swa->batch != kv->batch) return CSA2_ERR_INVALID_ARG;
        if (!aligned(swa->codes, 16) || !aligned(swa->scale, 4)) return CSA2_ERR_INVALID_ARG;
        if ((int64_t)swa_len + Tq - 1 > swa->window_cap) return CSA2_ERR_CAPACITY;
    }
    const int64_t BT = (int64_t)kv->batch * Tq;

    AttnArgs a;
    memset(&a, 0, sizeof(a));
    a.codes = kv->codes;
    a.scales = kv->scales;
    a.cap = kv->cap;
    a.ratio = kv->ratio;
    a.pm = kv->pm;
    if (swa_len > 0) {
        a.swa_codes = swa->codes;
        a.swa_scale = swa->scale;
        a.wcap = swa->window_cap;
    } else {
        a.wcap = 1;
    }
    a.q = (const uint16_t *)q_bf16;
    a.q_pos = q_pos;
    a.Tq = Tq;
    a.H = H;
    a.topk = topk;
    a.top_k = top_k;
    a.swa_len = swa_len;
    a.softmax_scale = softmax_scale;
    a.swa_new = (const uint16_t *)swa_new_bf16;
    st = rope_args(rope, &a.rope);
    if (st != CSA2_OK) return st;
    a.out = out;
    a.lse = lse;
    a.dev_err = dev_err;
    a.wait = current_wait_cfg();
    a.settled = settled ? 1 : 0;
    return launched(launch_sparse_attn(a, (int)BT, (cudaStream_t)stream));
}

csa2_status csa2_sparse_attn_decode(const csa2_global_kv *kv, const csa2_swa *swa,
                                    const void *q_bf16, const int32_t *q_pos, int32_t Tq,
                                    int32_t H, const int32_t *topk, int32_t top_k,
                                    int32_t swa_len, float softmax_scale, float *out,
                                    float *lse, void *workspace, size_t ws_bytes,
                                    int32_t *dev_err, csa2_stream_t stream) {
    (void)workspace;
    (void)ws_bytes;
    KvView v;
    return sparse_attn(view_of(kv, &v), swa, nullptr, q_bf16, q_pos, Tq, H, topk, top_k, swa_len,
                       softmax_scale, nullptr, out, lse, dev_err, stream);
}

csa2_status csa2_sparse_attn_decode_append(const csa2_global_kv *kv, const csa2_swa *swa,
                                           const void *swa_bf16, const void *q_bf16,
                                           const int32_t *q_pos, int32_t Tq, int32_t H,
                                           const int32_t *topk, int32_t top_k, int32_t swa_len,
                                           float softmax_scale, float *out, float *lse,
                                           void *workspace, size_t ws_bytes, int32_t *dev_err,
                                           csa2_stream_t stream) {
    return csa2_sparse_attn_decode_append_rope(kv, swa, swa_bf16, q_bf16, q_pos, Tq, H, topk, top_k,
                                               swa_len, softmax_scale, nullptr, out, lse, workspace,
                                               ws_bytes, dev_err, stream);
}

csa2_status csa2_sparse_attn_decode_append_rope(
    const csa2_global_kv *kv, const csa2_swa *swa, const void *swa_bf16, const void *q_bf16,
    const int32_t *q_pos, int32_t Tq, int32_t H, const int32_t *topk, int32_t top_k,
    int32_t swa_len, float softmax_scale, const csa2_rope *rope, float *out, float *lse,
    void *workspace, size_t ws_bytes, int32_t *dev_err, csa2_stream_t stream) {
    (void)workspace;
    (void)ws_bytes;
    if (Tq != 1) return CSA2_ERR_UNSUPPORTED;
    if (swa_len <= 0 || !swa || !swa_bf16) return CSA2_ERR_INVALID_ARG;
    if (!aligned(swa_bf16, 16)) return CSA2_ERR_INVALID_ARG;
    KvView v;
    return sparse_attn(view_of(kv, &v), swa, swa_bf16, q_bf16, q_pos, Tq, H, topk, top_k, swa_len,
                       softmax_scale, rope, out, lse, dev_err, stream);
}

csa2_status csa2_sparse_attn_decode_reuse(const csa2_global_kv *kv, const csa2_swa *swa,
                                          const void *swa_bf16, const void *q_bf16,
                                          const int32_t *q_pos, int32_t Tq, int32_t H,
                                          const int32_t *topk, int32_t top_k, int32_t swa_len,
                                          float softmax_scale, const csa2_rope *rope, float *out,
                                          float *lse, int32_t *dev_err, csa2_stream_t stream) {
    if (swa_bf16) {
        if (Tq != 1) return CSA2_ERR_UNSUPPORTED;
        if (swa_len <= 0 || !swa || !aligned(swa_bf16, 16)) return CSA2_ERR_INVALID_ARG;
    } else if (rope) {
        return CSA2_ERR_INVALID_ARG;
    }
    KvView v;
    return sparse_attn(view_of(kv, &v), swa, swa_bf16, q_bf16, q_pos, Tq, H, topk, top_k, swa_len,
                       softmax_scale, rope, out, lse, dev_err, stream, true);
}

// ---- paged cache: the same calls over a csa2_paged_kv ----------------------------------
csa2_status csa2_quantize_append_paged(const csa2_paged_kv *kv, const void *kv_bf16,
                                       const void *idxk_bf16, int32_t T_kv, const int32_t *kv_start,
                                       const csa2_swa *swa, const void *swa_bf16, int32_t T_swa,
                                       const int32_t *swa_start, const csa2_rope *rope,
                                       int32_t *dev_err, csa2_stream_t stream) {
    KvView v;
    const KvView *pv;
    csa2_status st = paged_view(kv, &v, &pv);
    if (st != CSA2_OK) return st;
    return quantize_append(pv, kv_bf16, idxk_bf16, T_kv, kv_start, swa, swa_bf16, T_swa, swa_start,
                           rope, dev_err, stream);
}

csa2_status csa2_index_full_paged(const csa2_paged_kv *kv, const void *q_idx_bf16, const float *w,
                                  const int32_t *q_pos, int32_t Tq, int32_t H_I, int32_t n_max,
                                  int32_t pool_blocks, int32_t top_k, int32_t *pool_out,
                                  int32_t *topk_out, int32_t *topk_count, void *workspace,
                                  size_t ws_bytes, int32_t *dev_err, csa2_stream_t stream) {
    KvView v;
    const KvView *pv;
    csa2_status st = paged_view(kv, &v, &pv);
    if (st != CSA2_OK) return st;
    return index_full(pv, q_idx_bf16, w, q_pos, Tq, H_I, n_max, pool_blocks, top_k, pool_out, topk_out,
                      topk_count, workspace, ws_bytes, dev_err, stream, false);
}

static csa2_status reindex_paged(const csa2_paged_kv *kv, const void *q_idx_bf16, const float *w,
                                 const int32_t *q_pos, int32_t Tq, int32_t H_I, const int32_t *pool,
                                 int32_t pool_blocks, int32_t top_k, int32_t *topk_out,
                                 int32_t *topk_count, void *workspace, size_t ws_bytes,
                                 int32_t *dev_err, csa2_stream_t stream, bool settled) {
    KvView v;
    const KvView *pv;
    csa2_status st = paged_view(kv, &v, &pv);
    if (st != CSA2_OK) return st;
    return index_reindex(pv, q_idx_bf16, w, q_pos, Tq, H_I, pool, pool_blocks, top_k, topk_out,
                         topk_count, workspace, ws_bytes, dev_err, stream, settled);
}

csa2_status csa2_index_reindex_paged(const csa2_paged_kv *kv, const void *q_idx_bf16, const float *w,
                                     const int32_t *q_pos, int32_t Tq, int32_t H_I, const int32_t *pool,
                                     int32_t pool_blocks, int32_t top_k, int32_t *topk_out,
                                     int32_t *topk_count, void *workspace, size_t ws_bytes,
                                     int32_t *dev_err, csa2_stream_t stream) {
    return reindex_paged(kv, q_idx_bf16, w, q_pos, Tq, H_I, pool, pool_blocks, top_k, topk_out, topk_count,
                         workspace, ws_bytes, dev_err, stream, false);
}

csa2_status csa2_index_reindex_paged_settled(const csa2_paged_kv *kv, const void *q_idx_bf16,
                                             const float *w, const int32_t *q_pos, int32_t Tq,
                                             int32_t H_I, const int32_t *pool, int32_t pool_blocks,
                                             int32_t top_k, int32_t *topk_out, int32_t *topk_count,
                                             void *workspace, size_t ws_bytes, int32_t *dev_err,
                                             csa2_stream_t stream) {
    return reindex_paged(kv, q_idx_bf16, w, q_pos, Tq, H_I, pool, pool_blocks, top_k, topk_out, topk_count,
                         workspace, ws_bytes, dev_err, stream, true);
}

static csa2_status attn_paged(const csa2_paged_kv *kv, const csa2_swa *swa, const void *swa_bf16,
                              const void *q_bf16, const int32_t *q_pos, int32_t Tq, int32_t H,
                              const int32_t *topk, int32_t top_k, int32_t swa_len, float softmax_scale,
                              const csa2_rope *rope, float *out, float *lse, int32_t *dev_err,
                              csa2_stream_t stream, bool settled) {
    KvView v;
    const KvView *pv;
    csa2_status st = paged_view(kv, &v, &pv);
    if (st != CSA2_OK) return st;
    if (swa_bf16) {
        if (Tq != 1) return CSA2_ERR_UNSUPPORTED;
        if (swa_len <= 0 || !swa) return CSA2_ERR_INVALID_ARG;
        if (!aligned(swa_bf16, 16)) return CSA2_ERR_INVALID_ARG;
    } else if (rope) {
        return CSA2_ERR_INVALID_ARG;
    }
    return sparse_attn(pv, swa, swa_bf16, q_bf16, q_pos, Tq, H, topk, top_k, swa_len, softmax_scale,
                       rope, out, lse, dev_err, stream, settled);
}

csa2_status csa2_sparse_attn_decode_paged(const csa2_paged_kv *kv, const csa2_swa *swa,
                                          const void *swa_bf16, const void *q_bf16,
                                          const int32_t *q_pos, int32_t Tq, int32_t H,
                                          const int32_t *topk, int32_t top_k, int32_t swa_len,
                                          float softmax_scale, const csa2_rope *rope, float *out,
                                          float *lse, int32_t *dev_err, csa2_stream_t stream) {
    return attn_paged(kv, swa, swa_bf16, q_bf16, q_pos, Tq, H, topk, top_k, swa_len, softmax_scale, rope, out,
                      lse, dev_err, stream, false);
}

csa2_status csa2_sparse_attn_decode_paged_reuse(const csa2_paged_kv *kv, const csa2_swa *swa,
                                                const void *swa_bf16, const void *q_bf16,
                                                const int32_t *q_pos, int32_t Tq, int32_t H,
                                                const int32_t *topk, int32_t top_k, int32_t swa_len,
                                                float softmax_scale, const csa2_rope *rope, float *out,
                                                float *lse, int32_t *dev_err, csa2_stream_t stream) {
    return attn_paged(kv, swa, swa_bf16, q_bf16, q_pos, Tq, H, topk, top_k, swa_len, softmax_scale, rope, out,
                      lse, dev_err, stream, true);
}

csa2_status csa2_read_device_error(int32_t *dev_err, int32_t *bits_out, csa2_stream_t stream) {
    if (!dev_err) return CSA2_ERR_INVALID_ARG;
    int32_t bits = 0;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&bits, dev_err, sizeof(bits), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return launched(cudaErrorUnknown);
    if (cudaMemsetAsync(dev_err, 0, sizeof(int32_t), s) != cudaSuccess) return launched(cudaErrorUnknown);
    if (cudaStreamSynchronize(s) != cudaSuccess) return launched(cudaErrorUnknown);
    if (bits_out) *bits_out = bits;
    return bits ? CSA2_ERR_DEVICE_BOUNDS : CSA2_OK;
}

}  // extern "C"
