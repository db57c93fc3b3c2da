// csa2_internal.h -- kernel argument blocks and launchers shared by the .cu files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace csa2 {

// Paged cache: entry e of request b lives in row table[b][e >> shift] << shift |
// (e & (2^shift - 1)) of the planes (pages of 2^shift entries); table == nullptr is the
// contiguous layout, row b * cap + e.
struct PageMap {
    const int32_t *table;     // [batch][max_pages] page ids, or null
    int32_t shift;
    int32_t max_pages;
    int32_t n_pages;
};

// Bounded waits.  Every spin of a kernel on an mbarrier gives up after `limit_ns` of
// wall time (%globaltimer); the kernel then flags CSA2_DEVERR_TIMEOUT, waits (bounded
// by kDrainLimitNs) for the tensor-core work and copies it has in flight, frees its
// TMEM and returns.  `stuck` is a test hook: with it set, the instrumented kernels'
// first wait of every CTA is on a barrier that nothing ever signals, so that wait
// always runs out.  Both come from csa2_debug_set_waits (defaults 0.5 s, off).
struct WaitCfg {
    uint64_t limit_ns;
    int32_t stuck;
};
constexpr uint64_t kDefaultWaitLimitNs = 500000000ull;
constexpr uint64_t kDrainLimitNs = 500000000ull;
WaitCfg current_wait_cfg();

// RoPE table of the _rope calls (cs == nullptr: no rotation); see csa2_rope.
struct RopeArgs {
    const float2 *cs;        // [n_pos][pairs] (cos, sin)
    int32_t n_pos;
    int32_t start;
    int32_t pairs;
};

struct QuantArgs {
    // main KV group (FP4 + FP8 indexer K)
    uint8_t *codes;
    uint8_t *scales;
    uint8_t *idx_codes;
    float *idx_scale;
    int32_t cap;
    int32_t d_idx;
    int32_t ratio;           // main entry in slot e sits at token position ratio * e + ratio - 1
    RopeArgs rope;
    const uint16_t *kv_bf16;
    const uint16_t *idxk_bf16;
    int32_t T_kv;
    const int32_t *kv_start;
    // SWA ring
    uint8_t *swa_codes;
    float *swa_scale;
    int32_t wcap;
    const uint16_t *swa_bf16;
    int32_t T_swa;
    const int32_t *swa_start;
    // work split: warps of each kind
    int64_t n_main, n_idx, n_swa;
    int32_t *dev_err;
    PageMap pm;
};

struct IndexArgs {
    const uint8_t *idx_codes;
    const float *idx_scale;
    int32_t cap;
    int32_t d_idx;
    int32_t ratio;
    const uint16_t *q_idx;   // [BT][H_I][d_idx] bf16 bits
    const float *w;          // [BT][H_I]
    const int32_t *q_pos;    // [BT]
    int32_t Tq;
    int32_t H_I;
    int64_t n_max;
    float *scores;           // workspace [BT][score_stride]
    int64_t score_stride;
    float *bmax;             // workspace [BT][bmax_stride] or null: max of each 8 positions
    int64_t bmax_stride;
    float *bmax64;           // workspace [BT][bmax64_stride] or null: max of each 64 positions
    int64_t bmax64_stride;
    const int32_t *pool;     // reindex input [BT][pool_blocks]
    int32_t pool_blocks;
    int32_t *pool_out;       // full output [BT][pool_blocks] or null
    int32_t top_k;
    int32_t *topk_out;
    int32_t *topk_count;
    int32_t *dev_err;
    WaitCfg wait;
    // slice form (context parallel): the cache holds entries [entry_lo, entry_lo + cap)
    // of each request (entry_lo a multiple of 64; 0 otherwise), and the selections are
    // written as candidate keys (order key << 32 | ~global id) instead of ids
    int64_t entry_lo;
    uint64_t *pool_keys_out;   // [BT][pool_blocks] or null
    uint64_t *topk_keys_out;   // [BT][top_k] or null
    PageMap pm;
    // Reindex scoring: 1 when every input was written at least two launches earlier on
    // the stream; the kernel then waits for the previous launch only before it lets the
    // next one start
    int32_t settled;
};

struct AttnArgs {
    const uint8_t *codes;
    const uint8_t *scales;
    int32_t cap;
    int32_t ratio;
    uint8_t *swa_codes;      // written only by the fused append (swa_new != null)
    float *swa_scale;
    int32_t wcap;
    const uint16_t *swa_new; // fused append: [BT][512] bf16 new SWA row per query (Tq = 1), or null
    RopeArgs rope;           // fused append: RoPE of the new row at its token position
    const uint16_t *q;       // [BT][H][512] bf16 bits
    const int32_t *q_pos;
    int32_t Tq;
    int32_t H;
    const int32_t *topk;     // [BT][top_k]
    int32_t top_k;
    int32_t swa_len;
    float softmax_scale;
    float *out;
    float *lse;
    int32_t *dev_err;
    WaitCfg wait;
    PageMap pm;
    // 1: every input was written at least two launches earlier on the stream (a Reuse
    // layer), so the kernel reads them before its dependency wait and waits only before
    // it lets the next launch start
    int32_t settled;
};

// Every kernel of the library asks for the largest shared-memory carveout, so that
// consecutive kernels of a step never make an SM re-partition L1 and shared memory.
template <class Kernel>
inline cudaError_t prefer_max_smem(Kernel kernel) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                (int)cudaSharedmemCarveoutMaxShared);
}

// Kernel attributes (dynamic shared-memory limit, carveout) belong to a device: a
// launcher sets its kernel's attributes once on every device it launches on.
// `done` holds one bit per device ordinal 0..63 (beyond that the attributes are set
// on every launch).  Two host threads may both set them the first time; that is
// harmless, the calls being idempotent.
template <class Kernel>
inline cudaError_t config_kernel_once(Kernel kernel, size_t dyn_smem, std::atomic<uint64_t> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t)1 << dev : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    if (dyn_smem > 0) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn_smem);
        if (e != cudaSuccess) return e;
    }
    e = prefer_max_smem(kernel);
    if (e != cudaSuccess) return e;
    done.fetch_or(bit, std::memory_order_acq_rel);
    return cudaSuccess;
}

// Number of SMs of the current device (148 on B200 if the query fails).
inline int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        (void)cudaGetLastError();
        n = 148;
    }
    return n;
}

// Launch with programmatic stream serialisation (see grid_dep_wait / grid_dep_launch).
template <class... KArgs, class... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

cudaError_t launch_quantize_append(const QuantArgs &a, cudaStream_t st);
cudaError_t launch_index_scan(const IndexArgs &a, int BT, cudaStream_t st);
cudaError_t launch_index_scan_tc(const IndexArgs &a, int B, cudaStream_t st);
cudaError_t launch_select_full(const IndexArgs &a, int BT, cudaStream_t st);
cudaError_t launch_reindex_score(const IndexArgs &a, int BT, cudaStream_t st);
cudaError_t launch_select_reindex(const IndexArgs &a, int BT, cudaStream_t st);
cudaError_t launch_sparse_attn(const AttnArgs &a, int BT, cudaStream_t st);
cudaError_t launch_index_merge(const uint64_t *lists, int BT, int n_lists, int list_len, int k,
                               int64_t lo, int64_t hi, int32_t *ids_out, int32_t *count_out,
                               int32_t *local_out, cudaStream_t st);
cudaError_t launch_attn_combine(const float *o_parts, const float *lse_parts, int n_parts, int64_t rows,
                                float *out, float *lse_out, cudaStream_t st);

}  // namespace csa2
