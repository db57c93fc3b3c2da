// csa2_noalloc.cu -- csa2_index_full_noalloc: the Full-layer index call for callers
// that cannot allocate device memory.
//
// Some hosts own every byte of device memory and give a plugin no way to call
// cudaMalloc (an inference-server backend that must run inside the server's
// execute callback, a runtime with a fixed memory budget), and some loops cannot
// afford cudaMalloc's device-wide synchronisation.  This entry point keeps the
// scratch it needs (per-position scores and block maxima) in a fixed array that
// lives in this library's device image, so the caller passes only inputs and
// outputs.  The array is allocated once per GPU when the library's device code
// is loaded and held until the process exits.
#include <mutex>

#include "csa2.h"

namespace {

__device__ __align__(256) uint8_t g_index_scratch[CSA2_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_index_scratch on the current device.  The first call on a
// device looks it up (this is the set-up step); later calls reuse it.  The host
// name of the array is not a device address and must never reach a kernel.
csa2_status scratch_for_current_device(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        (void)cudaGetLastError();
        return CSA2_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_index_scratch) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return CSA2_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return CSA2_OK;
}

}  // namespace

extern "C" csa2_status csa2_index_full_noalloc(const csa2_global_kv *kv, const void *q_idx_bf16,
                                               const float *w, const int32_t *q_pos, int32_t Tq,
                                               int32_t H_I, int32_t n_max, int32_t pool_blocks,
                                               int32_t top_k, int32_t *pool_out,
                                               int32_t *topk_out, int32_t *topk_count,
                                               int32_t *dev_err, csa2_stream_t stream) {
    if (!kv || kv->batch <= 0 || Tq <= 0 || n_max < 0) return CSA2_ERR_INVALID_ARG;
    const size_t need = csa2_workspace_size(CSA2_OP_INDEX_FULL, kv->batch, Tq, n_max, 0, top_k,
                                            pool_blocks);
    if (need > (size_t)CSA2_NOALLOC_SCRATCH_BYTES) return CSA2_ERR_WORKSPACE;
    void *scratch = nullptr;
    csa2_status st = scratch_for_current_device(&scratch);
    if (st != CSA2_OK) return st;
    return csa2_index_full(kv, q_idx_bf16, w, q_pos, Tq, H_I, n_max, pool_blocks, top_k, pool_out,
                           topk_out, topk_count, scratch, CSA2_NOALLOC_SCRATCH_BYTES, dev_err,
                           stream);
}
