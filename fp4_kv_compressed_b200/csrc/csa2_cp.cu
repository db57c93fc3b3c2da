// csa2_cp.cu -- context parallel: the combine of partial attention results.
//
// DeepSeek V4.1 Flash study notes, section 2 (report Figure 5): the Full-layer scan
// is the only per-query cost that grows with the context, so a single long request is
// split by entry range across GPUs.  Each shard attends over the selected entries it
// holds (and the shard holding the window, over the window too) and returns a
// normalised partial output o_s with its log-sum-exp lse_s.  The softmax over the
// union is recovered exactly (up to rounding) by
//   lse = log sum_s exp(lse_s),   o = sum_s exp(lse_s - lse) o_s,
// parts with lse_s = -inf contributing nothing.  One thread per 4 channels of a row.
#include <stdint.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

__global__ void __launch_bounds__(256)
attn_combine_kernel(const float *o_parts, const float *lse_parts, int n_parts, int64_t rows,
                    float *out, float *lse_out) {
    grid_dep_wait();
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = t / (kDim / 4);
    if (row >= rows) return;
    const int c4 = (int)(t % (kDim / 4));
    float m = -INFINITY;
    for (int p = 0; p < n_parts; ++p) m = fmaxf(m, __ldg(lse_parts + (int64_t)p * rows + row));
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float l = 0.0f;
    if (m != -INFINITY) {
        for (int p = 0; p < n_parts; ++p) {
            const float lp = __ldg(lse_parts + (int64_t)p * rows + row);
            if (lp == -INFINITY) continue;
            const float wgt = __expf(lp - m);
            l += wgt;
            const float4 o = __ldg(reinterpret_cast<const float4 *>(o_parts + ((int64_t)p * rows + row) * kDim) + c4);
            acc.x = fmaf(wgt, o.x, acc.x);
            acc.y = fmaf(wgt, o.y, acc.y);
            acc.z = fmaf(wgt, o.z, acc.z);
            acc.w = fmaf(wgt, o.w, acc.w);
        }
        const float inv = 1.0f / l;
        acc.x *= inv;
        acc.y *= inv;
        acc.z *= inv;
        acc.w *= inv;
    }
    grid_dep_launch();
    reinterpret_cast<float4 *>(out + row * kDim)[c4] = acc;
    if (c4 == 0) lse_out[row] = m == -INFINITY ? -INFINITY : m + logf(l);
}

cudaError_t launch_attn_combine(const float *o_parts, const float *lse_parts, int n_parts, int64_t rows,
                                float *out, float *lse_out, cudaStream_t st) {
    const int64_t threads = rows * (kDim / 4);
    if (threads == 0) return cudaSuccess;
    static std::atomic<uint64_t> configured{0};   // per device
    {
        cudaError_t e = config_kernel_once(attn_combine_kernel, 0, configured);
        if (e != cudaSuccess) return e;
    }
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    cudaError_t e = launch_pdl(attn_combine_kernel, dim3(blocks), dim3(256), 0, st, o_parts, lse_parts,
                               n_parts, rows, out, lse_out);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace csa2
