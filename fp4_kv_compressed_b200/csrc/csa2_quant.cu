// csa2_quant.cu -- a1/a2 quantise-append of main KV (FP4), indexer K and SWA (FP8).
//
// DeepSeek V4.1 Flash study notes, section 4, and myzaker "cache precision and
// tiering": the main KV cache is E2M1 with one E4M3 scale per 16 channels
// (4 + 8/16 = 4.5 bits per value) and no second-level global scale; it is
// quantised after RoPE.  The more quantisation-sensitive SWA window stays FP8.
// Readings fixed for this build: scale = E4M3_RNE(amax / 6), codes =
// E2M1_RNE(x / scale) with saturation (a zero scale stores zero codes); FP8 rows
// use sigma = amax / 448 and codes = E4M3_RNE(x / sigma).
//
// With a RoPE table (csa2_quantize_append_rope) the main and SWA rows are rotated in
// registers first (rope_lane16), the rotated values rounded to bf16, so the codes are
// those of the plain call given the rotated rows.
//
// One warp per row.  FP4 entry: lane l owns scale group l (16 channels, two
// 16-byte loads) and writes 8 code bytes + 1 scale byte, so a warp writes the
// entry's 256 + 32 bytes with coalesced stores.
#include <stdint.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

__device__ void quant_fp4_entry(const QuantArgs &a, int64_t row, int lane) {
    const int b = (int)(row / a.T_kv), i = (int)(row % a.T_kv);
    const int64_t slot = (int64_t)a.kv_start[b] + i;
    if (slot < 0 || slot >= a.cap) {
        if (lane == 0) set_dev_err(a.dev_err, CSA2_DEVERR_SLOT);
        return;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(a.kv_bf16 + row * kDim + 16 * lane);
    float x[16];
    unpack_bf16x8(src[0], x);
    unpack_bf16x8(src[1], x + 8);
    if (!rope_lane16(x, lane, a.rope.cs, a.rope.n_pos, a.rope.start, a.rope.pairs,
                     slot * a.ratio + a.ratio - 1) && lane == 0)
        set_dev_err(a.dev_err, CSA2_DEVERR_ROPE);
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < 16; ++c) amax = fmaxf(amax, fabsf(x[c]));
    const uint32_t s8 = cvt_e4m3x2(__fdiv_rn(amax, 6.0f), 0.0f) & 0xFFu;
    const float sd = e4m3_to_f32(s8);
    uint2 codes = make_uint2(0u, 0u);
    if (sd != 0.0f) {
        float r[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) r[c] = __fdiv_rn(x[c], sd);
        codes.x = cvt_e2m1x8(r);
        codes.y = cvt_e2m1x8(r + 8);
    }
    const int64_t e = cache_row(a.pm, a.cap, b, slot);
    if (e < 0) {
        if (lane == 0) set_dev_err(a.dev_err, CSA2_DEVERR_PAGE);
        return;
    }
    reinterpret_cast<uint2 *>(a.codes + e * kCodeBytes)[lane] = codes;
    a.scales[e * kScaleBytes + lane] = (uint8_t)s8;
}

__global__ void __launch_bounds__(256) quantize_append_kernel(QuantArgs a) {
    grid_dep_wait();
    grid_dep_launch();
    int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp < a.n_main) {
        quant_fp4_entry(a, warp, lane);
        return;
    }
    warp -= a.n_main;
    if (warp < a.n_idx) {
        const int b = (int)(warp / a.T_kv), i = (int)(warp % a.T_kv);
        const int64_t slot = (int64_t)a.kv_start[b] + i;
        if (slot < 0 || slot >= a.cap) {
            if (lane == 0) set_dev_err(a.dev_err, CSA2_DEVERR_SLOT);
            return;
        }
        const int64_t e = cache_row(a.pm, a.cap, b, slot);
        if (e < 0) {
            if (lane == 0) set_dev_err(a.dev_err, CSA2_DEVERR_PAGE);
            return;
        }
        const uint16_t *src = a.idxk_bf16 + warp * a.d_idx;
        if (a.d_idx == 128)
            quant_fp8_row<128>(src, a.idx_codes + e * 128, a.idx_scale + e, lane);
        else
            quant_fp8_row<64>(src, a.idx_codes + e * 64, a.idx_scale + e, lane);
        return;
    }
    warp -= a.n_idx;
    if (warp < a.n_swa) {
        const int b = (int)(warp / a.T_swa), i = (int)(warp % a.T_swa);
        const int64_t pos = (int64_t)a.swa_start[b] + i;
        if (pos < 0) {
            if (lane == 0) set_dev_err(a.dev_err, CSA2_DEVERR_SLOT);
            return;
        }
        const int64_t e = (int64_t)b * a.wcap + pos % a.wcap;
        const uint4 *src = reinterpret_cast<const uint4 *>(a.swa_bf16 + warp * kDim + 16 * lane);
        float x[16];
        unpack_bf16x8(src[0], x);
        unpack_bf16x8(src[1], x + 8);
        if (!rope_lane16(x, lane, a.rope.cs, a.rope.n_pos, a.rope.start, a.rope.pairs, pos) &&
            lane == 0)
            set_dev_err(a.dev_err, CSA2_DEVERR_ROPE);
        quant_fp8_lanes<512>(x, a.swa_codes + e * kDim, a.swa_scale + e, lane);
    }
}

cudaError_t launch_quantize_append(const QuantArgs &a, cudaStream_t st) {
    int64_t warps = a.n_main + a.n_idx + a.n_swa;
    if (warps == 0) return cudaSuccess;
    int64_t blocks = (warps * 32 + 255) / 256;
    static std::atomic<uint64_t> configured{0};   // per device
    {
        cudaError_t e = config_kernel_once(quantize_append_kernel, 0, configured);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = launch_pdl(quantize_append_kernel, dim3((unsigned)blocks), dim3(256), 0, st, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace csa2
