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
// One warp per row.  FP4 entry: lane l owns scale group l (16 channels, two
// 16-byte loads) and writes 8 code bytes + 1 scale byte, so a warp writes the
// entry's 256 + 32 bytes with coalesced stores.
#include <stdint.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

__device__ __forceinline__ void unpack_bf16x8(uint4 v, float *x) {
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        x[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

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
    const int64_t e = (int64_t)b * a.cap + slot;
    reinterpret_cast<uint2 *>(a.codes + e * kCodeBytes)[lane] = codes;
    a.scales[e * kScaleBytes + lane] = (uint8_t)s8;
}

// FP8 row of `width` channels (64, 128 or 512), one warp.
template <int WIDTH>
__device__ void quant_fp8_row(const uint16_t *src, uint8_t *dst_codes, float *dst_scale, int lane) {
    constexpr int PER = WIDTH / 32;      // channels per lane: 2, 4 or 16
    float x[PER];
    if constexpr (PER == 16) {
        const uint4 *s4 = reinterpret_cast<const uint4 *>(src + 16 * lane);
        unpack_bf16x8(s4[0], x);
        unpack_bf16x8(s4[1], x + 8);
    } else if constexpr (PER == 4) {
        uint2 v = reinterpret_cast<const uint2 *>(src)[lane];
        x[0] = bf16_bits_to_f32(v.x & 0xFFFFu);
        x[1] = bf16_bits_to_f32(v.x >> 16);
        x[2] = bf16_bits_to_f32(v.y & 0xFFFFu);
        x[3] = bf16_bits_to_f32(v.y >> 16);
    } else {
        uint32_t v = reinterpret_cast<const uint32_t *>(src)[lane];
        x[0] = bf16_bits_to_f32(v & 0xFFFFu);
        x[1] = bf16_bits_to_f32(v >> 16);
    }
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < PER; ++c) amax = fmaxf(amax, fabsf(x[c]));
    amax = warp_max(amax);
    const float sigma = __fdiv_rn(amax, 448.0f);
    uint32_t pk[PER / 2];
#pragma unroll
    for (int j = 0; j < PER / 2; ++j)
        pk[j] = sigma != 0.0f ? cvt_e4m3x2(__fdiv_rn(x[2 * j], sigma), __fdiv_rn(x[2 * j + 1], sigma))
                              : 0u;
    if constexpr (PER == 16) {
        uint4 o = make_uint4(pk[0] | (pk[1] << 16), pk[2] | (pk[3] << 16), pk[4] | (pk[5] << 16),
                             pk[6] | (pk[7] << 16));
        reinterpret_cast<uint4 *>(dst_codes)[lane] = o;
    } else if constexpr (PER == 4) {
        reinterpret_cast<uint32_t *>(dst_codes)[lane] = pk[0] | (pk[1] << 16);
    } else {
        reinterpret_cast<uint16_t *>(dst_codes)[lane] = (uint16_t)pk[0];
    }
    if (lane == 0) *dst_scale = sigma;
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
        const int64_t e = (int64_t)b * a.cap + slot;
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
        quant_fp8_row<512>(a.swa_bf16 + warp * kDim, a.swa_codes + e * kDim, a.swa_scale + e, lane);
    }
}

cudaError_t launch_quantize_append(const QuantArgs &a, cudaStream_t st) {
    int64_t warps = a.n_main + a.n_idx + a.n_swa;
    if (warps == 0) return cudaSuccess;
    int64_t blocks = (warps * 32 + 255) / 256;
    static bool attr_set = false;  // once per process (one device per process)
    if (!attr_set) {
        cudaError_t e = prefer_max_smem(quantize_append_kernel);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    cudaError_t e = launch_pdl(quantize_append_kernel, dim3((unsigned)blocks), dim3(256), 0, st, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace csa2
