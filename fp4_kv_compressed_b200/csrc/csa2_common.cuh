// csa2_common.cuh -- shared device helpers of libcsa2 (number formats, order keys).
//
// Formats (DeepSeek V4.1 Flash study notes, section 4; myzaker "cache precision
// and tiering"): the main KV is E2M1 with one E4M3 scale per 16 channels; the
// SWA window and the indexer K are E4M3 with one fp32 scale per token.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "csa2.h"

namespace csa2 {

constexpr int kDim = CSA2_KV_DIM;          // 512-channel K=V entry
constexpr int kCodeBytes = kDim / 2;       // 256 B of E2M1 codes per entry
constexpr int kScaleBytes = kDim / 16;     // 32 E4M3 scales per entry

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) {
    return __uint_as_float(h << 16);
}

// Eight fp32 values -> four bytes of E2M1 codes, round-to-nearest-even with
// saturation; value 2j goes to the low nibble of byte j.  (cvt puts its first
// source in the upper half.)
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float *v) {
    uint32_t out;
    asm("{\n.reg .b8 b0, b1, b2, b3;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
        "mov.b32 %0, {b0, b1, b2, b3};\n}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
          "f"(v[7]));
    return out;
}

// Two fp32 values -> two E4M3 bytes (lo in the low byte), RNE, saturating.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(out) : "f"(lo), "f"(hi));
    return out;
}

// Exact E4M3 -> fp32.  The code's 7 magnitude bits placed at fp32 bit 20 give
// the value times 2^-120 (the E4M3 subnormals land on fp32 subnormals), so one
// exact multiply by 2^120 finishes it.  Needs denormals preserved (no FTZ).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    uint32_t bits = ((b & 0x7Fu) << 20) | ((b & 0x80u) << 24);
    return __uint_as_float(bits) * 0x1p120f;
}

// Two E4M3 bytes (low 16 bits of w) -> f16x2, exact (low byte -> low half).
__device__ __forceinline__ uint32_t cvt_e4m3x2_f16x2(uint32_t w) {
    uint32_t out;
    uint16_t in = (uint16_t)w;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(out) : "h"(in));
    return out;
}

// Four bytes of E2M1 codes -> four f16x2 words (exact), byte j -> word j.
__device__ __forceinline__ void cvt_e2m1x8_f16x2(uint32_t w, uint32_t *out) {
    asm("{\n.reg .b8 b0, b1, b2, b3;\n"
        "mov.b32 {b0, b1, b2, b3}, %4;\n"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
        : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
        : "r"(w));
}

// d = a * b + c on two fp32 lanes, each lane an IEEE fma (round to nearest even).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(reinterpret_cast<unsigned long long &>(d))
        : "l"(reinterpret_cast<unsigned long long &>(a)),
          "l"(reinterpret_cast<unsigned long long &>(b)),
          "l"(reinterpret_cast<unsigned long long &>(c)));
    return d;
}

// Order key of a score: larger score -> larger key; -0 == +0; NaN -> 1 (below
// every number); 0 is reserved for "not a candidate".
__device__ __forceinline__ uint32_t score_key(float f) {
    if (f != f) return 1u;
    uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

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

// FP8 row of WIDTH channels (64, 128 or 512), one warp: sigma = amax / 448 (IEEE
// division), codes = E4M3_RNE_satfinite(x / sigma), a zero row stores zero codes.
// quant_fp8_lanes takes the lane's PER = WIDTH / 32 consecutive channels already in
// registers (lane l holds channels PER l ..); quant_fp8_row loads them first.
template <int WIDTH>
__device__ void quant_fp8_lanes(const float *x, uint8_t *dst_codes, float *dst_scale, int lane) {
    constexpr int PER = WIDTH / 32;      // channels per lane: 2, 4 or 16
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
    quant_fp8_lanes<WIDTH>(x, dst_codes, dst_scale, lane);
}

// RoPE of one 512-channel row inside the append (csa2_rope): lane l holds channels
// [16 l, 16 l + 16) as fp32 in x; the rotated pairs among them become
//   y0 = fma(x0, c, -(x1 * s)),  y1 = fma(x0, s, x1 * c),
// with (c, s) = cs[pos][i] for pair i = (channel - start) / 2, each rounded to bf16.
// cs == nullptr rotates nothing; a position outside [0, n_pos) rotates nothing and
// returns false.
__device__ __forceinline__ bool rope_lane16(float *x, int lane, const float2 *cs, int n_pos,
                                            int start, int pairs, int64_t pos) {
    if (cs == nullptr) return true;
    if (pos < 0 || pos >= n_pos) return false;
    const float2 *row = cs + pos * pairs;
    float2 t[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {             // every table load in flight together
        const int ch = 16 * lane + 2 * k;
        t[k] = ch >= start && ch < start + 2 * pairs ? __ldg(row + ((ch - start) >> 1))
                                                      : make_float2(1.0f, 0.0f);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int ch = 16 * lane + 2 * k;
        if (ch >= start && ch < start + 2 * pairs) {
            const float x0 = x[2 * k], x1 = x[2 * k + 1];
            const float y0 = fmaf(x0, t[k].x, -__fmul_rn(x1, t[k].y));
            const float y1 = fmaf(x0, t[k].y, __fmul_rn(x1, t[k].x));
            x[2 * k] = __bfloat162float(__float2bfloat16_rn(y0));
            x[2 * k + 1] = __bfloat162float(__float2bfloat16_rn(y1));
        }
    }
    return true;
}

// Programmatic dependent launch.  Every kernel of the library is launched so that the
// next kernel of the stream may be scheduled while it finishes: grid_dep_wait() blocks
// until the previous grid has completed with its memory visible (each kernel calls it
// before its first global memory access), grid_dep_launch() lets the next grid start
// launching (called once a CTA's main work is done).
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void set_dev_err(int32_t *dev_err, int bit) {
    if (dev_err) atomicOr(dev_err, bit);
}

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// Row of entry e of request b in the cache planes (see PageMap): -1 when the block
// table names a page outside [0, n_pages) (the caller skips the entry and flags it).
template <class PM>
__device__ __forceinline__ int64_t cache_row(const PM &pm, int64_t cap, int64_t b, int64_t e) {
    if (pm.table == nullptr) return b * cap + e;
    const int32_t pg = __ldg(pm.table + b * pm.max_pages + (e >> pm.shift));
    if (pg < 0 || pg >= pm.n_pages) return -1;
    return ((int64_t)pg << pm.shift) | (e & (((int64_t)1 << pm.shift) - 1));
}

__device__ __forceinline__ int64_t visible_entries(int32_t t, int32_t ratio) {
    return t < 0 ? 0 : ((int64_t)t + 1) / ratio;
}

}  // namespace csa2
