// csa2_attn.cu -- a8 sparse decode attention over FP4 entries + the FP8 SWA window.
//
// DeepSeek V4.1 Flash study notes, sections 1, 2 and 4: each layer attends, with
// its own query, over at most 512 selected global entries (FP4, dequantised on
// read -- "saves storage, does not make the attention matmul FP4") together with
// its own 128-token FP8 window.  K = V = the 512-channel entry (MQA, fixed for
// this build); one softmax over the union.
//
// Design: one CTA per (query, group of 32 heads), 8 warps.  Keys stream through
// shared memory in tiles of 32: a cp.async gather of the raw rows (double
// buffered), a dequantisation pass that writes K as bf16 and V as fp16 (both
// exact for FP4: e2m1 x e4m3 has at most 6 significant bits; the SWA V row is
// rounded once to fp16), then tensor-core tiles: S = Q K^T with bf16 operands
// and P V with fp16 operands, fp32 accumulation, online softmax in fp32.
// Warp (hg, cq) keeps Q[16 heads x 128 channels] in registers for S and owns
// O[16 heads x 128 channels] for P V; the four channel quarters of S are summed
// through shared memory in a fixed order.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

constexpr int kAttnThreads = 256;
constexpr int kHeadsCta = 32;
constexpr int kKeyTile = 32;
constexpr int kRawRow = 512;
constexpr int kPRow = kKeyTile + 8;   // padded fp16 row of P (80 bytes)

struct AttnSmem {
    uint8_t k[kKeyTile * 1024];           // bf16 [key][512], 16-byte units swizzled
    uint8_t v[kKeyTile * 1024];           // fp16 [key][512], same layout
    uint8_t raw[2][kKeyTile * kRawRow];   // gathered rows
    float s[4][kHeadsCta][kKeyTile];      // partial logits per channel quarter
    uint16_t p[kHeadsCta][kPRow];         // fp16 probabilities
    float alpha[kHeadsCta];
    float sigma[2][kKeyTile];
    int kind[2][kKeyTile];                // 0 none, 1 FP4 entry, 2 SWA row
    float lfin[kHeadsCta];
    float mfin[kHeadsCta];
};

__device__ __forceinline__ int kswz(int key, int unit) { return unit ^ (key & 7); }

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem));
}

__device__ __forceinline__ void ldsm_x4(uint32_t *r, const void *p) {
    uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t *r, const void *p) {
    uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}

__device__ __forceinline__ void mma_bf16(float *c, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float *c, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t f2_to_bf16x2(float2 f) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t f2_to_f16x2(float2 f) {
    __half2 h = __floats2half2_rn(f.x, f.y);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float2 f16x2_to_f2(uint32_t w) {
    return __half22float2(*reinterpret_cast<__half2 *>(&w));
}

struct KeyList {
    const int32_t *topk;   // this query's ids
    int top_k;
    int64_t w0;            // first window position
    int n_keys;            // top_k + window length
    int64_t n_vis;         // entries visible to the query
};

// Issue the cp.async gather of key tile `tile` into raw buffer `buf`.
__device__ __forceinline__ void gather_tile(AttnSmem &s, const AttnArgs &a, const KeyList &kl,
                                            int b, int tile, int buf) {
    const int row = threadIdx.x >> 3, sub = threadIdx.x & 7;
    const int kg = tile * kKeyTile + row;
    int kind = 0;
    float sigma = 0.0f;
    const uint8_t *src_codes = nullptr;
    const uint8_t *src_scales = nullptr;
    if (kg < kl.top_k) {
        int e = kl.topk[kg];
        if (e >= 0 && e < kl.n_vis) {
            kind = 1;
            sigma = 1.0f;
            int64_t off = (int64_t)b * a.cap + e;
            src_codes = a.codes + off * kCodeBytes;
            src_scales = a.scales + off * kScaleBytes;
        } else if (e >= 0 && sub == 0) {
            set_dev_err(a.dev_err, CSA2_DEVERR_INDEX);
        }
    } else if (kg < kl.n_keys) {
        int64_t pos = kl.w0 + (kg - kl.top_k);
        int64_t slot = (int64_t)b * a.wcap + pos % a.wcap;
        kind = 2;
        sigma = a.swa_scale[slot];
        src_codes = a.swa_codes + slot * kDim;
    }
    uint8_t *dst = s.raw[buf] + row * kRawRow;
    if (kind == 1) {
        for (int u = sub; u < 18; u += 8)
            cp_async16(dst + 16 * u, u < 16 ? src_codes + 16 * u : src_scales + 16 * (u - 16));
    } else if (kind == 2) {
        for (int u = sub; u < 32; u += 8) cp_async16(dst + 16 * u, src_codes + 16 * u);
    }
    if (sub == 0) {
        s.kind[buf][row] = kind;
        s.sigma[buf][row] = sigma;
    }
    asm volatile("cp.async.commit_group;\n");
}

// Dequantise raw buffer `buf` into s.k (bf16) and s.v (fp16).  Thread = (key row,
// 64-channel part).
__device__ __forceinline__ void dequant_tile(AttnSmem &s, const AttnArgs &a, int buf) {
    const int row = threadIdx.x >> 3, part = threadIdx.x & 7;
    const int kind = s.kind[buf][row];
    const uint8_t *raw = s.raw[buf] + row * kRawRow;
    uint8_t *krow = s.k + row * 1024;
    uint8_t *vrow = s.v + row * 1024;
    if (kind == 1) {
        const uint4 c0 = *reinterpret_cast<const uint4 *>(raw + 32 * part);
        const uint4 c1 = *reinterpret_cast<const uint4 *>(raw + 32 * part + 16);
        const uint32_t sc4 = *reinterpret_cast<const uint32_t *>(raw + 256 + 4 * part);
        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int g = 0; g < 4; ++g) {              // 16-channel scale group
            uint32_t sb = (sc4 >> (8 * g)) & 0xFFu;
            uint32_t sh = cvt_e4m3x2_f16x2(sb | (sb << 8));
            __half2 scale2 = *reinterpret_cast<__half2 *>(&sh);
#pragma unroll
            for (int hu = 0; hu < 2; ++hu) {       // 8-channel unit
                uint32_t vals[4];
                cvt_e2m1x8_f16x2(cw[2 * g + hu], vals);
                uint32_t vv[4], kk[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    __half2 v2 = __hmul2(*reinterpret_cast<__half2 *>(&vals[j]), scale2);
                    vv[j] = *reinterpret_cast<uint32_t *>(&v2);
                    kk[j] = f2_to_bf16x2(__half22float2(v2));
                }
                const int unit = 8 * part + 2 * g + hu;
                *reinterpret_cast<uint4 *>(vrow + 16 * kswz(row, unit)) = make_uint4(vv[0], vv[1], vv[2], vv[3]);
                *reinterpret_cast<uint4 *>(krow + 16 * kswz(row, unit)) = make_uint4(kk[0], kk[1], kk[2], kk[3]);
            }
        }
    } else if (kind == 2) {
        const float sigma = s.sigma[buf][row];
        if (part == 0 && sigma * 448.0f > 65504.0f) set_dev_err(a.dev_err, CSA2_DEVERR_RANGE);
#pragma unroll
        for (int q = 0; q < 4; ++q) {              // 16 channels per load
            const uint4 c = *reinterpret_cast<const uint4 *>(raw + 64 * part + 16 * q);
            const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int hu = 0; hu < 2; ++hu) {
                uint32_t vv[4], kk[4];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    uint32_t w = cw[2 * hu + j];
                    float2 lo = f16x2_to_f2(cvt_e4m3x2_f16x2(w & 0xFFFFu));
                    float2 hi = f16x2_to_f2(cvt_e4m3x2_f16x2(w >> 16));
                    kk[2 * j] = f2_to_bf16x2(lo);
                    kk[2 * j + 1] = f2_to_bf16x2(hi);
                    vv[2 * j] = f2_to_f16x2(make_float2(lo.x * sigma, lo.y * sigma));
                    vv[2 * j + 1] = f2_to_f16x2(make_float2(hi.x * sigma, hi.y * sigma));
                }
                const int unit = 8 * part + 2 * q + hu;
                *reinterpret_cast<uint4 *>(vrow + 16 * kswz(row, unit)) = make_uint4(vv[0], vv[1], vv[2], vv[3]);
                *reinterpret_cast<uint4 *>(krow + 16 * kswz(row, unit)) = make_uint4(kk[0], kk[1], kk[2], kk[3]);
            }
        }
    } else {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            *reinterpret_cast<uint4 *>(vrow + 16 * (8 * part + u)) = z;
            *reinterpret_cast<uint4 *>(krow + 16 * (8 * part + u)) = z;
        }
    }
}

__global__ void __launch_bounds__(kAttnThreads, 1)
sparse_attn_kernel(AttnArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    AttnSmem &s = *reinterpret_cast<AttnSmem *>(smem_raw);
    const int qi = blockIdx.y;
    const int b = qi / a.Tq;
    const int h0 = blockIdx.x * kHeadsCta;
    const int hcta = min(kHeadsCta, a.H - h0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hg = warp & 1, cq = warp >> 1;
    const int g = lane >> 2, t4 = lane & 3;
    const bool hg_on = 16 * hg < hcta;

    const int64_t t = a.q_pos[qi];
    KeyList kl;
    kl.topk = a.topk + (int64_t)qi * a.top_k;
    kl.top_k = a.top_k;
    kl.w0 = max64(0, t - a.swa_len + 1);
    const int n_win = a.swa_len > 0 ? (int)(t - kl.w0 + 1) : 0;
    kl.n_keys = a.top_k + n_win;
    kl.n_vis = min64(visible_entries((int32_t)t, a.ratio), a.cap);
    const int n_tiles = (kl.n_keys + kKeyTile - 1) / kKeyTile;

    if (n_tiles > 0) gather_tile(s, a, kl, b, 0, 0);

    // Q fragments: heads h0 + 16 hg + {g, g+8}, channels 128 cq + 16 ks + ...
    uint32_t qa[8][4];
    {
        const uint16_t *q = a.q + ((int64_t)qi * a.H + h0 + 16 * hg) * kDim + 128 * cq;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const int c = 16 * ks + 2 * t4;
            qa[ks][0] = hg_on ? *reinterpret_cast<const uint32_t *>(q + g * kDim + c) : 0u;
            qa[ks][1] = hg_on ? *reinterpret_cast<const uint32_t *>(q + (g + 8) * kDim + c) : 0u;
            qa[ks][2] = hg_on ? *reinterpret_cast<const uint32_t *>(q + g * kDim + c + 8) : 0u;
            qa[ks][3] = hg_on ? *reinterpret_cast<const uint32_t *>(q + (g + 8) * kDim + c + 8) : 0u;
        }
    }
    float oacc[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.0f;

    // softmax state of head (threadIdx.x >> 3), replicated over its 8 threads
    const int sm_h = threadIdx.x >> 3, sm_part = threadIdx.x & 7;
    float m_run = -INFINITY, l_run = 0.0f;
    const float log2e = 1.4426950408889634f;

    for (int tile = 0; tile < n_tiles; ++tile) {
        const int buf = tile & 1;
        asm volatile("cp.async.wait_all;\n" ::: "memory");
        __syncthreads();
        if (tile + 1 < n_tiles) gather_tile(s, a, kl, b, tile + 1, buf ^ 1);
        dequant_tile(s, a, buf);
        __syncthreads();

        // ---- S partial = Q[16 heads x 128 ch] K[32 keys x 128 ch]^T ----
        if (hg_on) {
            float sacc[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.0f;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int mi = lane >> 3, ri = lane & 7;
                    const int key = 8 * nt + ri;
                    const int unit = 16 * cq + 4 * kk + mi;
                    uint32_t bf[4];
                    ldsm_x4(bf, s.k + key * 1024 + 16 * kswz(key, unit));
                    mma_bf16(sacc[nt], qa[2 * kk], bf[0], bf[1]);
                    mma_bf16(sacc[nt], qa[2 * kk + 1], bf[2], bf[3]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                *reinterpret_cast<float2 *>(&s.s[cq][16 * hg + g][8 * nt + 2 * t4]) =
                    make_float2(sacc[nt][0], sacc[nt][1]);
                *reinterpret_cast<float2 *>(&s.s[cq][16 * hg + g + 8][8 * nt + 2 * t4]) =
                    make_float2(sacc[nt][2], sacc[nt][3]);
            }
        }
        __syncthreads();

        // ---- online softmax: head sm_h, keys 4 sm_part .. +3 ----
        {
            float lg[4];
            float tmax = -INFINITY;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int key = 4 * sm_part + j;
                const int kind = s.kind[buf][key];
                float v = ((s.s[0][sm_h][key] + s.s[1][sm_h][key]) + s.s[2][sm_h][key]) +
                          s.s[3][sm_h][key];
                lg[j] = kind ? v * (a.softmax_scale * log2e * s.sigma[buf][key]) : -INFINITY;
                tmax = fmaxf(tmax, lg[j]);
            }
            tmax = fmaxf(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, 1));
            tmax = fmaxf(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, 2));
            tmax = fmaxf(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, 4));
            const float m_new = fmaxf(m_run, tmax);
            float alpha = 1.0f, psum = 0.0f;
            float p[4];
            if (m_new == -INFINITY) {
                p[0] = p[1] = p[2] = p[3] = 0.0f;
            } else {
                alpha = exp2f(m_run - m_new);
#pragma unroll
                for (int j = 0; j < 4; ++j) { p[j] = exp2f(lg[j] - m_new); psum += p[j]; }
            }
            psum += __shfl_xor_sync(0xFFFFFFFFu, psum, 1);
            psum += __shfl_xor_sync(0xFFFFFFFFu, psum, 2);
            psum += __shfl_xor_sync(0xFFFFFFFFu, psum, 4);
            l_run = l_run * alpha + psum;
            m_run = m_new;
            __half2 p01 = __floats2half2_rn(p[0], p[1]);
            __half2 p23 = __floats2half2_rn(p[2], p[3]);
            *reinterpret_cast<uint2 *>(&s.p[sm_h][4 * sm_part]) =
                make_uint2(*reinterpret_cast<uint32_t *>(&p01), *reinterpret_cast<uint32_t *>(&p23));
            if (sm_part == 0) s.alpha[sm_h] = alpha;
        }
        __syncthreads();

        // ---- O[16 heads x 128 ch] = alpha * O + P[16 x 32] V[32 x 128] ----
        if (hg_on) {
            const float al = s.alpha[16 * hg + g], ah = s.alpha[16 * hg + g + 8];
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                oacc[nt][0] *= al; oacc[nt][1] *= al;
                oacc[nt][2] *= ah; oacc[nt][3] *= ah;
            }
            const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                uint32_t pa[4];
                ldsm_x4(pa, &s.p[16 * hg + ri + 8 * (mi & 1)][16 * ks + 8 * (mi >> 1)]);
#pragma unroll
                for (int np = 0; np < 8; ++np) {
                    const int key = 16 * ks + ri + 8 * (mi & 1);
                    const int unit = 16 * cq + 2 * np + (mi >> 1);
                    uint32_t vb[4];
                    ldsm_x4_t(vb, s.v + key * 1024 + 16 * kswz(key, unit));
                    mma_f16(oacc[2 * np], pa, vb[0], vb[1]);
                    mma_f16(oacc[2 * np + 1], pa, vb[2], vb[3]);
                }
            }
        }
    }

    if (sm_part == 0) {
        s.lfin[sm_h] = l_run;
        s.mfin[sm_h] = m_run;
    }
    __syncthreads();
    if (hg_on) {
        const int ha = 16 * hg + g, hb = ha + 8;
        const float la = s.lfin[ha], lb = s.lfin[hb];
        const float ia = la > 0.0f ? 1.0f / la : 0.0f;
        const float ib = lb > 0.0f ? 1.0f / lb : 0.0f;
        float *oa = a.out + ((int64_t)qi * a.H + h0 + ha) * kDim + 128 * cq;
        float *ob = a.out + ((int64_t)qi * a.H + h0 + hb) * kDim + 128 * cq;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            *reinterpret_cast<float2 *>(oa + 8 * nt + 2 * t4) = make_float2(oacc[nt][0] * ia, oacc[nt][1] * ia);
            *reinterpret_cast<float2 *>(ob + 8 * nt + 2 * t4) = make_float2(oacc[nt][2] * ib, oacc[nt][3] * ib);
        }
    }
    if (threadIdx.x < hcta) {
        const float l = s.lfin[threadIdx.x], m = s.mfin[threadIdx.x];
        a.lse[(int64_t)qi * a.H + h0 + threadIdx.x] =
            l > 0.0f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
}

cudaError_t launch_sparse_attn(const AttnArgs &a, int BT, cudaStream_t st) {
    size_t smem = sizeof(AttnSmem);
    static bool attr_set = false;  // once per process (one device per process)
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid((a.H + kHeadsCta - 1) / kHeadsCta, BT);
    sparse_attn_kernel<<<grid, kAttnThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace csa2
