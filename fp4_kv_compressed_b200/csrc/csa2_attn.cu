// csa2_attn_tc.cu -- a8 sparse decode attention on the 5th-generation tensor cores.
//
// DeepSeek V4.1 Flash study notes, sections 1, 2 and 4: each layer attends, with
// its own query, over at most 512 selected global entries (FP4, dequantised on
// read; the cache format saves storage, the attention matmul itself is not FP4)
// together with its own 128-token FP8 SWA window; one softmax over the union.
// K = V = the 512-channel entry (MQA, fixed for this build).
//
// One CTA per (query, group of 64 heads); 16 warps, specialised:
//   warp 0      TMEM allocation + the single MMA-issuing thread;
//   warps 4-7   softmax, one per TMEM lane quadrant (warp w reads lanes 32(w%4)..);
//   warps 8-15  producers: gather the tile's rows (FP4 entry or FP8 SWA row) into
//               registers one tile ahead, dequantise to fp16 into shared memory.
// Data layout: one fp16 tile of 64 keys x 512 channels serves both MMAs -- as the
// K-major B operand of S = Q K^T and as the MN-major B operand of O = P V -- in
// the 128-byte-swizzled layout [channel block of 64][key][128 B].  fp16 holds the
// FP4 values exactly (e2m1 x e4m3 has at most 6 significant bits); an SWA row is
// stored as its exact E4M3 codes and its scale sigma is applied in fp32, to the
// logit and folded into P for the P V product.  Q is converted to fp16 after an exact
// power-of-two scaling that keeps max|q| below 2^15.
// TMEM (512 columns): O = 64 x 512 fp32 in lanes 0-15 of each quadrant (M = 64
// layout), the two S buffers (64 x 64 fp32) at lane offset 16, columns 0..127.
// Online softmax in the log2 domain with lazy rescaling: O is rescaled only when
// a head's running max grows by more than 8 (p stays <= 2^8, safe in fp16).
// Every wait is bounded: on timeout the kernel flags CSA2_DEVERR_TIMEOUT, drains
// its MMAs, frees TMEM and returns.
#include <cuda_fp16.h>
#include <stdint.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {
namespace tc {

constexpr int kThreads = 512;
constexpr int kTK = 64;                        // keys per tile
constexpr int kHeads = 64;                     // heads per CTA (MMA M)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSpinLimit = 1u << 24;      // polls per wait before giving up

struct __align__(1024) Smem {
    uint8_t q[64 * 1024];            // Q fp16, [8 cb][64 heads][128 B] swizzled
    uint8_t kv[2][64 * 1024];        // K=V fp16 tiles, [8 cb][64 keys][128 B] swizzled
    uint8_t p[kHeads * 128];         // P fp16, [64 heads][64 keys] swizzled (K-major)
    int32_t ids[CSA2_TOPK_MAX];      // compacted selected entry ids
    float sig[2][kTK];               // per-key scale of each stage (1 FP4, sigma SWA, 0 none)
    uint64_t kv_full[2], kv_empty[2], s_full[2], p_full, pv_done, drain;
    uint32_t tmem_base;
    int32_t n_sel;
    int32_t abort;
    float qmax[16];
    int32_t warp_cnt[16];
};

// ---- small PTX wrappers ---------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}

// Bounded wait for the phase with the given parity; returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity) {
    uint32_t addr = smem_u32(b);
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n.reg .pred p;\n"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            "selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(addr), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ bool aborted(const Smem &s) {
    return *reinterpret_cast<const volatile int32_t *>(&s.abort) != 0;
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;                  // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                  // 128-byte swizzle
    return d;
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n.reg .pred p;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t *b) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(b))
                 : "memory");
}

// 16 lanes x 32 columns x 2 halves: thread t reads lane (t % 16) at columns
// [col, col+32) for t < 16 and [col + HALF, col + HALF + 32) for t >= 16.
template <int HALF>
__device__ __forceinline__ void tmem_ld16x32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], %33;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr), "n"(HALF));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

template <int HALF>
__device__ __forceinline__ void tmem_st16x32(uint32_t taddr, const float *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], %1, "
        "{%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
        "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33};" ::"r"(taddr),
        "n"(HALF), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
        "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])),
        "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
        "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
        "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
        "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
        "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
        "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

// Byte offset of (row, channel) in a [8 cb][64 rows][128 B] 128B-swizzled fp16 tile.
__device__ __forceinline__ uint32_t tile_off(int row, int ch) {
    int cb = ch >> 6, chunk = (ch >> 3) & 7;
    return (uint32_t)(cb * 8192 + row * 128 + ((chunk ^ (row & 7)) << 4) + ((ch & 7) << 1));
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// ---- producer: raw rows in registers -------------------------------------------------
struct Raw {
    uint4 c[8];      // FP4: c[0..3] = 64 code bytes (128 channels); SWA: 128 code bytes
    uint2 s;         // FP4: 8 scale bytes of the 128 channels
    float sigma;     // SWA scale
    int kind;        // 0 none, 1 FP4 entry, 2 SWA row
};

__device__ __forceinline__ void load_raw(Raw &r, const AttnArgs &a, const Smem &s, int b,
                                         int64_t w0, int n_keys, int tile, int row, int quarter) {
    const int kg = tile * kTK + row;
    r.kind = 0;
    if (kg < s.n_sel) {
        const int e = s.ids[kg];
        const int64_t off = (int64_t)b * a.cap + e;
        const uint4 *src = reinterpret_cast<const uint4 *>(a.codes + off * kCodeBytes + 64 * quarter);
#pragma unroll
        for (int i = 0; i < 4; ++i) r.c[i] = __ldg(src + i);
        r.s = __ldg(reinterpret_cast<const uint2 *>(a.scales + off * kScaleBytes + 8 * quarter));
        r.kind = 1;
    } else if (kg < n_keys) {
        const int64_t pos = w0 + (kg - s.n_sel);
        const int64_t slot = (int64_t)b * a.wcap + pos % a.wcap;
        const uint4 *src = reinterpret_cast<const uint4 *>(a.swa_codes + slot * kDim + 128 * quarter);
#pragma unroll
        for (int i = 0; i < 8; ++i) r.c[i] = __ldg(src + i);
        r.sigma = __ldg(a.swa_scale + slot);
        r.kind = 2;
    }
}

// Dequantise the thread's 128 channels of one key into the fp16 tile.
__device__ __forceinline__ void store_dequant(const Raw &r, uint8_t *tile, int row, int quarter,
                                              int32_t *dev_err) {
    const int ch0 = 128 * quarter;
    if (r.kind == 1) {
        const uint32_t cw[16] = {r.c[0].x, r.c[0].y, r.c[0].z, r.c[0].w, r.c[1].x, r.c[1].y,
                                 r.c[1].z, r.c[1].w, r.c[2].x, r.c[2].y, r.c[2].z, r.c[2].w,
                                 r.c[3].x, r.c[3].y, r.c[3].z, r.c[3].w};
        const uint32_t sc[2] = {r.s.x, r.s.y};
#pragma unroll
        for (int u = 0; u < 16; ++u) {                 // 8 channels per 32-bit code word
            const uint32_t sb = (sc[u >> 3] >> (8 * ((u >> 1) & 3))) & 0xFFu;
            const uint32_t sh = cvt_e4m3x2_f16x2(sb | (sb << 8));
            const __half2 scale2 = *reinterpret_cast<const __half2 *>(&sh);
            uint32_t v[4];
            cvt_e2m1x8_f16x2(cw[u], v);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __half2 x = __hmul2(*reinterpret_cast<__half2 *>(&v[j]), scale2);
                v[j] = *reinterpret_cast<uint32_t *>(&x);
            }
            *reinterpret_cast<uint4 *>(tile + tile_off(row, ch0 + 8 * u)) =
                make_uint4(v[0], v[1], v[2], v[3]);
        }
    } else if (r.kind == 2) {
        // exact E4M3 codes; the row scale is applied in fp32 on the logit and on P
        if (quarter == 0 && r.sigma * 256.0f > 65504.0f) set_dev_err(dev_err, CSA2_DEVERR_RANGE);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w4[4] = {r.c[i].x, r.c[i].y, r.c[i].z, r.c[i].w};
#pragma unroll
            for (int hu = 0; hu < 2; ++hu) {           // 8 channels
                const uint32_t w0 = w4[2 * hu], w1 = w4[2 * hu + 1];
                *reinterpret_cast<uint4 *>(tile + tile_off(row, ch0 + 16 * i + 8 * hu)) =
                    make_uint4(cvt_e4m3x2_f16x2(w0 & 0xFFFFu), cvt_e4m3x2_f16x2(w0 >> 16),
                               cvt_e4m3x2_f16x2(w1 & 0xFFFFu), cvt_e4m3x2_f16x2(w1 >> 16));
            }
        }
    } else {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < 16; ++u) *reinterpret_cast<uint4 *>(tile + tile_off(row, ch0 + 8 * u)) = z;
    }
}

// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(AttnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem &s = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qi = blockIdx.x;
    const int b = qi / a.Tq;
    const int h0 = blockIdx.y * kHeads;
    const int hcta = min(kHeads, a.H - h0);
    const int64_t t = a.q_pos[qi];
    const int64_t w0 = max64(0, t - a.swa_len + 1);
    const int n_win = a.swa_len > 0 ? (int)(t - w0 + 1) : 0;
    const int64_t n_vis = min64(visible_entries((int32_t)t, a.ratio), a.cap);

    // ---- set-up ------------------------------------------------------------------------
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.kv_full[i], 8);
            mbar_init(&s.kv_empty[i], 1);
            mbar_init(&s.s_full[i], 1);
        }
        mbar_init(&s.p_full, 4);
        mbar_init(&s.pv_done, 1);
        mbar_init(&s.drain, 1);
        s.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&s.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    // compact the valid selected ids (ids must be visible entries), warps 8-15
    if (warp >= 8) {
        const int pt = threadIdx.x - 256;                     // 0..255, two ids each
        const int32_t *src = a.topk + (int64_t)qi * a.top_k;
        int e0 = (2 * pt < a.top_k) ? src[2 * pt] : -1;
        int e1 = (2 * pt + 1 < a.top_k) ? src[2 * pt + 1] : -1;
        const bool ok0 = e0 >= 0 && e0 < n_vis, ok1 = e1 >= 0 && e1 < n_vis;
        if ((e0 >= 0 && !ok0) || (e1 >= 0 && !ok1)) set_dev_err(a.dev_err, CSA2_DEVERR_INDEX);
        const int mine = (int)ok0 + (int)ok1;
        int incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) s.warp_cnt[warp - 8] = incl;
        asm volatile("bar.sync 1, 256;" ::: "memory");
        int base = 0;
        for (int w = 0; w < warp - 8; ++w) base += s.warp_cnt[w];
        int pos = base + incl - mine;
        if (ok0) s.ids[pos++] = e0;
        if (ok1) s.ids[pos] = e1;
        if (threadIdx.x == 511) s.n_sel = base + incl;
        // Q: max |q| over the CTA's heads, then fp16 with a power-of-two scale
        const uint16_t *q = a.q + ((int64_t)qi * a.H + h0) * kDim;
        float m = 0.0f;
        for (int i = pt; i < hcta * kDim / 8; i += 256) {
            uint4 v = __ldg(reinterpret_cast<const uint4 *>(q) + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                m = fmaxf(m, fmaxf(fabsf(bf16_bits_to_f32(w[j] & 0xFFFFu)),
                                   fabsf(bf16_bits_to_f32(w[j] >> 16))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) s.qmax[warp - 8] = m;
        asm volatile("bar.sync 1, 256;" ::: "memory");
        float qm = 0.0f;
        for (int w = 0; w < 8; ++w) qm = fmaxf(qm, s.qmax[w]);
        const int e = qm > 0.0f ? max(0, ilogbf(qm) - 14) : 0;
        const float inv = exp2f((float)-e);
        for (int i = pt; i < kHeads * kDim / 8; i += 256) {
            const int row = i / 64, ch = (i % 64) * 8;
            uint4 o = make_uint4(0u, 0u, 0u, 0u);
            if (row < hcta) {
                uint4 v = __ldg(reinterpret_cast<const uint4 *>(q) + i);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                uint32_t h[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    h[j] = pack_h2(bf16_bits_to_f32(w[j] & 0xFFFFu) * inv,
                                   bf16_bits_to_f32(w[j] >> 16) * inv);
                o = make_uint4(h[0], h[1], h[2], h[3]);
            }
            *reinterpret_cast<uint4 *>(s.q + tile_off(row, ch)) = o;
        }
        if (threadIdx.x == 256) s.qmax[8] = (float)e;
        fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int n_sel = s.n_sel;
    const int n_keys = n_sel + n_win;
    const int n_tiles = (n_keys + kTK - 1) / kTK;
    const uint32_t tmem = s.tmem_base;
    const uint32_t idesc_s = (1u << 4) | ((uint32_t)(kTK >> 3) << 17) | ((uint32_t)(kHeads >> 4) << 24);
    const uint32_t idesc_pv = (1u << 4) | (1u << 16) | (32u << 17) | ((uint32_t)(kHeads >> 4) << 24);

    if (warp == 0) {
        // ---------------- MMA issuer ----------------
        if (lane == 0 && n_tiles > 0) {
            const uint32_t q_base = smem_u32(s.q);
            const uint32_t p_base = smem_u32(s.p);
            bool ok = true;
            auto issue_s = [&](int i) {
                const uint32_t kv = smem_u32(s.kv[i & 1]);
                const uint32_t d = tmem + (16u << 16) + (uint32_t)(i & 1) * kTK;
#pragma unroll
                for (int kk = 0; kk < 32; ++kk) {
                    const uint32_t off = (uint32_t)(kk >> 2) * 8192u + (uint32_t)(kk & 3) * 32u;
                    mma_f16(d, sw128_desc(q_base + off, 16, 1024), sw128_desc(kv + off, 16, 1024),
                            idesc_s, kk > 0);
                }
                mma_commit(&s.s_full[i & 1]);
            };
            ok = mbar_wait(&s.kv_full[0], 0);
            if (ok) {
                tc_fence_after();
                issue_s(0);
            }
            for (int i = 0; ok && i < n_tiles; ++i) {
                if (i + 1 < n_tiles) {
                    ok = mbar_wait(&s.kv_full[(i + 1) & 1], ((i + 1) >> 1) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    issue_s(i + 1);
                }
                ok = mbar_wait(&s.p_full, i & 1);
                if (!ok) break;
                tc_fence_after();
                const uint32_t kv = smem_u32(s.kv[i & 1]);
#pragma unroll
                for (int nh = 0; nh < 2; ++nh)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16(tmem + 256u * nh, sw128_desc(p_base + 32u * ks, 16, 1024),
                                sw128_desc(kv + 4u * 8192u * nh + 2048u * ks, 8192, 1024),
                                idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
                mma_commit(&s.kv_empty[i & 1]);
                mma_commit(&s.pv_done);
            }
            if (!ok) {
                atomicExch(&s.abort, 1);
                set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
            }
            // drain: every MMA issued so far has completed once this barrier flips
            mma_commit(&s.drain);
            mbar_wait(&s.drain, 0);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ---------------- softmax (TMEM quadrant warp % 4) ----------------
        const int qd = warp & 3;
        const int head = 16 * qd + (lane & 15);
        const int half = lane >> 4;
        const float c = a.softmax_scale * 1.4426950408889634f * exp2f(s.qmax[8]);
        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        const uint32_t s_lane = tmem + ((uint32_t)(32 * qd + 16) << 16);
        const uint32_t o_lane = tmem + ((uint32_t)(32 * qd) << 16);
        for (int i = 0; i < n_tiles; ++i) {
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s.s_full[i & 1], (i >> 1) & 1) && !aborted(s));
            if (!ok) break;
            tc_fence_after();
            // the stage's per-key scales: kv_full of this tile has completed (the
            // MMA waited on it) and cannot advance before this warp releases P
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s.kv_full[i & 1], (i >> 1) & 1));
            if (!ok) break;
            float x[32], sg[32];
            tmem_ld16x32<32>(s_lane + (uint32_t)(i & 1) * kTK, x);
            float mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int key = i * kTK + 32 * half + j;
                sg[j] = s.sig[i & 1][32 * half + j];
                x[j] = (key < n_keys && sg[j] > 0.0f) ? x[j] * (c * sg[j]) : -INFINITY;
                mt = fmaxf(mt, x[j]);
            }
            mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, 16));
            if (i > 0) {
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s.pv_done, (i - 1) & 1) && !aborted(s));
                if (!ok) break;
                tc_fence_after();
            }
            float alpha = 1.0f;
            if (i == 0) {
                m_run = mt;
            } else if (mt > m_run + 8.0f) {
                alpha = exp2f(m_run - mt);
                m_run = mt;
                l_run *= alpha;
            }
            if (__any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
#pragma unroll 1
                for (int cc = 0; cc < 256; cc += 32) {
                    float o[32];
                    tmem_ld16x32<256>(o_lane + (uint32_t)cc, o);
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] *= alpha;
                    tmem_st16x32<256>(o_lane + (uint32_t)cc, o);
                }
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            }
            float ps = 0.0f;
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float p0 = exp2f(x[2 * j] - m_run), p1 = exp2f(x[2 * j + 1] - m_run);
                ps += p0 + p1;
                pk[j] = pack_h2(p0 * sg[2 * j], p1 * sg[2 * j + 1]);   // V = code, so P carries sigma
            }
            l_run += ps;
#pragma unroll
            for (int cq = 0; cq < 4; ++cq) {
                const int chunk = 4 * half + cq;
                *reinterpret_cast<uint4 *>(s.p + head * 128 + ((chunk ^ (head & 7)) << 4)) =
                    make_uint4(pk[4 * cq], pk[4 * cq + 1], pk[4 * cq + 2], pk[4 * cq + 3]);
            }
            tc_fence_before();
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.p_full);
        }
        if (ok && n_tiles > 0) {
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s.pv_done, (n_tiles - 1) & 1) && !aborted(s));
            tc_fence_after();
        }
        if (!ok) {
            atomicExch(&s.abort, 1);
            set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
        }
        const float l_tot = l_run + __shfl_xor_sync(0xFFFFFFFFu, l_run, 16);
        const bool valid = ok && n_tiles > 0 && head < hcta && l_tot > 0.0f;
        const float inv = valid ? 1.0f / l_tot : 0.0f;
        float *orow = a.out + ((int64_t)qi * a.H + h0 + head) * kDim;
        if (ok && n_tiles > 0) {
#pragma unroll 1
            for (int cc = 0; cc < 256; cc += 32) {
                float o[32];
                tmem_ld16x32<256>(o_lane + (uint32_t)cc, o);
                if (head < hcta) {
                    float4 *dst = reinterpret_cast<float4 *>(orow + 256 * half + cc);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        dst[j] = make_float4(o[4 * j] * inv, o[4 * j + 1] * inv,
                                             o[4 * j + 2] * inv, o[4 * j + 3] * inv);
                }
            }
        } else if (head < hcta) {
            for (int cc = 0; cc < 256; ++cc) orow[256 * half + cc] = 0.0f;
        }
        if (half == 0 && head < hcta)
            a.lse[(int64_t)qi * a.H + h0 + head] =
                valid ? (m_run + log2f(l_tot)) * 0.6931471805599453f : -INFINITY;
        tc_fence_before();
    } else if (warp >= 8) {
        // ---------------- producers ----------------
        const int pt = threadIdx.x - 256;
        const int row = pt >> 2, quarter = pt & 3;
        Raw cur, nxt;
        if (n_tiles > 0) load_raw(nxt, a, s, b, w0, n_keys, 0, row, quarter);
        bool ok = true;
        for (int i = 0; i < n_tiles; ++i) {
            cur = nxt;
            if (i + 1 < n_tiles) load_raw(nxt, a, s, b, w0, n_keys, i + 1, row, quarter);
            if (i >= 2) {
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s.kv_empty[i & 1], ((i >> 1) - 1) & 1) && !aborted(s));
                if (!ok) break;
            }
            store_dequant(cur, s.kv[i & 1], row, quarter, a.dev_err);
            if (quarter == 0)
                s.sig[i & 1][row] = cur.kind == 1 ? 1.0f : (cur.kind == 2 ? cur.sigma : 0.0f);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.kv_full[i & 1]);
        }
        if (!ok) {
            atomicExch(&s.abort, 1);
            set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

}  // namespace tc

size_t attn_tc_smem_bytes() { return sizeof(tc::Smem) + 1024; }

cudaError_t launch_sparse_attn(const AttnArgs &a, int BT, cudaStream_t st) {
    const size_t smem = attn_tc_smem_bytes();
    static bool attr_set = false;  // once per process (one device per process)
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(tc::attn_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid(BT, (a.H + tc::kHeads - 1) / tc::kHeads);
    tc::attn_tc_kernel<<<grid, tc::kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace csa2
