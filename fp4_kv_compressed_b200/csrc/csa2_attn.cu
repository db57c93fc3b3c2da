// csa2_attn.cu -- a8 sparse decode attention on the 5th-generation tensor cores
// (and, for decode, the a2 append of the layer's SWA row, fused in).
//
// DeepSeek V4.1 Flash study notes, sections 1, 2 and 4: each layer attends, with
// its own query, over at most 512 selected global entries (FP4, dequantised on
// read; the cache format saves storage, the attention matmul itself is not FP4)
// together with its own 128-token FP8 SWA window; one softmax over the union.
// K = V = the 512-channel entry (MQA, fixed for this build).
//
// A 2-CTA cluster per (query, group of 64 heads); each CTA takes half of the
// query's key tiles and the two partial results are merged through distributed
// shared memory (each CTA writes half of the output channels).  16 warps, specialised:
//   warp 0      TMEM allocation + the MMA loop (whole warp, one elected lane issues);
//   warp 1      fused append only: quantises the query token's new SWA row;
//   warps 4-7   softmax, one per TMEM lane quadrant (warp w reads lanes 32(w%4)..);
//   warps 8-15  producers: gather the tile's rows (FP4 entry or FP8 SWA row) into
//               registers one tile ahead, dequantise to fp16 into shared memory,
//               channels 0-255 first (own mbarrier), then 256-511.
// Data layout: one fp16 tile of 64 keys x 512 channels serves both MMAs -- as the
// K-major B operand of S = Q K^T and as the MN-major B operand of O = P V -- in
// the 128-byte-swizzled layout [channel block of 64][key][128 B].  fp16 holds the
// FP4 values exactly (e2m1 x e4m3 has at most 6 significant bits); an SWA row is
// stored as its exact E4M3 codes and its scale sigma is applied in fp32, to the
// logit and folded into P for the P V product.  Q is converted to fp16 after an exact
// power-of-two scaling that keeps max|q| below 2^15.
// TMEM (512 columns): O = 64 x 512 fp32 in lanes 0-15 of each quadrant (M = 64
// layout); at lane offset 16, the two S buffers, each as 2 partial 64 x 64 fp32
// accumulators over channel halves (the low half's MMAs start as soon as the
// producers have written channels 0-255 of the tile; the softmax adds the two),
// columns 0..255.
// Online softmax in the log2 domain with lazy rescaling: O is rescaled only when
// a head's running max grows by more than 8 (p stays <= 2^8, safe in fp16).
// The MMA warp issues P V(i) and S(i+1) as soon as each is ready.  The combine
// moves the peer's half of O with bulk copies between the two CTAs' shared memory.
// Every wait is bounded: on timeout the kernel flags CSA2_DEVERR_TIMEOUT, drains its
// MMAs, frees TMEM and returns.
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
constexpr int kSPart = 2;                      // partial S accumulators per tile (K split)
constexpr uint32_t kXferBytes = 32 * 256 * 4;  // half (32 heads) of one CTA's O for the peer
constexpr uint64_t kWaitLimitNs = 500000000ull; // a wait gives up after 0.5 s of wall time

struct __align__(1024) Smem {
    uint8_t q[64 * 1024];            // Q fp16, [8 cb][64 heads][128 B] swizzled
    uint8_t kv[2][64 * 1024];        // K=V fp16 tiles, [8 cb][64 keys][128 B] swizzled
    uint8_t p[kHeads * 128];         // P fp16, [64 heads][64 keys] swizzled (K-major)
    int32_t ids[CSA2_TOPK_MAX];      // compacted selected entry ids
    float sig[2][kTK];               // per-key scale of each stage (1 FP4, sigma SWA, 0 none)
    alignas(16) uint8_t swa_new[kDim];   // fused append: the query token's new SWA row (E4M3)
    float swa_new_sigma;
    uint64_t kv_lo[2], kv_hi[2], kv_empty[2], s_full[2], p_full, pv_done, drain, xfer[2];
    uint32_t tmem_base;
    int32_t abort;
    float wred[16];
    int32_t wcnt[16];
    float cm[kHeads], cl[kHeads];    // this CTA's partial softmax max / sum per head
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

__device__ __forceinline__ uint64_t wall_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait for the phase with the given parity: false once kWaitLimitNs of wall
// time has passed without it completing.
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity) {
    const uint32_t addr = smem_u32(b);
    const uint64_t t0 = wall_ns();
    while (true) {
        uint32_t done;
        asm volatile(
            "{\n.reg .pred p;\n"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            "selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(addr), "r"(parity)
            : "memory");
        if (done) return true;
        if (wall_ns() - t0 > kWaitLimitNs) return false;
    }
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

__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
                 : "memory");
}

// Asynchronous bulk copy from this CTA's shared memory into another CTA's of the
// cluster (dst and bar are shared::cluster addresses); bar receives complete_tx.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst, const void *src, uint32_t bytes,
                                                  uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "r"(smem_u32(src)), "r"(bytes), "r"(bar)
        : "memory");
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

// One lane of a converged warp (the same lane on every call).
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile(
        "{\n.reg .pred p;\n.reg .b32 r;\n"
        "elect.sync r|p, 0xffffffff;\n"
        "selp.u32 %0, 1, 0, p;\n}"
        : "=r"(pred));
    return pred != 0;
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

// The same 16-column load without the wait: the caller issues several, then calls
// tmem_wait_ld() once before reading any of the registers.
template <int HALF>
__device__ __forceinline__ void tmem_ld16x16_nw(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], %17;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr), "n"(HALF));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

template <int HALF>
__device__ __forceinline__ void tmem_ld16x16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], %17;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr), "n"(HALF));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
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
// Producer thread (row, quarter q) handles channels [64q, 64q + 64) of the low half
// (channels 0-255) and [256 + 64q, 256 + 64q + 64) of the high half of one key, so
// that a tile's low half can be complete (and its S MMAs start) before the high half.
struct Raw {
    uint4 c[8];      // FP4: c[0..1] low-half codes, c[2..3] high-half codes (32 B each);
                     // SWA: c[0..3] low-half codes, c[4..7] high-half codes (64 B each)
    uint2 s;         // FP4: 4 scale bytes of each half (x low, y high)
    float sigma;     // SWA scale
    int kind;        // 0 none, 1 FP4 entry, 2 SWA row
};

// new_row / new_sigma: the window's newest row already quantised in shared memory
// (fused append), or null.
__device__ __forceinline__ void load_raw(Raw &r, const AttnArgs &a, const int32_t *ids, int n_sel,
                                         int b, int64_t w0, int n_keys, int tile, int row,
                                         int quarter, const uint8_t *new_row, float new_sigma) {
    const int kg = tile * kTK + row;
    r.kind = 0;
    if (kg < n_sel) {
        const int e = ids[kg];
        const int64_t off = (int64_t)b * a.cap + e;
        const uint8_t *codes = a.codes + off * kCodeBytes;
        const uint8_t *scales = a.scales + off * kScaleBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 *src = reinterpret_cast<const uint4 *>(codes + 128 * h + 32 * quarter);
            r.c[2 * h] = __ldg(src);
            r.c[2 * h + 1] = __ldg(src + 1);
        }
        r.s.x = __ldg(reinterpret_cast<const uint32_t *>(scales + 4 * quarter));
        r.s.y = __ldg(reinterpret_cast<const uint32_t *>(scales + 16 + 4 * quarter));
        r.kind = 1;
    } else if (kg < n_keys && new_row != nullptr && kg == n_keys - 1) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 *src = reinterpret_cast<const uint4 *>(new_row + 256 * h + 64 * quarter);
#pragma unroll
            for (int i = 0; i < 4; ++i) r.c[4 * h + i] = src[i];
        }
        r.sigma = new_sigma;
        r.kind = 2;
    } else if (kg < n_keys) {
        const int64_t pos = w0 + (kg - n_sel);
        const int64_t slot = (int64_t)b * a.wcap + pos % a.wcap;
        const uint8_t *codes = a.swa_codes + slot * kDim;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 *src = reinterpret_cast<const uint4 *>(codes + 256 * h + 64 * quarter);
#pragma unroll
            for (int i = 0; i < 4; ++i) r.c[4 * h + i] = __ldg(src + i);
        }
        r.sigma = __ldg(a.swa_scale + slot);
        r.kind = 2;
    }
}

// Dequantise the thread's 64 channels of half h of one key into the fp16 tile.
__device__ __forceinline__ void store_dequant_half(const Raw &r, uint8_t *tile, int row, int quarter,
                                                   int h, int32_t *dev_err) {
    const int ch0 = 256 * h + 64 * quarter;
    if (r.kind == 1) {
        const uint4 c0 = r.c[2 * h], c1 = r.c[2 * h + 1];
        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const uint32_t sw = h ? r.s.y : r.s.x;         // scales of channel groups 0..3 (16 each)
        uint32_t scale2[4];                            // one f16x2 scale per 16 channels
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const uint32_t hh = cvt_e4m3x2_f16x2((sw >> (16 * g)) & 0xFFFFu);
            scale2[2 * g] = (hh & 0xFFFFu) * 0x10001u;
            scale2[2 * g + 1] = (hh >> 16) * 0x10001u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {                  // 8 channels per 32-bit code word
            const __half2 sv = *reinterpret_cast<const __half2 *>(&scale2[u >> 1]);
            uint32_t v[4];
            cvt_e2m1x8_f16x2(cw[u], v);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __half2 x = __hmul2(*reinterpret_cast<__half2 *>(&v[j]), sv);
                v[j] = *reinterpret_cast<uint32_t *>(&x);
            }
            *reinterpret_cast<uint4 *>(tile + tile_off(row, ch0 + 8 * u)) = make_uint4(v[0], v[1], v[2], v[3]);
        }
    } else if (r.kind == 2) {
        // exact E4M3 codes; the row scale is applied in fp32 on the logit and on P
        if (h == 0 && quarter == 0 && r.sigma * 256.0f > 65504.0f) set_dev_err(dev_err, CSA2_DEVERR_RANGE);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 cv = r.c[4 * h + i];
            const uint32_t w4[4] = {cv.x, cv.y, cv.z, cv.w};
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
        for (int u = 0; u < 8; ++u) *reinterpret_cast<uint4 *>(tile + tile_off(row, ch0 + 8 * u)) = z;
    }
}

// ---- cluster helpers (2 CTAs per query split its keys; partials combine via DSMEM) ----
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t peer_addr(const void *local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
    return r;
}
__device__ __forceinline__ float ld_peer(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void st_peer4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t *b, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n.reg .pred p;\n"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(smem_u32(b)), "r"(parity)
        : "memory");
    return done != 0;
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------------------------------
// kRope: the fused append rotates the new SWA row first (a separate instantiation, so
// that the plain kernel carries none of its code).
template <bool kRope>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
attn_tc_kernel(AttnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem &s = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int qi = blockIdx.x >> 1;
    const int b = qi / a.Tq;
    const int h0 = blockIdx.y * kHeads;
    const int hcta = min(kHeads, a.H - h0);
    // ---- set-up (all threads) -------------------------------------------------------------
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.kv_lo[i], 8);
            mbar_init(&s.kv_hi[i], 8);
            mbar_init(&s.kv_empty[i], 1);
            mbar_init(&s.s_full[i], 1);
        }
        mbar_init(&s.p_full, 4);
        mbar_init(&s.pv_done, 1);
        mbar_init(&s.drain, 1);
        mbar_init(&s.xfer[0], 1);
        mbar_init(&s.xfer[1], 1);
        s.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&s.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    // barriers and TMEM above touch no global memory; everything below may read what the
    // previous kernel of the stream wrote
    grid_dep_wait();
    // every independent global load first (one memory round trip): the position, this
    // thread's Top-K entry, its Q chunks and (warp 1, fused append) the new SWA row
    const int32_t t32 = a.q_pos[qi];
    const int32_t *tk = a.topk + (int64_t)qi * a.top_k;
    const int e_id = (int)threadIdx.x < a.top_k ? tk[threadIdx.x] : -1;
    // Q chunks of 8 channels: thread t holds chunks t + 512 j
    const uint16_t *q = a.q + ((int64_t)qi * a.H + h0) * kDim;
    uint4 qv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int i = threadIdx.x + kThreads * j;
        qv[j] = (i / 64 < hcta) ? __ldg(reinterpret_cast<const uint4 *>(q) + i) : make_uint4(0u, 0u, 0u, 0u);
    }
    uint4 xraw[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
    if (a.swa_new != nullptr && warp == 1) {
        const uint4 *src = reinterpret_cast<const uint4 *>(a.swa_new + (int64_t)qi * kDim + 16 * lane);
        xraw[0] = __ldg(src);
        xraw[1] = __ldg(src + 1);
    }
    const int64_t t = t32;
    const int64_t w0 = max64(0, t - a.swa_len + 1);
    const int n_win = a.swa_len > 0 ? (int)(t - w0 + 1) : 0;
    const int64_t n_vis = min64(visible_entries((int32_t)t, a.ratio), a.cap);
    // selected ids: thread t checks topk[t]; valid ids are compacted in order
    const bool e_ok = e_id >= 0 && e_id < n_vis;
    if (e_id >= 0 && !e_ok) set_dev_err(a.dev_err, CSA2_DEVERR_INDEX);
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, e_ok);
    // fused SWA append (decode, Tq = 1): the token's new bf16 row, read above by warp 1
    const bool fuse = a.swa_new != nullptr && n_win > 0;
    float xnew[16];
    unpack_bf16x8(xraw[0], xnew);
    unpack_bf16x8(xraw[1], xnew + 8);
    float qm = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t w[4] = {qv[j].x, qv[j].y, qv[j].z, qv[j].w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
            qm = fmaxf(qm, fmaxf(fabsf(bf16_bits_to_f32(w[k] & 0xFFFFu)), fabsf(bf16_bits_to_f32(w[k] >> 16))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qm = fmaxf(qm, __shfl_xor_sync(0xFFFFFFFFu, qm, o));
    if (lane == 0) {
        s.wcnt[warp] = __popc(bal);
        s.wred[warp] = qm;
    }
    __syncthreads();
    int base = 0, n_sel = 0;
    float qmax = 0.0f;
#pragma unroll
    for (int w = 0; w < 16; ++w) {
        base += w < warp ? s.wcnt[w] : 0;
        n_sel += s.wcnt[w];
        qmax = fmaxf(qmax, s.wred[w]);
    }
    if (e_ok) s.ids[base + __popc(bal & ((1u << lane) - 1u))] = e_id;
    if (fuse && warp == 1) {
        // The same FP8 row quantiser as csa2_quantize_append: codes and sigma go to
        // shared memory (this CTA's producers read the window's newest key from there)
        // and, from head group 0's CTA that owns that key, to the ring slot t % wcap.
        if constexpr (kRope) {
            if (!rope_lane16(xnew, lane, a.rope.cs, a.rope.n_pos, a.rope.start, a.rope.pairs, t) &&
                lane == 0)
                set_dev_err(a.dev_err, CSA2_DEVERR_ROPE);
        }
        quant_fp8_lanes<kDim>(xnew, s.swa_new, &s.swa_new_sigma, lane);
        const int last_tile = (n_sel + n_win - 1) / kTK;
        const int n_all0 = (n_sel + n_win + kTK - 1) / kTK;
        const uint32_t owner = last_tile < (n_all0 + 1) / 2 ? 0u : 1u;
        __syncwarp();
        if (blockIdx.y == 0 && rank == owner) {
            const int64_t slot = (int64_t)b * a.wcap + t % a.wcap;
            reinterpret_cast<uint4 *>(a.swa_codes + slot * kDim)[lane] =
                reinterpret_cast<const uint4 *>(s.swa_new)[lane];
            if (lane == 0) a.swa_scale[slot] = s.swa_new_sigma;
        }
    }
    const int qexp = qmax > 0.0f ? max(0, ilogbf(qmax) - 14) : 0;   // max|q| * 2^-qexp < 2^15
    {
        const float inv = exp2f((float)-qexp);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = threadIdx.x + kThreads * j;
            const uint32_t w[4] = {qv[j].x, qv[j].y, qv[j].z, qv[j].w};
            uint32_t h[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                h[k] = pack_h2(bf16_bits_to_f32(w[k] & 0xFFFFu) * inv, bf16_bits_to_f32(w[k] >> 16) * inv);
            *reinterpret_cast<uint4 *>(s.q + tile_off(i / 64, (i % 64) * 8)) = make_uint4(h[0], h[1], h[2], h[3]);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int n_keys = n_sel + n_win;
    const int n_all = (n_keys + kTK - 1) / kTK;            // tiles of the query
    const int t_split = (n_all + 1) / 2;
    const int tile_lo = rank == 0 ? 0 : t_split;
    const int nt = (rank == 0 ? t_split : n_all) - tile_lo; // tiles of this CTA
    const uint32_t tmem = s.tmem_base;
    const uint32_t idesc_s = (1u << 4) | ((uint32_t)(kTK >> 3) << 17) | ((uint32_t)(kHeads >> 4) << 24);
    const uint32_t idesc_pv = (1u << 4) | (1u << 16) | (32u << 17) | ((uint32_t)(kHeads >> 4) << 24);
    const int qd = warp & 3;
    const int head = 16 * qd + (lane & 15);
    const int half = lane >> 4;
    float m_run = -INFINITY, l_run = 0.0f;

    if (warp == 0) {
        // ---------------- MMA issuer ----------------
        // The whole warp runs the loop (warp-uniform control flow and descriptors);
        // one elected lane issues the MMAs and commits.
        if (nt > 0) {
            const uint64_t qd0 = sw128_desc(smem_u32(s.q), 16, 1024);
            const uint64_t pd0 = sw128_desc(smem_u32(s.p), 16, 1024);
            const uint64_t kd0 = sw128_desc(smem_u32(s.kv[0]), 16, 1024);
            const uint64_t kd1 = sw128_desc(smem_u32(s.kv[1]), 16, 1024);
            const uint64_t vd0 = sw128_desc(smem_u32(s.kv[0]), 8192, 1024);
            const uint64_t vd1 = sw128_desc(smem_u32(s.kv[1]), 8192, 1024);
            int s_next = 0, pv_next = 0, s_half = 0;
            uint64_t idle_since = wall_ns();
            bool stalled = false;
            while (pv_next < nt && !stalled) {
                bool progressed = false;
                // P V first: it frees a K/V stage for the producers and O for the softmax
                int go = 0;
                if (lane == 0) go = pv_next < s_next && mbar_test(&s.p_full, pv_next & 1);
                if (__shfl_sync(0xFFFFFFFFu, go, 0)) {
                    tc_fence_after();
                    const uint64_t vb = (pv_next & 1) ? vd1 : vd0;
                    if (elect_one()) {
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                            for (int nh = 0; nh < 2; ++nh)
                                mma_f16(tmem + 256u * nh, pd0 + (uint64_t)(2 * ks),
                                        vb + (uint64_t)(nh * 2048 + ks * 128), idesc_pv,
                                        (pv_next > 0 || ks > 0) ? 1u : 0u);
                        mma_commit(&s.kv_empty[pv_next & 1]);
                        mma_commit(&s.pv_done);
                    }
                    __syncwarp();
                    ++pv_next;
                    progressed = true;
                }
                // S(s_next) in two halves: the accumulators of channels 0-255 once the
                // tile's low half has landed, those of channels 256-511 once its high half has
                go = 0;
                if (lane == 0)
                    go = s_next < nt && s_next <= pv_next + 1 &&
                         mbar_test(s_half ? &s.kv_hi[s_next & 1] : &s.kv_lo[s_next & 1], (s_next >> 1) & 1);
                if (__shfl_sync(0xFFFFFFFFu, go, 0)) {
                    tc_fence_after();
                    // S as kSPart partial sums over channel slices (kSPart / 2 per half),
                    // issued round-robin over the half's accumulators
                    const uint32_t d = tmem + (16u << 16) + (uint32_t)(s_next & 1) * (kSPart * kTK);
                    const uint64_t kb = (s_next & 1) ? kd1 : kd0;
                    if (elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < 32 / kSPart; ++kk)
#pragma unroll
                            for (int p2 = 0; p2 < kSPart / 2; ++p2) {
                                const int pp = (kSPart / 2) * s_half + p2;
                                const int k16 = pp * (32 / kSPart) + kk;      // K-step of 16 channels
                                const uint64_t off = (uint64_t)((k16 >> 2) * 512 + (k16 & 3) * 2);  // 16-byte units
                                mma_f16(d + (uint32_t)(pp * kTK), qd0 + off, kb + off, idesc_s, kk > 0);
                            }
                        if (s_half) mma_commit(&s.s_full[s_next & 1]);
                    }
                    __syncwarp();
                    if (s_half) ++s_next;
                    s_half ^= 1;
                    progressed = true;
                }
                if (progressed)
                    idle_since = wall_ns();
                else
                    stalled = __shfl_sync(0xFFFFFFFFu, (int)(wall_ns() - idle_since > kWaitLimitNs), 0) != 0;
            }
            if (pv_next < nt && lane == 0) {
                atomicExch(&s.abort, 1);
                set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
            }
            if (elect_one()) mma_commit(&s.drain);   // completes once every MMA issued above has
            __syncwarp();
            if (lane == 0) mbar_wait(&s.drain, 0);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ---------------- softmax (TMEM quadrant warp % 4) ----------------
        const float c = a.softmax_scale * 1.4426950408889634f * exp2f((float)qexp);
        const uint32_t s_lane = tmem + ((uint32_t)(32 * qd + 16) << 16);
        const uint32_t o_lane = tmem + ((uint32_t)(32 * qd) << 16);
        bool ok = true;
        for (int i = 0; i < nt; ++i) {
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s.s_full[i & 1], (i >> 1) & 1) &&
                                             mbar_wait(&s.kv_hi[i & 1], (i >> 1) & 1) && !aborted(s));
            if (!ok) break;
            tc_fence_after();
            float x[32], sg[32];
            {
                // all partial sums of 16 columns are loaded, then waited for once
                const uint32_t sb = s_lane + (uint32_t)(i & 1) * (kSPart * kTK);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t y[kSPart][16];
#pragma unroll
                    for (int pp = 0; pp < kSPart; ++pp) tmem_ld16x16_nw<32>(sb + (uint32_t)(pp * kTK + 16 * c), y[pp]);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float v = __uint_as_float(y[0][j]);
#pragma unroll
                        for (int pp = 1; pp < kSPart; ++pp) v += __uint_as_float(y[pp][j]);
                        x[16 * c + j] = v;
                    }
                }
            }
            const int key0 = (tile_lo + i) * kTK + 32 * half;
            float mt = -INFINITY;
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
                const float4 g4 = reinterpret_cast<const float4 *>(&s.sig[i & 1][32 * half])[j4];
                sg[4 * j4] = g4.x; sg[4 * j4 + 1] = g4.y; sg[4 * j4 + 2] = g4.z; sg[4 * j4 + 3] = g4.w;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                x[j] = (key0 + j < n_keys && sg[j] > 0.0f) ? x[j] * (c * sg[j]) : -INFINITY;
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
                alpha = ex2(m_run - mt);
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
                const float p0 = ex2(x[2 * j] - m_run), p1 = ex2(x[2 * j + 1] - m_run);
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
        if (ok && nt > 0) {
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s.pv_done, (nt - 1) & 1) && !aborted(s));
            tc_fence_after();
        }
        if (!ok) {
            atomicExch(&s.abort, 1);
            set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
        }
        l_run += __shfl_xor_sync(0xFFFFFFFFu, l_run, 16);
        if (half == 0) {
            s.cm[head] = (ok && nt > 0) ? m_run : -INFINITY;
            s.cl[head] = (ok && nt > 0) ? l_run : 0.0f;
        }
    } else if (warp >= 8) {
        // ---------------- producers ----------------
        const int pt = threadIdx.x - 256;
        const int row = pt >> 2, quarter = pt & 3;
        Raw cur, nxt;
        const uint8_t *new_row = fuse ? s.swa_new : nullptr;
        const float new_sigma = fuse ? s.swa_new_sigma : 0.0f;
        if (nt > 0) load_raw(nxt, a, s.ids, n_sel, b, w0, n_keys, tile_lo, row, quarter, new_row, new_sigma);
        bool ok = true;
        for (int i = 0; i < nt; ++i) {
            cur = nxt;
            if (i + 1 < nt) load_raw(nxt, a, s.ids, n_sel, b, w0, n_keys, tile_lo + i + 1, row, quarter, new_row, new_sigma);
            if (i >= 2) {
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s.kv_empty[i & 1], ((i >> 1) - 1) & 1) && !aborted(s));
                if (!ok) break;
            }
            store_dequant_half(cur, s.kv[i & 1], row, quarter, 0, a.dev_err);
            if (quarter == 0)
                s.sig[i & 1][row] = cur.kind == 1 ? 1.0f : (cur.kind == 2 ? cur.sigma : 0.0f);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.kv_lo[i & 1]);      // channels 0-255 of the tile ready
            store_dequant_half(cur, s.kv[i & 1], row, quarter, 1, a.dev_err);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.kv_hi[i & 1]);      // channels 256-511 ready
        }
        if (!ok) {
            atomicExch(&s.abort, 1);
            set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
        }
    }

    // ---- combine the two key halves of the query through distributed shared memory ----
    // CTA r outputs channels [256 r, 256 r + 256); a softmax thread (head, half) holds
    // O[head][256 half .. +256) of its CTA in TMEM.
    __syncwarp();                          // converged warps for the cluster barrier
    if (threadIdx.x == 0) {                // the peer's part, two halves of 32 heads, armed early
        mbar_expect_tx(&s.xfer[0], kXferBytes);
        mbar_expect_tx(&s.xfer[1], kXferBytes);
    }
    tc_fence_before();
    cluster_sync();                        // partial stats published; all MMAs of both CTAs done
    tc_fence_after();
    grid_dep_launch();
    // Both CTAs derive the same weights.  Every thread scales a 64-column piece of one
    // head's half-row of O (TMEM quadrant warp % 4, column quarter warp / 4) and stores
    // it into local staging: `own` for the channels this CTA writes, `send` for the
    // peer's.  One bulk copy moves `send` into the peer's `recv`; then all threads add
    // own + recv and write coalesced.
    float *own = reinterpret_cast<float *>(s.q);           // [64 heads][256] this CTA's part
    float *send = reinterpret_cast<float *>(s.kv[1]);      // [64 heads][256] for the peer
    float *recv = reinterpret_cast<float *>(s.kv[0]);      // [64 heads][256] from the peer
    const uint32_t peer = rank ^ 1u;
    {
        const int qw = warp & 3, sub = warp >> 2;
        const int hd = 16 * qw + (lane & 15), hf = lane >> 4;
        const float m_self = s.cm[hd], l_self = s.cl[hd];
        const float m_peer = ld_peer(peer_addr(&s.cm[hd], peer));
        const float l_peer = ld_peer(peer_addr(&s.cl[hd], peer));
        const float m_all = fmaxf(m_self, m_peer);
        float f_self = 0.0f, f_peer = 0.0f;
        if (m_all != -INFINITY) {
            f_self = m_self == -INFINITY ? 0.0f : ex2(m_self - m_all);
            f_peer = m_peer == -INFINITY ? 0.0f : ex2(m_peer - m_all);
        }
        const float l_all = l_self * f_self + l_peer * f_peer;
        const bool valid = hd < hcta && l_all > 0.0f;
        const float w = valid ? f_self / l_all : 0.0f;
        // warp-uniform: tcgen05.ld is a whole-warp instruction (lanes 0-15 read the low
        // half-row, lanes 16-31 the high one)
        const bool have = __shfl_sync(0xFFFFFFFFu, (int)(nt > 0 && !aborted(s)), 0) != 0;
        const uint32_t o_lane = tmem + ((uint32_t)(32 * qw) << 16);
        const bool keep = (uint32_t)hf == rank;
        float4 *dst = reinterpret_cast<float4 *>((keep ? own : send) + hd * 256);
#pragma unroll 1
        for (int cc = 64 * sub; cc < 64 * sub + 64; cc += 32) {
            float o[32];
            if (have) {
                tmem_ld16x32<256>(o_lane + (uint32_t)cc, o);
#pragma unroll
                for (int j = 0; j < 32; ++j) o[j] *= w;
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) o[j] = 0.0f;
            }
            // float4 f of head hd's row is stored at f ^ (hd % 16): the 16 heads of a
            // quarter-warp then hit different bank groups
#pragma unroll
            for (int j = 0; j < 8; ++j)
                dst[(cc / 4 + j) ^ (hd & 15)] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
        }
        if (keep && sub == 0 && rank == 0 && hd < hcta)
            a.lse[(int64_t)qi * a.H + h0 + hd] =
                valid ? (m_all + log2f(l_all)) * 0.6931471805599453f : -INFINITY;
    }
    fence_async_smem();                    // generic-proxy writes of `send` -> the bulk copy
    __syncthreads();
    if (threadIdx.x == 0) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t dst = peer_addr(recv + hh * 32 * 256, peer), bar = peer_addr(&s.xfer[hh], peer);
            bulk_copy_to_peer(dst, send + hh * 32 * 256, kXferBytes / 2, bar);
            bulk_copy_to_peer(dst + kXferBytes / 2, reinterpret_cast<uint8_t *>(send + hh * 32 * 256) + kXferBytes / 2,
                              kXferBytes / 2, bar);
        }
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    // add the peer's part as each half of the heads lands; write coalesced
    const float4 *o4 = reinterpret_cast<const float4 *>(own);
    const float4 *r4 = reinterpret_cast<const float4 *>(recv);
    float *obase = a.out + ((int64_t)qi * a.H + h0) * kDim + 256 * rank;
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
        const bool got = __syncthreads_and(mbar_wait(&s.xfer[hh], 0)) != 0;
        if (!got && threadIdx.x == 0) set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
#pragma unroll 2
        for (int i = hh * 32 * 64 + threadIdx.x; i < (hh + 1) * 32 * 64; i += kThreads) {
            const int h = i >> 6, c4 = i & 63;
            if (h < hcta) {
                const int f = h * 64 + (c4 ^ (h & 15));
                const float4 x = o4[f];
                const float4 y = got ? r4[f] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                reinterpret_cast<float4 *>(obase + (int64_t)h * kDim)[c4] =
                    make_float4(x.x + y.x, x.y + y.y, x.z + y.z, x.w + y.w);
            }
        }
    }
    // this CTA's outgoing copy has finished reading `send` before the CTA may exit
    if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

}  // namespace tc

size_t attn_tc_smem_bytes() { return sizeof(tc::Smem) + 1024; }

template <bool kRope>
static cudaError_t launch_attn_t(const AttnArgs &a, int BT, cudaStream_t st) {
    const size_t smem = attn_tc_smem_bytes();
    static std::atomic<uint64_t> configured{0};   // per device
    {
        cudaError_t e = config_kernel_once(tc::attn_tc_kernel<kRope>, smem, configured);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(2 * BT, (a.H + tc::kHeads - 1) / tc::kHeads);   // 2-CTA clusters
    cudaError_t e = launch_pdl(tc::attn_tc_kernel<kRope>, grid, dim3(tc::kThreads), smem, st, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_sparse_attn(const AttnArgs &a, int BT, cudaStream_t st) {
    return a.swa_new != nullptr && a.rope.cs != nullptr ? launch_attn_t<true>(a, BT, st)
                                                         : launch_attn_t<false>(a, BT, st);
}

}  // namespace csa2
