// csa2_attn.cu -- a8 sparse decode attention on the 5th-generation tensor cores
// (and, for decode, the a2 append of the layer's SWA row, fused in).
//
// DeepSeek V4.1 Flash study notes, sections 1, 2 and 4: each layer attends, with
// its own query, over at most 512 selected global entries (FP4, dequantised on
// read; the cache format saves storage, the attention matmul itself is not FP4)
// together with its own 128-token FP8 SWA window; one softmax over the union.
// K = V = the 512-channel entry (MQA, fixed for this build).
//
// Work split: one CTA per (query, group of 32 heads), over all of the query's keys, so
// no two CTAs share a softmax and nothing is combined: each CTA writes its heads' rows
// of the output directly.  (The other split, keys over several CTAs, needs their
// partial outputs moved between SMs at the end; on this part that exchange cost more
// than the extra dequantisation of every key by both head groups of a query.)
//
// Transposed tiles.  A tile is 128 keys.  The scores are S^T = K Q^T with the keys
// as the MMA's M = 128 (one TMEM lane per key) and the 32 heads as N; the output is
// O^T = V^T P^T with the channels as M (four 128-channel blocks) and the heads as N.
// K and V are the same dequantised fp16 values: K is written into TMEM, where it is the
// A operand of S^T (so the score MMAs read no shared memory but Q, and the next tile's
// scores can run while this tile's softmax does), and V into a shared-memory tile of
// four stages of 128 channels x 128 keys, the MN-major A operand of O^T.  fp16 holds
// the FP4 values exactly (e2m1 x e4m3 has at most 6 significant bits); an SWA row is
// stored as its exact E4M3 codes and its scale sigma is applied in fp32, to the logit
// and folded into P.  Q (the K-major B operand of S^T) is converted to fp16 after an
// exact power-of-two scaling that keeps max|q| below 2^15.  P^T (the MN-major B
// operand of O^T) is [128 keys][32 heads] with the 64-byte swizzle.
//
// 12 warps, specialised:
//   warp 0       TMEM allocation + the MMA issue loop (one elected lane issues): S^T of
//                the next tile as soon as its K is in TMEM, then O^T of this tile;
//   warp 1       fused append only: quantises the query token's new SWA row;
//   warp 2       prefetches the entries of the later tiles into L2 (bulk prefetch; the
//                set-up prefetches the request's SWA ring);
//   warps 4-11   workers: warp w handles keys 32 (w % 4) .. (its TMEM lane quadrant) and
//                half hh = (w - 4) / 4: the producer's 256 channels, the softmax's 16
//                heads.  Per tile: wait for S^T(i); write K(i + 1) to TMEM; the softmax
//                of tile i -> P^T; V(i + 1) into the shared stages as O^T(i) releases
//                them; load the raw bytes of tile i + 2 (one thread per key, one memory
//                round trip for its two stages).
// TMEM (512 columns): O^T block j (channels 128 j .. 128 j + 127) at columns
// 32 j .. 32 j + 31 (column = head); the two S^T buffers at columns 128 and 160; K at
// columns 256 + channel / 2 (lane = key).
// Online softmax in the log2 domain with lazy rescaling: the running max of a head
// moves (and O, l are rescaled) only when a tile's logit exceeds it by more than 8,
// so p <= 2^8 stays safe in fp16.  The check is per tile and per head half; the exact
// tile max (a shuffle reduce-scatter within a warp, then across the four warps that
// share the heads) is formed only when it fires, and always on the first tile.
// Every wait is bounded (WaitCfg): on timeout the kernel flags CSA2_DEVERR_TIMEOUT,
// waits (bounded) for the MMAs it issued, frees TMEM and returns.  The four softmax
// warps of a head half agree on leaving the tile loop through a barrier reduction, so
// that no named barrier is ever left waiting for a warp that has gone.
#include <cuda_fp16.h>
#include <stdint.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {
namespace attn {

constexpr int kThreads = 384;
constexpr int kWarps = kThreads / 32;
constexpr int kQChunks = (32 * 64 + kThreads - 1) / kThreads;   // 16-byte Q chunks per thread
constexpr int kTK = 128;                       // keys per tile (S^T M, TMEM lanes)
constexpr int kHeads = 32;                     // heads per CTA (MMA N)
constexpr int kStages = 4;                     // 128-channel quarters of a tile
constexpr int kStageBytes = kTK * 128 * 2;     // 128 keys x 128 channels fp16
constexpr int kCbBytes = kTK * 128;            // one 64-channel block of a stage
constexpr int kQCbBytes = kHeads * 128;        // one 64-channel block of Q
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 128;                // S^T buffer b at columns 128 + 32 b
constexpr uint32_t kKCol = 256;                // K of the tile (A of S^T): channel c at column 256 + c / 2
constexpr int kWorkWarp0 = 4;                  // softmax + producer warps 4..11
constexpr int kWorkWarps = kWarps - kWorkWarp0;
constexpr float kLazy = 8.0f;                  // rescale threshold (log2 units)

struct __align__(1024) Smem {
    uint8_t q[8 * kQCbBytes];                  // Q fp16, [8 cb][32 heads][128 B] swizzled
    uint8_t kv[kStages][kStageBytes];          // stage j: [2 cb][128 keys][128 B] swizzled
    uint8_t pt[kTK * kHeads * 2];              // P^T fp16, [128 keys][32 heads], 64-byte swizzle
    int32_t ids[CSA2_TOPK_MAX];                // compacted selected entry ids
    float ksig[kTK];                           // per key of the tile: 1 FP4, sigma SWA, -1 none
    alignas(16) uint8_t swa_new[kDim];         // fused append: the new SWA row (E4M3 codes)
    float swa_new_sigma;
    alignas(16) float red[2][4][16];           // softmax half hh: per quadrant warp, 16 heads
    alignas(16) float mrun[kHeads];            // running max per head (log2 domain)
    alignas(16) float alpha[kHeads];           // factor of the last move of the running max
    float wfin[kHeads];                        // 1 / l per head (0: no key)
    uint64_t kv_full[kStages], kv_empty[kStages], s_full[2], k_full, p_full, pv_done, drain, never;
    uint64_t new_ready;                        // fused append: the new SWA row is in smem
    uint32_t tmem_base;
    int32_t abort;
    float wred[kWarps];
    int32_t wcnt[2 * kWarps];
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
__device__ __forceinline__ bool aborted(const Smem &s) {
    return *reinterpret_cast<const volatile int32_t *>(&s.abort) != 0;
}
// Bounded wait for the phase with the given parity: false once limit_ns of wall time
// has passed without it completing or (kHonorAbort) as soon as a role of the CTA has
// aborted.
template <bool kHonorAbort = true>
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity, uint64_t limit_ns,
                                          const Smem &s) {
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
        if ((kHonorAbort && aborted(s)) || wall_ns() - t0 > limit_ns) return false;
    }
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
// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 version field).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// The same descriptor with the 64-byte swizzle (layout type 4).
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (sw128_desc(saddr, lbo, sbo) & ~((uint64_t)7 << 61)) | ((uint64_t)4 << 61);
}
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n.reg .pred p;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
// The same with A read from TMEM (a_tmem: lane 0, first column of the K-step).
__device__ __forceinline__ void mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n.reg .pred p;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate));
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
// 32 lanes x 16 columns: thread t of the warp reads TMEM lane (base + t), 16 columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 16 columns, in place: v *= f (per column), read and written back.
__device__ __forceinline__ void tmem_scale16(uint32_t taddr, const float *f) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f[i]);
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Named barrier of the four softmax warps that share head half hh (ids 1, 2).
__device__ __forceinline__ void group_sync(int hh) {
    asm volatile("bar.sync %0, 128;" ::"r"(1 + hh) : "memory");
}
// The same barrier with an OR over the four warps' predicates: every thread of the
// group receives the same answer.
__device__ __forceinline__ bool group_any(int hh, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n.reg .pred p, q;\n"
        "setp.ne.u32 p, %1, 0;\n"
        "bar.red.or.pred q, %2, 128, p;\n"
        "selp.u32 %0, 1, 0, q;\n}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(1 + hh)
        : "memory");
    return r != 0;
}
// L2 prefetch of [p, p + bytes) (p 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Byte offset of (row, 16-byte chunk c of a 128-byte row) in a 128B-swizzled block.
__device__ __forceinline__ uint32_t swz(int row, int c) {
    return (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4));
}
// The same for 64-byte rows with the 64-byte swizzle (chunk c of row r at c ^ (r / 2 % 4)).
__device__ __forceinline__ uint32_t swz64(int row, int c) {
    return (uint32_t)(row * 64 + ((c ^ ((row >> 1) & 3)) << 4));
}

// ---- producer: one thread per key of the tile -------------------------------------------
// Worker warp w (quadrant q = w % 4, half h = (w - 4) / 4): thread t handles key 32 q + t
// of the tile and channels 256 h .. 256 h + 255 (stages 2 h and 2 h + 1).  The key's
// row of K goes to TMEM lane 32 q + t (the A operand of S^T, columns kKCol + channel / 2)
// and its row of V to the shared-memory tile (the A operand of O^T); both come from the
// same raw bytes, held in registers a whole tile ahead and dequantised twice.
struct Raw {
    uint4 c[2][8];   // stage 2 h + s: FP4: c[s][0..3] = the 64 code bytes; SWA: c[s][0..7] = 128 codes
    uint2 sc[2];     // FP4: the stage's 8 scale bytes (E4M3, one per 16 channels)
    float sigma;     // 1 for an FP4 entry, the row scale of an SWA row, -1 for no key
    int kind;        // 1 FP4 entry, 2 SWA row, 3 the fused new SWA row (not yet read), 0 zero row,
                     // -1 nothing
};

struct KeyMap {      // the query's keys and where each comes from
    const int32_t *ids;
    int n_sel;
    int64_t w0;      // first window position
    int n_keys;      // keys of the query (selection + window)
    int64_t b;
    int64_t ring_base;
    const uint8_t *new_row;   // fused append: the newest window key is this row (smem)
    const float *new_sigma;
    uint64_t *new_ready;      // ... written once this completes
    const Smem *smem;
};

// Issue every load of key kg's two stages (one memory round trip).  The fused new SWA
// row is only marked here (kind 3): see take_new_row.
__device__ __forceinline__ void load_key(Raw &r, const AttnArgs &a, const KeyMap &km, int kg, bool zrow, int h) {
    r.kind = zrow ? 0 : -1;
    r.sigma = -1.0f;
    if (kg >= km.n_keys) return;
    if (kg < km.n_sel) {
        const int64_t off = cache_row(a.pm, a.cap, km.b, km.ids[kg]);   // checked when compacted
        const uint4 *src = reinterpret_cast<const uint4 *>(a.codes + off * kCodeBytes + 128 * h);
        const uint2 *sc = reinterpret_cast<const uint2 *>(a.scales + off * kScaleBytes + 16 * h);
#pragma unroll
        for (int st = 0; st < 2; ++st) {
#pragma unroll
            for (int u = 0; u < 4; ++u) r.c[st][u] = __ldg(src + 4 * st + u);
            r.sc[st] = __ldg(sc + st);
        }
        r.kind = 1;
        r.sigma = 1.0f;
    } else if (km.new_row != nullptr && kg == km.n_keys - 1) {
        r.kind = 3;
    } else {
        const int64_t pos = km.w0 + (kg - km.n_sel);
        const int64_t slot = km.ring_base + pos % a.wcap;
        const uint4 *src = reinterpret_cast<const uint4 *>(a.swa_codes + slot * kDim + 256 * h);
#pragma unroll
        for (int st = 0; st < 2; ++st)
#pragma unroll
            for (int u = 0; u < 8; ++u) r.c[st][u] = __ldg(src + 8 * st + u);
        r.sigma = __ldg(a.swa_scale + slot);
        r.kind = 2;
    }
}

// Kind 3 -> 2: the fused new SWA row, once warp 1 has quantised it into shared memory
// (bounded wait; on timeout the key is dropped as a zero row and flagged).
__device__ __forceinline__ void take_new_row(Raw &r, const AttnArgs &a, const KeyMap &km, int h, bool &new_ok) {
    if (!new_ok) new_ok = mbar_wait(km.new_ready, 0, a.wait.limit_ns, *km.smem);
    if (!new_ok) {
        set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
        r.kind = 0;
        r.sigma = -1.0f;
        return;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(km.new_row + 256 * h);
#pragma unroll
    for (int st = 0; st < 2; ++st)
#pragma unroll
        for (int u = 0; u < 8; ++u) r.c[st][u] = src[8 * st + u];
    r.sigma = *km.new_sigma;
    r.kind = 2;
}

// Channels 8 u .. 8 u + 7 of the thread's stage st as four f16x2 words (zeros for no key).
__device__ __forceinline__ void dq8(const Raw &r, int st, int u, uint32_t v[4]) {
    if (r.kind == 1) {
        const uint4 cv = r.c[st][u >> 2];
        const uint32_t w = (u & 3) == 0 ? cv.x : (u & 3) == 1 ? cv.y : (u & 3) == 2 ? cv.z : cv.w;
        // scale byte u / 2 (one per 16 channels): byte pair (u / 4) % 2 of word u / 8
        const uint32_t sw = (u >> 3) == 0 ? r.sc[st].x : r.sc[st].y;
        const uint32_t hs = cvt_e4m3x2_f16x2((sw >> (16 * ((u >> 2) & 1))) & 0xFFFFu);
        const uint32_t s2 = (((u >> 1) & 1) ? (hs >> 16) : (hs & 0xFFFFu)) * 0x10001u;
        const __half2 sv = *reinterpret_cast<const __half2 *>(&s2);
        cvt_e2m1x8_f16x2(w, v);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            __half2 x = __hmul2(*reinterpret_cast<__half2 *>(&v[k]), sv);
            v[k] = *reinterpret_cast<uint32_t *>(&x);
        }
    } else if (r.kind == 2) {
        // exact E4M3 codes; the row scale is applied in fp32 on the logit and on P
        const uint4 cv = r.c[st][u >> 1];
        const uint32_t w0 = (u & 1) ? cv.z : cv.x, w1 = (u & 1) ? cv.w : cv.y;
        v[0] = cvt_e4m3x2_f16x2(w0 & 0xFFFFu);
        v[1] = cvt_e4m3x2_f16x2(w0 >> 16);
        v[2] = cvt_e4m3x2_f16x2(w1 & 0xFFFFu);
        v[3] = cvt_e4m3x2_f16x2(w1 >> 16);
    } else {
        v[0] = v[1] = v[2] = v[3] = 0u;
    }
}

// The thread's K row of stage st into TMEM (taddr: lane 32 q, column of the stage's
// channel 0): 64 columns in four 16-column stores.
__device__ __forceinline__ void store_k(const Raw &r, int st, uint32_t taddr) {
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
        uint32_t v[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) dq8(r, st, 4 * qq + c, v + 4 * c);
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
            "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr + 16u * (uint32_t)qq),
            "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
            "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
            : "memory");
    }
}

// The thread's V row of stage st into row `row` of the shared-memory stage (fp16, swizzled).
__device__ __forceinline__ void store_v(const Raw &r, int st, uint8_t *stage, int row) {
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        uint32_t v[4];
        dq8(r, st, u, v);
        *reinterpret_cast<uint4 *>(stage + (u >> 3) * kCbBytes + swz(row, u & 7)) = make_uint4(v[0], v[1], v[2], v[3]);
    }
}

// Max (kMax) or sum over the warp's 32 lanes of each of 16 values; lane l ends with the
// reduction of value l % 16 (a butterfly reduce-scatter over 16 lanes, then one more
// exchange with the other half-warp).
template <bool kMax>
__device__ __forceinline__ float reduce_scatter16(const float *x, int lane) {
    float a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const bool hi = lane & 8;
        const float mine = hi ? x[8 + k] : x[k], other = hi ? x[k] : x[8 + k];
        const float o = __shfl_xor_sync(0xFFFFFFFFu, other, 8);
        a[k] = kMax ? fmaxf(mine, o) : mine + o;
    }
#pragma unroll
    for (int st = 4; st >= 1; st >>= 1) {
#pragma unroll
        for (int k = 0; k < st; ++k) {
            const bool hi = lane & st;
            const float mine = hi ? a[st + k] : a[k], other = hi ? a[k] : a[st + k];
            const float o = __shfl_xor_sync(0xFFFFFFFFu, other, st);
            a[k] = kMax ? fmaxf(mine, o) : mine + o;
        }
    }
    const float o = __shfl_xor_sync(0xFFFFFFFFu, a[0], 16);
    return kMax ? fmaxf(a[0], o) : a[0] + o;
}

// ---------------------------------------------------------------------------------------
// kRope: the fused append rotates the new SWA row first (a separate instantiation, so
// that the plain kernel carries none of its code).  Grid: (n32 * BT), n32 = ceil(H / 32).
template <bool kRope>
__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(AttnArgs a, int n32) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem &s = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qi = blockIdx.x / n32, hgrp = blockIdx.x % n32;
    const int b = qi / a.Tq;
    const int h0 = hgrp * kHeads;
    const int hcta = min(kHeads, a.H - h0);
    const uint64_t lim = a.wait.limit_ns;
    // ---- set-up -----------------------------------------------------------------------------
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&s.kv_full[i], kWorkWarps / 2);   // stage j: the 4 warps of channel half j / 2
            mbar_init(&s.kv_empty[i], 1);
        }
        mbar_init(&s.s_full[0], 1);
        mbar_init(&s.s_full[1], 1);
        mbar_init(&s.k_full, kWorkWarps);
        mbar_init(&s.p_full, kWorkWarps);
        mbar_init(&s.pv_done, 1);
        mbar_init(&s.drain, 1);
        mbar_init(&s.never, 1);
        mbar_init(&s.new_ready, 1);
        s.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&s.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    // The caller's inputs q, q_pos and swa_new are read before the dependency wait (no
    // kernel of this library writes them; see the header): Q is loaded, scaled and
    // staged while the previous kernel of the stream finishes.
    const int32_t t32 = a.q_pos[qi];
    const uint16_t *q = a.q + ((int64_t)qi * a.H + h0) * kDim;
    uint4 qv[kQChunks];   // chunk i = threadIdx.x + kThreads k: head i / 64, channels 8 (i % 64) .. + 7
#pragma unroll
    for (int k = 0; k < kQChunks; ++k) {
        const int i = threadIdx.x + kThreads * k;
        qv[k] = (i < kHeads * 64 && i / 64 < hcta) ? __ldg(reinterpret_cast<const uint4 *>(q) + i)
                                                   : make_uint4(0u, 0u, 0u, 0u);
    }
    uint4 xraw[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
    if (a.swa_new != nullptr && warp == 1) {
        const uint4 *src = reinterpret_cast<const uint4 *>(a.swa_new + (int64_t)qi * kDim + 16 * lane);
        xraw[0] = __ldg(src);
        xraw[1] = __ldg(src + 1);
    }
    {
        float qm = 0.0f;
#pragma unroll
        for (int k = 0; k < kQChunks; ++k) {
            const uint32_t w[4] = {qv[k].x, qv[k].y, qv[k].z, qv[k].w};
#pragma unroll
            for (int c = 0; c < 4; ++c)
                qm = fmaxf(qm, fmaxf(fabsf(bf16_bits_to_f32(w[c] & 0xFFFFu)), fabsf(bf16_bits_to_f32(w[c] >> 16))));
        }
        qm = warp_max(qm);
        if (lane == 0) s.wred[warp] = qm;
    }
    __syncthreads();
    float qmax = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) qmax = fmaxf(qmax, s.wred[w]);
    const int qexp = qmax > 0.0f ? max(0, ilogbf(qmax) - 14) : 0;   // max|q| * 2^-qexp < 2^15
    {
        const float inv = exp2f((float)-qexp);
#pragma unroll
        for (int k = 0; k < kQChunks; ++k) {
            const int i = threadIdx.x + kThreads * k;
            if (i >= kHeads * 64) break;
            const int hd = i / 64, ch8 = i % 64;
            const uint32_t w[4] = {qv[k].x, qv[k].y, qv[k].z, qv[k].w};
            uint32_t h[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                h[c] = pack_h2(bf16_bits_to_f32(w[c] & 0xFFFFu) * inv, bf16_bits_to_f32(w[c] >> 16) * inv);
            *reinterpret_cast<uint4 *>(s.q + (ch8 >> 3) * kQCbBytes + swz(hd, ch8 & 7)) =
                make_uint4(h[0], h[1], h[2], h[3]);
        }
    }
    // everything below may read what the previous kernel of the stream wrote (the Top-K)
    grid_dep_wait();
    const int *tk = a.topk + (int64_t)qi * a.top_k;
    const int e_id0 = (int)threadIdx.x < a.top_k ? tk[threadIdx.x] : -1;
    const int e_id1 = (int)threadIdx.x + kThreads < a.top_k ? tk[threadIdx.x + kThreads] : -1;
    const int64_t t = t32;
    const int64_t w0 = max64(0, t - a.swa_len + 1);
    const int n_win = a.swa_len > 0 ? (int)(t - w0 + 1) : 0;
    const int64_t n_vis = min64(visible_entries((int32_t)t, a.ratio), a.cap);
    auto entry_ok = [&](int e) {
        bool ok = e >= 0 && e < n_vis;
        if (e >= 0 && !ok && hgrp == 0) set_dev_err(a.dev_err, CSA2_DEVERR_INDEX);
        if (ok && cache_row(a.pm, a.cap, b, e) < 0) {
            if (hgrp == 0) set_dev_err(a.dev_err, CSA2_DEVERR_PAGE);
            ok = false;
        }
        return ok;
    };
    const bool e_ok0 = entry_ok(e_id0), e_ok1 = entry_ok(e_id1);
    if (threadIdx.x == 32 * 3 && a.swa_len > 0 && hgrp == 0) {
        // the request's whole SWA ring (rows are contiguous) and its scales
        prefetch_l2(a.swa_codes + (int64_t)b * a.wcap * kDim, (uint32_t)a.wcap * kDim);
        const float *sg = a.swa_scale + (int64_t)b * a.wcap;   // only whole 16-byte units
        if ((reinterpret_cast<uintptr_t>(sg) & 15) == 0 && (a.wcap & 3) == 0)
            prefetch_l2(sg, (uint32_t)a.wcap * 4);
    }
    const uint32_t bal0 = __ballot_sync(0xFFFFFFFFu, e_ok0), bal1 = __ballot_sync(0xFFFFFFFFu, e_ok1);
    if (lane == 0) {
        s.wcnt[warp] = __popc(bal0);
        s.wcnt[kWarps + warp] = __popc(bal1);
    }
    __syncthreads();
    // compaction in Top-K slot order: slots [0, kThreads) by warp, then [kThreads, 2 kThreads)
    int base0 = 0, base1 = 0, n_sel = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        base0 += w < warp ? s.wcnt[w] : 0;
        base1 += w < warp ? s.wcnt[kWarps + w] : 0;
        n_sel += s.wcnt[w];
    }
    base1 += n_sel;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) n_sel += s.wcnt[kWarps + w];
    const uint32_t below = (1u << lane) - 1u;
    if (e_ok0) s.ids[base0 + __popc(bal0 & below)] = e_id0;
    if (e_ok1) s.ids[base1 + __popc(bal1 & below)] = e_id1;
    const int n_keys = n_sel + n_win;         // the selected entries, then the window
    const int nt = (n_keys + kTK - 1) / kTK;
    const bool fuse = a.swa_new != nullptr && n_win > 0;
    KeyMap km;
    km.ids = s.ids;
    km.n_sel = n_sel;
    km.w0 = w0;
    km.n_keys = n_keys;
    km.b = b;
    km.ring_base = (int64_t)b * a.wcap;
    km.new_row = fuse ? s.swa_new : nullptr;
    km.new_sigma = &s.swa_new_sigma;
    km.new_ready = &s.new_ready;
    km.smem = &s;
    const bool worker = warp >= kWorkWarp0;
    // worker: key quadrant, and half (the softmax's 16 heads, the producer's 256 channels)
    const int qd = warp & 3, hh = (warp - kWorkWarp0) >> 2;
    const int r = 32 * qd + lane;                              // worker: key of the tile
    // rows of the tile's last 16-key group of valid keys are read by the output MMAs
    // and so written (zeros past the keys); rows after that group are not written
    auto zlim_of = [&](int i) { return ((min(kTK, n_keys - i * kTK) + 15) / 16) * 16; };
    bool new_ok = false;
    Raw raw;
    __syncthreads();                       // s.ids complete
    if (worker && nt > 0) load_key(raw, a, km, r, r < zlim_of(0), hh);   // tile 0, in flight
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = s.tmem_base;
    if (warp == 0) {
        // ---------------- MMA issuer (whole warp runs the loop; one lane issues) ----------------
        if (nt > 0) {
            bool ok = true;
            // S^T = K Q^T: A = stage (K-major, 128 keys), B = Q (K-major, 32 heads), M 128 N 32
            const uint32_t idesc_s = (1u << 4) | ((uint32_t)(kHeads >> 3) << 17) | ((uint32_t)(kTK >> 4) << 24);
            // O^T = V^T P^T: A = stage (MN-major, 128 channels), B = P^T (MN-major, 32 heads)
            const uint32_t idesc_o = (1u << 4) | (1u << 15) | (1u << 16) | ((uint32_t)(kHeads >> 3) << 17) |
                                     ((uint32_t)(kTK >> 4) << 24);
            const uint64_t qd_desc = sw128_desc(smem_u32(s.q), 16, 1024);
            // P^T rows are 64 bytes (32 heads): 8-row groups 512 bytes apart
            const uint64_t pd = sw64_desc(smem_u32(s.pt), 4096, 512);
            // S^T(i) once K(i) is in TMEM (A from TMEM: the 8 columns of 16 channels per step)
            auto issue_s = [&](int i) -> bool {
                const bool got = __shfl_sync(0xFFFFFFFFu, (int)mbar_wait(&s.k_full, i & 1, lim, s), 0) != 0;
                if (!got) return false;
                tc_fence_after();
                if (elect_one()) {
                    const uint32_t sd = tmem + kSCol + (uint32_t)kHeads * (uint32_t)(i & 1);
#pragma unroll 4
                    for (int k = 0; k < 32; ++k) {      // K-steps of 16 channels
                        const uint64_t boff = (uint64_t)((k >> 2) * (kQCbBytes >> 4) + (k & 3) * 2);
                        mma_f16_ta(sd, tmem + kKCol + 8u * (uint32_t)k, qd_desc + boff, idesc_s, k != 0 ? 1u : 0u);
                    }
                    mma_commit(&s.s_full[i & 1]);
                }
                __syncwarp();
                return true;
            };
            ok = issue_s(0);
            for (int i = 0; ok && i < nt; ++i) {
                // the next tile's scores first: they run while the softmax of this tile does
                if (i + 1 < nt && !(ok = issue_s(i + 1))) break;
                // P^T(i) from the softmax (the test hook makes the first of these waits stuck)
                const bool got = a.wait.stuck && i == 0 ? mbar_wait(&s.never, 0, lim, s)
                                                        : mbar_wait(&s.p_full, i & 1, lim, s);
                ok = __shfl_sync(0xFFFFFFFFu, (int)got, 0) != 0;
                if (!ok) break;
                tc_fence_after();
                const int nk = (min(kTK, n_keys - i * kTK) + 15) / 16;   // K-steps of valid keys
#pragma unroll 1
                for (int j = 0; j < kStages; ++j) {
                    ok = __shfl_sync(0xFFFFFFFFu, (int)mbar_wait(&s.kv_full[j], i & 1, lim, s), 0) != 0;
                    if (!ok) break;
                    tc_fence_after();
                    if (elect_one()) {
                        const uint64_t vd = sw128_desc(smem_u32(s.kv[j]), kCbBytes, 1024);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)    // 16 keys per step: 2048 B of V^T, 1024 B of P^T
                            if (kk < nk)
                                mma_f16(tmem + (uint32_t)kHeads * (uint32_t)j, vd + (uint64_t)(kk * 128),
                                        pd + (uint64_t)(kk * 64), idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(&s.kv_empty[j]);
                        if (j == kStages - 1) mma_commit(&s.pv_done);
                    }
                    __syncwarp();
                }
            }
            if (!ok && lane == 0) {
                atomicExch(&s.abort, 1);
                set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
            }
            // every MMA issued above has completed once this arrives
            if (elect_one()) mma_commit(&s.drain);
            __syncwarp();
            const bool drained = mbar_wait<false>(&s.drain, 0, kDrainLimitNs, s);
            (void)drained;
        }
    } else if (warp == 1) {
        if (fuse) {
            // The same FP8 row quantiser as csa2_quantize_append: codes and sigma go to
            // shared memory (the workers read the window's newest key from there, after
            // new_ready) and, from head group 0, to the ring slot t % wcap.
            float xnew[16];
            unpack_bf16x8(xraw[0], xnew);
            unpack_bf16x8(xraw[1], xnew + 8);
            if constexpr (kRope) {
                if (!rope_lane16(xnew, lane, a.rope.cs, a.rope.n_pos, a.rope.start, a.rope.pairs, t) &&
                    lane == 0 && hgrp == 0)
                    set_dev_err(a.dev_err, CSA2_DEVERR_ROPE);
            }
            quant_fp8_lanes<kDim>(xnew, s.swa_new, &s.swa_new_sigma, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.new_ready);
            if (hgrp == 0) {
                const int64_t slot = (int64_t)b * a.wcap + t % a.wcap;
                reinterpret_cast<uint4 *>(a.swa_codes + slot * kDim)[lane] =
                    reinterpret_cast<const uint4 *>(s.swa_new)[lane];
                if (lane == 0) a.swa_scale[slot] = s.swa_new_sigma;
            }
        }
    } else if (warp == 2) {
        // L2 prefetch of the entries of the later tiles (tile 0 is already in flight), by
        // one head group (the others read the same rows)
        if (hgrp == 0) {
            for (int kg = kTK + lane; kg < n_sel; kg += 32) {
                const int64_t row = cache_row(a.pm, a.cap, b, s.ids[kg]);
                prefetch_l2(a.codes + row * kCodeBytes, kCodeBytes);
                prefetch_l2(a.scales + row * kScaleBytes, kScaleBytes);
            }
        }
    } else if (worker) {
        // ---------------- workers ----------------
        // Tile i: wait for S^T(i); write K(i + 1) into TMEM (S^T(i) no longer reads it), so
        // that S^T(i + 1) runs during this softmax; the softmax of tile i (keys 32 qd ..,
        // heads 16 hh ..) -> P^T(i); V(i + 1) into the shared-memory stages as O^T(i)
        // releases them; then the raw bytes of tile i + 2.
        const float c0 = a.softmax_scale * 1.4426950408889634f * exp2f((float)qexp);
        const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
        const float4 *mrun4 = reinterpret_cast<const float4 *>(&s.mrun[16 * hh]);
        float lsum = 0.0f;   // head 16 hh + lane % 16: this warp's keys' share of l
        bool ok = true, stop = false;
        // K of the thread's key and channel half into TMEM; arrive k_full
        auto put_k = [&]() {
            if (raw.kind == 3) take_new_row(raw, a, km, hh, new_ok);
#pragma unroll
            for (int st = 0; st < 2; ++st)
                store_k(raw, st, tmem + lane_base + kKCol + 64u * (uint32_t)(2 * hh + st));
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.k_full);
        };
        // V of the thread's key and channel half into stages 2 hh, 2 hh + 1 of tile i (after
        // O^T(i - 1) has released them); s.ksig of the tile; arrive kv_full
        auto put_v = [&](int i) -> bool {
#pragma unroll
            for (int st = 0; st < 2; ++st) {
                const int j = 2 * hh + st;
                if (i > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(&s.kv_empty[j], (i - 1) & 1, lim, s))) return false;
                if (raw.kind >= 0) store_v(raw, st, s.kv[j], r);
                if (st == 0 && hh == 0) {
                    s.ksig[r] = raw.sigma;
                    // P carries sigma in fp16: p <= 2^8 needs sigma <= 65504 / 256
                    if (raw.kind == 2 && raw.sigma * 256.0f > 65504.0f && hgrp == 0)
                        set_dev_err(a.dev_err, CSA2_DEVERR_RANGE);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.kv_full[j]);
            }
            return true;
        };
        if (nt > 0) {
            put_k();
            ok = put_v(0);
            if (ok && nt > 1) load_key(raw, a, km, kTK + r, r < zlim_of(1), hh);
        }
        for (int i = 0; i < nt; ++i) {
            // ---- S^T(i) and the tile's key scales; the four warps of the half agree ----
            // (kv_full[2 hh] of tile i: the ksig writes of this half's... every h = 0 warp;
            // kv_full[0] covers them)
            const bool w_ok = ok && __all_sync(0xFFFFFFFFu, mbar_wait(&s.s_full[i & 1], (i >> 1) & 1, lim, s) &&
                                                                mbar_wait(&s.kv_full[0], i & 1, lim, s));
            stop = group_any(hh, !w_ok || aborted(s));
            if (stop) break;
            tc_fence_after();
            float x[16];
            tmem_ld16(tmem + lane_base + kSCol + (uint32_t)kHeads * (uint32_t)(i & 1) + 16u * (uint32_t)hh, x);
            // ---- K(i + 1) into TMEM: every lane of this warp has read S^T(i), which was
            // the last reader of K(i) ----
            tc_fence_before();
            if (i + 1 < nt) put_k();
            // ---- softmax of tile i ----
            const float sig = s.ksig[r];
            const bool valid = sig >= 0.0f;
            const float ck = c0 * sig;
            float dmax = -INFINITY;
#pragma unroll
            for (int h = 0; h < 16; ++h) x[h] = valid ? x[h] * ck : -INFINITY;   // logits, log2 units
            if (i > 0) {
                // x -> x - m in place: the lazy check, and (common case) the exponent of p
#pragma unroll
                for (int h4 = 0; h4 < 4; ++h4) {
                    const float4 mv = mrun4[h4];
                    x[4 * h4] -= mv.x; x[4 * h4 + 1] -= mv.y; x[4 * h4 + 2] -= mv.z; x[4 * h4 + 3] -= mv.w;
                    dmax = fmaxf(dmax, fmaxf(fmaxf(x[4 * h4], x[4 * h4 + 1]), fmaxf(x[4 * h4 + 2], x[4 * h4 + 3])));
                }
            }
            const bool upd = group_any(hh, i == 0 || dmax > kLazy);
            if (upd) {
                if (i > 0) {   // back to the logits (one rounding; p's exponent stays consistent)
#pragma unroll
                    for (int h4 = 0; h4 < 4; ++h4) {
                        const float4 mv = mrun4[h4];
                        x[4 * h4] += mv.x; x[4 * h4 + 1] += mv.y; x[4 * h4 + 2] += mv.z; x[4 * h4 + 3] += mv.w;
                    }
                }
                // exact tile max per head, then the running max moves
                const float wm = reduce_scatter16<true>(x, lane);   // head 16 hh + lane % 16
                if (lane < 16) s.red[hh][qd][lane] = wm;
                group_sync(hh);
                if (qd == 0 && lane < 16) {
                    const float tm = fmaxf(fmaxf(s.red[hh][0][lane], s.red[hh][1][lane]),
                                           fmaxf(s.red[hh][2][lane], s.red[hh][3][lane]));
                    const float old = i > 0 ? s.mrun[16 * hh + lane] : -INFINITY;
                    const float mn = fmaxf(old, tm);
                    s.mrun[16 * hh + lane] = mn;
                    s.alpha[16 * hh + lane] = old == -INFINITY ? 0.0f : ex2(old - mn);
                }
                group_sync(hh);
                lsum *= s.alpha[16 * hh + (lane & 15)];
#pragma unroll
                for (int h4 = 0; h4 < 4; ++h4) {
                    const float4 mv = mrun4[h4];
                    x[4 * h4] -= mv.x; x[4 * h4 + 1] -= mv.y; x[4 * h4 + 2] -= mv.z; x[4 * h4 + 3] -= mv.w;
                }
            }
            // p = 2^(x - m); P^T carries the key's scale (V holds SWA codes, not values)
            const float sv = valid ? sig : 0.0f;
            uint32_t pk[8];
#pragma unroll
            for (int h2 = 0; h2 < 8; ++h2) {
                const float p0 = ex2(x[2 * h2]), p1 = ex2(x[2 * h2 + 1]);
                x[2 * h2] = p0;
                x[2 * h2 + 1] = p1;
                pk[h2] = pack_h2(p0 * sv, p1 * sv);
            }
#pragma unroll
            for (int c = 0; c < 2; ++c)   // heads 16 hh + 8 c .. : chunk 2 hh + c of the key's row
                *reinterpret_cast<uint4 *>(s.pt + swz64(r, 2 * hh + c)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            if (upd && i > 0) {
                // the running max moved: wait for O^T(i - 1) (issued after S^T(i + 1), so not
                // implied by s_full(i)), then scale this warp's 16 head columns of every block
                // before O^T(i) accumulates on them
                const bool pv = __all_sync(0xFFFFFFFFu, mbar_wait(&s.pv_done, (i - 1) & 1, lim, s));
                if (!pv && lane == 0) {
                    atomicExch(&s.abort, 1);
                    set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
                }
                tc_fence_after();
                float f[16];
#pragma unroll
                for (int h = 0; h < 16; ++h) f[h] = s.alpha[16 * hh + h];
#pragma unroll 1
                for (int j = 0; j < kStages; ++j)
                    tmem_scale16(tmem + lane_base + (uint32_t)kHeads * (uint32_t)j + 16u * (uint32_t)hh, f);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.p_full);
            lsum += reduce_scatter16<false>(x, lane);   // this tile's 32 keys, after P^T is released
            // ---- V(i + 1) into the stages as O^T(i) releases them; raw bytes of tile i + 2 ----
            if (ok && i + 1 < nt) {
                ok = put_v(i + 1);
                if (ok && i + 2 < nt) load_key(raw, a, km, (i + 2) * kTK + r, r < zlim_of(i + 2), hh);
            }
        }
        ok = ok && !stop;
        if (ok && nt > 0) {
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s.pv_done, (nt - 1) & 1, lim, s));
            tc_fence_after();
        }
        if (!ok && lane == 0) {
            atomicExch(&s.abort, 1);
            set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
        }
        // the sum per head over the four quadrants; 1 / l and the log-sum-exp (the group
        // barrier is taken by all four warps of the half, aborted or not)
        if (lane < 16) s.red[hh][qd][lane] = lsum;
        group_sync(hh);
        if (qd == 0 && lane < 16) {
            const int h = 16 * hh + lane;
            const bool have = nt > 0 && !aborted(s);
            const float l = have ? s.red[hh][0][lane] + s.red[hh][1][lane] + s.red[hh][2][lane] + s.red[hh][3][lane]
                                 : 0.0f;
            const bool valid = h < hcta && l > 0.0f;
            s.wfin[h] = valid ? 1.0f / l : 0.0f;
            if (h < hcta)
                a.lse[(int64_t)qi * a.H + h0 + h] =
                    valid ? (s.mrun[h] + log2f(l)) * 0.6931471805599453f : -INFINITY;
        }
    }

    // ---- output: O^T / l, straight from TMEM --------------------------------------------------
    __syncwarp();
    tc_fence_before();
    __syncthreads();                       // 1 / l written; every MMA of the CTA has completed
    tc_fence_after();
    grid_dep_launch();
    // Task u (32; warp u % 12 takes u, so the TMEM lane quadrant u % 4 is the warp's):
    // channels 32 (u % 4) .. of block (u >> 2) & 3, heads 16 (u >> 4) .. .  A thread holds
    // one channel of 16 heads; a warp store covers 32 consecutive channels of one head.
    const bool have = __shfl_sync(0xFFFFFFFFu, (int)(nt > 0 && !aborted(s)), 0) != 0;
#pragma unroll 1
    for (int u = warp; u < 32; u += kWarps) {
        const int cq = u & 3, blk = (u >> 2) & 3, hp = u >> 4;
        float o[16];
        if (have) {
            tmem_ld16(tmem + ((uint32_t)(32 * cq) << 16) + (uint32_t)kHeads * (uint32_t)blk + 16u * (uint32_t)hp, o);
        } else {
#pragma unroll
            for (int h = 0; h < 16; ++h) o[h] = 0.0f;
        }
        float *dst = a.out + ((int64_t)qi * a.H + h0) * kDim + 128 * blk + 32 * cq + lane;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int h = 16 * hp + k;
            if (h < hcta) dst[(int64_t)h * kDim] = o[k] * s.wfin[h];
        }
    }
    tc_fence_before();
    __syncthreads();                       // every TMEM load of the CTA has completed
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

}  // namespace attn

size_t attn_smem_bytes() { return sizeof(attn::Smem) + 1024; }

template <bool kRope>
static cudaError_t launch_attn_t(const AttnArgs &a, int BT, cudaStream_t st) {
    const size_t smem = attn_smem_bytes();
    static std::atomic<uint64_t> configured{0};   // per device
    {
        cudaError_t e = config_kernel_once(attn::attn_kernel<kRope>, smem, configured);
        if (e != cudaSuccess) return e;
    }
    const int n32 = (a.H + attn::kHeads - 1) / attn::kHeads;
    cudaError_t e = launch_pdl(attn::attn_kernel<kRope>, dim3(n32 * BT), dim3(attn::kThreads), smem, st, a, n32);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_sparse_attn(const AttnArgs &a, int BT, cudaStream_t st) {
    return a.swa_new != nullptr && a.rope.cs != nullptr ? launch_attn_t<true>(a, BT, st)
                                                         : launch_attn_t<false>(a, BT, st);
}

}  // namespace csa2
