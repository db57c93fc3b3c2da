// csa2_attn.cu -- a8 sparse decode attention on the 5th-generation tensor cores
// (and, for decode, the a2 append of the layer's SWA row, fused in).
//
// DeepSeek V4.1 Flash study notes, sections 1, 2 and 4: each layer attends, with
// its own query, over at most 512 selected global entries (FP4, dequantised on
// read; the cache format saves storage, the attention matmul itself is not FP4)
// together with its own 128-token FP8 SWA window; one softmax over the union.
// K = V = the 512-channel entry (MQA, fixed for this build).
//
// Work split: a cluster of CS CTAs per (query, group of 64 heads), CS = 4 when the
// grid still fits the SMs (small batches), else 2.  The query's keys (selected entries
// first, then the window) are cut in CS chunks of a multiple of 16; each CTA runs an
// independent online softmax over its chunk.  At the end the partial maxima and sums
// are exchanged through distributed shared memory, and each CTA finalises 4 / CS of
// the four 128-channel output blocks from its own partial and the others' (bulk
// copies between the CTAs' shared memories).
//
// Transposed tiles.  A tile is 64 keys.  The scores are S^T = K Q^T with the keys as
// the MMA's M = 64 (TMEM lanes 32 q .. 32 q + 15 hold keys 16 q .. 16 q + 15) and the
// 64 heads as N; the output is O^T = V^T P^T with the channels as M (four 128-channel
// blocks, M = 128) and the heads as N.  One fp16 tile in shared memory serves both:
// four stages of 128 channels x 64 keys, each the K-major A operand of S^T (rows =
// keys) and the MN-major A operand of O^T (M = channels contiguous in a row).  fp16
// holds the FP4 values exactly (e2m1 x e4m3 has at most 6 significant bits); an SWA
// row is stored as its exact E4M3 codes and its scale sigma is applied in fp32, to the
// logit and folded into P.  Q (the K-major B operand of S^T) is converted to fp16
// after an exact power-of-two scaling that keeps max|q| below 2^15.
//
// Two tiles in flight.  The worker warps form two sets of four; set s owns the tiles
// h with h % 2 == s and its own tile buffer, S^T accumulator and P^T buffer.  The MMA
// warp issues S^T(h) and then O^T(h - 1), so the score MMAs of one set's tile run
// while the other set takes the softmax of its own, and the output MMAs of a tile run
// while the next tile is being written.  The running max is handed from tile to tile
// (an mbarrier per set); each thread keeps its row-sum partial against the max it last
// saw, so neither set ever rescales the other's sums.
//
// 12 warps, specialised:
//   warp 0       TMEM allocation + the MMA issue loop (one elected lane issues);
//   warp 1       fused append only: quantises the query token's new SWA row;
//   warp 2       prefetches the entries of this CTA's later tiles into L2 (bulk prefetch;
//                the set-up prefetches the request's SWA ring);
//   warps 4-11   workers: set (w - 4) / 4, TMEM lane quadrant w % 4.  Producer: the warp
//                gathers keys 16 (w % 4) .. + 15 of its set's next tile warp-cooperatively
//                (one load instruction = one 64-byte stage slice of 8 keys), all four
//                stages in registers before the softmax of the set's current tile, and
//                dequantises stage j as soon as O^T of the set's previous tile has read
//                it.  Softmax: the warp reads its 16 keys x 64 heads with one
//                tcgen05.ld.16x256b.x8 (a thread: 2 keys x 16 heads).
// TMEM (512 columns): O^T block j (channels 128 j .. 128 j + 127) at columns
// 64 j .. 64 j + 63 (column = head); the two sets' S^T at columns 256 and 320.
// Online softmax in the log2 domain with lazy rescaling: the running max of a head
// moves (and O is rescaled) only when a tile's logit exceeds it by more than 8, so
// p <= 2^8 stays safe in fp16.  The check is per tile; the exact tile max (a shuffle
// reduce-scatter within a warp, then across the set's four warps) is formed only when
// it fires, and always on the first tile.
// Every wait is bounded (WaitCfg): on timeout the kernel flags CSA2_DEVERR_TIMEOUT,
// waits (bounded) for the MMAs it issued, still takes part in both cluster barriers
// of the combine, frees TMEM and returns.  The four warps of a set agree on leaving
// the tile loop through a barrier reduction, so that no named barrier is ever left
// waiting for a warp that has gone.
#include <cuda_fp16.h>
#include <stdint.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {
namespace attn {

constexpr int kThreads = 384;
constexpr int kWarps = kThreads / 32;
constexpr int kQChunks = (64 * 64 + kThreads - 1) / kThreads;   // 16-byte Q chunks per thread
constexpr int kTK = 64;                        // keys per tile (S^T M)
constexpr int kSets = 2;                       // worker sets = tiles in flight
constexpr int kCh = 128;                       // channels per O^T block (its M, TMEM lanes)
constexpr int kHeads = 64;                     // heads per CTA (MMA N)
constexpr int kStages = 4;                     // 128-channel quarters of a tile
constexpr int kStageBytes = kTK * 128 * 2;     // 64 keys x 128 channels fp16
constexpr int kCbBytes = kTK * 128;            // one 64-channel block of a stage
constexpr int kQCbBytes = kHeads * 128;        // one 64-channel block of Q
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 256;                // S^T of set s at columns 256 + 64 s
constexpr int kWorkWarp0 = 4;                  // softmax + producer warps 4..11
constexpr int kSetWarps = 4;                   // warps per set (one per TMEM lane quadrant)
constexpr float kLazy = 8.0f;                  // rescale threshold (log2 units)
constexpr int kMaxCS = 4;                      // CTAs per query (cluster size): 2 or 4

struct __align__(1024) Smem {
    uint8_t q[8 * kQCbBytes];                  // Q fp16, [8 cb][64 heads][128 B] swizzled
    uint8_t kv[kSets][kStages][kStageBytes];   // set s, stage j: [2 cb][64 keys][128 B] swizzled
    uint8_t pt[kSets][kTK * 128];              // P^T fp16 of set s, [64 keys][64 heads] swizzled
    int32_t ids[CSA2_TOPK_MAX];                // compacted selected entry ids
    float ksig[kSets][kTK];                    // per key of the tile: 1 FP4, sigma SWA, -1 none
    alignas(16) uint8_t swa_new[kDim];         // fused append: the new SWA row (E4M3 codes)
    float swa_new_sigma;
    alignas(16) float red[kSets][kSetWarps][kHeads];    // per set and warp: tile max / row sums
    alignas(16) float mref[kSets][kSetWarps][kHeads];   // the max the row sums are taken against
    alignas(16) float mrun[kHeads];            // running max per head (log2 domain)
    alignas(16) float alpha[kSets][kHeads];    // factor of the last move of the running max
    float cm[kHeads], cl[kHeads];              // this CTA's partial max / sum per head
    float pm[kMaxCS][kHeads], pl[kMaxCS][kHeads];   // every CTA's partial max / sum, by rank
    float wself[kHeads];                       // combine: weight of this CTA's partial
    uint64_t kv_full[kSets][kStages], kv_empty[kSets][kStages];
    uint64_t s_full[kSets], p_full[kSets], pv_done[kSets], m_ready[kSets], drain, never;
    uint64_t new_ready;                        // fused append: the new SWA row is in smem
    uint64_t xfer[2];                          // combine: the peers' parts of head half h have landed
    uint32_t tmem_base;
    int32_t abort;
    float wred[kWarps];
    int32_t wcnt[2 * kWarps];
};

static_assert(sizeof(Smem) + 1024 <= 227 * 1024, "one CTA per SM: at most 227 KB of shared memory");

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
// 32 lanes x 32 columns: thread t of the warp reads TMEM lane (base + t), 32 columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 16 lanes x 64 columns (16x256b, 8 repeats): thread t reads lanes base + t / 4 and
// base + t / 4 + 8, columns 8 r + 2 (t % 4) and + 1 of repeat r, as
// v[4 r] v[4 r + 1] (first lane) and v[4 r + 2] v[4 r + 3] (second lane).
__device__ __forceinline__ void tmem_ld16x64(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
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
// Named barrier of the four warps of worker set `set` (ids 1, 2).
__device__ __forceinline__ void group_sync(int set) {
    asm volatile("bar.sync %0, 128;" ::"r"(1 + set) : "memory");
}
// The same barrier with an OR over the four warps' predicates: every thread of the
// set receives the same answer.
__device__ __forceinline__ bool group_any(int set, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n.reg .pred p, q;\n"
        "setp.ne.u32 p, %1, 0;\n"
        "bar.red.or.pred q, %2, 128, p;\n"
        "selp.u32 %0, 1, 0, q;\n}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(1 + set)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
                 : "memory");
}
// Bulk copy from this CTA's shared memory into the peer CTA's (dst and bar are
// shared::cluster addresses; completes as bytes on bar).  No multicast.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "r"(smem_u32(src)), "r"(bytes), "r"(bar)
        : "memory");
}
// L2 prefetch of [p, p + bytes) (p 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
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
__device__ __forceinline__ void st_peer(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Byte offset of (row, 16-byte chunk c of a 128-byte row) in a 128B-swizzled block.
__device__ __forceinline__ uint32_t swz(int row, int c) {
    return (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4));
}

// ---- producer: warp-cooperative gather, a whole tile ahead ------------------------------
// Worker warp wi (0..7) produces keys 16 wi .. 16 wi + 15 of a tile, as two groups of 8.
// Lane l of a group handles key 4 ((l >> 3) & 1) + ((l & 7) >> 1) of the group and piece
// p = 2 (l >> 4) + (l & 1) of every 128-channel stage: channels 32 p .. 32 p + 31, i.e.
// chunks 4 (p & 1) .. + 3 of block p >> 1.  So one load instruction reads one 64-byte
// stage slice of 8 keys (8 cache lines, not 32), and a quarter-warp's 16-byte shared
// stores hit 4 consecutive rows x 2 chunk halves: 8 distinct bank groups.
constexpr int kGroups = 2;         // key groups of 8 per worker warp and tile

__device__ __forceinline__ int prod_key(int wi, int g, int lane) {   // key of the tile
    return 16 * wi + 8 * g + 4 * ((lane >> 3) & 1) + ((lane & 7) >> 1);
}
__device__ __forceinline__ int prod_piece(int lane) { return 2 * (lane >> 4) + (lane & 1); }

struct Raw {
    uint4 c[kGroups][kStages][2];   // FP4: c[g][j][0] = 32 codes of stage j; SWA: 32 E4M3 codes
    uint32_t sc[kGroups][2];        // FP4: the 2 scale bytes of stage j at bits 16 (j & 1) of sc[g][j >> 1]
    float sigma[kGroups];           // 1 for an FP4 entry, the row scale of an SWA row, -1 for no key
    int kind[kGroups];              // 1 FP4 entry, 2 SWA row, 3 the fused new SWA row (not yet read),
                                    // 0 zero row, -1 nothing
};

struct KeyMap {      // this CTA's keys and where each comes from
    const int32_t *ids;
    int n_sel;
    int64_t w0;      // first window position
    int n_keys;      // keys of the query (selection + window)
    int k_end;       // end of this CTA's key range
    int64_t b;
    int64_t ring_base;
    const uint8_t *new_row;   // fused append: the newest window key is this row (smem)
    const float *new_sigma;
    uint64_t *new_ready;      // ... written once this completes
    const Smem *smem;
};

// Issue every load of the lane's two keys (all four stages: one memory round trip).
// kg0: the tile's first key; zlim: keys of the tile below zlim are written (zero rows
// past the valid keys).  The fused new SWA row is only marked here (kind 3).
__device__ __forceinline__ void load_keys(Raw &r, const AttnArgs &a, const KeyMap &km, int kg0, int zlim,
                                          int wi, int lane) {
    const int p = prod_piece(lane);
#pragma unroll
    for (int g = 0; g < kGroups; ++g) {
        const int kt = prod_key(wi, g, lane), kg = kg0 + kt;
        r.kind[g] = kt < zlim ? 0 : -1;
        r.sigma[g] = -1.0f;
        if (kg >= km.k_end) continue;
        if (kg < km.n_sel) {
            const int64_t off = cache_row(a.pm, a.cap, km.b, km.ids[kg]);   // checked when compacted
            const uint4 *src = reinterpret_cast<const uint4 *>(a.codes + off * kCodeBytes + 16 * p);
            const uint16_t *sc = reinterpret_cast<const uint16_t *>(a.scales + off * kScaleBytes + 2 * p);
#pragma unroll
            for (int j = 0; j < kStages; ++j) r.c[g][j][0] = __ldg(src + 4 * j);
            r.sc[g][0] = (uint32_t)__ldg(sc) | ((uint32_t)__ldg(sc + 4) << 16);
            r.sc[g][1] = (uint32_t)__ldg(sc + 8) | ((uint32_t)__ldg(sc + 12) << 16);
            r.kind[g] = 1;
            r.sigma[g] = 1.0f;
        } else if (km.new_row != nullptr && kg == km.n_keys - 1) {
            r.kind[g] = 3;
        } else {
            const int64_t pos = km.w0 + (kg - km.n_sel);
            const int64_t slot = km.ring_base + pos % a.wcap;
            const uint4 *src = reinterpret_cast<const uint4 *>(a.swa_codes + slot * kDim + 32 * p);
#pragma unroll
            for (int j = 0; j < kStages; ++j) {
                r.c[g][j][0] = __ldg(src + 8 * j);
                r.c[g][j][1] = __ldg(src + 8 * j + 1);
            }
            r.sigma[g] = __ldg(a.swa_scale + slot);
            r.kind[g] = 2;
        }
    }
}

// Kind 3 -> 2: the fused new SWA row, once warp 1 has quantised it into shared memory
// (bounded wait; on timeout the key is dropped as a zero row and flagged).
__device__ __forceinline__ void take_new_row(Raw &r, int g, const AttnArgs &a, const KeyMap &km, int lane,
                                             bool &new_ok) {
    if (!new_ok) new_ok = mbar_wait(km.new_ready, 0, a.wait.limit_ns, *km.smem);
    if (!new_ok) {
        set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
        r.kind[g] = 0;
        r.sigma[g] = -1.0f;
        return;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(km.new_row + 32 * prod_piece(lane));
#pragma unroll
    for (int j = 0; j < kStages; ++j) {
        r.c[g][j][0] = src[8 * j];
        r.c[g][j][1] = src[8 * j + 1];
    }
    r.sigma[g] = *km.new_sigma;
    r.kind[g] = 2;
}

// Dequantise stage j of the lane's piece of key row `row` (fp16, swizzled).
__device__ __forceinline__ void store_piece(const Raw &r, int g, int j, uint8_t *stage, int row, int lane) {
    const int p = prod_piece(lane);
    uint8_t *blk = stage + (p >> 1) * kCbBytes;
    const int c0 = 4 * (p & 1);
    const int kind = r.kind[g];
    if (kind == 1) {
        const uint32_t two = (r.sc[g][j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
        const uint32_t hs = cvt_e4m3x2_f16x2(two);
        const uint32_t scale2[2] = {(hs & 0xFFFFu) * 0x10001u, (hs >> 16) * 0x10001u};   // per 16 channels
        const uint4 cv = r.c[g][j][0];
#pragma unroll
        for (int c = 0; c < 4; ++c) {                  // 8 channels per 32-bit code word
            const uint32_t w = c == 0 ? cv.x : c == 1 ? cv.y : c == 2 ? cv.z : cv.w;
            const __half2 sv = *reinterpret_cast<const __half2 *>(&scale2[c >> 1]);
            uint32_t v[4];
            cvt_e2m1x8_f16x2(w, v);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                __half2 x = __hmul2(*reinterpret_cast<__half2 *>(&v[k]), sv);
                v[k] = *reinterpret_cast<uint32_t *>(&x);
            }
            *reinterpret_cast<uint4 *>(blk + swz(row, c0 + c)) = make_uint4(v[0], v[1], v[2], v[3]);
        }
    } else if (kind == 2) {
        // exact E4M3 codes; the row scale is applied in fp32 on the logit and on P
#pragma unroll
        for (int c = 0; c < 4; ++c) {                  // 8 channels = 8 code bytes
            const uint4 cv = r.c[g][j][c >> 1];
            const uint32_t w0 = (c & 1) ? cv.z : cv.x, w1 = (c & 1) ? cv.w : cv.y;
            *reinterpret_cast<uint4 *>(blk + swz(row, c0 + c)) =
                make_uint4(cvt_e4m3x2_f16x2(w0 & 0xFFFFu), cvt_e4m3x2_f16x2(w0 >> 16),
                           cvt_e4m3x2_f16x2(w1 & 0xFFFFu), cvt_e4m3x2_f16x2(w1 >> 16));
        }
    } else if (kind == 0) {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4 *>(blk + swz(row, c0 + c)) = z;
    }
}

// Max (kMax) or sum over the 16 keys of a softmax warp, per head.  A thread holds
// x[4 r + e] (its first key) and x[4 r + 2 + e] (its second key) of head 8 r + 2 (lane
// % 4) + e; value i = 2 r + e is the reduction of that head over the thread's two keys,
// then over the eight lanes that share lane % 4.  The lane ends with values 2 (lane / 4)
// and 2 (lane / 4) + 1 (a butterfly reduce-scatter over lane bits 4, 3, 2: 14 shuffles).
template <bool kMax>
__device__ __forceinline__ float2 reduce_keys16(const float *x, int lane) {
    auto val = [&](int i) {
        const float p = x[4 * (i >> 1) + (i & 1)], q = x[4 * (i >> 1) + 2 + (i & 1)];
        return kMax ? fmaxf(p, q) : p + q;
    };
    float a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const bool hi = lane & 16;
        const float lo_v = val(k), hi_v = val(8 + k);
        const float mine = hi ? hi_v : lo_v, other = hi ? lo_v : hi_v;
        const float o = __shfl_xor_sync(0xFFFFFFFFu, other, 16);
        a[k] = kMax ? fmaxf(mine, o) : mine + o;
    }
#pragma unroll
    for (int st = 4; st >= 2; st >>= 1) {
#pragma unroll
        for (int k = 0; k < st; ++k) {
            const bool hi = lane & (2 * st);
            const float mine = hi ? a[st + k] : a[k], other = hi ? a[k] : a[st + k];
            const float o = __shfl_xor_sync(0xFFFFFFFFu, other, 2 * st);
            a[k] = kMax ? fmaxf(mine, o) : mine + o;
        }
    }
    return make_float2(a[0], a[1]);
}

// ---------------------------------------------------------------------------------------
// kRope: the fused append rotates the new SWA row first (a separate instantiation, so
// that the plain kernel carries none of its code).  CS: CTAs per query (the cluster,
// set at launch), 2 or 4.
template <bool kRope, int CS>
__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(AttnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem &s = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Settled: the next launch may start at once; it computes from its queries only after
    // this kernel has completed, and this kernel completes only after its MMA warp has
    // waited for the previous launch (below), so the layers' compute stays in order.
    if (a.settled) grid_dep_launch();
    const uint32_t rank = cluster_rank();
    const int qi = blockIdx.x / CS;
    const int b = qi / a.Tq;
    const int h0 = blockIdx.y * kHeads;
    const int hcta = min(kHeads, a.H - h0);
    const uint64_t lim = a.wait.limit_ns;
    // ---- set-up -----------------------------------------------------------------------------
    if (threadIdx.x == 0) {
        for (int st = 0; st < kSets; ++st) {
            for (int i = 0; i < kStages; ++i) {
                mbar_init(&s.kv_full[st][i], kSetWarps);
                mbar_init(&s.kv_empty[st][i], 1);
            }
            mbar_init(&s.s_full[st], 1);
            mbar_init(&s.p_full[st], kSetWarps);
            mbar_init(&s.pv_done[st], 1);
            mbar_init(&s.m_ready[st], kSetWarps);
        }
        mbar_init(&s.drain, 1);
        mbar_init(&s.never, 1);
        mbar_init(&s.new_ready, 1);
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
    // Everything below may read what the previous kernel of the stream wrote (the
    // Top-K), unless the caller settled every input before the most recent ordinary
    // launch (an ordinary launch waits for its predecessor before it lets the next one
    // start, so whatever was written before it is complete here).  Settled, the set-up
    // and the first tiles' gathers and dequantisation run at once and the wait moves to
    // the MMA warp, before the first score MMA: nothing computed from this layer's
    // queries starts before the previous launch has completed (in the model a layer's
    // queries come from the previous layer's output).
    if (!a.settled) {
        grid_dep_wait();
        grid_dep_launch();   // the previous launch has completed: the next may start
    }
    const int *tk = a.topk + (int64_t)qi * a.top_k;
    const int e_id0 = (int)threadIdx.x < a.top_k ? tk[threadIdx.x] : -1;
    const int e_id1 = (int)threadIdx.x + kThreads < a.top_k ? tk[threadIdx.x + kThreads] : -1;
    const int64_t t = t32;
    const int64_t w0 = max64(0, t - a.swa_len + 1);
    const int n_win = a.swa_len > 0 ? (int)(t - w0 + 1) : 0;
    const int64_t n_vis = min64(visible_entries((int32_t)t, a.ratio), a.cap);
    auto entry_ok = [&](int e) {
        bool ok = e >= 0 && e < n_vis;
        if (e >= 0 && !ok) set_dev_err(a.dev_err, CSA2_DEVERR_INDEX);
        if (ok && cache_row(a.pm, a.cap, b, e) < 0) {
            set_dev_err(a.dev_err, CSA2_DEVERR_PAGE);
            ok = false;
        }
        return ok;
    };
    const bool e_ok0 = entry_ok(e_id0), e_ok1 = entry_ok(e_id1);
    if (threadIdx.x == 32 * 3 && a.swa_len > 0 && rank == 0) {
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
    // this CTA's key range: the query's keys cut in CS chunks of a multiple of 16
    const int n_keys = n_sel + n_win;
    const int chunk = ((n_keys + CS - 1) / CS + 15) / 16 * 16;
    const int k0 = min(n_keys, (int)rank * chunk), k1 = min(n_keys, k0 + chunk);
    const int nt = (k1 - k0 + kTK - 1) / kTK;   // tiles; tile h belongs to worker set h % 2
    const bool fuse = a.swa_new != nullptr && n_win > 0;
    const uint32_t owner = n_keys > 0 ? (uint32_t)((n_keys - 1) / chunk) : 0u;   // holds the newest key
    KeyMap km;
    km.ids = s.ids;
    km.n_sel = n_sel;
    km.w0 = w0;
    km.n_keys = n_keys;
    km.k_end = k1;
    km.b = b;
    km.ring_base = (int64_t)b * a.wcap;
    km.new_row = fuse && rank == owner ? s.swa_new : nullptr;
    km.new_sigma = &s.swa_new_sigma;
    km.new_ready = &s.new_ready;
    km.smem = &s;
    const bool worker = warp >= kWorkWarp0;
    const int set = (warp - kWorkWarp0) >> 2;   // worker: set, its tiles h = set, set + 2, ..
    const int qd = warp & 3;                     // worker: TMEM lane quadrant, keys 16 qd .. of a tile
    // rows of the tile's last 16-key group of valid keys are read by the output MMAs
    // and so written (zeros past the keys); rows after that group are not written
    auto zlim_of = [&](int i) { return ((min(kTK, k1 - k0 - i * kTK) + 15) / 16) * 16; };
    bool new_ok = false;
    Raw raw;
    __syncthreads();                       // s.ids complete
    if (worker && set < nt) load_keys(raw, a, km, k0 + set * kTK, zlim_of(set), qd, lane);   // in flight
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = s.tmem_base;
    if (warp == 0) {
        // ---------------- MMA issuer (whole warp runs the loop; one lane issues) ----------------
        // Issue order S^T(0), S^T(1), O^T(0), S^T(2), O^T(1), ..: the scores of the next
        // tile go ahead of the output of this one.
        if (nt > 0) {
            bool ok = true;
            // S^T = K Q^T: A = stage (K-major, 64 keys), B = Q (K-major, 64 heads), M 64 N 64
            const uint32_t idesc_s = (1u << 4) | ((uint32_t)(kHeads >> 3) << 17) | ((uint32_t)(kTK >> 4) << 24);
            // O^T = V^T P^T: A = stage (MN-major, 128 channels), B = P^T (MN-major, 64 heads)
            const uint32_t idesc_o = (1u << 4) | (1u << 15) | (1u << 16) | ((uint32_t)(kHeads >> 3) << 17) |
                                     ((uint32_t)(kCh >> 4) << 24);
            const uint64_t qd_desc = sw128_desc(smem_u32(s.q), 16, 1024);
            if (a.settled) grid_dep_wait();
            for (int h = 0; ok && h <= nt; ++h) {
                if (h < nt) {
                    const int bs = h & 1;
                    const uint32_t sd = tmem + kSCol + 64u * (uint32_t)bs;
#pragma unroll 1
                    for (int j = 0; j < kStages; ++j) {
                        ok = __shfl_sync(0xFFFFFFFFu, (int)mbar_wait(&s.kv_full[bs][j], (h >> 1) & 1, lim, s), 0) != 0;
                        if (!ok) break;
                        tc_fence_after();
                        if (elect_one()) {
                            const uint64_t kd = sw128_desc(smem_u32(s.kv[bs][j]), 16, 1024);
#pragma unroll
                            for (int k = 0; k < 8; ++k) {       // K-steps of 16 channels
                                const uint64_t aoff = (uint64_t)((k >> 2) * (kCbBytes >> 4) + (k & 3) * 2);
                                const uint64_t boff = (uint64_t)((2 * j + (k >> 2)) * (kQCbBytes >> 4) + (k & 3) * 2);
                                mma_f16(sd, kd + aoff, qd_desc + boff, idesc_s, (j | k) != 0 ? 1u : 0u);
                            }
                            if (j == kStages - 1) mma_commit(&s.s_full[bs]);
                        }
                        __syncwarp();
                    }
                    if (!ok) break;
                }
                if (h == 0) continue;
                // O^T(h - 1) once its P^T is written (the test hook makes the first of these
                // waits stuck)
                const int ho = h - 1, bo = ho & 1;
                const bool got = a.wait.stuck && ho == 0 ? mbar_wait(&s.never, 0, lim, s)
                                                         : mbar_wait(&s.p_full[bo], (ho >> 1) & 1, lim, s);
                ok = __shfl_sync(0xFFFFFFFFu, (int)got, 0) != 0;
                if (!ok) break;
                tc_fence_after();
                const int nk = (min(kTK, k1 - k0 - ho * kTK) + 15) / 16;   // K-steps of valid keys
                if (elect_one()) {
                    const uint64_t pd = sw128_desc(smem_u32(s.pt[bo]), 8192, 1024);
#pragma unroll 1
                    for (int j = 0; j < kStages; ++j) {
                        const uint64_t vd = sw128_desc(smem_u32(s.kv[bo][j]), kCbBytes, 1024);
                        for (int kk = 0; kk < nk; ++kk)
                            mma_f16(tmem + 64u * (uint32_t)j, vd + (uint64_t)(kk * 128), pd + (uint64_t)(kk * 128),
                                    idesc_o, (ho > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(&s.kv_empty[bo][j]);
                    }
                    mma_commit(&s.pv_done[bo]);
                }
                __syncwarp();
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
        if (fuse && rank == owner) {
            // The same FP8 row quantiser as csa2_quantize_append: codes and sigma go to
            // shared memory (this CTA's workers read the window's newest key from there,
            // after new_ready) and, from head group 0, to the ring slot t % wcap.
            float xnew[16];
            unpack_bf16x8(xraw[0], xnew);
            unpack_bf16x8(xraw[1], xnew + 8);
            if constexpr (kRope) {
                if (!rope_lane16(xnew, lane, a.rope.cs, a.rope.n_pos, a.rope.start, a.rope.pairs, t) &&
                    lane == 0)
                    set_dev_err(a.dev_err, CSA2_DEVERR_ROPE);
            }
            quant_fp8_lanes<kDim>(xnew, s.swa_new, &s.swa_new_sigma, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.new_ready);
            if (blockIdx.y == 0) {
                const int64_t slot = (int64_t)b * a.wcap + t % a.wcap;
                reinterpret_cast<uint4 *>(a.swa_codes + slot * kDim)[lane] =
                    reinterpret_cast<const uint4 *>(s.swa_new)[lane];
                if (lane == 0) a.swa_scale[slot] = s.swa_new_sigma;
            }
        }
    } else if (warp == 2) {
        // L2 prefetch of the entries of this CTA's later tiles (tiles 0 and 1 are in flight)
        for (int kg = k0 + kSets * kTK + lane; kg < min(k1, n_sel); kg += 32) {
            const int64_t row = cache_row(a.pm, a.cap, b, s.ids[kg]);
            prefetch_l2(a.codes + row * kCodeBytes, kCodeBytes);
            prefetch_l2(a.scales + row * kScaleBytes, kScaleBytes);
        }
    } else if (worker) {
        // ---------------- workers: produce tile h, take its softmax, load tile h + 2 ----------------
        // Softmax: thread (ii, cc) = (lane / 4, lane % 4) holds keys kA = 16 qd + ii and
        // kA + 8 of the tile and heads 8 r + 2 cc + e (r < 8, e < 2): x[4 r + e] (kA) and
        // x[4 r + 2 + e] (kA + 8).  Its row sums are for heads 8 ii + 2 cc + e.
        const float c0 = a.softmax_scale * 1.4426950408889634f * exp2f((float)qexp);
        const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
        const int ii = lane >> 2, cc = lane & 3;
        const int kA = 16 * qd + ii;
        // row sums of this warp's keys of this set's tiles, heads 8 ii + 2 cc + e, as sums of
        // 2^(x - mref) with mref in the thread's own slot of s.mref
        float lsum[2] = {0.0f, 0.0f};
        float2 *mref = reinterpret_cast<float2 *>(&s.mref[set][qd][8 * ii + 2 * cc]);
        *mref = make_float2(-INFINITY, -INFINITY);
        bool ok = true, stop = false;
        for (int h = set; h < nt; h += kSets) {
            // ---- produce tile h (its stages are free once O^T(h - 2) has read them) ----
            if (ok) {
#pragma unroll
                for (int g = 0; g < kGroups; ++g)
                    if (raw.kind[g] == 3) take_new_row(raw, g, a, km, lane, new_ok);
#pragma unroll
                for (int j = 0; j < kStages; ++j) {   // unrolled: raw.c[.][j] stays in registers
                    if (h >= kSets) {
                        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s.kv_empty[set][j], ((h - kSets) >> 1) & 1, lim, s));
                        if (!ok) break;
                    }
#pragma unroll
                    for (int g = 0; g < kGroups; ++g) {
                        const int kt = prod_key(qd, g, lane);
                        store_piece(raw, g, j, s.kv[set][j], kt, lane);
                        if (j == 0 && prod_piece(lane) == 0) {
                            const float sg = raw.sigma[g];
                            s.ksig[set][kt] = sg;
                            // P carries sigma in fp16: p <= 2^8 needs sigma <= 65504 / 256
                            if (raw.kind[g] == 2 && sg * 256.0f > 65504.0f) set_dev_err(a.dev_err, CSA2_DEVERR_RANGE);
                        }
                    }
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.kv_full[set][j]);
                }
                if (ok && h + kSets < nt) load_keys(raw, a, km, k0 + (h + kSets) * kTK, zlim_of(h + kSets), qd, lane);
            }
            // ---- softmax of tile h: every wait first; the four warps of the set agree ----
            // (kv_full[set][0]: every warp's s.ksig of the tile is written; m_ready: the
            // previous tile has fixed the running max)
            const bool w_ok =
                ok && __all_sync(0xFFFFFFFFu, mbar_wait(&s.s_full[set], (h >> 1) & 1, lim, s) &&
                                                  mbar_wait(&s.kv_full[set][0], (h >> 1) & 1, lim, s) &&
                                                  (h == 0 || mbar_wait(&s.m_ready[set ^ 1], ((h - 1) >> 1) & 1, lim, s)));
            stop = group_any(set, !w_ok || aborted(s));
            if (stop) break;
            tc_fence_after();
            float x[32];
            tmem_ld16x64(tmem + lane_base + kSCol + 64u * (uint32_t)set, x);
            const float sgA = s.ksig[set][kA], sgB = s.ksig[set][kA + 8];
            const bool vA = sgA >= 0.0f, vB = sgB >= 0.0f;
            const float ckA = c0 * sgA, ckB = c0 * sgB;
#pragma unroll
            for (int r = 0; r < 8; ++r) {   // logits, log2 units
                x[4 * r] = vA ? x[4 * r] * ckA : -INFINITY;
                x[4 * r + 1] = vA ? x[4 * r + 1] * ckA : -INFINITY;
                x[4 * r + 2] = vB ? x[4 * r + 2] * ckB : -INFINITY;
                x[4 * r + 3] = vB ? x[4 * r + 3] * ckB : -INFINITY;
            }
            float dmax = -INFINITY;
            if (h > 0) {
                // x -> x - m in place: the lazy check, and (common case) the exponent of p
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const float2 mv = *reinterpret_cast<const float2 *>(&s.mrun[8 * r + 2 * cc]);
                    x[4 * r] -= mv.x; x[4 * r + 1] -= mv.y; x[4 * r + 2] -= mv.x; x[4 * r + 3] -= mv.y;
                    dmax = fmaxf(dmax, fmaxf(fmaxf(x[4 * r], x[4 * r + 1]), fmaxf(x[4 * r + 2], x[4 * r + 3])));
                }
            }
            const bool upd = group_any(set, h == 0 || dmax > kLazy);
            if (upd) {
                if (h > 0) {   // back to the logits (one rounding; p's exponent stays consistent)
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const float2 mv = *reinterpret_cast<const float2 *>(&s.mrun[8 * r + 2 * cc]);
                        x[4 * r] += mv.x; x[4 * r + 1] += mv.y; x[4 * r + 2] += mv.x; x[4 * r + 3] += mv.y;
                    }
                }
                // exact tile max per head, then the running max moves
                const float2 wm = reduce_keys16<true>(x, lane);   // heads 8 ii + 2 cc, + 1
                *reinterpret_cast<float2 *>(&s.red[set][qd][8 * ii + 2 * cc]) = wm;
                group_sync(set);
                if (qd == 0) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int hd = 2 * lane + e;
                        const float tm = fmaxf(fmaxf(s.red[set][0][hd], s.red[set][1][hd]),
                                               fmaxf(s.red[set][2][hd], s.red[set][3][hd]));
                        const float old = h > 0 ? s.mrun[hd] : -INFINITY;
                        const float mn = fmaxf(old, tm);
                        s.mrun[hd] = mn;
                        s.alpha[set][hd] = old == -INFINITY ? 0.0f : ex2(old - mn);
                    }
                }
                group_sync(set);
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const float2 mv = *reinterpret_cast<const float2 *>(&s.mrun[8 * r + 2 * cc]);
                    x[4 * r] -= mv.x; x[4 * r + 1] -= mv.y; x[4 * r + 2] -= mv.x; x[4 * r + 3] -= mv.y;
                }
            }
            // bring the row sums to this tile's running max; then the next tile may move it
            {
                const float2 mt = *reinterpret_cast<const float2 *>(&s.mrun[8 * ii + 2 * cc]);
                const float2 mr = *mref;
                if (mt.x != mr.x) lsum[0] = lsum[0] > 0.0f ? lsum[0] * ex2(mr.x - mt.x) : 0.0f;   // the max only grows
                if (mt.y != mr.y) lsum[1] = lsum[1] > 0.0f ? lsum[1] * ex2(mr.y - mt.y) : 0.0f;
                *mref = mt;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.m_ready[set]);
            // p = 2^(x - m); P^T carries the key's scale (V holds SWA codes, not values).
            // Row kA (and kA + 8) of P^T, 16-byte chunk r: word cc = heads 8 r + 2 cc, + 1.
            const float svA = vA ? sgA : 0.0f, svB = vB ? sgB : 0.0f;
            uint8_t *pt = s.pt[set];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
#pragma unroll
                for (int k = 0; k < 4; ++k) x[4 * r + k] = ex2(x[4 * r + k]);
                const uint32_t off = (uint32_t)(((r ^ ii) << 4) + 4 * cc);
                *reinterpret_cast<uint32_t *>(pt + kA * 128 + off) = pack_h2(x[4 * r] * svA, x[4 * r + 1] * svA);
                *reinterpret_cast<uint32_t *>(pt + (kA + 8) * 128 + off) =
                    pack_h2(x[4 * r + 2] * svB, x[4 * r + 3] * svB);
            }
            // The row sums are taken after P is released (off the output MMAs' critical
            // path), except when O must be rescaled first: then before, so that x is no
            // longer live during the rescale.
            float2 ls;
            if (upd && h > 0) {
                ls = reduce_keys16<false>(x, lane);   // heads 8 ii + 2 cc, + 1
                // the running max moved: once O^T(h - 1) has landed, scale this warp's lanes
                // (32 channels of every block) before O^T(h) accumulates on them
                const bool landed =
                    __all_sync(0xFFFFFFFFu, mbar_wait(&s.pv_done[set ^ 1], ((h - 1) >> 1) & 1, lim, s));
                if (landed) {
                    tc_fence_after();
#pragma unroll 1
                    for (int j = 0; j < 4 * kStages; ++j) {    // block j / 4, 16 head columns at a time
                        float f[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) f[k] = s.alpha[set][16 * (j & 3) + k];
                        tmem_scale16(tmem + lane_base + 64u * (uint32_t)(j >> 2) + 16u * (uint32_t)(j & 3), f);
                    }
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                } else if (lane == 0) {
                    atomicExch(&s.abort, 1);
                    set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
                }
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.p_full[set]);
            } else {
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.p_full[set]);
                ls = reduce_keys16<false>(x, lane);
            }
            lsum[0] += ls.x;
            lsum[1] += ls.y;
        }
        ok = ok && !stop;
        if (ok && set < nt) {
            // O^T of this set's last tile has landed.  (Only the set's own pv_done: its
            // previous phase is known complete, so the parity wait cannot alias; the MMA
            // warp's drain covers every MMA before the combine.)
            const int hl = set + ((nt - 1 - set) / kSets) * kSets;
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s.pv_done[set], (hl >> 1) & 1, lim, s));
            tc_fence_after();
        }
        if (!ok && lane == 0) {
            atomicExch(&s.abort, 1);
            set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
        }
        // this warp's row sums (the max they are taken against is in s.mref)
        *reinterpret_cast<float2 *>(&s.red[set][qd][8 * ii + 2 * cc]) = make_float2(lsum[0], lsum[1]);
    }

    // ---- combine the two key halves of the query through distributed shared memory ----
    // CTA r writes channels [256 r, 256 r + 256) = O^T blocks 2 r, 2 r + 1.  Every thread
    // of both CTAs takes every cluster barrier, whatever happened above.
    __syncwarp();
    tc_fence_before();
    __syncthreads();                       // row sums written; this CTA's MMAs have completed
    tc_fence_after();
    const bool have = __shfl_sync(0xFFFFFFFFu, (int)(nt > 0 && !aborted(s)), 0) != 0;
    if (threadIdx.x < kHeads) {
        // this CTA's partial max and sum per head: the eight warps' sums brought to the
        // final running max, in a fixed order
        const int h = threadIdx.x;
        const float m = s.mrun[h];
        float l = 0.0f;
#pragma unroll
        for (int st = 0; st < kSets; ++st)
#pragma unroll
            for (int w = 0; w < kSetWarps; ++w) {
                const float ls = s.red[st][w][h];
                if (ls > 0.0f) l += ls * ex2(s.mref[st][w][h] - m);
            }
        s.cl[h] = have ? l : 0.0f;
        s.cm[h] = have ? m : -INFINITY;
    }
    __syncthreads();
    // Every CTA owns NB = 4 / CS of the four 128-channel blocks (blocks NB r ..): it sends
    // its partial of every other CTA's blocks (scaled by its weight) into that CTA's
    // shared memory and adds what the others sent it to its own.
    constexpr int NB = 4 / CS;
    constexpr uint32_t kPiece = NB * kCh * (kHeads / 2) * 4;   // one peer's blocks, one head half, fp32
    constexpr int kPieceF = (int)(kPiece / 4);
    for (int i = threadIdx.x; i < CS * kHeads; i += kThreads) {   // stats to every CTA, own slot `rank`
        const int r2 = i / kHeads, h = i % kHeads;
        if (r2 == (int)rank) {
            s.pm[rank][h] = s.cm[h];
            s.pl[rank][h] = s.cl[h];
        } else {
            st_peer(peer_addr(&s.pm[rank][h], (uint32_t)r2), s.cm[h]);
            st_peer(peer_addr(&s.pl[rank][h], (uint32_t)r2), s.cl[h]);
        }
    }
    if (threadIdx.x == 0) {                // armed before any peer can send
        mbar_expect_tx(&s.xfer[0], (CS - 1) * kPiece);
        mbar_expect_tx(&s.xfer[1], (CS - 1) * kPiece);
    }
    cluster_sync();                        // stats exchanged; every CTA's tiles are free
    if (a.settled && nt == 0) grid_dep_wait();   // (a CTA without keys did not wait above)
    if (threadIdx.x < kHeads) {
        const int h = threadIdx.x;
        float m_all = -INFINITY;
#pragma unroll
        for (int r2 = 0; r2 < CS; ++r2) m_all = fmaxf(m_all, s.pm[r2][h]);
        float l_all = 0.0f, f_self = 0.0f;
        if (m_all != -INFINITY) {
#pragma unroll
            for (int r2 = 0; r2 < CS; ++r2) {
                const float f = s.pm[r2][h] == -INFINITY ? 0.0f : ex2(s.pm[r2][h] - m_all);
                l_all += s.pl[r2][h] * f;
                if (r2 == (int)rank) f_self = f;
            }
        }
        const bool valid = h < hcta && l_all > 0.0f;
        s.wself[h] = valid ? f_self / l_all : 0.0f;
        if (rank == 0 && h < hcta)
            a.lse[(int64_t)qi * a.H + h0 + h] = valid ? (m_all + log2f(l_all)) * 0.6931471805599453f : -INFINITY;
    }
    __syncthreads();
    // Send slot j (0 .. CS - 2) holds the part for peer (rank + 1 + j) % CS; it lands in
    // that peer's receive slot CS - 2 - j (so receive slot i holds what CTA
    // (peer + 1 + i) % CS sent).  A slot is [2 head halves][NB blocks][128 channels][32
    // heads] fp32, float4 units swizzled by channel; receive slots fill s.kv from the
    // start, send slots follow them in s.kv and then s.q (both free by now).
    // Task u (warp u % 12 takes u, so the TMEM lane quadrant u % 4 is the warp's):
    // channels 32 (u % 4) .., head half (u >> 2) & 1, block bsel / send slot from u >> 3.
    auto recv_slot = [&](int i) { return reinterpret_cast<float *>(&s.kv[0][0][0]) + i * 2 * kPieceF; };
    auto send_slot = [&](int j) {
        const int k = (CS - 1) + j;        // slot index in the sequence s.kv, then s.q
        return k * 2 * kPieceF < (int)(sizeof(s.kv) / 4)
                   ? reinterpret_cast<float *>(&s.kv[0][0][0]) + k * 2 * kPieceF
                   : reinterpret_cast<float *>(s.q) + (k * 2 * kPieceF - (int)(sizeof(s.kv) / 4));
    };
#pragma unroll 1
    for (int u = warp; u < 8 * NB * (CS - 1); u += kWarps) {
        const int cq = u & 3, hp = (u >> 2) & 1, bsel = (u >> 3) % NB, j = (u >> 3) / NB;
        const int pr = ((int)rank + 1 + j) % CS;
        const int crow = 32 * cq + lane;             // channel within a block
        const uint32_t taddr = tmem + ((uint32_t)(32 * cq) << 16) + 32u * (uint32_t)hp;
        float o[32];
        if (have) {
            tmem_ld32(taddr + 64u * (uint32_t)(NB * pr + bsel), o);
        } else {
#pragma unroll
            for (int h = 0; h < 32; ++h) o[h] = 0.0f;
        }
        float4 *dst = reinterpret_cast<float4 *>(send_slot(j) + hp * kPieceF + (bsel * kCh + crow) * (kHeads / 2));
#pragma unroll
        for (int f = 0; f < 8; ++f) {                // float4 f = heads 32 hp + 4 f ..
            const int h = 32 * hp + 4 * f;
            dst[f ^ (crow & 7)] = make_float4(o[4 * f] * s.wself[h], o[4 * f + 1] * s.wself[h + 1],
                                              o[4 * f + 2] * s.wself[h + 2], o[4 * f + 3] * s.wself[h + 3]);
        }
    }
    fence_async_smem();                    // generic-proxy writes of `send` -> the bulk copy
    __syncthreads();
    if (threadIdx.x < 2 * (CS - 1)) {      // one copy per (peer, head half)
        const int j = threadIdx.x >> 1, hp = threadIdx.x & 1;
        const uint32_t pr = (uint32_t)(((int)rank + 1 + j) % CS);
        const uint32_t dst = peer_addr(recv_slot(CS - 2 - j) + hp * kPieceF, pr);
        bulk_copy_to_peer(dst, send_slot(j) + hp * kPieceF, kPiece, peer_addr(&s.xfer[hp], pr));
    }
    bool got_all = true;
#pragma unroll 1
    for (int u = warp; u < 8 * NB; u += kWarps) {
        const int cq = u & 3, hp = (u >> 2) & 1, bsel = u >> 3;
        const int crow = 32 * cq + lane;
        const uint32_t taddr = tmem + ((uint32_t)(32 * cq) << 16) + 32u * (uint32_t)hp;
        float own[32];
        if (have) {
            tmem_ld32(taddr + 64u * (uint32_t)(NB * (int)rank + bsel), own);
        } else {
#pragma unroll
            for (int h = 0; h < 32; ++h) own[h] = 0.0f;
        }
        const bool got = __all_sync(0xFFFFFFFFu, mbar_wait<false>(&s.xfer[hp], 0, kDrainLimitNs, s));
        got_all = got_all && got;
#pragma unroll
        for (int f = 0; f < 8; ++f) {
            const int h = 32 * hp + 4 * f;
#pragma unroll
            for (int k = 0; k < 4; ++k) own[4 * f + k] *= s.wself[h + k];
        }
#pragma unroll 1
        for (int i = 0; i < CS - 1; ++i) {           // the senders in a fixed order
            const float4 *src = reinterpret_cast<const float4 *>(recv_slot(i) + hp * kPieceF +
                                                                 (bsel * kCh + crow) * (kHeads / 2));
#pragma unroll
            for (int f = 0; f < 8; ++f) {
                const float4 pr = got ? src[f ^ (crow & 7)] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                own[4 * f] += pr.x; own[4 * f + 1] += pr.y; own[4 * f + 2] += pr.z; own[4 * f + 3] += pr.w;
            }
        }
        float *obase = a.out + ((int64_t)qi * a.H + h0) * kDim + 128 * (NB * (int)rank + bsel) + crow;
#pragma unroll
        for (int k = 0; k < 32; ++k)
            if (32 * hp + k < hcta) obase[(int64_t)(32 * hp + k) * kDim] = own[k];
    }
    if (!got_all && lane == 0) set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
    // A warp with no task for a head half still waits for it, so that every incoming
    // copy has landed before the closing barrier.
    if (!__all_sync(0xFFFFFFFFu, mbar_wait<false>(&s.xfer[0], 0, kDrainLimitNs, s) &&
                                     mbar_wait<false>(&s.xfer[1], 0, kDrainLimitNs, s)) &&
        lane == 0)
        set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
    // Every CTA has seen its incoming copies land, so every outgoing copy has finished
    // reading its send slot: only now may a CTA leave (and its shared memory be reused).
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

}  // namespace attn

size_t attn_smem_bytes() { return sizeof(attn::Smem) + 1024; }

template <bool kRope, int CS>
static cudaError_t launch_attn_t(const AttnArgs &a, int BT, int hg, cudaStream_t st) {
    const size_t smem = attn_smem_bytes();
    static std::atomic<uint64_t> configured{0};   // per device
    {
        cudaError_t e = config_kernel_once(attn::attn_kernel<kRope, CS>, smem, configured);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CS * BT, hg);
    cfg.blockDim = dim3(attn::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;   // the CS CTAs of a query
    attr[1].val.clusterDim.x = CS;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, attn::attn_kernel<kRope, CS>, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// 4 CTAs per query when the whole grid still fits the SMs once (small batches: shorter
// per-query latency), else 2.
cudaError_t launch_sparse_attn(const AttnArgs &a, int BT, cudaStream_t st) {
    const int hg = (a.H + attn::kHeads - 1) / attn::kHeads;
    const bool four = (int64_t)4 * BT * hg <= device_sm_count();
    const bool rope = a.swa_new != nullptr && a.rope.cs != nullptr;
    if (four) return rope ? launch_attn_t<true, 4>(a, BT, hg, st) : launch_attn_t<false, 4>(a, BT, hg, st);
    return rope ? launch_attn_t<true, 2>(a, BT, hg, st) : launch_attn_t<false, 2>(a, BT, hg, st);
}

}  // namespace csa2

