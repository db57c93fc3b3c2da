// csa2_index.cu -- Full-layer index scan, pool / Top-K selection, Reindex (sm_100a).
//
// DeepSeek V4.1 Flash study notes, section 2 (report Figure 5) and myzaker
// "CSA2 attention": the first Full layer scans all causally visible positions,
// scores them block by block and builds a shared candidate pool of at most
// 2048 blocks x 8 positions; it picks at most 512 positions; later Reindex
// layers re-score with their own index query only inside the pool.
//
// Score (fixed for this build): score(s) = sum_h w_h * relu(q_h . k_s), k_s the
// FP8 indexer K of entry s times its per-entry scale, evaluated in this fp32
// order so that Top-K membership is reproducible bit for bit:
//   per head: (even, odd) = fma chains over channel pairs (2j, 2j+1), one
//             packed fma.rn.f32x2 per pair; a_h = even + odd
//   t = fma chain over h of (w_h, max(a_h, 0));  score = t * sigma_s
// Selection order: score descending, ties to the lower position.
#include <cuda_fp16.h>
#include <stdint.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {

// ------------------------------------------------------------------------------
// Scoring core (score_rows_at): a group of NT threads scores a tile of NT * R rows
// staged in shared memory (thread t: rows t + NT r, r < R).  The Full scan runs it in
// small CTAs (kScoreThreads) that keep many tiles in flight per SM; so does the Reindex
// scoring, with the smaller tile.
// ------------------------------------------------------------------------------
constexpr int kScoreThreads = 64;
constexpr int kScanRows = 4;       // rows per thread, Full scan (256-row, 32 KB tiles)
constexpr int kReindexRows = 2;    // rows per thread, Reindex gather (128-row, 16 KB tiles)

// 16-byte unit u of row r lives at unit swz(r, u): a quarter-warp reading unit
// u of 8 consecutive rows hits 8 different 16-byte bank groups.
template <int D>
__device__ __forceinline__ int swz(int r, int u) {
    if constexpr (D == 128)
        return u ^ (r & 7);
    else
        return u ^ ((r >> 1) & 3);
}

template <int D, int HI, int R>
struct ScoreSmem {
    uint8_t rows[kScoreThreads * R * D];
    float2 q[D / 2][HI];     // q pairs (q[h][2j], q[h][2j+1]) as fp32
    float w[HI];
    float m64[kScoreThreads / 32][R];   // per warp and row group: max of its 32 rows
};

// Stage q (bf16 [HI][D]) and w into shared memory as fp32.
// All of a thread's loads are issued before any is used (one memory round trip).
template <int D, int HI, int R>
__device__ __forceinline__ void load_query(ScoreSmem<D, HI, R> &s, const uint16_t *q, const float *w) {
    constexpr int kPer = (HI * D / 2 + kScoreThreads - 1) / kScoreThreads;
    uint32_t two[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int e = threadIdx.x + k * kScoreThreads;
        two[k] = e < HI * D / 2 ? __ldg(reinterpret_cast<const uint32_t *>(q) + e) : 0u;
    }
    const float wv = threadIdx.x < HI ? __ldg(w + threadIdx.x) : 0.0f;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int e = threadIdx.x + k * kScoreThreads;
        if (e < HI * D / 2) {
            const int h = e / (D / 2), j = e % (D / 2);
            s.q[j][h] = make_float2(bf16_bits_to_f32(two[k] & 0xFFFFu), bf16_bits_to_f32(two[k] >> 16));
        }
    }
    if (threadIdx.x < HI) s.w[threadIdx.x] = wv;
}

// Copy one 16-byte unit global -> shared (bypassing L1).
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// Scores of rows tid + NT s (s < R) of a staged tile (swizzled rows of D bytes),
// before the per-entry scale, in the fixed order above.  Rows must be staged;
// invalid rows produce garbage the caller discards.
template <int D, int HI, int R, int NT>
__device__ __forceinline__ void score_rows_at(const uint8_t *rows, const float2 (*q)[HI], const float *w,
                                              int tid, float out[R]) {
    float2 acc[R][HI];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < HI; ++h) acc[r][h] = make_float2(0.0f, 0.0f);

#pragma unroll
    for (int u = 0; u < D / 16; ++u) {          // 16 channels = 8 pairs per unit
        uint32_t wv[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int row = tid + NT * r;
            const uint4 kw = *reinterpret_cast<const uint4 *>(rows + row * D + 16 * swz<D>(row, u));
            wv[r][0] = kw.x; wv[r][1] = kw.y; wv[r][2] = kw.z; wv[r][3] = kw.w;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {           // one 32-bit word = channel pairs 2i, 2i+1 of the unit
            float2 qa[HI], qb[HI];              // q is read per word: few live registers
#pragma unroll
            for (int h = 0; h < HI; ++h) {
                qa[h] = q[8 * u + 2 * i][h];
                qb[h] = q[8 * u + 2 * i + 1][h];
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                uint32_t h01 = cvt_e4m3x2_f16x2(wv[r][i] & 0xFFFFu);
                uint32_t h23 = cvt_e4m3x2_f16x2(wv[r][i] >> 16);
                float2 k01 = __half22float2(*reinterpret_cast<__half2 *>(&h01));
                float2 k23 = __half22float2(*reinterpret_cast<__half2 *>(&h23));
#pragma unroll
                for (int h = 0; h < HI; ++h) {
                    acc[r][h] = fma2(qa[h], k01, acc[r][h]);
                    acc[r][h] = fma2(qb[h], k23, acc[r][h]);
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        float t = 0.0f;
#pragma unroll
        for (int h = 0; h < HI; ++h) {
            float a = __fadd_rn(acc[r][h].x, acc[r][h].y);
            t = __fmaf_rn(w[h], a > 0.0f ? a : 0.0f, t);
        }
        out[r] = t;
    }
}

template <int D, int HI, int R>
__device__ __forceinline__ void score_rows(const ScoreSmem<D, HI, R> &s, float out[R]) {
    score_rows_at<D, HI, R, kScoreThreads>(s.rows, s.q, s.w, threadIdx.x, out);
}

// ------------------------------------------------------------------------------
// a3: Full scan.  grid (ceil(n_max / kTileRows), B*Tq), kScoreThreads threads.
// ------------------------------------------------------------------------------
template <int D, int HI>
__global__ void __launch_bounds__(kScoreThreads)
index_scan_kernel(IndexArgs a) {
    constexpr int R = kScanRows, kTileRows = kScoreThreads * R;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    ScoreSmem<D, HI, R> &s = *reinterpret_cast<ScoreSmem<D, HI, R> *>(smem_raw);
    grid_dep_wait();
    const int qi = blockIdx.y;
    const int b = qi / a.Tq;
    int64_t N = max64(0, visible_entries(a.q_pos[qi], a.ratio) - a.entry_lo);   // of this cache
    if (a.topk_keys_out) N = min64(N, a.cap);     // a slice: the query sees past its end
    if (N > a.n_max || N > a.cap) {
        if (threadIdx.x == 0 && blockIdx.x == 0) set_dev_err(a.dev_err, CSA2_DEVERR_NMAX);
        N = min64(min64(N, a.n_max), a.cap);
    }
    const int64_t p0 = (int64_t)blockIdx.x * kTileRows;
    if (p0 >= N) return;
    const int rows = (int)min64(kTileRows, N - p0);

    // the tile's rows are consecutive cache rows (a page holds whole tiles)
    const int64_t row0 = cache_row(a.pm, a.cap, b, p0);
    if (row0 < 0) {
        if (threadIdx.x == 0) set_dev_err(a.dev_err, CSA2_DEVERR_PAGE);
        return;
    }
    const uint8_t *src = a.idx_codes + row0 * D;
    constexpr int U = D / 16;
    for (int e = threadIdx.x; e < rows * U; e += kScoreThreads) {
        int r = e / U, u = e % U;
        cp_async16(s.rows + r * D + 16 * swz<D>(r, u), src + (int64_t)e * 16);
    }
    cp_async_commit();
    load_query<D, HI>(s, a.q_idx + (int64_t)qi * HI * D, a.w + (int64_t)qi * HI);
    // the rows' scales, fetched while the tile is in flight
    const float *sig = a.idx_scale + row0;
    float sgv[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int row = threadIdx.x + kScoreThreads * r;
        sgv[r] = __ldg(sig + min(row, rows - 1));   // branch-free: all R loads in flight
    }
    cp_async_wait_all();
    __syncthreads();

    float sc[R];
    score_rows<D, HI, R>(s, sc);
    grid_dep_launch();

    float *scores = a.scores + (int64_t)qi * a.score_stride;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        int row = threadIdx.x + kScoreThreads * r;
        int64_t p = p0 + row;
        float v = -INFINITY;
        if (row < rows) {
            v = __fmul_rn(sc[r], sgv[r]);
            scores[p] = v;
        }
        if (a.bmax) {
            // block of 8 positions = 8 consecutive lanes
            float m = v;
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
            if ((row & 7) == 0 && row < rows) a.bmax[(int64_t)qi * a.bmax_stride + p / 8] = m;
            if (a.bmax64) {
                // super-block of 64 positions = rows 64 r .. 64 r + 63 = both warps' r-th rows
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 8));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
                if ((threadIdx.x & 31) == 0) s.m64[threadIdx.x >> 5][r] = m;
            }
        }
    }
    if (a.bmax64) {
        __syncthreads();
        if (threadIdx.x < R && 64 * (int)threadIdx.x < rows)
            a.bmax64[(int64_t)qi * a.bmax64_stride + p0 / 64 + threadIdx.x] =
                fmaxf(s.m64[0][threadIdx.x], s.m64[1][threadIdx.x]);
    }
}

// ------------------------------------------------------------------------------
// a6: Reindex scoring of the pool.  grid (ceil(8 pool_blocks / kTileRows), B*Tq),
// kScoreThreads threads, kTileRows = kScoreThreads * kReindexRows (16 pool blocks).
// Candidate c = 8 * slot + r of the pool (slot < pool_blocks, r < 8) is position
// 8 * pool[slot] + r; its score goes to scores[qi][c] and the maximum of the slot's
// visible positions to bmax[qi][slot] (for the selection's block lemma).  Many small
// CTAs keep many scattered 1 KB blocks in flight per SM.
// ------------------------------------------------------------------------------
template <int D, int HI>
__global__ void __launch_bounds__(kScoreThreads)
reindex_score_kernel(IndexArgs a) {
    constexpr int R = kReindexRows, kTileRows = kScoreThreads * R;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    ScoreSmem<D, HI, R> &s = *reinterpret_cast<ScoreSmem<D, HI, R> *>(smem_raw);
    __shared__ int64_t row_of[kTileRows];   // cache row of each candidate, -1: not scored
    // Settled inputs (written before the most recent ordinary launch): the pool ids are
    // resolved and the rows staged at once, and the wait moves to just before the scoring,
    // so that nothing is computed from this layer's query before the previous launch has
    // completed (the scores go to a workspace the previous launch does not read).
    if (!a.settled) grid_dep_wait();
    const int qi = blockIdx.y;
    const int b = qi / a.Tq;
    int64_t N = visible_entries(a.q_pos[qi], a.ratio);
    N = min64(N, a.cap);
    const int slot0 = blockIdx.x * (kTileRows / 8);
    const int32_t *pool = a.pool + (int64_t)qi * a.pool_blocks;
    float sgv[R];   // row threadIdx.x + kScoreThreads i is handled by this thread below
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int r = threadIdx.x + kScoreThreads * i;
        const int slot = slot0 + r / 8;
        int blk = __ldg(pool + min(slot, a.pool_blocks - 1));
        if (slot >= a.pool_blocks) blk = -1;
        const int64_t p = (int64_t)blk * 8 + (r & 7);
        if (blk >= 0 && (int64_t)blk * 8 >= N && (r & 7) == 0) set_dev_err(a.dev_err, CSA2_DEVERR_INDEX);
        int64_t row = blk >= 0 && p < N ? cache_row(a.pm, a.cap, b, p) : -1;
        if (blk >= 0 && p < N && row < 0) set_dev_err(a.dev_err, CSA2_DEVERR_PAGE);
        row_of[r] = row;
        sgv[i] = __ldg(a.idx_scale + (row >= 0 ? row : 0));   // branch-free (row 0 always exists)
    }
    __syncthreads();
    constexpr int U = D / 16;
    for (int e = threadIdx.x; e < kTileRows * U; e += kScoreThreads) {
        const int r = e / U, u = e % U;
        if (row_of[r] >= 0)
            cp_async16(s.rows + r * D + 16 * swz<D>(r, u), a.idx_codes + row_of[r] * D + 16 * u);
    }
    cp_async_commit();
    load_query<D, HI>(s, a.q_idx + (int64_t)qi * HI * D, a.w + (int64_t)qi * HI);
    cp_async_wait_all();
    __syncthreads();
    if (a.settled) grid_dep_wait();

    float sc[R];
    score_rows<D, HI, R>(s, sc);
    grid_dep_launch();
    float *out = a.scores + (int64_t)qi * a.score_stride + (int64_t)slot0 * 8;
    float *bm = a.bmax + (int64_t)qi * a.bmax_stride + slot0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int row = threadIdx.x + kScoreThreads * r;
        const bool valid = row_of[row] >= 0;
        const float v = valid ? __fmul_rn(sc[r], sgv[r]) : -INFINITY;
        if (slot0 + row / 8 < a.pool_blocks) out[row] = valid ? v : 0.0f;
        // the slot's 8 candidates are 8 consecutive lanes
        float m = v;
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
        if ((row & 7) == 0 && slot0 + row / 8 < a.pool_blocks) bm[row / 8] = m;
    }
}

// ------------------------------------------------------------------------------
// Block-wide Top-K selection (one CTA per query).
// Keys are 32-bit order keys (0 = not a candidate).  Radix select, most significant
// digit first, over the bits where the valid keys differ: the digits start at the
// highest bit in which the smallest and largest valid keys differ (scores share
// their sign and most exponent bits, which would otherwise pile every key into a
// few bins), 11 bits per pass, stopping as soon as the remaining demand equals
// the population of the chosen bin.  The result is a masked threshold (T, mask)
// and a count `take`: selected = every key whose masked value exceeds T, plus
// the `take` lowest-indexed keys whose masked value equals T.  A compaction over
// per-warp contiguous segments then writes the selected ids in index order.
// ------------------------------------------------------------------------------
constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelStageMax = 16384;   // keys staged in shared memory up to this count
// Flat selections over more keys (prefill chunks, long encoder groups) use a second
// instantiation that stages up to kSelStageWide keys (192 KB, one CTA per SM) and so
// reads its row from HBM once instead of once per radix pass.
constexpr int kSelStageWide = 49152;
constexpr int kSelDigit = 11;         // bits per radix pass
// Flat rows longer than this select through the 64- and 8-position block maxima.
constexpr int kSelFlatDirect = 16384;

template <int kCap>
struct SelSmemT {
    uint32_t hist[1 << kSelDigit];
    int wa[kSelWarps], wb[kSelWarps], wc[kSelWarps];
    uint32_t wmin[kSelWarps], wmax[kSelWarps];
    int bcast[4];
    alignas(16) int pool[CSA2_POOL_MAX];
    int sup[CSA2_POOL_MAX];               // multi-level selection: the chosen super-blocks
    alignas(16) uint32_t keys[kCap];
};
using SelSmem = SelSmemT<kSelStageMax>;

// dst[0..n) = the raw 32-bit words src[0..n), copied into shared memory with 16-byte
// cp.async (src 16-byte aligned, as every workspace row is) so that no register or
// dependent round trip is involved; the caller converts in place after a barrier.
__device__ __forceinline__ void stage_raw(uint32_t *dst, const void *src, int n) {
    const uint32_t *s32 = reinterpret_cast<const uint32_t *>(src);
    const int n4 = n / 4;
    for (int c = threadIdx.x; c < n4; c += kSelThreads) cp_async16(dst + 4 * c, s32 + 4 * c);
    for (int i = 4 * n4 + (int)threadIdx.x; i < n; i += kSelThreads) dst[i] = __ldg(s32 + i);
    cp_async_commit();
    cp_async_wait_all();
}

// Inclusive scan over the warp's lanes.
__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// The bin (of nbins, visited from the top) holding the rem-th largest counted key:
// bin, number of counted keys in higher bins, population of the bin.  Each thread reads
// its bins and zeroes them for the next pass.  Every warp derives its own prefix from
// the warps' totals (no broadcast step): two barriers.
template <class S>
__device__ __forceinline__ void sel_find_bin(S &s, int nbins, int rem, int &bin, int &above,
                                             int &cnt) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int per = (nbins + kSelThreads - 1) / kSelThreads;   // 1 or 2 bins per thread
    int c[2] = {0, 0}, sum = 0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int bb = nbins - 1 - (threadIdx.x * per + j);
        if (j < per && bb >= 0) {
            c[j] = (int)s.hist[bb];
            s.hist[bb] = 0u;
        }
        sum += c[j];
    }
    const int incl = warp_incl_scan(sum, lane);
    if (lane == 31) s.wa[warp] = incl;
    __syncthreads();
    const int wt = s.wa[lane];
    const int wprefix = __shfl_sync(0xFFFFFFFFu, warp_incl_scan(wt, lane) - wt, warp);
    int run = wprefix + incl - sum;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        if (c[j] > 0 && run < rem && rem <= run + c[j]) {
            s.bcast[0] = nbins - 1 - (threadIdx.x * per + j);
            s.bcast[1] = run;
            s.bcast[2] = c[j];
        }
        run += c[j];
    }
    __syncthreads();
    bin = s.bcast[0];
    above = s.bcast[1];
    cnt = s.bcast[2];
}

// Top-k of n candidates (keys from key_at, 0 = not a candidate) -> ascending ids in
// out[0..cnt), cnt = min(k, #valid) returned.  Block barriers: one for the statistics,
// three per radix pass, two for the compaction.
template <class KeyAt, class IdAt, class S>
__device__ int block_topk(KeyAt key_at, IdAt id_at, int n, int k, int *out, S &s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // the first radix pass's bins start at zero (each pass's readers zero them for the next)
    for (int i = threadIdx.x; i < (1 << kSelDigit); i += kSelThreads) s.hist[i] = 0u;
    // valid count, smallest and largest valid key
    int nv = 0;
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int i = threadIdx.x; i < n; i += kSelThreads) {
        const uint32_t key = key_at(i);
        if (key != 0u) {
            ++nv;
            kmin = min(kmin, key);
            kmax = max(kmax, key);
        }
    }
    nv = __reduce_add_sync(0xFFFFFFFFu, nv);
    kmin = __reduce_min_sync(0xFFFFFFFFu, kmin);
    kmax = __reduce_max_sync(0xFFFFFFFFu, kmax);
    if (lane == 0) {
        s.wc[warp] = nv;
        s.wmin[warp] = kmin;
        s.wmax[warp] = kmax;
    }
    __syncthreads();
    // every warp reduces the warps' figures itself
    const int nvalid = __reduce_add_sync(0xFFFFFFFFu, s.wc[lane]);
    kmin = __reduce_min_sync(0xFFFFFFFFu, s.wmin[lane]);
    kmax = __reduce_max_sync(0xFFFFFFFFu, s.wmax[lane]);
    const int kk = min(k, nvalid);
    if (kk == 0) {
        __syncthreads();   // every warp has read the figures before the next selection writes them
        return 0;
    }

    // ---- threshold ----
    uint32_t T, mask;
    int take;
    if (kk == nvalid) {                 // everything valid is selected
        T = 0u;
        mask = 0u;
        take = kk;
    } else if (kmin == kmax) {          // all valid keys equal: the first kk in index order
        T = kmax;
        mask = 0xFFFFFFFFu;
        take = kk;
    } else {
        const int hi = 31 - __clz(kmin ^ kmax);
        uint32_t pmask = ~((2u << hi) - 1u);      // bits above hi are common to every valid key
        uint32_t prefix = kmax & pmask;
        int rem = kk, lo_bit = hi + 1;
        while (lo_bit > 0) {
            const int bits = min(kSelDigit, lo_bit), shift = lo_bit - bits, nbins = 1 << bits;
            for (int i = threadIdx.x; i < n; i += kSelThreads) {
                const uint32_t key = key_at(i);
                if (key != 0u && (key & pmask) == prefix)
                    atomicAdd(&s.hist[(key >> shift) & (uint32_t)(nbins - 1)], 1u);
            }
            __syncthreads();
            int bin, above, cnt;
            sel_find_bin(s, nbins, rem, bin, above, cnt);
            prefix |= (uint32_t)bin << shift;
            pmask |= (uint32_t)(nbins - 1) << shift;
            rem -= above;
            lo_bit = shift;
            if (cnt == rem) break;            // the whole bin is taken
        }
        T = prefix;
        mask = pmask;
        take = rem;
    }

    // ---- compaction in index order: warp w owns keys [w*seg, (w+1)*seg) ----
    const int seg = ((n + kSelThreads - 1) / kSelThreads) * 32;
    const int lo = warp * seg, hi_i = min(n, lo + seg);
    int ngt = 0, neq = 0;
    for (int i0 = lo; i0 < hi_i; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < hi_i ? key_at(i) : 0u;
        const uint32_t km = key & mask;
        ngt += __popc(__ballot_sync(0xFFFFFFFFu, key != 0u && km > T));
        neq += __popc(__ballot_sync(0xFFFFFFFFu, key != 0u && km == T));
    }
    if (lane == 0) {
        s.wa[warp] = ngt;
        s.wb[warp] = neq;
    }
    __syncthreads();
    // this warp's exclusive prefixes and the totals, from the warps' counts
    const int a_w = s.wa[lane], b_w = s.wb[lane];
    const int ia = warp_incl_scan(a_w, lane), ib = warp_incl_scan(b_w, lane);
    int gt_run = __shfl_sync(0xFFFFFFFFu, ia - a_w, warp), eq_run = __shfl_sync(0xFFFFFFFFu, ib - b_w, warp);
    const int total = __shfl_sync(0xFFFFFFFFu, ia, 31) + min(take, __shfl_sync(0xFFFFFFFFu, ib, 31));
    const uint32_t lt = (1u << lane) - 1u;
    for (int i0 = lo; i0 < hi_i; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < hi_i ? key_at(i) : 0u;
        const uint32_t km = key & mask;
        const bool gt = key != 0u && km > T, eq = key != 0u && km == T;
        const uint32_t bgt = __ballot_sync(0xFFFFFFFFu, gt), beq = __ballot_sync(0xFFFFFFFFu, eq);
        const int gt_before = gt_run + __popc(bgt & lt), eq_before = eq_run + __popc(beq & lt);
        if (gt || (eq && eq_before < take)) {
            const int r = gt_before + min(take, eq_before);
            if (r < kk) out[r] = id_at(i);
        }
        gt_run += __popc(bgt);
        eq_run += __popc(beq);
    }
    __syncthreads();
    return min(total, kk);
}

// keys[8 i + j] = order key of src[8 ids[i] + j] (i < n, j < 8), 0 for the entries at or
// past `limit`.  src rows are 32-byte aligned and long enough for whole groups of 8.
__device__ __forceinline__ void gather8_keys(uint32_t *keys, const float *src, const int *ids, int n,
                                             int64_t limit) {
    for (int c = threadIdx.x; c < 2 * n; c += kSelThreads)
        cp_async16(keys + 4 * c, src + (int64_t)ids[c >> 1] * 8 + 4 * (c & 1));
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    for (int i = threadIdx.x; i < 8 * n; i += kSelThreads) {
        const int64_t p = (int64_t)ids[i >> 3] * 8 + (i & 7);
        keys[i] = p < limit ? score_key(__uint_as_float(keys[i])) : 0u;
    }
    __syncthreads();
}

// a4 + a5: one CTA per query.
// Lemma (the pages' pool argument, for any k and any partition into contiguous groups):
// the k best items by (value desc, index asc) all lie in the k best groups by (group max
// desc, group asc) -- an item of another group is preceded by the maxima of k groups,
// each of which precedes it.  So:
//   Hierarchical: pool = the pool_blocks best 8-position blocks (from the 64-position
//     super-blocks first when there are more blocks than the stage holds); Top-K = the
//     top_k best positions of the top_k best pool blocks (top_k <= pool_blocks).
//   Flat: Top-K over all visible positions; for long rows from the top_k best
//     super-blocks, then their top_k best blocks, then those blocks' positions.
// Outputs ascending.
template <int kCap>
__global__ void __launch_bounds__(kSelThreads)
select_full_kernel(IndexArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    SelSmemT<kCap> &s = *reinterpret_cast<SelSmemT<kCap> *>(smem_raw);
    __shared__ int sel_out[CSA2_TOPK_MAX];
    __shared__ int sub[CSA2_TOPK_MAX];
    grid_dep_wait();
    // The next launch (the layer's attention) may start now: its CTAs take the SMs this
    // selection leaves free and stage their queries; they read the Top-K only after
    // this kernel has completed.
    grid_dep_launch();
    const int qi = blockIdx.x;
    int64_t N64 = max64(0, visible_entries(a.q_pos[qi], a.ratio) - a.entry_lo);
    N64 = min64(min64(N64, a.n_max), a.cap);
    const int N = (int)N64;
    const int nb = (N + 7) / 8, nb64 = (N + 63) / 64;
    const float *scores = a.scores + (int64_t)qi * a.score_stride;
    const float *bm = a.bmax ? a.bmax + (int64_t)qi * a.bmax_stride : nullptr;
    const float *bm64 = a.bmax64 ? a.bmax64 + (int64_t)qi * a.bmax64_stride : nullptr;
    // the top_k best 8-blocks among the candidate blocks ids[0..n) (ascending), into
    // sub[]; keys from bm
    auto best_blocks = [&](const int *ids, int n) -> int {
        for (int i = threadIdx.x; i < n; i += kSelThreads) s.keys[i] = score_key(__ldg(bm + ids[i]));
        __syncthreads();
        auto k = [&](int i) -> uint32_t { return s.keys[i]; };
        auto id = [&](int i) -> int { return ids[i]; };
        return block_topk(k, id, n, a.top_k, sub, s);
    };
    // Top-K over the positions of blocks sub[0..n) (ascending)
    auto best_positions = [&](int n) -> int {
        gather8_keys(s.keys, scores, sub, n, N);
        auto k = [&](int i) -> uint32_t { return s.keys[i]; };
        auto id = [&](int i) -> int { return sub[i >> 3] * 8 + (i & 7); };
        return block_topk(k, id, 8 * n, a.top_k, sel_out, s);
    };
    int cnt;
    if (a.pool_blocks > 0) {
        int np;
        if (nb <= kCap) {
            stage_raw(s.keys, bm, nb);
            __syncthreads();
            for (int i = threadIdx.x; i < nb; i += kSelThreads) s.keys[i] = score_key(__uint_as_float(s.keys[i]));
            __syncthreads();
            auto bkey = [&](int i) -> uint32_t { return s.keys[i]; };
            auto bid = [&](int i) -> int { return i; };
            np = block_topk(bkey, bid, nb, a.pool_blocks, s.pool, s);
        } else if (bm64 != nullptr && nb64 <= kCap) {
            // the pool_blocks best super-blocks, then the best 8-blocks inside them
            stage_raw(s.keys, bm64, nb64);
            __syncthreads();
            for (int i = threadIdx.x; i < nb64; i += kSelThreads) s.keys[i] = score_key(__uint_as_float(s.keys[i]));
            __syncthreads();
            auto gkey = [&](int i) -> uint32_t { return s.keys[i]; };
            auto gid = [&](int i) -> int { return i; };
            const int ns = block_topk(gkey, gid, nb64, a.pool_blocks, s.pool, s);
            __syncthreads();
            gather8_keys(s.keys, bm, s.pool, ns, nb);
            for (int i = threadIdx.x; i < ns; i += kSelThreads) s.sup[i] = s.pool[i];
            __syncthreads();
            auto ckey = [&](int i) -> uint32_t { return s.keys[i]; };
            auto cid = [&](int i) -> int { return s.sup[i >> 3] * 8 + (i & 7); };
            np = block_topk(ckey, cid, 8 * ns, a.pool_blocks, s.pool, s);
        } else {
            auto bkey = [&](int i) -> uint32_t { return score_key(bm[i]); };
            auto bid = [&](int i) -> int { return i; };
            np = block_topk(bkey, bid, nb, a.pool_blocks, s.pool, s);
        }
        __syncthreads();
        int32_t *pool_out = a.pool_out ? a.pool_out + (int64_t)qi * a.pool_blocks : nullptr;
        if (pool_out)
            for (int i = threadIdx.x; i < a.pool_blocks; i += blockDim.x)
                pool_out[i] = i < np ? s.pool[i] : -1;
        if (a.pool_keys_out) {
            uint64_t *pk = a.pool_keys_out + (int64_t)qi * a.pool_blocks;
            for (int i = threadIdx.x; i < a.pool_blocks; i += blockDim.x)
                pk[i] = i < np ? ((uint64_t)score_key(__ldg(bm + s.pool[i])) << 32) |
                                     (uint32_t)~(uint32_t)(s.pool[i] + a.entry_lo / 8)
                               : 0ull;
        }
        // the top_k best pool blocks hold the Top-K; their positions
        const int ns = best_blocks(s.pool, np);
        __syncthreads();
        cnt = best_positions(ns);
    } else if (N > kSelFlatDirect && bm != nullptr && bm64 != nullptr && nb64 <= kCap) {
        stage_raw(s.keys, bm64, nb64);
        __syncthreads();
        for (int i = threadIdx.x; i < nb64; i += kSelThreads) s.keys[i] = score_key(__uint_as_float(s.keys[i]));
        __syncthreads();
        auto gkey = [&](int i) -> uint32_t { return s.keys[i]; };
        auto gid = [&](int i) -> int { return i; };
        const int ns = block_topk(gkey, gid, nb64, a.top_k, s.pool, s);
        __syncthreads();
        // the blocks of those super-blocks, their top_k best, then their positions
        gather8_keys(s.keys, bm, s.pool, ns, nb);
        for (int i = threadIdx.x; i < ns; i += kSelThreads) s.sup[i] = s.pool[i];
        __syncthreads();
        auto ckey = [&](int i) -> uint32_t { return s.keys[i]; };
        auto cid = [&](int i) -> int { return s.sup[i >> 3] * 8 + (i & 7); };
        const int nsb = block_topk(ckey, cid, 8 * ns, a.top_k, sub, s);
        __syncthreads();
        cnt = best_positions(nsb);
    } else {
        const bool staged = N <= kCap;
        if (staged) {
            stage_raw(s.keys, scores, N);
            __syncthreads();
            for (int i = threadIdx.x; i < N; i += kSelThreads) s.keys[i] = score_key(__uint_as_float(s.keys[i]));
            __syncthreads();
        }
        auto key = [&](int i) -> uint32_t { return staged ? s.keys[i] : score_key(scores[i]); };
        auto id = [&](int i) -> int { return i; };
        cnt = block_topk(key, id, N, a.top_k, sel_out, s);
    }
    __syncthreads();
    if (a.topk_keys_out) {
        // slice form: the selected entries' candidate keys, global ids
        uint64_t *tk = a.topk_keys_out + (int64_t)qi * a.top_k;
        for (int i = threadIdx.x; i < a.top_k; i += blockDim.x)
            tk[i] = i < cnt ? ((uint64_t)score_key(__ldg(scores + sel_out[i])) << 32) |
                                  (uint32_t)~(uint32_t)(sel_out[i] + a.entry_lo)
                            : 0ull;
    }
    if (a.topk_out) {
        int32_t *topk = a.topk_out + (int64_t)qi * a.top_k;
        for (int i = threadIdx.x; i < a.top_k; i += blockDim.x) topk[i] = i < cnt ? sel_out[i] : -1;
    }
    if (threadIdx.x == 0 && a.topk_count) a.topk_count[qi] = cnt;
}

// a6 selection: Top-K of the scored pool candidates.  By the block lemma, the Top-K lies
// in the top_k best pool slots by their maxima: select those slots (<= 2048 keys), then
// the Top-K over their <= 8 top_k positions.  Slots are in pool order = position order.
__global__ void __launch_bounds__(kSelThreads)
select_reindex_kernel(IndexArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    SelSmem &s = *reinterpret_cast<SelSmem *>(smem_raw);
    __shared__ int sel_out[CSA2_TOPK_MAX];
    __shared__ int sub[CSA2_TOPK_MAX];
    grid_dep_wait();
    grid_dep_launch();   // as in select_full_kernel: the layer's attention may start
    const int qi = blockIdx.x;
    const int64_t N = min64(visible_entries(a.q_pos[qi], a.ratio), a.cap);
    const int32_t *pool = a.pool + (int64_t)qi * a.pool_blocks;
    const float *sc = a.scores + (int64_t)qi * a.score_stride;
    const float *bm = a.bmax + (int64_t)qi * a.bmax_stride;
    const int P = a.pool_blocks;
    for (int i = threadIdx.x; i < P; i += kSelThreads) {
        const int blk = __ldg(pool + i);
        s.pool[i] = blk;
        s.keys[i] = blk >= 0 && (int64_t)blk * 8 < N ? score_key(__ldg(bm + i)) : 0u;
        if (i > 0 && blk >= 0 && __ldg(pool + i - 1) >= blk) set_dev_err(a.dev_err, CSA2_DEVERR_INDEX);
    }
    __syncthreads();
    auto skey = [&](int i) -> uint32_t { return s.keys[i]; };
    auto sid = [&](int i) -> int { return i; };
    const int ns = block_topk(skey, sid, P, a.top_k, sub, s);
    __syncthreads();
    // the chosen slots' 8 scores each (32 bytes, 16-byte aligned rows), then their keys
    for (int c = threadIdx.x; c < 2 * ns; c += kSelThreads)
        cp_async16(s.keys + 4 * c, sc + (int64_t)sub[c >> 1] * 8 + 4 * (c & 1));
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    for (int i = threadIdx.x; i < 8 * ns; i += kSelThreads) {
        const int64_t p = (int64_t)s.pool[sub[i >> 3]] * 8 + (i & 7);
        s.keys[i] = p < N ? score_key(__uint_as_float(s.keys[i])) : 0u;
    }
    __syncthreads();
    auto key = [&](int i) -> uint32_t { return s.keys[i]; };
    auto id = [&](int i) -> int { return s.pool[sub[i >> 3]] * 8 + (i & 7); };
    const int cnt = block_topk(key, id, 8 * ns, a.top_k, sel_out, s);
    __syncthreads();
    int32_t *topk = a.topk_out + (int64_t)qi * a.top_k;
    for (int i = threadIdx.x; i < a.top_k; i += blockDim.x) topk[i] = i < cnt ? sel_out[i] : -1;
    if (threadIdx.x == 0) a.topk_count[qi] = cnt;
}

// ------------------------------------------------------------------------------
// Context parallel: merge of the shards' candidate lists.  One CTA per query; the lists
// [n_lists][BT][list_len] of candidate keys (order key << 32 | ~global id, 0 = empty;
// shard-major, as an all-gather lays them out) are given in ascending slice order and
// each is ascending in id, so candidate index order
// is id order and block_topk's (key desc, index asc) order is the (key desc, id asc)
// order.  Every item of the global Top-k is in its own shard's local Top-k, so the
// result is exact.  Outputs ascending ids, -1 padded; with local_out, also the ids in
// [lo, hi) shifted by -lo (others -1).
// ------------------------------------------------------------------------------
__global__ void __launch_bounds__(kSelThreads)
index_merge_kernel(const uint64_t *lists, int n_lists, int list_len, int k, int64_t lo, int64_t hi,
                   int32_t *ids_out, int32_t *count_out, int32_t *local_out) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    SelSmem &s = *reinterpret_cast<SelSmem *>(smem_raw);
    __shared__ int sel_out[CSA2_POOL_MAX];
    grid_dep_wait();
    const int qi = blockIdx.x, BT = gridDim.x;
    const int n = n_lists * list_len;
    auto at = [&](int i) -> const uint64_t * {
        return lists + ((int64_t)(i / list_len) * BT + qi) * list_len + i % list_len;
    };
    for (int i = threadIdx.x; i < n; i += kSelThreads) s.keys[i] = (uint32_t)(__ldg(at(i)) >> 32);
    __syncthreads();
    auto key = [&](int i) -> uint32_t { return s.keys[i]; };
    auto id = [&](int i) -> int { return (int)~(uint32_t)__ldg(at(i)); };
    const int cnt = block_topk(key, id, n, k, sel_out, s);
    __syncthreads();
    grid_dep_launch();
    for (int i = threadIdx.x; i < k; i += kSelThreads) {
        const int g = i < cnt ? sel_out[i] : -1;
        if (ids_out) ids_out[(int64_t)qi * k + i] = g;
        if (local_out) local_out[(int64_t)qi * k + i] = g >= 0 && g >= lo && g < hi ? (int)(g - lo) : -1;
    }
    if (threadIdx.x == 0 && count_out) count_out[qi] = cnt;
}

cudaError_t launch_index_merge(const uint64_t *lists, int BT, int n_lists, int list_len, int k,
                               int64_t lo, int64_t hi, int32_t *ids_out, int32_t *count_out,
                               int32_t *local_out, cudaStream_t st) {
    const size_t smem = sizeof(SelSmem);
    static std::atomic<uint64_t> configured{0};   // per device
    {
        cudaError_t e = config_kernel_once(index_merge_kernel, smem, configured);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = launch_pdl(index_merge_kernel, dim3(BT), dim3(kSelThreads), smem, st, lists, n_lists,
                               list_len, k, lo, hi, ids_out, count_out, local_out);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// ------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------
template <int D, int HI>
static cudaError_t launch_scan_t(const IndexArgs &a, int grid_x, int BT, cudaStream_t st) {
    size_t smem = sizeof(ScoreSmem<D, HI, kScanRows>);
    static std::atomic<uint64_t> configured{0};   // per device
    {
        cudaError_t e = config_kernel_once(index_scan_kernel<D, HI>, smem, configured);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = launch_pdl(index_scan_kernel<D, HI>, dim3(grid_x, BT), dim3(kScoreThreads), smem, st, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

#define CSA2_DISPATCH_HI(D, FN, ...)                                          \
    switch (a.H_I) {                                                          \
        case 1: return FN<D, 1>(__VA_ARGS__);                                 \
        case 2: return FN<D, 2>(__VA_ARGS__);                                 \
        case 4: return FN<D, 4>(__VA_ARGS__);                                 \
        case 8: return FN<D, 8>(__VA_ARGS__);                                 \
        case 16: return FN<D, 16>(__VA_ARGS__);                               \
        default: return cudaErrorInvalidValue;                                \
    }

cudaError_t launch_index_scan(const IndexArgs &a, int BT, cudaStream_t st) {
    constexpr int kTileRows = kScoreThreads * kScanRows;
    int grid_x = (int)((a.n_max + kTileRows - 1) / kTileRows);
    if (grid_x == 0) return cudaSuccess;
    if (a.d_idx == 128) { CSA2_DISPATCH_HI(128, launch_scan_t, a, grid_x, BT, st) }
    CSA2_DISPATCH_HI(64, launch_scan_t, a, grid_x, BT, st)
}

template <int kCap>
static cudaError_t launch_select_full_t(const IndexArgs &a, int BT, cudaStream_t st) {
    size_t smem = sizeof(SelSmemT<kCap>);
    static std::atomic<uint64_t> configured{0};   // per device
    {
        cudaError_t e = config_kernel_once(select_full_kernel<kCap>, smem, configured);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = launch_pdl(select_full_kernel<kCap>, dim3(BT), dim3(kSelThreads), smem, st, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_select_full(const IndexArgs &a, int BT, cudaStream_t st) {
    // flat rows longer than the default stage and without 64-position maxima (the
    // tensor-core scan): the wide stage, if they fit
    if (a.pool_blocks == 0 && a.n_max > kSelStageMax && a.bmax64 == nullptr)
        return launch_select_full_t<kSelStageWide>(a, BT, st);
    return launch_select_full_t<kSelStageMax>(a, BT, st);
}


template <int D, int HI>
static cudaError_t launch_reindex_t(const IndexArgs &a, int BT, cudaStream_t st) {
    size_t smem = sizeof(ScoreSmem<D, HI, kReindexRows>);
    static std::atomic<uint64_t> configured{0};   // per device
    {
        cudaError_t e = config_kernel_once(reindex_score_kernel<D, HI>, smem, configured);
        if (e != cudaSuccess) return e;
    }
    constexpr int kBlocksPerTile = kScoreThreads * kReindexRows / 8;
    int gx = (a.pool_blocks + kBlocksPerTile - 1) / kBlocksPerTile;
    cudaError_t e = launch_pdl(reindex_score_kernel<D, HI>, dim3(gx, BT), dim3(kScoreThreads), smem, st, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_reindex_score(const IndexArgs &a, int BT, cudaStream_t st) {
    if (a.d_idx == 128) { CSA2_DISPATCH_HI(128, launch_reindex_t, a, BT, st) }
    CSA2_DISPATCH_HI(64, launch_reindex_t, a, BT, st)
}

cudaError_t launch_select_reindex(const IndexArgs &a, int BT, cudaStream_t st) {
    size_t smem = sizeof(SelSmem);
    static std::atomic<uint64_t> configured{0};   // per device
    {
        cudaError_t e = config_kernel_once(select_reindex_kernel, smem, configured);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = launch_pdl(select_reindex_kernel, dim3(BT), dim3(kSelThreads), smem, st, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace csa2
