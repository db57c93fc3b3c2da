// csa2_index_tc.cu -- a3 Full-layer index scan on the tensor cores, for prefill
// chunks (many query tokens per request).
//
// DeepSeek V4.1 Flash study notes, section 2, and myzaker "CSA2 attention": the
// Full layer scores every causally visible entry with
//   score(s) = sigma_s * sum_h w_h * relu(q_h . c_s)
// (c_s the entry's E4M3 indexer-K codes, sigma_s its scale).  With Tq query tokens
// per request the scan is Tq * N * H_I * d_idx multiply-adds, a dense contraction:
// the products c_s . q_h of 128 entries (MMA M = 128, one TMEM lane per entry)
// against 256 / H_I query tokens x H_I heads (MMA N = 256 columns) are one tcgen05
// MMA chain over the d_idx channels (K).  Operands are bf16: the bf16 query is used
// as is and the E4M3 codes are exact in bf16, so every product is exact; only the
// fp32 accumulation order differs from the fixed order of the exact scan
// (csa2_index.cu), so scores agree to a few fp32 ulps and Top-K membership can
// differ only between near-tied positions.
//
// Persistent: one CTA (512 threads) per SM takes a contiguous range of work items
// (request, block of 256 / H_I query tokens, tile of 128 entries), so the query
// block -- the MMA's B operand, kept in shared memory -- changes at most a few
// times per CTA.  Per tile: every thread converts a share of the tile's codes to
// bf16 into a 128-byte-swizzled K-major A tile (double-buffered), one elected
// thread issues the MMAs into one of two TMEM accumulators, and while they run all
// 16 warps take the previous tile's accumulator: thread = entry, so relu, w_h and
// the sum over a token's heads stay in registers, then sigma and the causal mask;
// a warp stores 32 consecutive entries of a token (128 bytes).  Scores and
// 8-position block maxima go to the same workspace as the exact scan, whose
// selection kernel then runs unchanged.  Every wait is bounded (WaitCfg); a CTA whose
// wait runs out flags CSA2_DEVERR_TIMEOUT, waits for the MMAs it has issued, frees its
// TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {
namespace itc {

constexpr int kThreads = 512;
constexpr int kM = 128;                  // entries per tile (MMA M, TMEM lanes)
constexpr int kN = 256;                  // query tokens x index heads (MMA N)
constexpr uint32_t kTmemCols = 512;      // two 256-column fp32 accumulators

template <int D>
struct __align__(1024) Smem {
    uint8_t q[D / 64][kN * 128];         // B: query rows (token, head), bf16, [channel block][row][128 B]
    uint8_t a[2][D / 64][kM * 128];      // A: entry codes as bf16, same layout, 2 buffers
    alignas(16) float w[kN];             // w of each column (token, head)
    int32_t nvis[kN];                    // visible entries of each token of the block (-1: none)
    uint64_t mma_done[2];
    uint64_t drain;                      // abort path: completes once every issued MMA has
    uint64_t never;                      // test hook (WaitCfg::stuck): never signalled
    uint32_t tmem_base;
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t wall_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity, uint64_t limit_ns) {
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
        if (wall_ns() - t0 > limit_ns) return false;
    }
}
// 128-byte-swizzled K-major operand descriptor (SBO = 8 rows x 128 B).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)(16u >> 4) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
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
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile(
        "{\n.reg .pred p;\n.reg .b32 r;\n"
        "elect.sync r|p, 0xffffffff;\n"
        "selp.u32 %0, 1, 0, p;\n}"
        : "=r"(pred));
    return pred != 0;
}
// 32 lanes x 32 columns: thread t of the warp reads lane (base + t), columns [col, col + 32).
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
// Byte offset of (row, 16-byte unit u of a 64-channel block) in a swizzled block.
__device__ __forceinline__ uint32_t swz_off(int row, int u) {
    return (uint32_t)(row * 128 + ((u ^ (row & 7)) << 4));
}
// Two E4M3 codes (low byte first) -> bf16x2, exact (E4M3 -> f16 -> f32 -> bf16).
__device__ __forceinline__ uint32_t e4m3x2_bf16x2(uint32_t two) {
    const uint32_t h = cvt_e4m3x2_f16x2(two);
    const float lo = __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
    const float hi = __half2float(__ushort_as_half((unsigned short)(h >> 16)));
    const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&b);
}

// Work item it = (by, tile), by = b * n_qblk + y: request b, query block y (tokens
// y * QB ..), entry tile (entries tile * 128 ..).  CTA c takes items
// [c * W / G, (c + 1) * W / G).
template <int D, int HI>
__global__ void __launch_bounds__(kThreads, 1) index_scan_tc_kernel(IndexArgs a, int B, int n_qblk,
                                                                    int n_tiles) {
    constexpr int QB = kN / HI;          // query tokens per block
    constexpr int CB = D / 64;           // 64-channel blocks
    constexpr int TPC = 32 / HI;         // tokens per 32-column TMEM load
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem<D> &s = *reinterpret_cast<Smem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int my_ent = 32 * (warp & 3) + lane;   // this thread's entry (TMEM lane) in a tile
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&s.mma_done[i])));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&s.drain)));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&s.never)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    }
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = s.tmem_base;
    grid_dep_wait();
    // kind::f16 instruction descriptor: F32 accumulator, bf16 A and B, both K-major
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kN >> 3) << 17) |
                           ((uint32_t)(kM >> 4) << 24);
    const int64_t total = (int64_t)B * n_qblk * n_tiles;
    const int64_t lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;

    int cur_by = -1, b = 0, tq0 = 0, hi_vis = 0;
    uint32_t n_issued = 0;               // MMA groups issued: buffer = n & 1, use = n >> 1
    int pend = -1;                       // issue number of the tile awaiting its epilogue
    int64_t pend_e0 = 0;
    float pend_sig = 0.0f;
    bool ok = true;
    bool stuck = a.wait.stuck != 0;      // test hook: the first wait never completes

    // epilogue of the pending tile: scores of entries pend_e0 + my_ent for every token
    auto epilogue = [&]() {
        const uint32_t buf = (uint32_t)pend & 1u;
        ok = __syncthreads_and(ok && (stuck ? mbar_wait(&s.never, 0, a.wait.limit_ns)
                                            : mbar_wait(&s.mma_done[buf], ((uint32_t)pend >> 1) & 1u,
                                                        a.wait.limit_ns))) != 0;
        stuck = false;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (!ok) return;
        const int64_t ent = pend_e0 + my_ent;
        const int col0 = 64 * (warp >> 2);
#pragma unroll 1
        for (int cc = 0; cc < 64; cc += 32) {
            float v[32];
            tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + buf * kN + (uint32_t)(col0 + cc), v);
#pragma unroll
            for (int u = 0; u < TPC; ++u) {
                const int c = col0 + cc + u * HI;            // first column of the token
                float wt[HI];
                if constexpr (HI >= 4) {
#pragma unroll
                    for (int h = 0; h < HI; h += 4) {
                        const float4 w4 = *reinterpret_cast<const float4 *>(&s.w[c + h]);
                        wt[h] = w4.x; wt[h + 1] = w4.y; wt[h + 2] = w4.z; wt[h + 3] = w4.w;
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < HI; ++h) wt[h] = s.w[c + h];
                }
                float t = 0.0f;
#pragma unroll
                for (int h = 0; h < HI; ++h) t = fmaf(wt[h], fmaxf(v[u * HI + h], 0.0f), t);
                const int tl = c / HI, tk = tq0 + tl;
                const int nv = s.nvis[tl];
                const bool vis = ent < nv;
                const float sc = __fmul_rn(t, pend_sig);
                const int64_t qi = (int64_t)b * a.Tq + tk;
                if (vis) a.scores[qi * a.score_stride + ent] = sc;
                if (a.bmax) {
                    float m = vis ? sc : -INFINITY;
                    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
                    if ((lane & 7) == 0 && vis) a.bmax[qi * a.bmax_stride + ent / 8] = m;
                }
            }
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        pend = -1;
    };

    for (int64_t it = lo; ok; ++it) {
        const bool have = it < hi;
        const int by = have ? (int)(it / n_tiles) : -1;
        if (have && by == cur_by && (int64_t)(it % n_tiles) * kM >= hi_vis) {
            it = (int64_t)(by + 1) * n_tiles - 1;            // the rest of this block is not visible
            continue;
        }
        if (!have || by != cur_by) {
            if (pend >= 0) epilogue();
            if (!have || !ok) break;
            // new query block: rows n = token * HI + head are consecutive rows of q_idx
            __syncthreads();
            cur_by = by;
            b = by / n_qblk;
            tq0 = (by % n_qblk) * QB;
            if (threadIdx.x < kN) {
                const int tl = threadIdx.x / HI, h = threadIdx.x % HI, tk = tq0 + tl;
                int nv = -1;
                float wv = 0.0f;
                if (tk < a.Tq) {
                    const int64_t qi = (int64_t)b * a.Tq + tk;
                    int64_t N = visible_entries(a.q_pos[qi], a.ratio);
                    if (N > a.n_max || N > a.cap) {
                        if (h == 0) set_dev_err(a.dev_err, CSA2_DEVERR_NMAX);
                        N = min64(min64(N, a.n_max), a.cap);
                    }
                    nv = (int)N;
                    wv = __ldg(a.w + qi * HI + h);
                }
                s.nvis[tl] = nv;
                s.w[threadIdx.x] = wv;
            }
            const uint16_t *qsrc = a.q_idx + ((int64_t)b * a.Tq + tq0) * HI * D;
            const int rows_valid = min(kN, (a.Tq - tq0) * HI);
            for (int e = threadIdx.x; e < kN * CB * 8; e += kThreads) {
                const int r = e / (CB * 8), cb = (e / 8) % CB, u = e % 8;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (r < rows_valid) v = __ldg(reinterpret_cast<const uint4 *>(qsrc + (int64_t)r * D + cb * 64 + u * 8));
                *reinterpret_cast<uint4 *>(s.q[cb] + swz_off(r, u)) = v;
            }
            __syncthreads();
            hi_vis = 0;
            for (int tl = 0; tl < QB; ++tl) hi_vis = max(hi_vis, s.nvis[tl]);
            if ((int64_t)(it % n_tiles) * kM >= hi_vis) {
                it = (int64_t)(by + 1) * n_tiles - 1;
                continue;
            }
        }
        // tile (by, it % n_tiles): convert into buffer n_issued & 1, issue its MMAs
        const int64_t e0 = (it % n_tiles) * kM;
        // the tile's entries are consecutive cache rows (a page holds whole tiles); a
        // bad page reads the request's first page instead and flags it (scores invalid)
        int64_t row0 = cache_row(a.pm, a.cap, b, e0);
        if (row0 < 0) {
            if (threadIdx.x == 0) set_dev_err(a.dev_err, CSA2_DEVERR_PAGE);
            row0 = 0;
        }
        const uint8_t *codes = a.idx_codes + row0 * D;
        const uint32_t buf = n_issued & 1u;
        const int64_t my_e = e0 + my_ent;
        const float sig = my_e < a.cap ? __ldg(a.idx_scale + row0 + my_ent) : 0.0f;
        constexpr int kUnits = kM * (D / 16) / kThreads;   // 16-code units per thread
        uint4 cu[kUnits];
#pragma unroll
        for (int k = 0; k < kUnits; ++k) {                  // all loads in flight together
            const int e = threadIdx.x + k * kThreads, n = e / (D / 16), g = e % (D / 16);
            cu[k] = make_uint4(0u, 0u, 0u, 0u);
            if (e0 + n < a.cap) cu[k] = __ldg(reinterpret_cast<const uint4 *>(codes + (int64_t)n * D + g * 16));
        }
#pragma unroll
        for (int k = 0; k < kUnits; ++k) {
            const int e = threadIdx.x + k * kThreads, n = e / (D / 16), g = e % (D / 16);
            // 16 channels = units u, u + 1 of channel block cb; which of the two is stored
            // first alternates so that a quarter-warp's stores hit 8 different bank groups
            const int cb = g / 4, u = (g % 4) * 2;
            const int first = (g ^ (g >> 2)) & 1;
            const uint32_t w0 = first ? cu[k].z : cu[k].x, w1 = first ? cu[k].w : cu[k].y;
            const uint32_t w2 = first ? cu[k].x : cu[k].z, w3 = first ? cu[k].y : cu[k].w;
            uint8_t *blk = s.a[buf][cb];
            *reinterpret_cast<uint4 *>(blk + swz_off(n, u + first)) =
                make_uint4(e4m3x2_bf16x2(w0 & 0xFFFFu), e4m3x2_bf16x2(w0 >> 16),
                           e4m3x2_bf16x2(w1 & 0xFFFFu), e4m3x2_bf16x2(w1 >> 16));
            *reinterpret_cast<uint4 *>(blk + swz_off(n, u + 1 - first)) =
                make_uint4(e4m3x2_bf16x2(w2 & 0xFFFFu), e4m3x2_bf16x2(w2 >> 16),
                           e4m3x2_bf16x2(w3 & 0xFFFFu), e4m3x2_bf16x2(w3 >> 16));
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (warp == 0) {
            if (elect_one()) {
                const uint32_t d = tmem + buf * kN;
#pragma unroll
                for (int k16 = 0; k16 < D / 16; ++k16) {
                    const int cb = k16 / 4, kk = k16 % 4;
                    const uint64_t ad = sw128_desc(smem_u32(s.a[buf][cb])) + (uint64_t)(2 * kk);
                    const uint64_t bd = sw128_desc(smem_u32(s.q[cb])) + (uint64_t)(2 * kk);
                    mma_bf16(d, ad, bd, idesc, k16 > 0 ? 1u : 0u);
                }
                mma_commit(&s.mma_done[buf]);
            }
            __syncwarp();
        }
        const int issued = (int)n_issued++;
        if (pend >= 0) epilogue();
        pend = issued;
        pend_e0 = e0;
        pend_sig = sig;
    }
    if (!ok) {
        // a wait ran out: the MMAs issued so far may still be running.  The issuing
        // thread commits once more; that arrival comes after all of them.
        if (threadIdx.x == 0) set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
        if (warp == 0) {
            if (elect_one()) mma_commit(&s.drain);
            __syncwarp();
        }
        const bool drained = mbar_wait(&s.drain, 0, kDrainLimitNs);
        (void)drained;
    }
    grid_dep_launch();
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

template <int D, int HI>
static cudaError_t launch_t(const IndexArgs &a, int B, cudaStream_t st) {
    const size_t smem = sizeof(Smem<D>) + 1024;
    static std::atomic<uint64_t> configured{0};   // per device
    {
        cudaError_t e = config_kernel_once(index_scan_tc_kernel<D, HI>, smem, configured);
        if (e != cudaSuccess) return e;
    }
    const int n_tiles = (int)((a.n_max + kM - 1) / kM);
    const int n_qblk = (a.Tq + kN / HI - 1) / (kN / HI);
    const int64_t total = (int64_t)B * n_qblk * n_tiles;
    if (total == 0) return cudaSuccess;
    const int grid = (int)(total < device_sm_count() ? total : device_sm_count());
    cudaError_t e = launch_pdl(index_scan_tc_kernel<D, HI>, dim3(grid), dim3(kThreads), smem, st, a,
                               B, n_qblk, n_tiles);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace itc

cudaError_t launch_index_scan_tc(const IndexArgs &a, int B, cudaStream_t st) {
#define CSA2_TC_HI(D)                                                   \
    switch (a.H_I) {                                                    \
        case 1: return itc::launch_t<D, 1>(a, B, st);                       \
        case 2: return itc::launch_t<D, 2>(a, B, st);                       \
        case 4: return itc::launch_t<D, 4>(a, B, st);                       \
        case 8: return itc::launch_t<D, 8>(a, B, st);                       \
        case 16: return itc::launch_t<D, 16>(a, B, st);                     \
        default: return cudaErrorInvalidValue;                          \
    }
    if (a.d_idx == 128) { CSA2_TC_HI(128) }
    CSA2_TC_HI(64)
#undef CSA2_TC_HI
}

}  // namespace csa2
