// csa2_index_tc.cu -- a3 Full-layer index scan on the tensor cores, for prefill
// chunks (many query tokens per request).
//
// DeepSeek V4.1 Flash study notes, section 2, and myzaker "CSA2 attention": the
// Full layer scores every causally visible entry with
//   score(s) = sigma_s * sum_h w_h * relu(q_h . c_s)
// (c_s the entry's E4M3 indexer-K codes, sigma_s its scale).  With Tq query tokens
// per request the scan is Tq * N * H_I * d_idx multiply-adds, which the CUDA cores
// of the exact scan (csa2_index.cu) take ~1000x longer to do than this tensor-core
// form: the products q_h . c_s of 128 / H_I query tokens (M = 128 rows = tokens x
// heads) against 256 entries (N = 256) at a time are one tcgen05 MMA chain over the
// d_idx channels (K).  Operands are bf16: the bf16 query is used as is and the E4M3
// codes are exact in bf16, so every product is exact; only the fp32 accumulation
// order differs from the fixed order of the exact scan, so scores agree to a few
// fp32 ulps and Top-K membership can differ only between near-tied positions.
//
// One CTA (512 threads) = one request's block of 128 / H_I query tokens and up to
// kTilesPerCta tiles of 256 entries.  Per tile: every thread converts a share of
// the tile's codes to bf16 into a 128-byte-swizzled K-major tile (double-buffered),
// one elected thread issues the MMAs into one of two TMEM accumulators, and while
// they run all 16 warps take the previous tile's accumulator: relu, w_h, the sum
// over the H_I rows of a token (lane shuffles), sigma, the causal mask; scores and
// 8-position block maxima go to the same workspace as the exact scan, whose
// selection kernel then runs unchanged.  Every wait is bounded (0.5 s).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "csa2_common.cuh"
#include "csa2_internal.h"

namespace csa2 {
namespace itc {

constexpr int kThreads = 512;
constexpr int kM = 128;                  // MMA rows: query tokens x index heads
constexpr int kN = 256;                  // entries per tile (MMA N)
constexpr int kTilesPerCta = 8;
constexpr uint32_t kTmemCols = 512;      // two 256-column fp32 accumulators
constexpr uint64_t kWaitLimitNs = 500000000ull;

template <int D>
struct __align__(1024) Smem {
    uint8_t a[D / 64][kM * 128];         // q, bf16, [channel block][row][128 B] swizzled
    uint8_t b[2][D / 64][kN * 128];      // entry codes as bf16, same layout, 2 buffers
    float sig[3][kN];                    // entry scales of tile i in sig[i % 3] (see the loop)
    float w[kM];                         // w of each row (token, head)
    int32_t nvis[kM];                    // visible entries of each row's token (-1: no token)
    uint64_t mma_done[2];
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

template <int D, int HI>
__global__ void __launch_bounds__(kThreads, 1) index_scan_tc_kernel(IndexArgs a) {
    constexpr int QB = kM / HI;          // query tokens per CTA
    constexpr int CB = D / 64;           // 64-channel blocks
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem<D> &s = *reinterpret_cast<Smem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.z;
    const int tq0 = blockIdx.y * QB;     // first query token of the block
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&s.mma_done[i])));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    }
    grid_dep_wait();
    // rows r = token * HI + head; tokens past Tq are zero rows whose scores are dropped
    if (threadIdx.x < kM) {
        const int r = threadIdx.x, tk = tq0 + r / HI, h = r % HI;
        int nv = -1;
        float wv = 0.0f;
        if (tk < a.Tq) {
            const int qi = b * a.Tq + tk;
            int64_t N = visible_entries(a.q_pos[qi], a.ratio);
            if (N > a.n_max || N > a.cap) {
                if (h == 0) set_dev_err(a.dev_err, CSA2_DEVERR_NMAX);
                N = min64(min64(N, a.n_max), a.cap);
            }
            nv = (int)N;
            wv = __ldg(a.w + (int64_t)qi * HI + h);
        }
        s.nvis[r] = nv;
        s.w[r] = wv;
    }
    // q rows into the A operand (bf16 as is): unit (row, cb, u) of 8 channels
    for (int e = threadIdx.x; e < kM * CB * 8; e += kThreads) {
        const int r = e / (CB * 8), cb = (e / 8) % CB, u = e % 8;
        const int tk = tq0 + r / HI, h = r % HI;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (tk < a.Tq)
            v = __ldg(reinterpret_cast<const uint4 *>(a.q_idx + ((int64_t)(b * a.Tq + tk) * HI + h) * D + cb * 64 + u * 8));
        *reinterpret_cast<uint4 *>(s.a[cb] + swz_off(r, u)) = v;
    }
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // tiles past the largest visible count of the block's tokens are skipped
    int hi_vis = 0;
    for (int r = 0; r < kM; r += HI) hi_vis = max(hi_vis, s.nvis[r]);
    const int n_tiles_vis = (hi_vis + kN - 1) / kN;
    const int t_begin = blockIdx.x * kTilesPerCta;
    const int t_end = min(n_tiles_vis, t_begin + kTilesPerCta);
    const int nt = max(0, t_end - t_begin);
    const uint32_t tmem = s.tmem_base;
    // kind::f16 instruction descriptor: F32 accumulator, bf16 A and B, both K-major
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kN >> 3) << 17) |
                           ((uint32_t)(kM >> 4) << 24);
    const uint8_t *codes = a.idx_codes + (int64_t)b * a.cap * D;
    const float *sigma = a.idx_scale + (int64_t)b * a.cap;
    bool ok = true;
    // tile i: convert into buffer i & 1, issue its MMAs, then the epilogue of tile i - 1
    for (int i = 0; i <= nt; ++i) {
        if (i < nt) {
            const int64_t e0 = (int64_t)(t_begin + i) * kN;
            // entry row n, 16-byte unit of 16 codes -> two bf16 units of 8 channels
            for (int e = threadIdx.x; e < kN * (D / 16); e += kThreads) {
                const int n = e / (D / 16), g = e % (D / 16);
                const int64_t ent = e0 + n;
                uint4 c = make_uint4(0u, 0u, 0u, 0u);
                if (ent < a.cap) c = __ldg(reinterpret_cast<const uint4 *>(codes + ent * D + g * 16));
                const uint32_t w4[4] = {c.x, c.y, c.z, c.w};
                uint32_t o[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    o[2 * k] = e4m3x2_bf16x2(w4[k] & 0xFFFFu);
                    o[2 * k + 1] = e4m3x2_bf16x2(w4[k] >> 16);
                }
                const int ch = g * 16, cb = ch / 64, u = (ch % 64) / 8;
                uint8_t *blk = s.b[i & 1][cb];
                *reinterpret_cast<uint4 *>(blk + swz_off(n, u)) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4 *>(blk + swz_off(n, u + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
            }
            // three scale buffers: a thread here has passed the barrier that ends tile i - 3's
            // epilogue, while warps with no rows to write may still be in tile i - 2's
            for (int n = threadIdx.x; n < kN; n += kThreads)
                s.sig[i % 3][n] = e0 + n < a.cap ? __ldg(sigma + e0 + n) : 0.0f;
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncthreads();
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            if (warp == 0) {
                if (elect_one()) {
                    const uint32_t d = tmem + (uint32_t)((i & 1) * kN);
#pragma unroll
                    for (int k16 = 0; k16 < D / 16; ++k16) {
                        const int cb = k16 / 4, kk = k16 % 4;
                        const uint64_t ad = sw128_desc(smem_u32(s.a[cb])) + (uint64_t)(2 * kk);
                        const uint64_t bd = sw128_desc(smem_u32(s.b[i & 1][cb])) + (uint64_t)(2 * kk);
                        mma_bf16(d, ad, bd, idesc, k16 > 0 ? 1u : 0u);
                    }
                    mma_commit(&s.mma_done[i & 1]);
                }
                __syncwarp();
            }
        }
        if (i > 0) {
            // epilogue of tile j = i - 1: warp w reads TMEM lanes 32 (w % 4) .. (rows) and
            // columns 64 (w / 4) .. +64 (entries)
            const int j = i - 1;
            ok = __syncthreads_and(ok && mbar_wait(&s.mma_done[j & 1], (j >> 1) & 1)) != 0;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            if (!ok) break;
            const int r = 32 * (warp & 3) + lane;
            const int c0 = 64 * (warp >> 2);
            const int tk = tq0 + r / HI, h = r % HI;
            const int nv = s.nvis[r];
            const float wr = s.w[r];
            const int64_t e0 = (int64_t)(t_begin + j) * kN;
            const bool writer = h == 0 && tk < a.Tq;
            const int qi = b * a.Tq + tk;
            float *srow = a.scores + (int64_t)qi * a.score_stride;
#pragma unroll 1
            for (int cc = 0; cc < 64; cc += 32) {
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)((j & 1) * kN + c0 + cc), v);
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    float t = wr * fmaxf(v[x], 0.0f);
#pragma unroll
                    for (int o = 1; o < HI; o <<= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
                    v[x] = t;
                }
                if (writer) {
                    float sc[32];
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        const int64_t ent = e0 + c0 + cc + x;
                        sc[x] = ent < nv ? __fmul_rn(v[x], s.sig[j % 3][c0 + cc + x]) : -INFINITY;
                    }
#pragma unroll
                    for (int x = 0; x < 32; x += 4)
                        if (e0 + c0 + cc + x + 3 < a.score_stride)
                            *reinterpret_cast<float4 *>(srow + e0 + c0 + cc + x) =
                                make_float4(sc[x], sc[x + 1], sc[x + 2], sc[x + 3]);
                    if (a.bmax) {
#pragma unroll
                        for (int x = 0; x < 32; x += 8) {
                            float m = sc[x];
#pragma unroll
                            for (int y = 1; y < 8; ++y) m = fmaxf(m, sc[x + y]);
                            const int64_t blk = (e0 + c0 + cc + x) / 8;
                            if (blk * 8 < nv) a.bmax[(int64_t)qi * a.bmax_stride + blk] = m;
                        }
                    }
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        }
    }
    if (!ok && threadIdx.x == 0) set_dev_err(a.dev_err, CSA2_DEVERR_TIMEOUT);
    grid_dep_launch();
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

template <int D, int HI>
static cudaError_t launch_t(const IndexArgs &a, int B, cudaStream_t st) {
    const size_t smem = sizeof(Smem<D>) + 1024;
    static bool attr_set = false;   // once per process and instantiation
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(index_scan_tc_kernel<D, HI>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = prefer_max_smem(index_scan_tc_kernel<D, HI>);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int n_tiles = (int)((a.n_max + kN - 1) / kN);
    const dim3 grid((n_tiles + kTilesPerCta - 1) / kTilesPerCta, (a.Tq + kM / HI - 1) / (kM / HI), B);
    if (grid.x == 0) return cudaSuccess;
    cudaError_t e = launch_pdl(index_scan_tc_kernel<D, HI>, grid, dim3(kThreads), smem, st, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace itc

cudaError_t launch_index_scan_tc(const IndexArgs &a, int B, cudaStream_t st) {
#define CSA2_TC_HI(D)                                                   \
    switch (a.H_I) {                                                    \
        case 1: return itc::launch_t<D, 1>(a, B, st);                   \
        case 2: return itc::launch_t<D, 2>(a, B, st);                   \
        case 4: return itc::launch_t<D, 4>(a, B, st);                   \
        case 8: return itc::launch_t<D, 8>(a, B, st);                   \
        case 16: return itc::launch_t<D, 16>(a, B, st);                 \
        default: return cudaErrorInvalidValue;                          \
    }
    if (a.d_idx == 128) { CSA2_TC_HI(128) }
    CSA2_TC_HI(64)
#undef CSA2_TC_HI
}

}  // namespace csa2
