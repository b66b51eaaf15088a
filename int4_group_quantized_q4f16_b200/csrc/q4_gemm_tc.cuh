// q4_gemm_tc.cuh -- batched (prefill) product on the 5th-generation tensor cores.
//
// Zero-TVM write-up, limitations section: the project ships batched-prefill
// shaders (not wired into its decode loop), and its shaders compute in f16
// (WebGPU shader-f16).  For M tokens at once the product becomes a real GEMM,
// so it is split in two launches:
//
//   1. q4_dequant_f16_kernel  -- w16[n][k] = fp16((q - 7) * s), one correct
//      rounding per weight (HBM-bound: 0.5625 B read, 2 B written per weight);
//   2. q4_gemm_tc_kernel      -- y[m][n] = fp16(sum_k w16[n][k] x[m][k]) with
//      tcgen05.mma (kind::f16, fp32 accumulator in tensor memory).
//
// Dequantizing inside the GEMM would cost ~1.6 instructions per weight for
// every CTA that touches the weight, several times the tensor-core time of a
// 128 x 256 tile; writing w16 once and streaming it with TMA keeps the GEMM a
// plain fp16 contraction.
//
// GEMM layout: from 128 tokens on, the tokens are the MMA's M dimension (128
// or 256 per CTA as one or two 128-row MMAs, TMEM lane = token) and the weight
// rows its N dimension (64..256 per CTA, TMEM column = weight row).  Below 128
// tokens the roles swap ("swap AB": weight rows as M, tokens as N = 64 or
// 128), so a prefill of a few dozen tokens does not pad the 128-row MMA.  Both operands are K-major fp16 tiles of 64 k
// (one 128-byte row per weight row / token), loaded by TMA with the 128-byte
// swizzle that the UMMA shared-memory descriptor names.
//
// Roles (128 threads): thread 0 issues TMA loads into an S-stage ring, thread
// 32 issues the MMAs (4 or 8 x K=16 per stage) and frees each stage with
// tcgen05.commit; all four warps then read the accumulator (warp w owns TMEM
// lanes 32w..32w+31) and store y.  Every mbarrier wait is bounded (2 s of
// globaltimer); on expiry the thread sets bit 0 of *err, stops issuing, and
// the CTA still drains its loads and frees its tensor memory.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "q4_common.cuh"

namespace zt {

__device__ __forceinline__ float4 ldg_stream_f4(const float *p)
{
    const uint4 v = ldg_stream(reinterpret_cast<const uint4 *>(p));
    return make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w));
}

// ------------------------------------------------------------ dequant ----
// (1024 + q) is the fp16 pattern 0x6400 | q; subtracting 1031 = 0x6407 gives
// q - 7 exactly, and __hmul2 rounds (q - 7) * s once, to nearest even.
__device__ __forceinline__ uint32_t dq_pair(uint32_t codes2, __half2 s2)
{
    uint32_t v = codes2 | 0x64006400u;
    __half2 h = *reinterpret_cast<__half2 *>(&v);
    h = __hmul2(__hsub2(h, __half2half2(__ushort_as_half((unsigned short)0x6407))), s2);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint4 dq_word(uint32_t w, __half2 s2)
{
    const uint32_t a = dq_pair(w & 0x000F000Fu, s2);          // k 0, 4
    const uint32_t b = dq_pair((w >> 4) & 0x000F000Fu, s2);   // k 1, 5
    const uint32_t c = dq_pair((w >> 8) & 0x000F000Fu, s2);   // k 2, 6
    const uint32_t d = dq_pair((w >> 12) & 0x000F000Fu, s2);  // k 3, 7
    uint4 o;
    o.x = __byte_perm(a, b, 0x5410);   // k 0, 1
    o.y = __byte_perm(c, d, 0x5410);   // k 2, 3
    o.z = __byte_perm(a, b, 0x7632);   // k 4, 5
    o.w = __byte_perm(c, d, 0x7632);   // k 6, 7
    return o;
}

__device__ __forceinline__ uint32_t ldg_stream_u32(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// One warp per weight row (rows strided over the grid's warps); lane l takes
// the code words l, l + 32, ...: each load instruction reads 128 contiguous
// bytes of codes and each store writes 512 contiguous bytes of w16.
// qw [N][kw] words (kw = K/8), scales [N][K/group], w16 as uint4 [N][kw] (8
// halves per word).  gsh = log2(group / 32).  err (may be null) is cleared by
// thread 0 so the GEMM that follows on the stream starts with a clean error
// word.
__global__ void __launch_bounds__(256) q4_dequant_f16_kernel(const uint32_t *__restrict__ qw,
                                                             const __half *__restrict__ scales,
                                                             uint4 *__restrict__ w16, int N, int kw, int gsh,
                                                             unsigned int *err)
{
    constexpr int U = 4;   // words per lane per step: their loads are in flight together
    if (err && blockIdx.x == 0 && threadIdx.x == 0) *err = 0u;
    const int lane = threadIdx.x & 31;
    const int spr = (kw >> 2) >> gsh;                       // scales per row, K / group
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long n = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < N; n += warps) {
        const uint32_t *src = qw + n * kw;
        const __half *srow = scales + n * spr;
        uint4 *dst = w16 + n * kw;
        for (int w0 = lane; w0 < kw; w0 += 32 * U) {
            uint32_t q[U];
            __half sc[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int w = w0 + 32 * u;
                if (w < kw) {
                    q[u] = ldg_stream_u32(src + w);
                    sc[u] = srow[(w >> 2) >> gsh];          // word w holds k = 8w .. 8w + 7
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int w = w0 + 32 * u;
                if (w < kw) dst[w] = dq_word(q[u], __half2half2(sc[u]));
            }
        }
    }
}

// --------------------------------------------------------------- GEMM ----
constexpr int kTcMma = 128;       // rows of one MMA (M)
constexpr int kTcK = 64;          // k per stage: one 128-byte swizzle row of fp16
constexpr int kTcThreads = 128;
constexpr unsigned kErrTcWait = 1u;

// Operand tiles.  A: AM rows per CTA (128, or 256 as two 128-row MMAs that
// share the B tile, into two accumulators); B: BN rows per CTA (the MMA N).
// The 256-row A tile halves the bytes each SM takes in per MMA cycle (the
// limit of the 128-row tile), at the cost of half as many CTAs.
template <int AM, int BN>
struct TcCfg {
    static constexpr int kHalves = AM / kTcMma;
    static constexpr int kABytes = AM * kTcK * 2;                       // 16 or 32 KB
    static constexpr int kBBytes = BN * kTcK * 2;                       // 8, 16 or 32 KB
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = (192 * 1024) / kStageBytes;          // 3..8
    static constexpr int kTmemCols = kHalves * BN;
    static constexpr int kSmem = kStages * kStageBytes + 1024 + 256;    // + alignment + barriers
    // instruction descriptor, kind::f16: D f32 (bits 4-5 = 1), A and B f16
    // (bits 7-9, 10-12 = 0), both K-major (bits 15, 16 = 0), N >> 3 at bit 17,
    // M >> 4 at bit 24
    static constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kTcMma >> 4) << 24);
    static_assert(AM == 128 || AM == 256, "one or two MMAs per k step");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M = 128");
    static_assert((BN & (BN - 1)) == 0 && BN >= 32, "tensor memory is allocated in powers of two >= 32 columns");
    static_assert(kTmemCols <= 512, "tensor memory holds 512 columns");
    static_assert(kStages >= 2, "ring depth");
};

__device__ __forceinline__ unsigned long long tc_now()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of parity `par` of the mbarrier at shared address `bar`
// to complete; false after 2 s.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t par, bool nap)
{
    unsigned long long t0 = 0;
    for (uint32_t it = 0;; ++it) {
        uint32_t ok;
        asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                     : "=r"(ok) : "r"(bar), "r"(par) : "memory");
        if (ok) return true;
        if (it == 0) t0 = tc_now();
        else if ((it & 15u) == 0 && tc_now() - t0 > 2000000000ull) return false;
        if (nap) __nanosleep(256);
    }
}

// UMMA shared-memory descriptor for a K-major tile in the 128-byte swizzle:
// start address >> 4 (bits 0-13), leading byte offset 1 (unused for this
// layout, bits 16-29), stride byte offset 1024 >> 4 between 8-row groups
// (bits 32-45), version 1 (bits 46-47), base offset 0 (the tile is 1024-byte
// aligned), layout 2 = SWIZZLE_128B (bits 61-63).
__device__ __forceinline__ uint64_t tc_desc_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tc_tma_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar) : "memory");
}

// 32 consecutive TMEM columns of this warp's 32 lanes into r[0..31]; the wait
// names the registers so no use is scheduled before the data has arrived.
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// TOKA: the A operand holds tokens (x) and B weight rows (w16): TMEM lane =
// token m, column = weight row n, so each thread ends with 32 consecutive
// outputs of one token row and writes them as four 16-byte stores.  Otherwise
// ("swap AB", for fewer than 128 tokens) A holds weight rows and B tokens.
// tma_a / tma_b: fp16 [rows][K], boxes 64 x AM and 64 x BN, 128-byte swizzled,
// out-of-range rows and k read as zero.
//
// Split K (blockIdx.z = split, kb_per k blocks each): with part != null the
// CTA writes its fp32 partial tile to part[z][M][N] instead of y, and
// q4_splitk_reduce_kernel sums the splits in order.
// SILU (with TOKA, unsplit): the fused FFN (Zero-TVM write-up, kernel-fusion
// section: gate, up and SiLU in one pass) on the binary16 weights [2N][K],
// gate rows first.  The B tile is two half boxes -- gate rows n0 .. n0 + BN/2
// and up rows N + n0 .. -- so TMEM columns c and BN/2 + c hold g and u of the
// same output, and the epilogue writes y = SiLU(g) u for BN/2 outputs.
template <int AM, int BN, bool TOKA, bool SILU>
__global__ void __launch_bounds__(kTcThreads, 1) q4_gemm_tc_kernel(const __grid_constant__ CUtensorMap tma_a,
                                                                   const __grid_constant__ CUtensorMap tma_b,
                                                                   __half *__restrict__ y, float *__restrict__ part,
                                                                   int M, int N, int K, int kb_per,
                                                                   unsigned int *err)
{
    using C = TcCfg<AM, BN>;
    constexpr int S = C::kStages;
    extern __shared__ __align__(128) unsigned char tc_smem[];
    const uint32_t raw = smem_u32(tc_smem);
    const uint32_t ring = (raw + 1023u) & ~1023u;                     // swizzle atoms are 1024-byte aligned
    const uint32_t bars = ring + S * C::kStageBytes;                  // full[S], empty[S], acc
    const uint32_t slot = bars + (2 * S + 1) * 8;                     // TMEM base written by tcgen05.alloc
    auto full = [&](int s) { return bars + 8u * s; };
    auto empty = [&](int s) { return bars + 8u * (S + s); };
    const uint32_t accb = bars + 8u * (2 * S);
    volatile uint32_t *consumed_s = reinterpret_cast<volatile uint32_t *>(tc_smem + (slot + 8 - raw));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    static_assert(!SILU || TOKA, "the fused FFN epilogue needs tokens as the A operand");
    const int a0 = blockIdx.x * AM, b0 = blockIdx.y * (SILU ? BN / 2 : BN);
    const int kb_lo = blockIdx.z * kb_per;
    const int kb_n = min((K + kTcK - 1) / kTcK - kb_lo, kb_per);   // k blocks of this split (>= 1)

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full(s)) : "memory");
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(empty(s)) : "memory");
        }
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(accb) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        *consumed_s = 0u;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot),
                     "r"(C::kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    uint32_t tmem;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(slot) : "memory");

    int issued = 0;
    if (threadIdx.x == 0) {
        // producer: stage s of round r waits until round r - 1 of s was consumed
        for (int kb = 0; kb < kb_n; ++kb) {
            const int s = kb % S, r = kb / S;
            if (r > 0 && !tc_wait(empty(s), (uint32_t)((r - 1) & 1), false)) {
                atomicOr(err, kErrTcWait);
                break;
            }
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full(s)),
                         "r"(C::kStageBytes) : "memory");
            const uint32_t a = ring + s * C::kStageBytes;
            tc_tma_2d(a, &tma_a, (kb_lo + kb) * kTcK, a0, full(s));
            if (SILU) {
                // gate rows, then the matching up rows N further down the fused weight
                tc_tma_2d(a + C::kABytes, &tma_b, (kb_lo + kb) * kTcK, b0, full(s));
                tc_tma_2d(a + C::kABytes + (BN / 2) * kTcK * 2, &tma_b, (kb_lo + kb) * kTcK, N + b0, full(s));
            } else {
                tc_tma_2d(a + C::kABytes, &tma_b, (kb_lo + kb) * kTcK, b0, full(s));
            }
            issued = kb + 1;
        }
    } else if (threadIdx.x == 32) {
        // MMA issuer
        int kb = 0;
        for (; kb < kb_n; ++kb) {
            const int s = kb % S, r = kb / S;
            if (!tc_wait(full(s), (uint32_t)(r & 1), false)) {
                atomicOr(err, kErrTcWait);
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t a = ring + s * C::kStageBytes;
            const uint64_t da = tc_desc_sw128(a), db = tc_desc_sw128(a + C::kABytes);
#pragma unroll
            for (int j = 0; j < kTcK / 16; ++j) {
                // K = 16 fp16 = 32 bytes further along the swizzled row: +2 in the address field
                const uint32_t acc = (kb | j) ? 1u : 0u;
#pragma unroll
                for (int h = 0; h < C::kHalves; ++h) {
                    // rows 128h.. of the A tile start 16 KB (1024 in the address field) further
                    asm volatile(
                        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                        ::"r"(tmem + (uint32_t)(h * BN)), "l"(da + (uint64_t)(h * 1024) + 2 * j), "l"(db + 2 * j),
                        "r"(C::kIdesc), "r"(acc));
                }
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(empty(s))
                         : "memory");
        }
        *consumed_s = (uint32_t)kb;
        // all MMAs issued above complete before this arrives
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(accb)
                     : "memory");
    }
    __syncwarp();

    // epilogue: TMEM lane = A row, column = B row
    // warp-uniform, so the aligned tensor-memory loads below stay converged
    const bool ok = __all_sync(0xffffffffu, tc_wait(accb, 0u, true));
    if (!ok && lane == 0) atomicOr(err, kErrTcWait);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const bool vec = TOKA && (N % 8) == 0 && ((reinterpret_cast<uintptr_t>(y) & 15) == 0);
    const bool vecp = TOKA && (N % 4) == 0 && ((reinterpret_cast<uintptr_t>(part) & 15) == 0);
    float *pz = part ? part + (size_t)blockIdx.z * M * N : nullptr;
    if constexpr (SILU) {
#pragma unroll 1
        for (int h = 0; h < C::kHalves; ++h) {
            const int m = a0 + h * kTcMma + warp * 32 + lane;          // this thread's token
            const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(h * BN);
#pragma unroll 1
            for (int c = 0; c < BN / 64; ++c) {
                uint32_t g[32], u[32];
                tc_ld32(trow + (uint32_t)(c * 32), g);
                tc_ld32(trow + (uint32_t)(BN / 2 + c * 32), u);
                const int n = b0 + c * 32;
                if (ok && m < M) {   // a block, not a jump: the next aligned loads stay converged
                float o[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    // fast exp and divide: their error (a few fp32 ulp) is far below the fp16 output's
                    // rounding; e^-g overflowing to inf gives SiLU = 0, its limit
                    const float gv = __uint_as_float(g[j]);
                    o[j] = __fdividef(gv, 1.0f + __expf(-gv)) * __uint_as_float(u[j]);
                }
                __half *dst = y + (size_t)m * N + n;
                if (vec && n + 32 <= N) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 v;
                        uint32_t *pv = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __half2 h2 = __floats2half2_rn(o[8 * q + 2 * e], o[8 * q + 2 * e + 1]);
                            pv[e] = *reinterpret_cast<uint32_t *>(&h2);
                        }
                        *reinterpret_cast<uint4 *>(dst + 8 * q) = v;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (n + j < N) dst[j] = __float2half_rn(o[j]);
                }
                }
            }
        }
    } else {
#pragma unroll 1
    for (int h = 0; h < C::kHalves; ++h) {
        const int ra = a0 + h * kTcMma + warp * 32 + lane;           // this thread's A row
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(h * BN);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            uint32_t r[32];
            tc_ld32(trow + (uint32_t)(c * 32), r);
            if (!ok) continue;
            const int rb = b0 + c * 32;                                 // first B row of these columns
            if (pz) {
                // fp32 partials, [M][N] per split
                if (TOKA) {
                    if (ra < M) {
                        float *dst = pz + (size_t)ra * N + rb;
                        if (vecp && rb + 32 <= N) {
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                *reinterpret_cast<float4 *>(dst + 4 * q) =
                                    make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                                __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (rb + j < N) dst[j] = __uint_as_float(r[j]);
                        }
                    }
                } else if (ra < N) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (rb + j < M) pz[(size_t)(rb + j) * N + ra] = __uint_as_float(r[j]);
                }
            } else if (TOKA) {
                if (ra < M) {
                    __half *dst = y + (size_t)ra * N + rb;
                    if (vec && rb + 32 <= N) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 v;
                            uint32_t *pv = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                __half2 h2 = __floats2half2_rn(__uint_as_float(r[8 * q + 2 * e]),
                                                               __uint_as_float(r[8 * q + 2 * e + 1]));
                                pv[e] = *reinterpret_cast<uint32_t *>(&h2);
                            }
                            *reinterpret_cast<uint4 *>(dst + 8 * q) = v;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (rb + j < N) dst[j] = __float2half_rn(__uint_as_float(r[j]));
                    }
                }
            } else if (ra < N) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int m = rb + j;
                    if (m < M) y[(size_t)m * N + ra] = __float2half_rn(__uint_as_float(r[j]));
                }
            }
        }
    }

    }   // SILU

    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
        // loads issued but never consumed (only after an expired wait) land before the CTA exits
        for (int kb = (int)*consumed_s; kb < issued; ++kb)
            if (!tc_wait(full(kb % S), (uint32_t)((kb / S) & 1), false)) break;
    }
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols)
                     : "memory");
    }
}

// y[i] = fp16(sum_z part[z][i]), z = 0 .. splits-1 in order (deterministic);
// four elements per thread when mn % 4 == 0 and y is 8-byte aligned.
__global__ void __launch_bounds__(256) q4_splitk_reduce_kernel(const float *__restrict__ part,
                                                               __half *__restrict__ y, long long mn, int splits)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if ((mn & 3) == 0 && (reinterpret_cast<uintptr_t>(y) & 7) == 0) {
        for (long long i = t0; i < mn / 4; i += stride) {
            float4 a = ldg_stream_f4(part + 4 * i);
            for (int z = 1; z < splits; ++z) {
                const float4 b = ldg_stream_f4(part + (size_t)z * mn + 4 * i);
                a.x += b.x;
                a.y += b.y;
                a.z += b.z;
                a.w += b.w;
            }
            const __half2 lo = __floats2half2_rn(a.x, a.y), hi = __floats2half2_rn(a.z, a.w);
            uint2 v;
            v.x = *reinterpret_cast<const uint32_t *>(&lo);
            v.y = *reinterpret_cast<const uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(y + 4 * i) = v;
        }
    } else {
        for (long long i = t0; i < mn; i += stride) {
            float a = part[i];
            for (int z = 1; z < splits; ++z) a += part[(size_t)z * mn + i];
            y[i] = __float2half_rn(a);
        }
    }
}

}  // namespace zt
