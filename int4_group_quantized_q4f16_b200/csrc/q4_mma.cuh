// q4_mma.cuh -- the sm_100a dequantizing GEMV for M <= 16: codes unpacked two
// per logic instruction into fp16 subnormals, contracted on tensor cores with
// register-sourced mma.sync, fed from HBM by per-warp cp.async rings.
//
// Operation: the int4 dequantizing matrix product of the Zero-TVM write-up
// (section "完整的推理流水线": the baseline / subgroup-reduce / rows x4, x8
// variants and the f32-output LM head) and its fused FFN (section "内核融合",
// fused_ffn: gate, up and SiLU in one pass).
//
// Why tensor cores for a GEMV: on CUDA cores the unpack costs at least one
// integer/logic instruction per weight (one fp32 lane per code), and the
// integer pipe -- half rate on this part -- saturates long before HBM does.
// Packing two codes per 32-bit register (one per fp16 half) halves that, and
// the mma.sync contraction then takes the multiply-adds off the CUDA cores.
// mma.sync reads its A operand from registers, exactly where the unpacked
// codes are; a tcgen05 contraction would first have to write them to shared
// or tensor memory (4x the code bytes), for no gain on a bandwidth-bound
// product.
//
// Arithmetic (exact products, fp32 accumulation):
//   * An fp16 bit pattern below 0x0400 is the subnormal value pattern * 2^-24
//     (IEEE 754 binary16).  So (w & 0x000F000F) read as half2 is exactly
//     (q0 * 2^-24, q4 * 2^-24), and (w & 0x00F000F0) is (16 q1 * 2^-24,
//     16 q5 * 2^-24): one logic instruction dequantizes two codes, with no
//     bias to subtract.
//   * mma.sync.m16n8k16 (f16 x f16 -> f32) forms the products q * x * 2^-24
//     exactly (4-bit times 11-bit significands) and accumulates in fp32.  The
//     k axis inside a group is permuted consistently on the A and B sides (a
//     dot product does not depend on the order of its terms), so that each
//     thread's codes come from one 32-bit word: thread t of a quad owns word t
//     (codes 8t..8t+7) of the group; step 0 of the group takes codes
//     {0,4 | 2,6} of it (mask 0x000F000F on w and w >> 8), step 1 codes
//     {1,5 | 3,7} (mask 0x00F000F0, which carries a factor 16).  The
//     activations are staged once per CTA in that order, and those meeting
//     step 1 are staged divided by 16 -- exact for |x| >= 2^-10 (smaller ones
//     are rounded to fp16 after the division, an absolute error below 2^-25
//     per value).  So both steps accumulate into one fp32 tile.
//   * Zero point: sum_k (q_k - 7) x_k = sum_k q_k x_k - 7 X_g; the -7 X_g term
//     (X_g = sum of the group's activations, per column) enters as the C
//     operand of the group's first mma.  The group's result is scaled once:
//     acc += s * D, in fp32, and the final 2^24 is an exact power-of-two
//     multiply.
//
// Layout (mma tile = 16 weight rows x 8 columns of x):
//   * A warp tile is 16 weight rows (for the fused FFN: 8 gate rows + the 8 up
//     rows of the same outputs, so gate and up of an output meet in one
//     thread).  K is cut into chunks of 8 groups (256 k).  Item = (tile,
//     chunk) = 16 x 128 bytes of codes + 16 x 16 bytes of scales.
//   * Each CTA owns a contiguous, balanced range of outputs; its 8 warps form
//     WR x WK (WK warps split a tile's chunks when the CTA has few rows).
//   * Every warp streams its items through a private ring of S stages with
//     16-byte cp.async copies (hardware waits, no spin loops).  Rows outside
//     the CTA's range are never copied: a partial tile costs math, not bytes.
//   * Programmatic dependent launch: the first S - 1 items are issued before
//     griddepcontrol.wait, so weights stream while the previous kernel on the
//     stream finishes; activations are read and outputs written after it.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "q4_stream.cuh"

namespace zt {

constexpr int kMW = 8;                              // warps per CTA
constexpr int kMThreads = kMW * 32;
constexpr int kMTileRows = 16;                      // weight rows per warp tile (mma M)
constexpr int kMChunkG = 8;                         // groups per item
constexpr int kMRowStride = kMChunkG * 16 + 16;     // smem bytes per tile row (padded: conflict-free)
constexpr int kMScaleOff = kMTileRows * kMRowStride;
constexpr int kMStage = kMScaleOff + kMTileRows * kMChunkG * 2;   // 2560 bytes per warp per stage
constexpr int kMMaxStages = 8;

struct MmaArgs {
    const uint4 *qw;            // [rows][G] 16-byte chunks
    const __half *scales;       // [rows][G]
    const __half *x;            // [M][K]
    void *out;                  // fp16 [M][N] or f32 [M][N]
    float *ws_val;              // Logits: per-CTA maximum [gridDim.x][M]
    int *ws_idx;
    int M, N, K, G;
    int stages;                 // ring depth S per warp (2..kMMaxStages)
    int wk;                     // warps splitting K (1, 2, 4, 8); WR = 8 / wk
    int max_tiles;              // tiles of the largest CTA range (sizes the WK > 1 buffer)
    int scales_async;           // 1: scales copied with cp.async; 0: read from global
};

// Per-CTA shared memory: rings, permuted activations (n-stride G*64 + 32
// bytes), C-operand table [G][NT][4 quad threads][c0 c1 c0 c1] f32 (= -7 X_g
// 2^-24 of columns 8nt + 2t, + 1), WK > 1 partials, LM-head maxima.
__host__ __device__ inline size_t mma_smem_bytes(int M, int G, int stages, int wk, int max_tiles, int NT)
{
    const size_t ring = (size_t)kMW * stages * kMStage;
    const size_t xp = (size_t)M * ((size_t)G * 64 + 32);
    const size_t x7 = (size_t)G * NT * 64;
    const size_t red = wk > 1 ? (size_t)max_tiles * wk * kMTileRows * 8 * NT * 4 : 0;
    const size_t best = (size_t)kMThreads * 2 * NT * 8;
    return ring + ((xp + 15) & ~(size_t)15) + x7 + red + best;
}

// Shared-memory loads by 32-bit shared-window address (keeps address math
// 32-bit and the loads explicit LDS).
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint4 lds_u128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ void cp_async16_u32(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                          float c0, float c1, float c2, float c3)
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c0), "f"(c1), "f"(c2), "f"(c3));
}

// Stage x in mma-B order: for column n and group g, 64 bytes = for t = 0..3:
// step 0 (x[8t], x[8t+4], x[8t+2], x[8t+6]), step 1 (x[8t+1], x[8t+5],
// x[8t+3], x[8t+7]) / 16 (k relative to 32g).  The C table holds, for each
// (g, n-tile, quad thread t), (c, c', c, c') with c = -7 X_g 2^-24 of column
// 8 nt + 2t and c' of the next column (zero for columns >= M).
__device__ __forceinline__ void stage_x_mma(const __half *__restrict__ x, unsigned char *xp, float *x7, int M,
                                            int K, int G, int NT)
{
    const int K8 = K >> 3;
    const size_t nstride = (size_t)G * 64 + 32;
    const __half2 sixteenth = __float2half2_rn(0.0625f);
    for (int i = threadIdx.x; i < G * NT * 16; i += kMThreads) x7[i] = 0.f;
    __syncthreads();
    for (int m = 0; m < M; ++m) {
        for (int base = 0; base < K8; base += kMThreads) {
            const int kk = base + threadIdx.x;      // (g = kk / 4, t = kk % 4)
            float part = 0.f;
            if (kk < K8) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(x + (size_t)m * K + 8 * kk);
                const uint32_t v01 = raw.x, v23 = raw.y, v45 = raw.z, v67 = raw.w;   // half pairs
                uint4 o;
                o.x = __byte_perm(v01, v45, 0x5410);   // (x0, x4)
                o.y = __byte_perm(v23, v67, 0x5410);   // (x2, x6)
                uint32_t h15 = __byte_perm(v01, v45, 0x7632);   // (x1, x5)
                uint32_t h37 = __byte_perm(v23, v67, 0x7632);   // (x3, x7)
                __half2 q15 = __hmul2(*reinterpret_cast<__half2 *>(&h15), sixteenth);
                __half2 q37 = __hmul2(*reinterpret_cast<__half2 *>(&h37), sixteenth);
                o.z = *reinterpret_cast<uint32_t *>(&q15);
                o.w = *reinterpret_cast<uint32_t *>(&q37);
                *reinterpret_cast<uint4 *>(xp + (size_t)m * nstride + (size_t)kk * 16) = o;
                const __half2 *h = reinterpret_cast<const __half2 *>(&raw);
                float v[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = __half22float2(h[j]);
                    v[2 * j] = f.x;
                    v[2 * j + 1] = f.y;
                }
                part = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
            }
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            if (kk < K8 && (kk & 3) == 0) {
                const float c = part * (-7.0f * pow2f(-24));
                const int g = kk >> 2, nt = m >> 3, t = (m & 7) >> 1, e = m & 1;
                float *cv = x7 + (((size_t)g * NT + nt) * 4 + t) * 4;
                cv[e] = c;
                cv[2 + e] = c;
            }
        }
    }
}

#ifndef ZT_MMA_MIN_CTAS
#define ZT_MMA_MIN_CTAS 2
#endif

template <int NT, int EPI>
__global__ void __launch_bounds__(kMThreads, ZT_MMA_MIN_CTAS) q4_mma_kernel(const MmaArgs a)
{
    constexpr int ROUT = (EPI == kEpiGateUp) ? kMTileRows / 2 : kMTileRows;   // outputs per tile
    extern __shared__ __align__(128) unsigned char smem[];
    const int M = a.M, N = a.N, G = a.G, S = a.stages, wk = a.wk;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int qg = lane >> 2, qt = lane & 3;       // mma quad row / thread in quad

    unsigned char *ring = smem + (size_t)warp * S * kMStage;
    unsigned char *xp = smem + (size_t)kMW * S * kMStage;
    const size_t nstride = (size_t)G * 64 + 32;
    float *x7 = reinterpret_cast<float *>(xp + (((size_t)M * nstride + 15) & ~(size_t)15));
    float *red = x7 + (size_t)G * NT * 16;
    const size_t red_floats = wk > 1 ? (size_t)a.max_tiles * wk * kMTileRows * 8 * NT : 0;
    float *bvs = red + red_floats;
    int *bis = reinterpret_cast<int *>(bvs + kMThreads * 2 * NT);

    pdl_launch_dependents();

    const int o_begin = (int)(((long long)N * blockIdx.x) / gridDim.x);
    const int o_end = (int)(((long long)N * (blockIdx.x + 1)) / gridDim.x);
    const int n_tiles = (o_end - o_begin + ROUT - 1) / ROUT;
    const int n_chunks = (G + kMChunkG - 1) / kMChunkG;
    const int wr_n = kMW / wk;
    const int my_wk = warp % wk, my_wr = warp / wk;
    const int my_tiles = my_wr < n_tiles ? (n_tiles - my_wr + wr_n - 1) / wr_n : 0;
    const int my_chunks = my_wk < n_chunks ? (n_chunks - my_wk + wk - 1) / wk : 0;
    const int n_items = my_tiles * my_chunks;
    const bool scales_async = a.scales_async != 0;

    // weight row of tile slot r (and whether it lies in this CTA's range)
    auto slot_row = [&](int o0, int r, bool &valid) -> int {
        if (EPI == kEpiGateUp) {
            const int o = o0 + (r & 7);
            valid = o < o_end;
            return (r < 8 ? 0 : N) + min(o, N - 1);
        }
        const int o = o0 + r;
        valid = o < o_end;
        return min(o, N - 1);
    };

    // ---------------------------------------------------------- issue side --
    // Lane l copies pieces p = l + 32 i (i < 4) of an item: tile row
    // r = l / 8 + 4 i, group l % 8 of the chunk.  Its source rows change per
    // tile only; per item just the chunk offset moves.
    const int pg = lane & 7;
    int is_tl = 0, is_cl = 0, is_stage = 0, is_left = n_items;
    const uint4 *src_w[4];
    bool ok_w[4];
    const __half *src_s = a.scales;
    bool ok_s = false;
    auto set_tile = [&](int tl) {
        const int o0 = o_begin + (my_wr + wr_n * tl) * ROUT;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int row = slot_row(o0, (lane >> 3) + 4 * i, ok_w[i]);
            src_w[i] = a.qw + (size_t)row * G + pg;
        }
        if (lane < kMTileRows) {
            const int row = slot_row(o0, lane, ok_s);
            src_s = a.scales + (size_t)row * G;
        }
    };
    if (n_items > 0) set_tile(0);
    const uint32_t ring_u = smem_u32(ring);
    const uint32_t piece_u = ring_u + (lane >> 3) * kMRowStride + pg * 16;   // + stage, + 4 i rows
    const uint32_t scale_u = ring_u + kMScaleOff + lane * 16;
    auto issue_next = [&]() {
        if (is_left > 0) {
            const int c = my_wk + wk * is_cl;
            const bool full = (c + 1) * kMChunkG <= G;
            const int kc = full ? kMChunkG : G - c * kMChunkG;
            const uint32_t so = (uint32_t)is_stage * kMStage;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (ok_w[i] && pg < kc) cp_async16_u32(piece_u + so + 4 * i * kMRowStride, src_w[i] + c * kMChunkG);
            if (scales_async && ok_s && lane < kMTileRows) cp_async16_u32(scale_u + so, src_s + c * kMChunkG);
            --is_left;
            if (++is_cl == my_chunks) {
                is_cl = 0;
                if (++is_tl < my_tiles) set_tile(is_tl);
            }
        }
        cp_async_commit();
        if (++is_stage == S) is_stage = 0;
    };

    for (int j = 0; j < S - 1; ++j) issue_next();

    pdl_wait();
    stage_x_mma(a.x, xp, x7, M, a.K, G, NT);
    __syncthreads();

    // Byte offsets from the start of shared memory; loads index the shared
    // array directly, so the compiler sees shared-space, 32-bit addressing.
    const uint32_t *smw = reinterpret_cast<const uint32_t *>(smem);
    const uint4 *smq = reinterpret_cast<const uint4 *>(smem);
    const uint32_t ring_o = (uint32_t)(ring - smem);
    uint32_t xb[NT];       // B-operand column of this lane (columns >= M read column M-1: ignored)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) xb[nt] = (uint32_t)(xp - smem) + (uint32_t)(min(qg + 8 * nt, M - 1) * nstride) + qt * 16;
    const uint32_t x7_o = (uint32_t)(reinterpret_cast<unsigned char *>(x7) - smem) + qt * 16;
    const uint32_t wq_o = ring_o + qg * kMRowStride + qt * 4;          // + stage + group
    const uint32_t sc_o = ring_o + kMScaleOff + qg * 16;

    float acc[NT][4];
    float best_v[2 * NT];
    int best_i[2 * NT];
#pragma unroll
    for (int i = 0; i < 2 * NT; ++i) {
        best_v[i] = -INFINITY;
        best_i[i] = 0x7fffffff;
    }
    int tl = 0, cl = 0, stage = 0;

    for (int j = 0; j < n_items; ++j) {
        cp_async_wait_dyn(S - 2);
        __syncwarp();
        const int t = my_wr + wr_n * tl;
        const int c = my_wk + wk * cl;
        const int o0 = o_begin + t * ROUT;
        const int kc = min(kMChunkG, G - c * kMChunkG);
        if (cl == 0) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
        }
        const uint32_t so = (uint32_t)stage * kMStage;
        // scales of rows qg and qg + 8 for the item's 8 groups
        uint4 sg, sg8;
        if (scales_async) {
            sg = smq[(sc_o + so) >> 4];
            sg8 = smq[(sc_o + so + 8 * 16) >> 4];
        } else {
            bool v0, v1;
            const int r0 = slot_row(o0, qg, v0), r1 = slot_row(o0, qg + 8, v1);
            uint32_t u0[4] = {0, 0, 0, 0}, u1[4] = {0, 0, 0, 0};
            const unsigned short *p0 = reinterpret_cast<const unsigned short *>(a.scales) + (size_t)r0 * G + c * kMChunkG;
            const unsigned short *p1 = reinterpret_cast<const unsigned short *>(a.scales) + (size_t)r1 * G + c * kMChunkG;
            for (int gl = 0; gl < kc; ++gl) {
                u0[gl >> 1] |= (uint32_t)p0[gl] << (16 * (gl & 1));
                u1[gl >> 1] |= (uint32_t)p1[gl] << (16 * (gl & 1));
            }
            sg = make_uint4(u0[0], u0[1], u0[2], u0[3]);
            sg8 = make_uint4(u1[0], u1[1], u1[2], u1[3]);
        }
        const uint32_t sgw[4] = {sg.x, sg.y, sg.z, sg.w}, sg8w[4] = {sg8.x, sg8.y, sg8.z, sg8.w};
        const uint32_t wrow0 = wq_o + so;
        const uint32_t xb0 = (uint32_t)(c * kMChunkG) * 64u;                   // + xb[nt] + gl * 64
        const uint32_t x70 = x7_o + (uint32_t)(c * kMChunkG) * (NT * 64u);    // + (gl * NT + nt) * 64
        auto step = [&](int gl) {
            const uint32_t w0 = smw[(wrow0 + gl * 16) >> 2];
            const uint32_t w1 = smw[(wrow0 + 8 * kMRowStride + gl * 16) >> 2];
            const uint32_t w0s = w0 >> 8, w1s = w1 >> 8;
            const uint32_t A0[4] = {w0 & 0x000F000Fu, w1 & 0x000F000Fu, w0s & 0x000F000Fu, w1s & 0x000F000Fu};
            const uint32_t A1[4] = {w0 & 0x00F000F0u, w1 & 0x00F000F0u, w0s & 0x00F000F0u, w1s & 0x00F000F0u};
            const __half2 sh0 = *reinterpret_cast<const __half2 *>(&sgw[gl >> 1]);
            const __half2 sh1 = *reinterpret_cast<const __half2 *>(&sg8w[gl >> 1]);
            const float s0 = (gl & 1) ? __high2float(sh0) : __low2float(sh0);
            const float s1 = (gl & 1) ? __high2float(sh1) : __low2float(sh1);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint4 bb = smq[(xb[nt] + xb0 + gl * 64) >> 4];
                const uint4 czu = smq[(x70 + (gl * NT + nt) * 64) >> 4];
                float d[4];
                mma_16816(d, A0, bb.x, bb.y, __uint_as_float(czu.x), __uint_as_float(czu.y), __uint_as_float(czu.z),
                          __uint_as_float(czu.w));
                mma_16816(d, A1, bb.z, bb.w, d[0], d[1], d[2], d[3]);
                acc[nt][0] = fmaf(d[0], s0, acc[nt][0]);
                acc[nt][1] = fmaf(d[1], s0, acc[nt][1]);
                acc[nt][2] = fmaf(d[2], s1, acc[nt][2]);
                acc[nt][3] = fmaf(d[3], s1, acc[nt][3]);
            }
        };
        if (kc == kMChunkG) {
#pragma unroll
            for (int gl = 0; gl < kMChunkG; ++gl) step(gl);
        } else {
#pragma unroll
            for (int gl = 0; gl < kMChunkG; ++gl)
                if (gl < kc) step(gl);
        }
        __syncwarp();
        issue_next();
        if (++stage == S) stage = 0;

        if (cl == my_chunks - 1) {
            if (wk > 1) {
                // this warp's partial of tile t: [16 rows][8*NT columns]
                float *rp = red + ((size_t)t * wk + my_wk) * kMTileRows * 8 * NT;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    rp[qg * 8 * NT + 8 * nt + 2 * qt] = acc[nt][0];
                    rp[qg * 8 * NT + 8 * nt + 2 * qt + 1] = acc[nt][1];
                    rp[(qg + 8) * 8 * NT + 8 * nt + 2 * qt] = acc[nt][2];
                    rp[(qg + 8) * 8 * NT + 8 * nt + 2 * qt + 1] = acc[nt][3];
                }
            } else {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int m = 8 * nt + 2 * qt + e;
                        if (m >= M) continue;
                        if (EPI == kEpiGateUp) {
                            const int n = o0 + qg;
                            if (n < o_end) {
                                const float g = acc[nt][e] * pow2f(24), u = acc[nt][2 + e] * pow2f(24);
                                const float silu = g / (1.0f + expf(-g));
                                reinterpret_cast<__half *>(a.out)[(size_t)m * N + n] = __float2half_rn(silu * u);
                            }
                        } else {
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const int n = o0 + qg + 8 * h;
                                if (n >= o_end) continue;
                                const float y = acc[nt][2 * h + e] * pow2f(24);
                                if (EPI == kEpiF16) {
                                    reinterpret_cast<__half *>(a.out)[(size_t)m * N + n] = __float2half_rn(y);
                                } else {
                                    reinterpret_cast<float *>(a.out)[(size_t)m * N + n] = y;
                                    if (better(y, n, best_v[2 * nt + e], best_i[2 * nt + e])) {
                                        best_v[2 * nt + e] = isnan(y) ? -INFINITY : y;
                                        best_i[2 * nt + e] = n;
                                    }
                                }
                            }
                        }
                    }
                }
            }
        }
        if (++cl == my_chunks) {
            cl = 0;
            ++tl;
        }
    }
    cp_async_wait<0>();

    if (wk > 1) {
        // WK partials of each tile meet here; fixed summation order
        __syncthreads();
        const int VO = ROUT * 8 * NT;                         // (output row, column) pairs per tile
        for (int idx = tid; idx < n_tiles * VO; idx += kMThreads) {
            const int t = idx / VO, vo = idx - (idx / VO) * VO;
            const int r = vo / (8 * NT), m = vo - (vo / (8 * NT)) * (8 * NT);
            const int n = o_begin + t * ROUT + r;
            if (n >= o_end || m >= M) continue;
            const float *rp = red + (size_t)t * wk * kMTileRows * 8 * NT;
            float y = 0.f, u = 0.f;
            for (int k2 = 0; k2 < wk; ++k2) {
                y += rp[(size_t)k2 * kMTileRows * 8 * NT + r * 8 * NT + m];
                if (EPI == kEpiGateUp) u += rp[(size_t)k2 * kMTileRows * 8 * NT + (r + 8) * 8 * NT + m];
            }
            y *= pow2f(24);
            if (EPI == kEpiF16) {
                reinterpret_cast<__half *>(a.out)[(size_t)m * N + n] = __float2half_rn(y);
            } else if (EPI == kEpiGateUp) {
                u *= pow2f(24);
                const float silu = y / (1.0f + expf(-y));
                reinterpret_cast<__half *>(a.out)[(size_t)m * N + n] = __float2half_rn(silu * u);
            } else {
                reinterpret_cast<float *>(a.out)[(size_t)m * N + n] = y;
                // thread tid handles m = idx % (8 NT) = tid % (8 NT): slot 0 of its table
                if (better(y, n, best_v[0], best_i[0])) {
                    best_v[0] = isnan(y) ? -INFINITY : y;
                    best_i[0] = n;
                }
            }
        }
    }

    if (EPI == kEpiLogits) {
#pragma unroll
        for (int i = 0; i < 2 * NT; ++i) {
            bvs[tid * 2 * NT + i] = best_v[i];
            bis[tid * 2 * NT + i] = best_i[i];
        }
        __syncthreads();
        if (tid < M) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
            for (int th = 0; th < kMThreads; ++th) {
                for (int i = 0; i < 2 * NT; ++i) {
                    int tm;
                    if (wk > 1) {
                        if (i != 0) continue;
                        tm = th % (8 * NT);
                    } else {
                        tm = 8 * (i >> 1) + 2 * (th & 3) + (i & 1);
                    }
                    if (tm == tid && better(bvs[th * 2 * NT + i], bis[th * 2 * NT + i], bv, bi)) {
                        bv = bvs[th * 2 * NT + i];
                        bi = bis[th * 2 * NT + i];
                    }
                }
            }
            a.ws_val[(size_t)blockIdx.x * M + tid] = bv;
            a.ws_idx[(size_t)blockIdx.x * M + tid] = bi;
        }
    }
}

}  // namespace zt
