// q4_mma.cuh -- building blocks of the sm_100a dequantizing GEMV for M <= 16
// (the kernel itself is q4_pass.cuh): codes unpacked two per logic instruction
// into fp16 subnormals, contracted on tensor cores with register-sourced
// mma.sync, fed from HBM by per-warp cp.async rings.
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
//   * Each CTA owns a contiguous, balanced range of outputs; its 16 (or 8)
//     warps form WR x WK (WK warps split a tile's chunks when the CTA has few
//     rows).
//   * Every warp streams its items through a private ring of S stages with
//     16-byte cp.async copies (hardware waits, no spin loops).  Rows outside
//     the CTA's range are never copied: a partial tile costs math, not bytes.
//   * Programmatic dependent launch: the first S - 1 items are issued before
//     griddepcontrol.wait, so weights stream while the previous kernel on the
//     stream finishes; activations are read and outputs written after it.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "q4_common.cuh"

namespace zt {

// Math warps per CTA: 16 (one CTA per SM) or 8 (one or two CTAs per SM), a
// launch-plan choice.  The staging helpers below take the CTA's size from
// blockDim; kMWMax sizes per-warp tables.
constexpr int kMWMax = 16;

// Barrier among all threads of the CTA as named barrier 1 (the same as
// __syncthreads(), kept apart from barrier 0).
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"r"(blockDim.x) : "memory"); }
constexpr int kMTileRows = 16;                      // weight rows per warp tile (mma M)
constexpr int kMChunkG = 8;                         // groups per item
// A ring stage holds an item: codes [16 rows][128 B] with the 128-byte XOR
// swizzle (16-byte chunk j of row r at r * 128 + (j ^ (r & 7)) * 16 -- the
// layout a TMA box with 128-byte swizzling writes; the 8 quad rows of an mma
// then read 8 distinct bank groups), and, in a separate region, the tile's
// scales [16 rows][16 B].
constexpr int kMCodeStage = kMTileRows * kMChunkG * 16;   // 2048 bytes
constexpr int kMScaleStage = kMTileRows * kMChunkG * 2;   // 256 bytes
constexpr int kMStage = kMCodeStage + kMScaleStage;       // 2304 bytes per warp per stage
constexpr int kMMaxStages = 8;

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
__device__ __forceinline__ void cp_async8_u32(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4_u32(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
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

// Single-column (M = 1) staging for the block-diagonal contraction of
// q4_pass.cuh.  A lane's mma B operand is a register pair (b0, b1) of which at
// most one is non-zero: b0 for a lane whose column is an even group of its
// pair of groups, b1 for an odd one, neither for the other lanes.  So that one
// 16-byte load gives two such pairs ready for two mma steps, each word w_s of
// a group (mma step s) is staged next to a zero: groups 2p and 2p + 1 form a
// 288-byte block, the even group as [w_0, 0, w_1, 0, ...] (128 bytes), 16
// bytes apart, the odd one as [0, w_0, 0, w_1, ...].  The area starts with a
// 224-byte zero region (the other lanes read 128 bytes of it, at 32 bytes per
// quarter-warp); with these offsets the three addresses a quarter-warp reads
// fall in distinct 16-byte bank groups.  Groups are padded with zeros to a
// multiple of 8 (one item).
// That paired layout serves the 16-warp CTAs of a pass.  The CTAs of single calls (8
// warps, several per SM, where the staging is a larger share of the call) use the plain
// one: a 64-byte zero block, then group g's four 16-byte pieces at 64 + 80 g (80, not
// 64: the lanes reading groups 2t and 2t + 1 then hit distinct banks), and one C float
// per group; their b0 and b1 come from two loads.
constexpr int kBdZero = 224;
constexpr int kBdPair = 288;
constexpr int kBdGroup = kBdPair / 2;   // bytes per group, for sizes and chunk steps
constexpr int kBd1Zero = 64;
constexpr int kBd1Group = 80;
__host__ __device__ constexpr uint32_t bd_slot(int kk)   // the 32 bytes of piece kk (4 words, 4 zeros)
{
    return kBdZero + (kk >> 3) * kBdPair + ((kk >> 2) & 1) * (kBdPair / 2) + (kk & 3) * 32;
}
__host__ __device__ constexpr uint32_t bd1_piece(int kk) { return kBd1Zero + (kk >> 2) * kBd1Group + (kk & 3) * 16; }
// bytes of the single-column area and of its C table for g_stage groups
__host__ __device__ constexpr size_t bd_area_bytes(int g8, bool paired)
{
    return paired ? (size_t)kBdZero + (size_t)g8 * kBdGroup : (size_t)kBd1Zero + (size_t)g8 * kBd1Group;
}
__host__ __device__ constexpr size_t bd_ctable_bytes(int g8, bool paired) { return (size_t)g8 * (paired ? 8 : 4); }
__host__ __device__ constexpr int round8(int g) { return (g + 7) & ~7; }
// The single-column C table.  Paired layout: per pair of groups (2p, 2p + 1) four floats (c_2p, c_2p+1,
// c_2p, c_2p+1), the C operand quad of the lanes that hold that pair, in one 16-byte load.  Plain layout:
// one float per group.
__device__ __forceinline__ void bd_c(float *x7, int g, float c, bool paired)
{
    if (paired) {
        x7[(g >> 1) * 4 + (g & 1)] = c;
        x7[(g >> 1) * 4 + (g & 1) + 2] = c;
    } else {
        x7[g] = c;
    }
}

// the four words o of piece kk, each beside a zero (after it in an even group, before it in an odd one)
__device__ __forceinline__ void bd_store(unsigned char *xp, int kk, uint4 o, bool paired)
{
    if (!paired) {
        *reinterpret_cast<uint4 *>(xp + bd1_piece(kk)) = o;
        return;
    }
    uint4 *d = reinterpret_cast<uint4 *>(xp + bd_slot(kk));
    if ((kk >> 2) & 1) {
        d[0] = make_uint4(0u, o.x, 0u, o.y);
        d[1] = make_uint4(0u, o.z, 0u, o.w);
    } else {
        d[0] = make_uint4(o.x, 0u, o.y, 0u);
        d[1] = make_uint4(o.z, 0u, o.w, 0u);
    }
}

// zero x and C of groups [Gw, round8(Gw)) in the single-column layout
__device__ __forceinline__ void bd_pad(unsigned char *xp, float *x7, int Gw, bool paired)
{
    for (int j = threadIdx.x; j < (round8(Gw) - Gw) * 4; j += (int)blockDim.x) {
        bd_store(xp, Gw * 4 + j, make_uint4(0, 0, 0, 0), paired);
        if ((j & 3) == 0) bd_c(x7, Gw + (j >> 2), 0.f, paired);
    }
}

// Byte offset of piece kk (8 activations) of column m in the staged area; with a
// single column (compact) the first 16 bytes of the piece's slot, where the norm
// prologue keeps h until the same thread turns it into x.
__device__ __forceinline__ size_t x_piece(int m, int kk, size_t nstride, bool compact, bool paired)
{
    return compact ? (size_t)(paired ? bd_slot(kk) : bd1_piece(kk)) : (size_t)m * nstride + (size_t)kk * 16;
}

// Stage x in mma-B order: for column n and group g, 64 bytes = for t = 0..3:
// step 0 (x[8t], x[8t+4], x[8t+2], x[8t+6]), step 1 (x[8t+1], x[8t+5],
// x[8t+3], x[8t+7]) / 16 (k relative to 32g).  The C table holds, for each
// (g, n-tile, quad thread t), (c, c', c, c') with c = -7 X_g 2^-24 of column
// 8 nt + 2t and c' of the next column (zero for columns >= M).  With a single
// column (compact) the layout is the block-diagonal one above and the table
// holds c per group.  Thread i of
// the CTA takes 8 activations of one column per round; the 4 threads of a
// group are adjacent lanes.  Callers synchronise before reading.
__device__ __forceinline__ void stage_x_one(const uint4 raw, int m, int kk, bool valid, unsigned char *xp,
                                            float *x7, size_t nstride, int NT, bool compact, bool paired)
{
    const __half2 sixteenth = __float2half2_rn(0.0625f);
    float part = 0.f;
    if (valid) {
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
        if (compact) bd_store(xp, kk, o, paired);
        else *reinterpret_cast<uint4 *>(xp + x_piece(m, kk, nstride, false, false)) = o;
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
    if (valid && (kk & 3) == 0) {
        const float c = part * (-7.0f * pow2f(-24));
        if (compact) {
            bd_c(x7, kk >> 2, c, paired);
        } else {
            const int g = kk >> 2, nt = m >> 3, t = (m & 7) >> 1, e = m & 1;
            float *cv = x7 + (((size_t)g * NT + nt) * 4 + t) * 4;
            cv[e] = c;
            cv[2 + e] = c;
        }
    }
}

// x: the first of the Gw groups to stage in row 0; row m starts ldx halves
// further.  Gs: groups per staged column (the n-stride is Gs * 64 + 32 bytes);
// the whole K is Gw = Gs = K / 32, a K window fewer groups.
__device__ __forceinline__ void stage_x_mma(const __half *__restrict__ x, int ldx, unsigned char *xp, float *x7,
                                            int M, int Gw, int Gs, int NT, bool paired = false)
{
    const int K8 = Gw * 4;                     // 8-element pieces per row: groups never straddle a column
    const int total = M * K8;
    const size_t nstride = (size_t)Gs * 64 + 32;
    // C entries of the padding columns M .. 8 NT - 1 are zero
    const bool compact = M == 1;
    const int pad = compact ? 0 : 8 * NT - M;
    for (int j = threadIdx.x; j < Gw * pad; j += (int)blockDim.x) {
        const int g = j / pad, m = M + (j - (j / pad) * pad);
        const int nt = m >> 3, t = (m & 7) >> 1, e = m & 1;
        float *cv = x7 + (((size_t)g * NT + nt) * 4 + t) * 4;
        cv[e] = 0.f;
        cv[2 + e] = 0.f;
    }
    // two rounds per iteration: both loads in flight before either is used.
    // L2-coherent loads: x may be an output of an earlier phase of the same launch.
    for (int base = 0; base < total; base += 2 * (int)blockDim.x) {
        const int i0 = base + threadIdx.x, i1 = i0 + (int)blockDim.x;
        const bool v0 = i0 < total, v1 = i1 < total;
        const int m0 = v0 ? i0 / K8 : 0, m1 = v1 ? i1 / K8 : 0;
        const int k0 = i0 - m0 * K8, k1 = i1 - m1 * K8;
        uint4 r0 = make_uint4(0, 0, 0, 0), r1 = make_uint4(0, 0, 0, 0);
        if (v0) r0 = __ldcg(reinterpret_cast<const uint4 *>(x + (size_t)m0 * ldx + 8 * k0));
        if (v1) r1 = __ldcg(reinterpret_cast<const uint4 *>(x + (size_t)m1 * ldx + 8 * k1));
        stage_x_one(r0, m0, k0, v0, xp, x7, nstride, NT, compact, paired);
        if (base + (int)blockDim.x < total) stage_x_one(r1, m1, k1, v1, xp, x7, nstride, NT, compact, paired);
    }
    if (compact) bd_pad(xp, x7, Gw, paired);
}

// Residual add + RMSNorm ahead of a projection (the pages' add_norm step:
// residual connection and RMSNorm in one kernel), staged like stage_x_mma:
//   h = fp16(res + dlt) (dlt may be null), r = 1 / sqrt(sum_k h^2 / K + eps)
//   per row, x = fp16(h * r * gamma).
// Pass 1 writes h into the activation area (plain order) and sums squares
// (fp32, fixed order: per-thread strided sums, warp butterfly, warps in
// order); pass 2 turns each thread's own 16 bytes of h into x in the mma-B
// order.  res_out / x_out (plain [M][K] fp16) are written when non-null.
// scratch: kMWMax + M floats of shared memory.  All threads of the CTA call it.
__device__ __forceinline__ uint32_t hadd2_u32(uint32_t a, uint32_t b)
{
    __half2 r = __hadd2(*reinterpret_cast<const __half2 *>(&a), *reinterpret_cast<const __half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ void stage_x_norm(const __half *res, const __half *dlt, const __half *gamma, float eps,
                                             __half *res_out, __half *x_out, unsigned char *xp, float *x7,
                                             float *scratch, int M, int K, int G, int NT, bool paired = false)
{
    const int K8 = K >> 3;
    const size_t nstride = (size_t)G * 64 + 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int m = 0; m < M; ++m) {
        float part = 0.f;
        for (int kk = threadIdx.x; kk < K8; kk += (int)blockDim.x) {
            uint4 h = __ldcg(reinterpret_cast<const uint4 *>(res + (size_t)m * K + 8 * kk));
            if (dlt) {
                const uint4 d = __ldcg(reinterpret_cast<const uint4 *>(dlt + (size_t)m * K + 8 * kk));
                h.x = hadd2_u32(h.x, d.x);
                h.y = hadd2_u32(h.y, d.y);
                h.z = hadd2_u32(h.z, d.z);
                h.w = hadd2_u32(h.w, d.w);
            }
            *reinterpret_cast<uint4 *>(xp + x_piece(m, kk, nstride, M == 1, paired)) = h;
            if (res_out) *reinterpret_cast<uint4 *>(res_out + (size_t)m * K + 8 * kk) = h;
            const __half2 *hh = reinterpret_cast<const __half2 *>(&h);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __half22float2(hh[j]);
                part = fmaf(f.x, f.x, part);
                part = fmaf(f.y, f.y, part);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) scratch[warp] = part;
        consumer_sync();
        if (threadIdx.x == 0) {
            float ss = 0.f;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) ss += scratch[w];
            scratch[kMWMax + m] = 1.0f / sqrtf(ss / (float)K + eps);
        }
        consumer_sync();
    }
    const int total = M * K8;
    const bool compact = M == 1;
    const int pad = compact ? 0 : 8 * NT - M;
    for (int j = threadIdx.x; j < G * pad; j += (int)blockDim.x) {
        const int g = j / pad, m = M + (j - (j / pad) * pad);
        const int nt = m >> 3, t = (m & 7) >> 1, e = m & 1;
        float *cv = x7 + (((size_t)g * NT + nt) * 4 + t) * 4;
        cv[e] = 0.f;
        cv[2 + e] = 0.f;
    }
    auto normalise = [&](int m, int kk) {
        const uint4 h = *reinterpret_cast<const uint4 *>(xp + x_piece(m, kk, nstride, compact, paired));
        const uint4 g = __ldcg(reinterpret_cast<const uint4 *>(gamma + 8 * kk));
        const float r = scratch[kMWMax + m];
        const __half2 *hh = reinterpret_cast<const __half2 *>(&h);
        const __half2 *gg = reinterpret_cast<const __half2 *>(&g);
        uint4 x;
        __half2 *xx = reinterpret_cast<__half2 *>(&x);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 hf = __half22float2(hh[j]), gf = __half22float2(gg[j]);
            xx[j] = __floats2half2_rn(hf.x * r * gf.x, hf.y * r * gf.y);
        }
        if (x_out) *reinterpret_cast<uint4 *>(x_out + (size_t)m * K + 8 * kk) = x;
        return x;
    };
    for (int base = 0; base < total; base += 2 * (int)blockDim.x) {
        const int i0 = base + threadIdx.x, i1 = i0 + (int)blockDim.x;
        const bool v0 = i0 < total, v1 = i1 < total;
        const int m0 = v0 ? i0 / K8 : 0, m1 = v1 ? i1 / K8 : 0;
        const int k0 = i0 - m0 * K8, k1 = i1 - m1 * K8;
        uint4 r0 = make_uint4(0, 0, 0, 0), r1 = make_uint4(0, 0, 0, 0);
        if (v0) r0 = normalise(m0, k0);
        if (v1) r1 = normalise(m1, k1);
        stage_x_one(r0, m0, k0, v0, xp, x7, nstride, NT, compact, paired);
        if (base + (int)blockDim.x < total) stage_x_one(r1, m1, k1, v1, xp, x7, nstride, NT, compact, paired);
    }
    if (compact) bd_pad(xp, x7, G, paired);
}

// The same prologue for a projection whose activations are staged in K
// windows (they do not fit in shared memory whole).  norm_rows takes the sums
// of squares over all of K once per segment, in exactly stage_x_norm's order
// (so r is bit-identical), writes h to res_out when non-null and r[m] to rn;
// stage_x_norm_window then stages groups [g0, g0 + Gw) of x = fp16(h r gamma),
// recomputing h = fp16(res + dlt) for just those k.  scratch: kMWMax floats.
__device__ __forceinline__ void norm_rows(const __half *res, const __half *dlt, float eps, __half *res_out,
                                          float *rn, float *scratch, int M, int K)
{
    const int K8 = K >> 3;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int m = 0; m < M; ++m) {
        float part = 0.f;
        for (int kk = threadIdx.x; kk < K8; kk += (int)blockDim.x) {
            uint4 h = __ldcg(reinterpret_cast<const uint4 *>(res + (size_t)m * K + 8 * kk));
            if (dlt) {
                const uint4 d = __ldcg(reinterpret_cast<const uint4 *>(dlt + (size_t)m * K + 8 * kk));
                h.x = hadd2_u32(h.x, d.x);
                h.y = hadd2_u32(h.y, d.y);
                h.z = hadd2_u32(h.z, d.z);
                h.w = hadd2_u32(h.w, d.w);
            }
            if (res_out) *reinterpret_cast<uint4 *>(res_out + (size_t)m * K + 8 * kk) = h;
            const __half2 *hh = reinterpret_cast<const __half2 *>(&h);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __half22float2(hh[j]);
                part = fmaf(f.x, f.x, part);
                part = fmaf(f.y, f.y, part);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) scratch[warp] = part;
        consumer_sync();
        if (threadIdx.x == 0) {
            float ss = 0.f;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) ss += scratch[w];
            rn[m] = 1.0f / sqrtf(ss / (float)K + eps);
        }
        consumer_sync();
    }
}

__device__ __forceinline__ void stage_x_norm_window(const __half *res, const __half *dlt, const __half *gamma,
                                                    __half *x_out, const float *rn, unsigned char *xp, float *x7,
                                                    int M, int K, int g0, int Gw, int Gs, int NT,
                                                    bool paired = false)
{
    const int K8 = Gw * 4, k8_0 = g0 * 4;
    const int total = M * K8;
    const size_t nstride = (size_t)Gs * 64 + 32;
    const bool compact = M == 1;
    const int pad = compact ? 0 : 8 * NT - M;
    for (int j = threadIdx.x; j < Gw * pad; j += (int)blockDim.x) {
        const int g = j / pad, m = M + (j - (j / pad) * pad);
        const int nt = m >> 3, t = (m & 7) >> 1, e = m & 1;
        float *cv = x7 + (((size_t)g * NT + nt) * 4 + t) * 4;
        cv[e] = 0.f;
        cv[2 + e] = 0.f;
    }
    auto normalise = [&](int m, int kk) {
        const size_t off = (size_t)m * K + 8 * (size_t)(k8_0 + kk);
        uint4 h = __ldcg(reinterpret_cast<const uint4 *>(res + off));
        if (dlt) {
            const uint4 d = __ldcg(reinterpret_cast<const uint4 *>(dlt + off));
            h.x = hadd2_u32(h.x, d.x);
            h.y = hadd2_u32(h.y, d.y);
            h.z = hadd2_u32(h.z, d.z);
            h.w = hadd2_u32(h.w, d.w);
        }
        const uint4 g = __ldcg(reinterpret_cast<const uint4 *>(gamma + 8 * (size_t)(k8_0 + kk)));
        const float r = rn[m];
        const __half2 *hh = reinterpret_cast<const __half2 *>(&h);
        const __half2 *gg = reinterpret_cast<const __half2 *>(&g);
        uint4 x;
        __half2 *xx = reinterpret_cast<__half2 *>(&x);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 hf = __half22float2(hh[j]), gf = __half22float2(gg[j]);
            xx[j] = __floats2half2_rn(hf.x * r * gf.x, hf.y * r * gf.y);
        }
        if (x_out) *reinterpret_cast<uint4 *>(x_out + off) = x;
        return x;
    };
    for (int base = 0; base < total; base += 2 * (int)blockDim.x) {
        const int i0 = base + threadIdx.x, i1 = i0 + (int)blockDim.x;
        const bool v0 = i0 < total, v1 = i1 < total;
        const int m0 = v0 ? i0 / K8 : 0, m1 = v1 ? i1 / K8 : 0;
        const int k0 = i0 - m0 * K8, k1 = i1 - m1 * K8;
        uint4 r0 = make_uint4(0, 0, 0, 0), r1 = make_uint4(0, 0, 0, 0);
        if (v0) r0 = normalise(m0, k0);
        if (v1) r1 = normalise(m1, k1);
        stage_x_one(r0, m0, k0, v0, xp, x7, nstride, NT, compact, paired);
        if (base + (int)blockDim.x < total) stage_x_one(r1, m1, k1, v1, xp, x7, nstride, NT, compact, paired);
    }
    if (compact) bd_pad(xp, x7, Gw, paired);
}

}  // namespace zt
