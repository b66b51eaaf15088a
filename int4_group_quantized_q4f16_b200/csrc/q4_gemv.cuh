// q4_gemv.cuh -- sm_100a kernels for the q4f16 dequantizing matrix-vector
// product (int4 codes, fp16 group-32 scales, fp16 activations, fp32 accumulate).
//
// Operation: the int4 dequantizing matrix product of the Zero-TVM write-up
// (section "完整的推理流水线": baseline / subgroup-reduce / rows x4, rows x8
// variants and the f32 LM-head variant) and its fused FFN (section "内核融合").
// One templated kernel covers all of them; the epilogue differs.
//
// Work decomposition (CUDA cores; the path is HBM-bound at M = 1):
//   * A CTA is WK x WR warps.  The WK warps split K: warp kw, lane l owns the
//     groups g = 32*kw + l, + 32*WK, ...  A group is exactly one 16-byte chunk
//     of packed codes, so a warp reads 512 contiguous bytes per row: fully
//     coalesced 128-bit loads straight from HBM.
//   * Each warp computes R weight rows at once, so every activation value it
//     fetches from shared memory is reused R times (the pages' rows x4 / x8
//     tiling).
//   * Lane partials are combined with a transposing warp-shuffle butterfly
//     (the pages' subgroup reduction) and the WK warps through shared memory,
//     in a fixed order: results are deterministic.
//   * The grid is persistent (SM count x resident CTAs); CTAs stride over
//     row tiles.
//
// Arithmetic (exact products, no conversion instructions):
//   For a binary32 bit pattern below 2^24 the value is exactly
//   pattern * 2^-149 (subnormals, and exponent field 1, are linear in the bit
//   pattern -- IEEE 754 binary32 encoding).  So masking a 4-bit code in place,
//   (word & (0xF << 4p)), and reinterpreting the bits as a float gives exactly
//   q * 2^(4p) * 2^-149 with one logic instruction.  The activation is
//   pre-scaled once per CTA to x * 2^(90 - 4p), so every product equals
//   q * x * 2^-59 exactly (4-bit times 11-bit significands fit in 24 bits) and
//   stays a normal number for every finite fp16 x.  Codes 6 and 7 of a word sit
//   above bit 23 and are taken from (word >> 12) at p = 3, 4.  The zero point
//   is applied per group with the identity
//       sum_k (q_k - 7) x_k = sum_k q_k x_k - 7 * X_g,   X_g = sum_{k in g} x_k,
//   X_g being computed once per CTA.  Products pair up into packed
//   fma.rn.f32x2 (sm_100).  The group sum is scaled by s in fp32, and the final
//   2^59 is an exact power-of-two multiply.  Denormals must not be flushed:
//   this file is compiled without -ftz / --use_fast_math.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace zt {

constexpr int kGroup = 32;                 // k values per scale
constexpr int kMaxWarps = 8;               // per CTA
constexpr int kThreadsMax = kMaxWarps * 32;
constexpr int kMaxCtas = 4096;             // grid cap (sizes the LM-head workspace)

enum EpiKind : int { kEpiF16 = 0, kEpiGateUp = 1, kEpiLogits = 2 };

struct Q4Args {
    const uint4 *qw;        // [rows][G]: one 16-byte chunk = the 32 codes of one group
    const __half *scales;   // [rows][G]
    const __half *x;        // [M][K]
    void *out;              // fp16 [M][N] (F16, GateUp) or f32 [M][N] (Logits)
    float *ws_val;          // Logits: per-CTA maximum   [gridDim.x][M]
    int *ws_idx;            // Logits: per-CTA arg-max   [gridDim.x][M]
    int M, N, K, G;         // N = output features; G = K / 32
    int wk, wr;             // warps along K, warps along rows (wk * wr <= 8)
    int n_tiles;            // row tiles of wr * (outputs per warp) outputs
};

// exponent (of 2) applied to x for the code at position j = k % 8 of its word
__host__ __device__ constexpr int xscale_exp(int j) { return j <= 5 ? 90 - 4 * j : 90 - 4 * (j - 3); }

__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// 128-bit streaming load: weights are read exactly once, keep them out of L1.
__device__ __forceinline__ uint4 ldg_stream(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float bits_f(uint32_t u) { return __uint_as_float(u); }

// sum over the 8 codes of one word of q_j * x''_j (scaled by 2^-59), into acc
__device__ __forceinline__ float2 word_dot(uint32_t w, const float4 &xa, const float4 &xb, float2 acc)
{
    const uint32_t h = w >> 12;
    acc = __ffma2_rn(make_float2(bits_f(w & 0xFu), bits_f(w & 0xF0u)), make_float2(xa.x, xa.y), acc);
    acc = __ffma2_rn(make_float2(bits_f(w & 0xF00u), bits_f(w & 0xF000u)), make_float2(xa.z, xa.w), acc);
    acc = __ffma2_rn(make_float2(bits_f(w & 0xF0000u), bits_f(w & 0xF00000u)), make_float2(xb.x, xb.y), acc);
    acc = __ffma2_rn(make_float2(bits_f(h & 0xF000u), bits_f(h & 0xF0000u)), make_float2(xb.z, xb.w), acc);
    return acc;
}

// Transposing butterfly over the 32 lanes of a warp: on return every lane holds
// in v[0] the warp-wide sum of value number `vid` (a function of the lane id).
template <int V>
__device__ __forceinline__ void warp_transpose_reduce(float (&v)[V], int lane, int &vid)
{
    vid = 0;
#pragma unroll
    for (int s = 0; s < 5; ++s) {
        const int o = 16 >> s;
        const int half = V >> (s + 1);
        if (half >= 1) {
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < (half >= 1 ? half : 1); ++i) {
                const float send = up ? v[i] : v[i + half];
                const float keep = up ? v[i + half] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
            if (up) vid += half;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
        }
    }
}

// greater value wins; equal values -> lower index; NaN counts as -inf
__device__ __forceinline__ bool better(float v, int i, float bv, int bi)
{
    v = isnan(v) ? -INFINITY : v;
    bv = isnan(bv) ? -INFINITY : bv;
    return v > bv || (v == bv && i < bi);
}

// Dynamic shared memory layout (bytes):
//   xs   float [M][G][32]  pre-scaled activations, float4 slots XOR-swizzled by g&7
//   xg   float [M][G]      7 * X_g * 2^-59
//   red  float [wr][wk][V] per-warp partial sums
//   bv   float [256], bi int [256]   (Logits: per-thread running maxima)
__host__ __device__ inline size_t q4_smem_bytes(int M, int G, int wk, int wr, int V)
{
    return (size_t)M * G * 32 * 4 + (size_t)M * G * 4 + (size_t)wr * wk * V * 4 +
           (size_t)kThreadsMax * 8;
}

template <int R, int MT, int EPI>
__global__ void __launch_bounds__(kThreadsMax) q4_gemv_kernel(const Q4Args a)
{
    constexpr int V = R * MT;                                // partial sums per lane
    constexpr int ROUT = (EPI == kEpiGateUp) ? R / 2 : R;    // outputs per warp
    static_assert(V <= 32 && (V & (V - 1)) == 0, "R*MT must be a power of two <= 32");
    static_assert(EPI != kEpiGateUp || (R % 2 == 0), "gate/up needs an even row count");

    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int M = a.M, K = a.K, G = a.G, N = a.N, wk = a.wk, wr = a.wr;
    float *xs = reinterpret_cast<float *>(smem_raw);
    float *xg = xs + (size_t)M * G * 32;
    float *red = xg + (size_t)M * G;
    float *bvs = red + wr * wk * V;
    int *bis = reinterpret_cast<int *>(bvs + kThreadsMax);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int kw = warp % wk;
    const int wri = warp / wk;
    const int nthreads = blockDim.x;

    // ---- stage pre-scaled activations once per CTA ----
    for (int idx = tid; idx < M * K; idx += nthreads) {
        const int m = idx / K, k = idx - m * K;
        const int g = k >> 5, c = (k & 31) >> 2, e = k & 3;
        const float v = __half2float(a.x[idx]) * pow2f(xscale_exp(k & 7));
        xs[(((size_t)m * G + g) * 8 + (c ^ (g & 7))) * 4 + e] = v;
    }
    for (int idx = tid; idx < M * G; idx += nthreads) {
        const __half *xp = a.x + (size_t)idx * kGroup;   // (m, g) -> x[m][32g ...]
        float s = 0.f;
#pragma unroll 8
        for (int j = 0; j < kGroup; ++j) s += __half2float(xp[j]);
        xg[idx] = s * (7.0f * pow2f(-59));
    }
    __syncthreads();

    float best_v = -INFINITY;
    int best_i = 0x7fffffff;
    const int rows_per_tile = wr * ROUT;
    const int n_out = wr * V / (EPI == kEpiGateUp ? 2 : 1);   // outputs per tile (incl. m)

    for (int tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x) {
        const int obase = tile * rows_per_tile + wri * ROUT;   // first output row of this warp

        // weight rows of this warp (clamped: rows past N are loaded but never stored)
        int wrow[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            if (EPI == kEpiGateUp) {
                const int o = min(obase + (r % ROUT), N - 1);
                wrow[r] = (r < ROUT) ? o : N + o;
            } else {
                wrow[r] = min(obase + r, N - 1);
            }
        }

        float part[V];
#pragma unroll
        for (int i = 0; i < V; ++i) part[i] = 0.f;

        for (int g = kw * 32 + lane; g < G; g += wk * 32) {
            uint4 w[R];
            float s[R];
#pragma unroll
            for (int r = 0; r < R; ++r) w[r] = ldg_stream(a.qw + (size_t)wrow[r] * G + g);
#pragma unroll
            for (int r = 0; r < R; ++r) s[r] = __half2float(a.scales[(size_t)wrow[r] * G + g]);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < M) {
                    const float4 *xv4 = reinterpret_cast<const float4 *>(xs + ((size_t)m * G + g) * 32);
                    const int sw = g & 7;
                    float4 xv[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) xv[c] = xv4[c ^ sw];
                    const float xgm = xg[m * G + g];
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        float2 acc = make_float2(0.f, 0.f);
                        acc = word_dot(w[r].x, xv[0], xv[1], acc);
                        acc = word_dot(w[r].y, xv[2], xv[3], acc);
                        acc = word_dot(w[r].z, xv[4], xv[5], acc);
                        acc = word_dot(w[r].w, xv[6], xv[7], acc);
                        part[r * MT + m] = fmaf(s[r], (acc.x + acc.y) - xgm, part[r * MT + m]);
                    }
                }
            }
        }

        int vid;
        warp_transpose_reduce<V>(part, lane, vid);
        if ((lane & (32 / V - 1)) == 0) red[(wri * wk + kw) * V + vid] = part[0];
        __syncthreads();

        if (tid < n_out) {
            // output (wri_o, r, m) of this tile
            constexpr int VO = ROUT * MT;
            const int wri_o = tid / VO, vo = tid - wri_o * VO;
            const int r = vo / MT, m = vo - r * MT;
            const int n = tile * rows_per_tile + wri_o * ROUT + r;
            const float *rp = red + wri_o * wk * V;
            float t0 = 0.f, t1 = 0.f;
            for (int k2 = 0; k2 < wk; ++k2) {
                t0 += rp[k2 * V + r * MT + m];
                if (EPI == kEpiGateUp) t1 += rp[k2 * V + (r + ROUT) * MT + m];
            }
            if (n < N && m < M) {
                const float y = t0 * pow2f(59);
                if (EPI == kEpiF16) {
                    reinterpret_cast<__half *>(a.out)[(size_t)m * N + n] = __float2half_rn(y);
                } else if (EPI == kEpiGateUp) {
                    const float u = t1 * pow2f(59);
                    const float silu = y / (1.0f + expf(-y));
                    reinterpret_cast<__half *>(a.out)[(size_t)m * N + n] = __float2half_rn(silu * u);
                } else {
                    reinterpret_cast<float *>(a.out)[(size_t)m * N + n] = y;
                    if (better(y, n, best_v, best_i)) { best_v = isnan(y) ? -INFINITY : y; best_i = n; }
                }
            }
        }
        __syncthreads();   // red[] is reused by the next tile
    }

    if (EPI == kEpiLogits) {
        // per-CTA maximum for each m; thread t always handled m = t % MT
        bvs[tid] = best_v;
        bis[tid] = best_i;
        __syncthreads();
        if (tid < M) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
            const int lim = min(n_out, nthreads);
            for (int t = tid; t < lim; t += MT)
                if (better(bvs[t], bis[t], bv, bi)) { bv = bvs[t]; bi = bis[t]; }
            a.ws_val[(size_t)blockIdx.x * M + tid] = bv;
            a.ws_idx[(size_t)blockIdx.x * M + tid] = bi;
        }
    }
}

// Second pass of the LM head: reduce the per-CTA maxima to one index per row
// of x.  One CTA per m; a total order (value, then lower index), so the result
// does not depend on the reduction order.
__global__ void __launch_bounds__(256) q4_argmax_reduce_kernel(const float *ws_val, const int *ws_idx,
                                                               int n_cta, int M, int32_t *argmax)
{
    __shared__ float sv[256];
    __shared__ int si[256];
    const int m = blockIdx.x;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int c = threadIdx.x; c < n_cta; c += blockDim.x) {
        const float v = ws_val[(size_t)c * M + m];
        const int i = ws_idx[(size_t)c * M + m];
        if (better(v, i, bv, bi)) { bv = isnan(v) ? -INFINITY : v; bi = i; }
    }
    sv[threadIdx.x] = bv;
    si[threadIdx.x] = bi;
    __syncthreads();
    for (int s = blockDim.x / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) {
            if (better(sv[threadIdx.x + s], si[threadIdx.x + s], sv[threadIdx.x], si[threadIdx.x])) {
                sv[threadIdx.x] = sv[threadIdx.x + s];
                si[threadIdx.x] = si[threadIdx.x + s];
            }
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) argmax[m] = (si[0] == 0x7fffffff) ? 0 : si[0];
}

}  // namespace zt
