// q4_gemv.cuh -- sm_100a kernels for the q4f16 dequantizing matrix-vector
// product (int4 codes, fp16 group-32 scales, fp16 activations, fp32 accumulate).
//
// Operation: the int4 dequantizing matrix product of the Zero-TVM write-up
// (section "完整的推理流水线": baseline / subgroup-reduce / rows x4, rows x8
// variants and the f32 LM-head variant) and its fused FFN (section "内核融合").
// One templated kernel covers all of them; the epilogue differs.
//
// Work decomposition (CUDA cores; the path is HBM-bound at M = 1):
//   * Persistent grid: one CTA of 16 warps per SM (or as many as fit), each
//     CTA stages the activations once into shared memory.
//   * A warp owns a tile of R weight rows over the whole of K and needs no
//     block-wide synchronisation: lane l handles the groups g = l, l + 32, ...
//     A group is exactly one 16-byte chunk of packed codes, so each load
//     instruction of a warp reads 512 contiguous bytes of one row: fully
//     coalesced 128-bit loads straight from HBM, U groups x R rows in flight
//     per lane.
//   * Every activation value a lane fetches from shared memory serves R rows
//     (the pages' rows x4 / rows x8 tiling).
//   * Lane partials are combined with a transposing warp-shuffle butterfly
//     (the pages' subgroup reduction) in a fixed order, so results are
//     deterministic and identical rows give identical outputs.
//   * Tiles are dealt to CTAs first, then to warps, so consecutive tiles land
//     on different SMs.
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
constexpr int kMaxCtas = 4096;             // grid cap (sizes the LM-head workspace)

enum EpiKind : int { kEpiF16 = 0, kEpiGateUp = 1, kEpiLogits = 2, kEpiRope = 3 };   // RoPE: pass kernel only

struct Q4Args {
    const uint4 *qw;        // [rows][G]: one 16-byte chunk = the 32 codes of one group
    const __half *scales;   // [rows][G]
    const __half *x;        // [M][K]
    void *out;              // fp16 [M][N] (F16, GateUp) or f32 [M][N] (Logits)
    float *ws_val;          // Logits: per-CTA maximum   [gridDim.x][M]
    int *ws_idx;            // Logits: per-CTA arg-max   [gridDim.x][M]
    int M, N, K, G;         // N = output features; G = K / 32
    int n_tiles;            // warp tiles (of R weight rows = R or R/2 outputs)
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

// sum over the 32 codes of one group (16 bytes) of q_k * x''_k, scaled by 2^-59
__device__ __forceinline__ float group_dot(const uint4 &w, const float4 (&xv)[8])
{
#ifdef ZT_SCALAR_FMA
    float acc0 = 0.f, acc1 = 0.f;
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t u = ws[i], h = u >> 12;
        const float4 xa = xv[2 * i], xb = xv[2 * i + 1];
        acc0 = fmaf(bits_f(u & 0xFu), xa.x, acc0);
        acc1 = fmaf(bits_f(u & 0xF0u), xa.y, acc1);
        acc0 = fmaf(bits_f(u & 0xF00u), xa.z, acc0);
        acc1 = fmaf(bits_f(u & 0xF000u), xa.w, acc1);
        acc0 = fmaf(bits_f(u & 0xF0000u), xb.x, acc0);
        acc1 = fmaf(bits_f(u & 0xF00000u), xb.y, acc1);
        acc0 = fmaf(bits_f(h & 0xF000u), xb.z, acc0);
        acc1 = fmaf(bits_f(h & 0xF0000u), xb.w, acc1);
    }
    return acc0 + acc1;
#else
    float2 acc = make_float2(0.f, 0.f);
    acc = word_dot(w.x, xv[0], xv[1], acc);
    acc = word_dot(w.y, xv[2], xv[3], acc);
    acc = word_dot(w.z, xv[4], xv[5], acc);
    acc = word_dot(w.w, xv[6], xv[7], acc);
    return acc.x + acc.y;
#endif
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

// Inverse of warp_transpose_reduce's lane -> value map: the value number a lane holds.
template <int V>
__device__ __forceinline__ int lane_vid(int lane)
{
    int vid = 0;
#pragma unroll
    for (int s = 0; s < 5; ++s) {
        const int half = V >> (s + 1);
        if (half >= 1 && (lane & (16 >> s))) vid += half;
    }
    return vid;
}

// greater value wins; equal values -> lower index; NaN counts as -inf
__device__ __forceinline__ bool better(float v, int i, float bv, int bi)
{
    v = isnan(v) ? -INFINITY : v;
    bv = isnan(bv) ? -INFINITY : bv;
    return v > bv || (v == bv && i < bi);
}

constexpr int kWarps = 16;                 // per CTA
constexpr int kThreads = kWarps * 32;

// Dynamic shared memory layout (bytes):
//   xs   float [M][G][32]  pre-scaled activations, float4 slots XOR-swizzled by g&7
//   xg   float [M][G]      7 * X_g * 2^-59
//   bv   float [kThreads], bi int [kThreads]   (Logits: per-lane running maxima)
__host__ __device__ inline size_t q4_smem_bytes(int M, int G)
{
    return (size_t)M * G * 32 * 4 + (size_t)M * G * 4 + (size_t)kThreads * 8;
}

// Stage x once per CTA: xs = x * 2^(90 - 4p(k)) (exact), xg = 7 * X_g * 2^-59.
// Each thread converts 8 consecutive k (one 16-byte load); the 4 threads of a
// group add their partial sums with two shuffles (fixed order).
__device__ __forceinline__ void stage_activations(const __half *__restrict__ x, float *xs, float *xg, int M,
                                                  int K, int G)
{
    const int K8 = K >> 3;
    for (int m = 0; m < M; ++m) {
        for (int base = 0; base < K8; base += kThreads) {
            const int kk = base + threadIdx.x;        // uniform trip count: shuffles see full warps
            float part = 0.f;
            if (kk < K8) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(x + (size_t)m * K + 8 * kk);
                const __half2 *h = reinterpret_cast<const __half2 *>(&raw);
                float v[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = __half22float2(h[j]);
                    v[2 * j] = f.x;
                    v[2 * j + 1] = f.y;
                }
                part = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
                const int g = kk >> 2, c0 = (kk & 3) * 2;
                float4 *dst = reinterpret_cast<float4 *>(xs + ((size_t)m * G + g) * 32);
                dst[c0 ^ (g & 7)] = make_float4(v[0] * pow2f(xscale_exp(0)), v[1] * pow2f(xscale_exp(1)),
                                                v[2] * pow2f(xscale_exp(2)), v[3] * pow2f(xscale_exp(3)));
                dst[(c0 + 1) ^ (g & 7)] = make_float4(v[4] * pow2f(xscale_exp(4)), v[5] * pow2f(xscale_exp(5)),
                                                      v[6] * pow2f(xscale_exp(6)), v[7] * pow2f(xscale_exp(7)));
            }
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            if (kk < K8 && (kk & 3) == 0) xg[(size_t)m * G + (kk >> 2)] = part * (7.0f * pow2f(-59));
        }
    }
}

template <int R, int MT, int U, int EPI>
__global__ void __launch_bounds__(kThreads, 1) q4_gemv_kernel(const Q4Args a)
{
    constexpr int V = R * MT;                                // partial sums per lane
    constexpr int ROUT = (EPI == kEpiGateUp) ? R / 2 : R;    // outputs per warp tile
    static_assert(V <= 32 && (V & (V - 1)) == 0, "R*MT must be a power of two <= 32");
    static_assert(EPI != kEpiGateUp || (R % 2 == 0), "gate/up needs an even row count");

    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int M = a.M, G = a.G, N = a.N;
    float *xs = reinterpret_cast<float *>(smem_raw);
    float *xg = xs + (size_t)M * G * 32;
    float *bvs = xg + (size_t)M * G;
    int *bis = reinterpret_cast<int *>(bvs + kThreads);

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;

    stage_activations(a.x, xs, xg, M, a.K, G);
    __syncthreads();

    const int vid = lane_vid<V>(lane);
    const bool rep = (lane & (32 / V - 1)) == 0;      // one lane per distinct value
    const int my_r = vid / MT, my_m = vid - (vid / MT) * MT;
    float best_v = -INFINITY;
    int best_i = 0x7fffffff;

    for (int tile = blockIdx.x + gridDim.x * warp; tile < a.n_tiles; tile += gridDim.x * kWarps) {
        const int obase = tile * ROUT;                    // first output row of the tile
        const uint4 *rowp[R];
        const __half *srow[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            int row;
            if (EPI == kEpiGateUp) {
                const int o = min(obase + (r % ROUT), N - 1);
                row = (r < ROUT) ? o : N + o;
            } else {
                row = min(obase + r, N - 1);              // rows past N are loaded, never stored
            }
            rowp[r] = a.qw + (size_t)row * G;
            srow[r] = a.scales + (size_t)row * G;
        }

        float part[V];
#pragma unroll
        for (int i = 0; i < V; ++i) part[i] = 0.f;

        for (int g0 = lane; g0 < G; g0 += 32 * U) {
            uint4 w[U][R];
            float s[U][R];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int g = g0 + 32 * u;
#pragma unroll
                for (int r = 0; r < R; ++r) w[u][r] = (g < G) ? ldg_stream(rowp[r] + g) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int g = g0 + 32 * u;
#pragma unroll
                for (int r = 0; r < R; ++r) s[u][r] = (g < G) ? __half2float(srow[r][g]) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int g = g0 + 32 * u;
                if (g < G) {
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
                                acc = word_dot(w[u][r].x, xv[0], xv[1], acc);
                                acc = word_dot(w[u][r].y, xv[2], xv[3], acc);
                                acc = word_dot(w[u][r].z, xv[4], xv[5], acc);
                                acc = word_dot(w[u][r].w, xv[6], xv[7], acc);
                                part[r * MT + m] = fmaf(s[u][r], (acc.x + acc.y) - xgm, part[r * MT + m]);
                            }
                        }
                    }
                }
            }
        }

        int v_unused;
        warp_transpose_reduce<V>(part, lane, v_unused);
        const float y = part[0] * pow2f(59);              // this lane's value: (row my_r, m my_m)
        if (EPI == kEpiGateUp) {
            const float u = __shfl_xor_sync(0xffffffffu, y, 16);   // the up row's value
            const int n = obase + my_r;
            if (rep && vid < V / 2 && n < N && my_m < M) {
                const float silu = y / (1.0f + expf(-y));
                reinterpret_cast<__half *>(a.out)[(size_t)my_m * N + n] = __float2half_rn(silu * u);
            }
        } else {
            const int n = obase + my_r;
            if (rep && n < N && my_m < M) {
                if (EPI == kEpiF16) {
                    reinterpret_cast<__half *>(a.out)[(size_t)my_m * N + n] = __float2half_rn(y);
                } else {
                    reinterpret_cast<float *>(a.out)[(size_t)my_m * N + n] = y;
                    if (better(y, n, best_v, best_i)) { best_v = isnan(y) ? -INFINITY : y; best_i = n; }
                }
            }
        }
    }

    if (EPI == kEpiLogits) {
        // per-CTA maximum for each m over all its lanes' running maxima
        bvs[threadIdx.x] = best_v;
        bis[threadIdx.x] = best_i;
        __syncthreads();
        if (threadIdx.x < M) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
            for (int t = 0; t < kThreads; ++t) {
                const int tv = lane_vid<V>(t & 31);
                if (tv - (tv / MT) * MT == (int)threadIdx.x && better(bvs[t], bis[t], bv, bi)) {
                    bv = bvs[t];
                    bi = bis[t];
                }
            }
            a.ws_val[(size_t)blockIdx.x * M + threadIdx.x] = bv;
            a.ws_idx[(size_t)blockIdx.x * M + threadIdx.x] = bi;
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
    asm volatile("griddepcontrol.wait;" ::: "memory");   // the first pass may still be running
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
