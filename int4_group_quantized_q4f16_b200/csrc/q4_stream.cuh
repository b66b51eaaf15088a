// q4_stream.cuh -- the streaming sm_100a kernel for the q4f16 dequantizing
// matrix-vector product at small batch (M <= 4): the HBM-bound hot path.
//
// Operation: the int4 dequantizing matrix product of the Zero-TVM write-up
// (section "完整的推理流水线": the baseline / subgroup-reduce / rows x4, x8
// variants and the f32-output LM head) and its fused FFN (section "内核融合",
// fused_ffn: gate, up and SiLU in one pass).  Arithmetic is the exact-product
// scheme of q4_gemv.cuh (codes masked in place and read as subnormal floats,
// pre-scaled activations, fp32 accumulation); this file is about feeding it
// from HBM at full rate.
//
// Data movement (CTA = 8 warps; persistent grid sized from occupancy):
//   * Each CTA owns a contiguous, balanced range of output rows, so every SM
//     streams the same number of bytes.
//   * The range is cut into tiles of 4 weight rows (rows x4; for the fused FFN
//     2 gate + 2 up rows) and K into chunks of 32 groups (1024 k, one group
//     per lane).  The 8 warps form WR x WK: WR warps deal the tiles, WK warps
//     split the chunks of a tile (WK > 1 when the CTA has few rows, e.g. the
//     3072-row projections), chosen on the host to balance items per warp.
//   * Every warp owns a private ring of S stages in shared memory and fills
//     it with 16-byte cp.async copies (LDGSTS, L2 only): lane l copies group l
//     of each of the tile's 4 rows, lanes 0..3 the chunk's 64 bytes of scales.
//     S - 1 items per warp are in flight while one is computed, i.e. tens of
//     KB per SM without registers.  cp.async.wait_group is a hardware wait:
//     the kernel contains no spin loops.
//   * The pre-scaled activations of a group are read once from shared memory
//     for all 4 rows of a tile.  Lane partials are combined by a warp-shuffle
//     butterfly; WK > 1 partials meet in shared memory and are summed in a
//     fixed order at the end: results are deterministic.
//   * Programmatic dependent launch: the kernel lets the next kernel on the
//     stream launch at once; each warp issues its first S - 1 weight copies
//     before griddepcontrol.wait, so weights stream while the previous kernel
//     finishes.  Activations are read and outputs written only after the wait.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "q4_gemv.cuh"

namespace zt {

constexpr int kAW = 8;                              // warps per CTA
constexpr int kAThreads = kAW * 32;
constexpr int kAR = 4;                              // weight rows per tile
constexpr int kAChunkG = 32;                        // groups per chunk (one per lane)
constexpr int kARowBytes = kAChunkG * 16;           // codes of one row of a chunk: 512 B
constexpr int kAScaleBytes = kAChunkG * 2;          // scales of one row of a chunk: 64 B
constexpr int kAStage = kAR * (kARowBytes + kAScaleBytes);   // 2304 B per warp per stage
constexpr int kAMaxStages = 8;

struct StreamArgs {
    const uint4 *qw;            // [rows][G] 16-byte chunks
    const __half *scales;       // [rows][G]
    const __half *x;            // [M][K]
    void *out;                  // fp16 [M][N] or f32 [M][N]
    float *ws_val;              // Logits: per-CTA maximum [gridDim.x][M]
    int *ws_idx;
    int M, N, K, G;
    int stages;                 // ring depth S per warp (2..kAMaxStages)
    int wk;                     // warps splitting K (1, 2, 4, 8); WR = 8 / wk
    int max_tiles;              // tiles of the largest CTA range (sizes the WK > 1 buffer)
    int scales_async;           // 1: scales copied with cp.async; 0: read from global
};

// R = weight rows per tile, V = R * MT partial sums per lane
__host__ __device__ inline size_t stream_smem_bytes(int M, int G, int stages, int wk, int max_tiles, int R, int V)
{
    const size_t ring = (size_t)kAW * stages * R * (kARowBytes + kAScaleBytes);
    const size_t xs = (size_t)M * G * 32 * 4;
    const size_t xg = ((size_t)M * G * 4 + 15) & ~(size_t)15;
    const size_t red = wk > 1 ? (size_t)max_tiles * wk * V * 4 : 0;
    return ring + xs + xg + ((red + 15) & ~(size_t)15) + (size_t)kAThreads * 8;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_dyn(int pending)
{
    // wait_group takes an immediate: dispatch the ring depths in use
    switch (pending) {
    case 0: cp_async_wait<0>(); break;
    case 1: cp_async_wait<1>(); break;
    case 2: cp_async_wait<2>(); break;
    case 3: cp_async_wait<3>(); break;
    case 4: cp_async_wait<4>(); break;
    case 5: cp_async_wait<5>(); break;
    default: cp_async_wait<6>(); break;
    }
}

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Stage x for the whole CTA (same values as stage_activations in q4_gemv.cuh).
__device__ __forceinline__ void stage_x_cta(const __half *__restrict__ x, float *xs, float *xg, int M, int K, int G)
{
    const int K8 = K >> 3;
    for (int m = 0; m < M; ++m) {
        for (int base = 0; base < K8; base += kAThreads) {
            const int kk = base + threadIdx.x;
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

template <int MT, int EPI, int R = kAR>
__global__ void __launch_bounds__(kAThreads, 2) q4_stream_kernel(const StreamArgs a)
{
    constexpr int V = R * MT;
    constexpr int ROUT = (EPI == kEpiGateUp) ? R / 2 : R;          // outputs per tile
    constexpr int STAGE = R * (kARowBytes + kAScaleBytes);
    static_assert(V <= 32 && (V & (V - 1)) == 0, "R*MT must be a power of two <= 32");

    extern __shared__ __align__(128) unsigned char smem[];
    const int M = a.M, N = a.N, G = a.G, S = a.stages, wk = a.wk;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned char *ring = smem + (size_t)warp * S * STAGE;
    float *xs = reinterpret_cast<float *>(smem + (size_t)kAW * S * STAGE);
    float *xg = xs + (size_t)M * G * 32;
    float *red = xg + (((size_t)M * G + 3) & ~(size_t)3);
    const size_t red_floats = wk > 1 ? (size_t)a.max_tiles * wk * V : 0;
    float *bvs = red + ((red_floats + 3) & ~(size_t)3);
    int *bis = reinterpret_cast<int *>(bvs + kAThreads);

    pdl_launch_dependents();

    // this CTA's outputs [o_begin, o_end), tiles of ROUT outputs, chunks of 32 groups
    const int o_begin = (int)(((long long)N * blockIdx.x) / gridDim.x);
    const int o_end = (int)(((long long)N * (blockIdx.x + 1)) / gridDim.x);
    const int n_tiles = (o_end - o_begin + ROUT - 1) / ROUT;
    const int n_chunks = (G + kAChunkG - 1) / kAChunkG;
    const int wr_n = kAW / wk;
    const int my_wk = warp % wk, my_wr = warp / wk;
    const int my_tiles = my_wr < n_tiles ? (n_tiles - my_wr + wr_n - 1) / wr_n : 0;
    const int my_chunks = my_wk < n_chunks ? (n_chunks - my_wk + wk - 1) / wk : 0;
    const int n_items = my_tiles * my_chunks;
    const bool scales_async = a.scales_async != 0;

    // Issue side: item counters advance without divisions.  Rows past the
    // CTA's range are clamped (copied, never stored).
    int is_tl = 0, is_cl = 0, is_stage = 0, is_left = n_items;
    const uint4 *is_w[R];
    const __half *is_s[R];
    auto set_rows = [&](const uint4 **wp, const __half **sp, int tl) {
        const int o0 = o_begin + (my_wr + wr_n * tl) * ROUT;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            int row;
            if (EPI == kEpiGateUp) {
                const int o = min(o0 + (r % ROUT), N - 1);
                row = (r < ROUT) ? o : N + o;
            } else {
                row = min(o0 + r, N - 1);
            }
            wp[r] = a.qw + (size_t)row * G;
            sp[r] = a.scales + (size_t)row * G;
        }
    };
    if (n_items > 0) set_rows(is_w, is_s, 0);
    auto issue_next = [&]() {
        if (is_left > 0) {
            const int c = my_wk + wk * is_cl;
            unsigned char *st = ring + (size_t)is_stage * STAGE;
            const int g = c * kAChunkG + lane;
            const int kc = min(kAChunkG, G - c * kAChunkG);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                if (lane < kc) cp_async16(st + r * kARowBytes + lane * 16, is_w[r] + g);
                if (scales_async && lane < (kc >> 3))
                    cp_async16(st + R * kARowBytes + r * kAScaleBytes + lane * 16, is_s[r] + c * kAChunkG + lane * 8);
            }
            --is_left;
            if (++is_cl == my_chunks) {
                is_cl = 0;
                if (++is_tl < my_tiles) set_rows(is_w, is_s, is_tl);
            }
        }
        cp_async_commit();     // one group per item slot, so wait counts stay uniform
        if (++is_stage == S) is_stage = 0;
    };

    // prologue: weights stream before the previous kernel has finished
    for (int j = 0; j < S - 1; ++j) issue_next();

    pdl_wait();
    stage_x_cta(a.x, xs, xg, M, a.K, G);
    __syncthreads();

    const int vid = lane_vid<V>(lane);
    const bool rep = (lane & (32 / V - 1)) == 0;
    const int my_r = vid / MT, my_m = vid - (vid / MT) * MT;
    float best_v = -INFINITY;
    int best_i = 0x7fffffff;
    float part[V];
    const __half *cs_s[R];
    const uint4 *cs_w_unused[R];
    int tl = 0, cl = 0, stage = 0;
    if (n_items > 0 && !scales_async) set_rows(cs_w_unused, cs_s, 0);

    for (int j = 0; j < n_items; ++j) {
        cp_async_wait_dyn(S - 2);          // item j's group has landed
        __syncwarp();
        const int t = my_wr + wr_n * tl;
        const int c = my_wk + wk * cl;
        const int o0 = o_begin + t * ROUT;
        if (cl == 0) {
#pragma unroll
            for (int v = 0; v < V; ++v) part[v] = 0.f;
        }
        const int g = c * kAChunkG + lane;
        if (g < G) {
            const unsigned char *st = ring + (size_t)stage * STAGE;
            float sc[R];
#pragma unroll
            for (int r = 0; r < R; ++r)
                sc[r] = scales_async
                            ? __half2float(reinterpret_cast<const __half *>(st + R * kARowBytes + r * kAScaleBytes)[lane])
                            : __half2float(cs_s[r][g]);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < M) {
                    const float4 *xv4 = reinterpret_cast<const float4 *>(xs + ((size_t)m * G + g) * 32);
                    const int swz = g & 7;
                    float4 xv[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) xv[q] = xv4[q ^ swz];
                    const float xgm = xg[m * G + g];
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(st + r * kARowBytes + lane * 16);
                        part[r * MT + m] = fmaf(sc[r], group_dot(w, xv) - xgm, part[r * MT + m]);
                    }
                }
            }
        }
        __syncwarp();                      // the stage is free again (scales were read by all lanes)
        issue_next();
        if (++stage == S) stage = 0;

        if (cl == my_chunks - 1) {
            int v_unused;
            warp_transpose_reduce<V>(part, lane, v_unused);
            if (wk > 1) {
                if (rep) red[((size_t)t * wk + my_wk) * V + vid] = part[0];
            } else {
                const float y = part[0] * pow2f(59);
                const int n = o0 + my_r;
                if (EPI == kEpiGateUp) {
                    const float u = __shfl_xor_sync(0xffffffffu, y, 16);
                    if (rep && vid < V / 2 && n < o_end && my_m < M) {
                        const float silu = y / (1.0f + expf(-y));
                        reinterpret_cast<__half *>(a.out)[(size_t)my_m * N + n] = __float2half_rn(silu * u);
                    }
                } else if (rep && n < o_end && my_m < M) {
                    if (EPI == kEpiF16) {
                        reinterpret_cast<__half *>(a.out)[(size_t)my_m * N + n] = __float2half_rn(y);
                    } else {
                        reinterpret_cast<float *>(a.out)[(size_t)my_m * N + n] = y;
                        if (better(y, n, best_v, best_i)) {
                            best_v = isnan(y) ? -INFINITY : y;
                            best_i = n;
                        }
                    }
                }
            }
        }
        if (++cl == my_chunks) {
            cl = 0;
            ++tl;
            if (!scales_async && tl < my_tiles) set_rows(cs_w_unused, cs_s, tl);
        }
    }
    cp_async_wait<0>();

    if (wk > 1) {
        // partials of the WK warps of each tile meet here; fixed summation order
        __syncthreads();
        constexpr int VO = ROUT * MT;
        for (int idx = tid; idx < n_tiles * VO; idx += kAThreads) {
            const int t = idx / VO, vo = idx - (idx / VO) * VO;
            const int r = vo / MT, m = vo - (vo / MT) * MT;
            const int n = o_begin + t * ROUT + r;
            const float *rp = red + (size_t)t * wk * V;
            float y = 0.f, u = 0.f;
            for (int k2 = 0; k2 < wk; ++k2) {
                y += rp[k2 * V + r * MT + m];
                if (EPI == kEpiGateUp) u += rp[k2 * V + (r + ROUT) * MT + m];
            }
            y *= pow2f(59);
            if (n < o_end && m < M) {
                if (EPI == kEpiF16) {
                    reinterpret_cast<__half *>(a.out)[(size_t)m * N + n] = __float2half_rn(y);
                } else if (EPI == kEpiGateUp) {
                    u *= pow2f(59);
                    const float silu = y / (1.0f + expf(-y));
                    reinterpret_cast<__half *>(a.out)[(size_t)m * N + n] = __float2half_rn(silu * u);
                } else {
                    reinterpret_cast<float *>(a.out)[(size_t)m * N + n] = y;
                    if (better(y, n, best_v, best_i)) {
                        best_v = isnan(y) ? -INFINITY : y;
                        best_i = n;
                    }
                }
            }
        }
    }

    if (EPI == kEpiLogits) {
        // per-CTA maximum per m.  Thread t holds maxima for m = (its vid) % MT
        // when the warp epilogue ran (wk == 1), or for m = idx % MT when the
        // shared-memory epilogue did (idx = t + 256 i, and 256 % MT == 0).
        bvs[tid] = best_v;
        bis[tid] = best_i;
        __syncthreads();
        if (tid < M) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
            for (int t = 0; t < kAThreads; ++t) {
                int tm;
                if (wk > 1) {
                    tm = t % MT;
                } else {
                    const int tv = lane_vid<V>(t & 31);
                    tm = tv - (tv / MT) * MT;
                }
                if (tm == tid && better(bvs[t], bis[t], bv, bi)) {
                    bv = bvs[t];
                    bi = bis[t];
                }
            }
            a.ws_val[(size_t)blockIdx.x * M + tid] = bv;
            a.ws_idx[(size_t)blockIdx.x * M + tid] = bi;
        }
    }
}

}  // namespace zt
