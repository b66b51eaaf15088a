// q4_stream.cuh -- the streaming sm_100a kernel for the q4f16 dequantizing
// matrix-vector product at small batch (M <= 4): the HBM-bound hot path.
//
// Operation: the int4 dequantizing matrix product of the Zero-TVM write-up
// (section "完整的推理流水线": the baseline / subgroup-reduce / rows x4, x8
// variants and the f32-output LM head) and its fused FFN (section "内核融合",
// fused_ffn: gate, up and SiLU in one pass).  Arithmetic is the exact-product
// scheme of q4_gemv.cuh (codes masked in place and read as subnormal floats,
// pre-scaled activations, fp32 accumulation); only the data movement differs.
//
// Data movement (one CTA = 1 producer warp + 8 consumer warps, 2 CTAs per SM):
//   * Each CTA owns a contiguous, balanced range of output rows, so every SM
//     streams the same number of bytes and all finish together.
//   * The rows are cut into tiles of 32 weight rows and each tile into chunks
//     of 1024 k.  One (tile, chunk) item = 32 row pieces of 512 contiguous
//     bytes of codes + 64 bytes of scales, moved by the producer with 1D TMA
//     bulk copies (cp.async.bulk, no multicast) into a ring of S stages in
//     shared memory, completion tracked by an mbarrier per stage.  With S - 1
//     stages in flight per CTA the memory system sees tens of KB outstanding
//     per SM without spending registers on it.
//   * A consumer warp owns 4 weight rows of the tile; lane l reads group l of
//     the chunk (16 bytes, conflict-free) and the 32 pre-scaled activations
//     of that group once for all 4 rows.  Lane partials are combined by a
//     warp-shuffle butterfly after the tile's last chunk.
//   * Programmatic dependent launch: the kernel lets the next kernel on the
//     stream launch at once, and its producer starts streaming weights before
//     the previous kernel has finished; only the activations are read after
//     griddepcontrol.wait.  Consequence (stated in the C header): qw and scales
//     must not be produced by a kernel that triggers dependent launches early.
//   * Every wait on an mbarrier is bounded by a time limit; on expiry the
//     kernel records an error code in a device word, drains its own copies in
//     flight (again bounded) and returns.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "q4_gemv.cuh"

namespace zt {

constexpr int kSC = 8;                              // consumer warps per CTA
constexpr int kSThreads = (kSC + 1) * 32;           // + one producer warp
constexpr int kSR = 4;                              // weight rows per consumer warp per tile
constexpr int kTileRows = kSC * kSR;                // weight rows per tile
constexpr int kKC = 1024;                           // k per chunk: one group per lane
constexpr int kChunkW = kKC / 2;                    // bytes of codes per row per chunk
constexpr int kChunkS = kKC / 16;                   // bytes of scales per row per chunk
constexpr int kStageBytes = kTileRows * (kChunkW + kChunkS);
constexpr int kMaxStages = 8;
constexpr int kBarBytes = 256;                      // barriers + flags at the front of smem
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s per wait

// device error codes (OR-ed into StreamArgs::err)
constexpr unsigned kErrFullTimeout = 1u;            // a consumer gave up waiting for data
constexpr unsigned kErrEmptyTimeout = 2u;           // the producer gave up waiting for a free stage
constexpr unsigned kErrDrainTimeout = 4u;           // copies still in flight at exit

struct StreamArgs {
    const uint8_t *qw;          // packed codes, [rows][K/2] bytes
    const __half *scales;       // [rows][G]
    const __half *x;            // [M][K]
    void *out;                  // fp16 [M][N] or f32 [M][N]
    float *ws_val;              // Logits: per-CTA maximum [gridDim.x][M]
    int *ws_idx;
    unsigned int *err;          // device error word
    int M, N, K, G;
    int stages;                 // ring depth S (2..kMaxStages)
    int scales_tma;             // 1: scales ride in the stage; 0: read from global
};

__host__ __device__ inline size_t stream_smem_bytes(int M, int G, int stages)
{
    return (size_t)kBarBytes + (size_t)stages * kStageBytes + (size_t)M * G * 32 * 4 +
           (((size_t)M * G * 4 + 15) & ~(size_t)15) + (size_t)kSC * 32 * 8;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of `bar` with parity `parity` to complete; false after
// kWaitLimitNs without completion.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
}

// 1D bulk copy global -> this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kSC * 32) : "memory"); }

// x staging for the consumer warps (same values as stage_activations).
__device__ __forceinline__ void stage_x_consumers(const __half *__restrict__ x, float *xs, float *xg, int M, int K,
                                                  int G, int tid)
{
    const int K8 = K >> 3;
    for (int m = 0; m < M; ++m) {
        for (int base = 0; base < K8; base += kSC * 32) {
            const int kk = base + tid;
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

template <int MT, int EPI>
__global__ void __launch_bounds__(kSThreads, 2) q4_stream_kernel(const StreamArgs a)
{
    constexpr int R = kSR;
    constexpr int V = R * MT;
    constexpr int ROUT = (EPI == kEpiGateUp) ? R / 2 : R;          // outputs per consumer warp
    constexpr int TOUT = kSC * ROUT;                               // outputs per tile
    static_assert(V <= 32 && (V & (V - 1)) == 0, "R*MT must be a power of two <= 32");

    extern __shared__ __align__(128) unsigned char smem[];
    const int S = a.stages;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty = full + kMaxStages;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kMaxStages);
    unsigned char *stage0 = smem + kBarBytes;
    float *xs = reinterpret_cast<float *>(stage0 + (size_t)S * kStageBytes);
    float *xg = xs + (size_t)a.M * a.G * 32;
    float *bvs = xg + (((size_t)a.M * a.G + 3) & ~(size_t)3);
    int *bis = reinterpret_cast<int *>(bvs + kSC * 32);

    const int M = a.M, N = a.N, K = a.K, G = a.G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // this CTA's output rows [o_begin, o_end)
    const int o_begin = (int)(((long long)N * blockIdx.x) / gridDim.x);
    const int o_end = (int)(((long long)N * (blockIdx.x + 1)) / gridDim.x);
    const int n_tiles = (o_end - o_begin + TOUT - 1) / TOUT;
    const int n_chunks = (K + kKC - 1) / kKC;
    const int n_items = n_tiles * n_chunks;

    if (tid == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kSC);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == kSC) {
        // ------------------------------------------------------ producer --
        if (lane == 0) {
            const size_t row_bytes = (size_t)K / 2;
            int issued = 0;
            for (int i = 0; i < n_items; ++i) {
                const int s = i % S;
                if (i >= S && !mbar_wait_bounded(&empty[s], ((i / S) - 1) & 1)) {
                    atomicOr(a.err, kErrEmptyTimeout);
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                const int t = i / n_chunks, c = i - t * n_chunks;
                const int o0 = o_begin + t * TOUT;
                const int rows = min(TOUT, o_end - o0);
                const int kcount = min(kKC, K - c * kKC);
                const uint32_t wbytes = (uint32_t)kcount / 2, sbytes = (uint32_t)kcount / 16;
                const int halves = (EPI == kEpiGateUp) ? 2 : 1;
                const uint32_t total = (uint32_t)(halves * rows) * (wbytes + (a.scales_tma ? sbytes : 0u));
                unsigned char *sw = stage0 + (size_t)s * kStageBytes;
                unsigned char *ss = sw + kTileRows * kChunkW;
                mbar_arrive_expect_tx(&full[s], total);
                for (int h = 0; h < halves; ++h) {
                    for (int r = 0; r < rows; ++r) {
                        const int slot = h * TOUT + r;
                        const size_t wrow = (size_t)(h * N + o0 + r);
                        bulk_g2s(sw + (size_t)slot * kChunkW, a.qw + wrow * row_bytes + (size_t)c * (kKC / 2), wbytes,
                                 &full[s]);
                        if (a.scales_tma)
                            bulk_g2s(ss + (size_t)slot * kChunkS, a.scales + wrow * G + (size_t)c * (kKC / 32), sbytes,
                                     &full[s]);
                    }
                }
                issued = i + 1;
            }
            // drain: every copy this CTA issued must land before it exits
            for (int i = max(0, issued - S); i < issued; ++i) {
                if (!mbar_wait_bounded(&full[i % S], (i / S) & 1)) {
                    atomicOr(a.err, kErrDrainTimeout);
                    break;
                }
            }
        }
    } else {
        // ----------------------------------------------------- consumers --
        pdl_wait();                                   // activations may come from the previous kernel
        stage_x_consumers(a.x, xs, xg, M, K, G, tid);
        consumers_sync();

        const int vid = lane_vid<V>(lane);
        const bool rep = (lane & (32 / V - 1)) == 0;
        const int my_r = vid / MT, my_m = vid - (vid / MT) * MT;
        float best_v = -INFINITY;
        int best_i = 0x7fffffff;
        float part[V];

        for (int i = 0; i < n_items; ++i) {
            const int s = i % S;
            if (*abort_flag) break;
            if (!mbar_wait_bounded(&full[s], (i / S) & 1)) {
                atomicOr(a.err, kErrFullTimeout);
                *abort_flag = 1;
                break;
            }
            const int t = i / n_chunks, c = i - t * n_chunks;
            const int o0 = o_begin + t * TOUT;
            const int rows = min(TOUT, o_end - o0);
            if (c == 0) {
#pragma unroll
                for (int v = 0; v < V; ++v) part[v] = 0.f;
            }
            const int g = c * 32 + lane;
            if (warp * ROUT < rows && g < G) {
                const unsigned char *sw = stage0 + (size_t)s * kStageBytes;
                const __half *ss = reinterpret_cast<const __half *>(sw + kTileRows * kChunkW);
                int slot[R];
#pragma unroll
                for (int r = 0; r < R; ++r)
                    slot[r] = (EPI == kEpiGateUp) ? (r < ROUT ? warp * ROUT + r : TOUT + warp * ROUT + (r - ROUT))
                                                  : warp * R + r;
                uint4 w[R];
                float sc[R];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    w[r] = *reinterpret_cast<const uint4 *>(sw + (size_t)slot[r] * kChunkW + lane * 16);
                    if (a.scales_tma) {
                        sc[r] = __half2float(ss[slot[r] * (kChunkS / 2) + lane]);
                    } else {
                        const int orow = min(o0 + (slot[r] % TOUT), N - 1);
                        const size_t wrow = (size_t)((slot[r] >= TOUT ? N : 0) + orow);
                        sc[r] = __half2float(a.scales[wrow * G + g]);
                    }
                }
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
                            float2 acc = make_float2(0.f, 0.f);
                            acc = word_dot(w[r].x, xv[0], xv[1], acc);
                            acc = word_dot(w[r].y, xv[2], xv[3], acc);
                            acc = word_dot(w[r].z, xv[4], xv[5], acc);
                            acc = word_dot(w[r].w, xv[6], xv[7], acc);
                            part[r * MT + m] = fmaf(sc[r], (acc.x + acc.y) - xgm, part[r * MT + m]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);

            if (c == n_chunks - 1) {
                int v_unused;
                warp_transpose_reduce<V>(part, lane, v_unused);
                const float y = part[0] * pow2f(59);
                const int n = o0 + warp * ROUT + my_r;
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

        if (EPI == kEpiLogits) {
            bvs[tid] = best_v;
            bis[tid] = best_i;
            consumers_sync();
            if (tid < M) {
                float bv = -INFINITY;
                int bi = 0x7fffffff;
                for (int t = 0; t < kSC * 32; ++t) {
                    const int tv = lane_vid<V>(t & 31);
                    if (tv - (tv / MT) * MT == tid && better(bvs[t], bis[t], bv, bi)) {
                        bv = bvs[t];
                        bi = bis[t];
                    }
                }
                a.ws_val[(size_t)blockIdx.x * M + tid] = bv;
                a.ws_idx[(size_t)blockIdx.x * M + tid] = bi;
            }
        }
    }
}

}  // namespace zt
