// q4_common.cuh -- constants and small device helpers shared by the q4f16
// decode kernels (q4_mma.cuh, q4_pass.cuh), and the second pass of the greedy
// argmax over the LM head's f32 logits.
//
// Operation: the int4 dequantizing matrix product of the Zero-TVM write-up
// (section "完整的推理流水线": the baseline / subgroup-reduce / rows x4, x8
// variants, the f32-output LM head, and greedy sampling as an argmax dispatch).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace zt {

constexpr int kGroup = 32;                 // k values per scale (the q4f16 format)
constexpr int kMaxCtas = 4096;             // grid cap (sizes the LM-head workspace)

// kEpiRope: a projection whose output feature pairs are rotated (RoPE epilogue)
enum EpiKind : int { kEpiF16 = 0, kEpiGateUp = 1, kEpiLogits = 2, kEpiRope = 3 };

__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// greater value wins; equal values -> lower index; NaN counts as -inf
__device__ __forceinline__ bool better(float v, int i, float bv, int bi)
{
    v = isnan(v) ? -INFINITY : v;
    bv = isnan(bv) ? -INFINITY : bv;
    return v > bv || (v == bv && i < bi);
}

// 128-bit streaming load: data read exactly once, kept out of L1.
__device__ __forceinline__ uint4 ldg_stream(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Programmatic dependent launch: let the next kernel on the stream launch now;
// wait until the kernel ahead of this one on the stream has completed.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Second pass of the LM head's argmax: one CTA per activation row m reduces
// the per-CTA (maximum, lowest index) pairs of the first pass with the total
// order of better(), so the result does not depend on the reduction order.
// It never triggers its dependents early: the next LM-head call on the stream
// may reuse the same partial-maximum scratch, and must not start writing it
// while this kernel still reads it.
__global__ void __launch_bounds__(256) q4_argmax_reduce_kernel(const float *ws_val, const int *ws_idx,
                                                               int n_cta, int M, int32_t *argmax)
{
    __shared__ float sv[256];
    __shared__ int si[256];
    pdl_wait();   // the first pass may still be running
    const int m = blockIdx.x;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int c = threadIdx.x; c < n_cta; c += blockDim.x) {
        const float v = ws_val[(size_t)c * M + m];
        const int i = ws_idx[(size_t)c * M + m];
        if (better(v, i, bv, bi)) {
            bv = isnan(v) ? -INFINITY : v;
            bi = i;
        }
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
