/*
 * zt_q4.h -- C ABI of the q4f16 dequantizing GEMV library for NVIDIA B200
 * (sm_100a): the int4 group-quantized matrix-vector products that dominate
 * single-token LLM decode.
 *
 * Source of the operations: the Zero-TVM forum write-up ("Zero-TVM：手写 WGSL
 * 着色器在浏览器中运行 Phi-3-mini，挑战编译器霸权"), section "完整的推理流水线"
 * (int4 反量化矩阵乘法 -- the int4 dequantizing matrix product, with an f32-output
 * variant for the LM head; greedy argmax sampling) and section "内核融合"
 * (fused_ffn: gate, up and SiLU in one pass).  Its performance section names the
 * weights "Phi-3-mini-q4f16_1".  The pages give no bit layout; this library
 * fixes the format below and every entry point uses it.
 *
 * FORMAT ("q4f16", group 32)
 *   W is n_rows x K (output features x input features), row-major.
 *   qw      uint32 [n_rows][K/8].  Element (n,k) is the 4-bit code in bits
 *           4*(k%8) .. 4*(k%8)+3 of qw[n][k/8] (low nibble first), 0..15.
 *   scales  IEEE binary16 bit patterns [n_rows][K/32]: one scale per 32 k.
 *   dequant w[n][k] = (code - 7) * scales[n][k/32]   (zero point 7).
 *   x       IEEE binary16 [M][K], M = number of tokens (1..16; the batched
 *           prefill entry points below take any M >= 1).
 *   Products are exact and accumulate in fp32; fp16 outputs are rounded once,
 *   to nearest even, at the store.
 *
 * CONVENTIONS (all compute entry points)
 *   - Pointers named qw, scales, x, y, logits, argmax, workspace are DEVICE
 *     pointers owned by the caller; the library never allocates, frees or
 *     keeps them after the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is launched asynchronously on it; no entry point
 *     synchronizes.  Errors inside a kernel surface at the caller's next
 *     synchronization, as for any CUDA launch.
 *   - Every argument is checked on the host BEFORE anything is launched; a
 *     call that returns a negative status launched nothing and wrote nothing.
 *   - Shapes (decode entry points): 1 <= M <= 16, N >= 1, K >= 32, K % 32 == 0, and the products
 *     n_rows*K and M*K fit in int64 (n_rows = N, or 2N for gate/up).
 *   - Alignment: qw and x 16 bytes; scales and y 2 bytes; logits and argmax
 *     4 bytes; workspace 16 bytes.
 *   - Inputs and outputs must not overlap.
 *   - Thread safety: calls on different streams may run concurrently.
 *   - Launch overlap: the kernels use programmatic dependent launch.  A call
 *     may start streaming qw and scales from HBM before the kernel ahead of it
 *     on the stream has finished; it reads x (and writes its outputs) only
 *     after that kernel completes.  So x may be produced by the preceding
 *     kernel, but qw and scales must not be written by a preceding kernel
 *     that itself triggers dependent launches early (weights are meant to be
 *     static; ordinary kernels, copies and the library's own calls are safe).
 */
#ifndef ZT_Q4_H
#define ZT_Q4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ZT_API __attribute__((visibility("default")))
#else
#define ZT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define ZT_OK                    0
#define ZT_ERR_INVALID_ARG      -1  /* null pointer, M/N/K out of range, K % 32 */
#define ZT_ERR_MISALIGNED       -2  /* a pointer violates its alignment rule */
#define ZT_ERR_WORKSPACE        -3  /* workspace smaller than the query says */
#define ZT_ERR_LAUNCH           -4  /* the CUDA launch failed (see zt_q4_last_cuda_error) */
#define ZT_ERR_UNSUPPORTED      -5  /* shape valid but beyond this build's limits */
#define ZT_ERR_DEVICE           -6  /* no usable sm_100 device / attribute query failed */

/*
 * y[m][n] = sum_k (q[n][k] - 7) * s[n][k/32] * x[m][k]        (fp16 out)
 *
 * The plain projection (Zero-TVM write-up, "完整的推理流水线": the baseline,
 * subgroup-reduce and rows x4 / rows x8 variants of the int4 dequantizing
 * matrix product -- one kernel here, with warp-shuffle K reduction and
 * row tiling chosen from the shape).
 *   qw [N][K/8], scales [N][K/32], x [M][K], y [M][N] (fp16 bit patterns).
 * Returns ZT_OK or a negative status.
 */
ZT_API int zt_q4_gemv(const uint32_t *qw, const uint16_t *scales, const uint16_t *x,
               uint16_t *y, int M, int N, int K, void *stream);

/*
 * Fused FFN input projection (Zero-TVM write-up, "内核融合": fused_ffn.wgsl,
 * gate, up and SiLU in one pass):
 *   g = gate row n . x_m,  u = up row n . x_m   (both fp32, never rounded)
 *   y[m][n] = fp16( SiLU(g) * u ),  SiLU(g) = g / (1 + exp(-g)).
 *   qw [2N][K/8] and scales [2N][K/32]: rows 0..N-1 are gate, N..2N-1 up.
 *   x [M][K], y [M][N].
 */
ZT_API int zt_q4_gate_up_silu(const uint32_t *qw, const uint16_t *scales, const uint16_t *x,
                       uint16_t *y, int M, int N, int K, void *stream);

/*
 * Bytes of device workspace zt_q4_lmhead_argmax needs for these shapes
 * (per-CTA partial maxima; 0 if the shapes are invalid).  The value depends
 * only on (M, N, K), never on the device.
 */
ZT_API size_t zt_q4_lmhead_workspace_bytes(int M, int N, int K);

/*
 * LM head with f32 logits and greedy argmax (Zero-TVM write-up,
 * "完整的推理流水线": the f32-output dequantizing matrix product "for sampling
 * stability", and greedy decoding as an argmax dispatch):
 *   logits[m][n] = sum_k (q[n][k] - 7) * s[n][k/32] * x[m][k]   (f32, not rounded to fp16)
 *   argmax[m]    = the lowest n among the maxima of logits[m][*]; NaN counts as
 *                  -infinity (a row of NaN gives 0).
 *   qw [N][K/8], scales [N][K/32], x [M][K], logits [M][N] f32, argmax [M] int32.
 *   workspace: device scratch of at least zt_q4_lmhead_workspace_bytes(M,N,K)
 *   bytes, 16-byte aligned, owned by the caller; its contents on entry do not
 *   matter.  Two launches on `stream` (logits + per-CTA maxima, then the
 *   final reduction); no device-side waits, no float atomics: the result is
 *   deterministic.
 */
ZT_API int zt_q4_lmhead_argmax(const uint32_t *qw, const uint16_t *scales, const uint16_t *x,
                        float *logits, int32_t *argmax, void *workspace, size_t ws_bytes,
                        int M, int N, int K, void *stream);

/*
 * zt_q4_lmhead_argmax without a caller-supplied workspace, for callers that
 * cannot allocate device memory: a plug-in running inside a host framework
 * that owns every device allocation, code being recorded into a CUDA graph
 * (where cudaMalloc is not allowed), or a latency-critical decode loop that
 * must not allocate (cudaMalloc can synchronize the device).  There is no
 * counterpart on the pages; it is an interface convenience of this library.
 *
 * Same arguments, results and checks as zt_q4_lmhead_argmax, minus the
 * workspace: the per-CTA maxima go to one static 512 KiB device array inside
 * the library (enough for every legal shape, M <= 16; a shape needing more
 * would return ZT_ERR_WORKSPACE).  Every GPU that loads the library holds that
 * array until the process exits.  Allocates nothing: no cudaMalloc/cudaFree.
 *   - The first call on a device looks the array's device address up
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - Every call on a device shares the array.  Calls whose kernels can
 *     overlap on the GPU (different streams without ordering) race on it and
 *     give wrong argmax; serialize them (one stream, or events).
 *   - Nothing in the array needs to start at zero: each call writes every
 *     entry it later reads.
 *   - Every check (null pointers, shapes, alignment, the array's size) runs
 *     before the first CUDA call.
 *   - The array's device address is looked up once per device and kept for
 *     the life of the process; after cudaDeviceReset the library must be
 *     reloaded before this entry point is used again.
 */
ZT_API int zt_q4_lmhead_argmax_noalloc(const uint32_t *qw, const uint16_t *scales, const uint16_t *x,
                                       float *logits, int32_t *argmax, int M, int N, int K, void *stream);

/*
 * A DECODE WEIGHT PASS in one launch: a list of projections run in order by one
 * persistent kernel (Zero-TVM write-up, "完整的推理流水线": per decoder layer the
 * QKV, output, fused FFN and down projections, then the f32 LM head; this is
 * that sequence of int4 dequantizing products with the weights streamed back to
 * back).  Each projection computes exactly what the single-call entry point of
 * its kind computes (zt_q4_gemv, zt_q4_gate_up_silu, zt_q4_lmhead_argmax), with
 * the same arguments and the same checks; M (tokens, 1..16) is shared.
 *
 * Ordering: a projection with `wait` != 0 reads its x only after every earlier
 * projection of the list has completed on the whole GPU (so x may be an earlier
 * projection's output); without `wait`, x must not be written by the list.  A
 * projection that writes a buffer an earlier projection reads needs `wait` too.
 * The weights of later projections stream while earlier ones compute.
 *
 * `wait` on any projection makes the launch cooperative (all CTAs resident);
 * the wait is bounded: after 2 s a CTA records bit 1 in the error word, stops
 * and exits (outputs are then incomplete); read it with zt_q4_pass_errors.
 *
 * workspace: device memory, 16-byte aligned, at least
 * zt_q4_pass_workspace_bytes(projs, n, M) bytes: barrier counters, the error
 * word, and the per-CTA maxima of each LM head.  Its contents on entry do not
 * matter (the call clears what it needs on `stream`).  Launches: one pass
 * kernel, plus one argmax reduction per LM-head projection.
 * projs is a HOST array of n entries (1..ZT_Q4_PASS_MAX), read during the call.
 */
#define ZT_Q4_GEMV 0
#define ZT_Q4_GATE_UP_SILU 1
#define ZT_Q4_LM_HEAD 2
#define ZT_Q4_PASS_MAX 192

/*
 * Optional prologue of a pass projection: residual add + RMSNorm (Zero-TVM
 * write-up, "内核融合": add_norm.wgsl joins the residual connection and the
 * RMSNorm layer normalisation; the pages give no formula, the standard RMSNorm
 * on the fp16 residual stream is read).  The projection's x is then not read;
 * instead, per row m (token) of [M][K]:
 *
 *   h[m][k] = fp16(residual[m][k] + delta[m][k])      (delta NULL: h = residual)
 *   x[m][k] = fp16(h[m][k] * gamma[k] / sqrt(sum_k h[m][k]^2 / K + eps))
 *
 * (h * gamma * r in fp32, the sum of squares in fp32, one rounding to fp16 at
 * the end, so an element can differ from the exactly rounded value by one
 * fp16 ulp.)  The kernel computes x while staging the projection's
 * activations -- no separate launch, x never goes through HBM.  h and x can be
 * written out (residual_out, x_out), once, by one CTA.  All pointers are
 * device memory, 16-byte aligned; residual_out must not overlap residual or
 * delta; a later projection that reads residual_out needs `wait`.
 */
typedef struct zt_q4_norm {
    const uint16_t *residual; /* [M][K] fp16 */
    const uint16_t *delta;    /* [M][K] fp16, or NULL */
    const uint16_t *gamma;    /* [K] fp16 */
    uint16_t *residual_out;   /* [M][K] fp16 receives h, or NULL */
    uint16_t *x_out;          /* [M][K] fp16 receives x, or NULL */
    float eps;                /* >= 0, finite */
} zt_q4_norm;

/*
 * Optional epilogue of a ZT_Q4_GEMV pass projection: rotary position
 * embedding (Zero-TVM write-up, "完整的推理流水线": RoPE is computed in place
 * inside the fused QKV kernel; the pages give no formula, the standard
 * rotation is read).  The N output rows form heads of head_dim features; for
 * head h, i < head_dim / 2, n = h * head_dim + i, n2 = n + head_dim / 2 and
 * token m at position pos[m]:
 *
 *   phi       = pos[m] * theta^(-2 i / head_dim)
 *   out[m][n]  = fp16(y[n] cos(phi) - y[n2] sin(phi))
 *   out[m][n2] = fp16(y[n2] cos(phi) + y[n] sin(phi))
 *
 * y is the projection's fp32 result (not rounded before the rotation); the
 * angle, sin, cos and the rotation are taken in double.  Use it for the Q and
 * K rows of a QKV projection and give the V rows their own plain projection
 * (same pass, same phase; ld_out lets both write one [M][3 * D] buffer).
 */
typedef struct zt_q4_rope {
    const int32_t *pos;       /* [M] device: position of token m, >= 0 */
    int head_dim;             /* even; N % head_dim == 0 */
    float theta;              /* frequency base, > 0 (10000 for Phi-3-mini) */
} zt_q4_rope;

typedef struct zt_q4_proj {
    const uint32_t *qw;       /* [n_rows][K/8], n_rows = N (2N for GATE_UP_SILU) */
    const uint16_t *scales;   /* [n_rows][K/32] fp16 */
    const uint16_t *x;        /* [M][K] fp16 (ignored, may be NULL, when norm is set) */
    void *out;                /* fp16 [M][ld_out], or f32 [M][ld_out] logits for LM_HEAD */
    int32_t *argmax;          /* LM_HEAD: [M]; ignored otherwise */
    int kind;                 /* ZT_Q4_GEMV, ZT_Q4_GATE_UP_SILU or ZT_Q4_LM_HEAD */
    int N, K;
    int wait;                 /* read x only after all earlier projections completed */
    int ld_out;               /* elements between output rows (tokens); 0 means N; else >= N */
    int group;                /* k per fp16 scale: 0 or 32 (the q4f16 format), 64 or 128; K % group == 0;
                                 scales are then [n_rows][K/group] */
    const zt_q4_norm *norm;   /* HOST pointer to the add + RMSNorm prologue, or NULL */
    const zt_q4_rope *rope;   /* HOST pointer to the RoPE epilogue (ZT_Q4_GEMV only), or NULL */
} zt_q4_proj;

ZT_API size_t zt_q4_pass_workspace_bytes(const zt_q4_proj *projs, int n, int M);
ZT_API int zt_q4_pass(const zt_q4_proj *projs, int n, int M, void *workspace, size_t ws_bytes, void *stream);

/*
 * Launch plan of the decode kernel (every decode entry point and zt_q4_pass run
 * it), from the shapes alone -- no device is touched, nothing is launched:
 * M tokens (1..16), K_max the largest K of the list (a multiple of 32), n the
 * number of projections (1 for a single call).  Writes the CTAs resident per SM
 * (1 or 2) and their warps (warps_per_cta: 16 with one CTA per SM, else 8),
 * the ring depth in weight items per warp (2..4), k_window: 0 when
 * each projection's activations are staged whole in shared memory, else the
 * length in k of the windows that projections with K > k_window are staged in
 * (a multiple of 256; the CTA then walks such a projection's rows in rounds and
 * stages the windows in turn), and column_blocks: 1, or 2 when M > 8 tokens whose
 * activations would not fit whole run as two CTAs per row share, one for the
 * first ceil(M/2) tokens and one for the rest (k_window then refers to ceil(M/2)
 * tokens).  Every legal shape has a plan.  Diagnostics.
 */
ZT_API int zt_q4_pass_plan(int M, int K_max, int n, int *ctas_per_sm, int *stages, int *k_window,
                           int *column_blocks, int *warps_per_cta);

/* Synchronous read of a finished pass's error word (0: no bounded wait expired). */
ZT_API int zt_q4_pass_errors(const void *workspace, int n, unsigned int *out);

/*
 * TEST HOOK for the error path (tests only): zt_q4_pass with CTA 0 not counting
 * phase 0 done, so every CTA's bounded wait before phase 1 runs out (about 2 s),
 * sets the error bit, drains its copies and returns; phase 0's outputs are
 * complete, later phases' are not.  The list must contain a projection with
 * `wait` set (else ZT_ERR_INVALID_ARG).  Nothing faults or hangs: the wait is
 * the kernel's own bounded one, and the context stays usable.
 */
ZT_API int zt_q4_pass_test_withhold(const zt_q4_proj *projs, int n, int M, void *workspace, size_t ws_bytes,
                                    void *stream);

/*
 * BOUNDS-CHECKED BUILD.  The same sources compiled with -DZT_Q4_CHECKED
 * (libzt_q4_checked.so beside libzt_q4.so) compare, in the pass kernel that
 * serves every decode entry point, each computed global index (weight and
 * scale copies and loads, output and LM-head workspace stores) and each read
 * and write of its shared partial buffer with the extent of its buffer.  An
 * index outside it sets bit ZT_Q4_ERR_BOUNDS (2) of the error word that
 * zt_q4_pass_errors reads (bit 0 is the expired bounded wait) and the access
 * is skipped: no assert, no trap, the context stays usable.  The activation
 * staging (m < M, k < K over x with row stride K) is not instrumented.
 *
 * zt_q4_build_flags: ZT_Q4_BUILD_CHECKED when this library is the checked
 * build, else 0.
 *
 * zt_q4_pass_test_cut (TEST HOOK, checked build only; ZT_ERR_UNSUPPORTED in
 * the default one): zt_q4_pass with the weight extent of every projection
 * taken `rows` rows short, so that the copies of its last rows fail their
 * check (and are skipped) while the buffers themselves stay whole: the error
 * bit is set and nothing out of bounds is read.  rows < 1: ZT_ERR_INVALID_ARG.
 */
#define ZT_Q4_BUILD_CHECKED 1
#define ZT_Q4_ERR_BOUNDS 2u
ZT_API int zt_q4_build_flags(void);
ZT_API int zt_q4_pass_test_cut(const zt_q4_proj *projs, int n, int M, void *workspace, size_t ws_bytes,
                               void *stream, int rows);

/*
 * BATCHED PREFILL (M > 16 tokens; any M >= 1 is accepted)
 *
 * Zero-TVM write-up, limitations section: the project ships shaders for
 * batched prefill (not wired into its decode loop), and its shaders compute
 * in f16 (WebGPU shader-f16).  For M tokens at once the weights are first
 * dequantized to binary16 the way an f16 shader forms them,
 *     w16[n][k] = fp16((code - 7) * scales[n][k/group])   (one rounding, to nearest even),
 * and then y[m][n] = fp16(sum_k w16[n][k] * x[m][k]) with fp32 accumulation on
 * the tensor cores (tcgen05, kind::f16).  This is NOT the decode entry points'
 * arithmetic (they use the exact products (code - 7) * s); the difference is
 * the rounding of each weight to binary16.
 *
 * zt_q4_dequant_f16: w16 (DEVICE, fp16 [N][K], 16-byte aligned) from qw [N][K/8]
 *     and scales [N][K/group].  group: 0 or 32, 64, 128 (K % group == 0).  HBM-bound
 *     streaming kernel; a caller that runs many prefill batches may keep w16 and
 *     call zt_q4_gemm_f16w directly.
 * zt_q4_gemm_f16w: y fp16 [M][N] = x fp16 [M][K] times w16^T.  workspace (DEVICE,
 *     16-byte aligned, zt_q4_gemm_f16w_workspace_bytes(M, N, K) bytes) holds an error
 *     word (cleared by the call, on the stream) and, for shapes whose tiles cover
 *     few SMs, fp32 partial sums of a split along K, added in a fixed order by a
 *     second launch (results are deterministic).  Bit 0 of the error word is set if
 *     one of the kernel's bounded waits (2 s) expired (outputs are then incomplete);
 *     read it with zt_q4_gemm_f16w_errors.  w16 and x 16-byte aligned, y 2 bytes.
 * zt_q4_gemm: both steps through one workspace of zt_q4_gemm_workspace_bytes(M, N, K)
 *     bytes (16-byte aligned): w16 first, then the GEMM's workspace; read its error
 *     word with zt_q4_gemm_errors.  Two or three launches on `stream`.
 * The tile plan (and so the workspace size) is a function of (M, N, K) alone.
 * Shapes: 1 <= M <= 2^22, N >= 1, K >= 32, K % 32 == 0, N*K <= 2^40.  Inputs and
 * outputs must not overlap.  Status codes as elsewhere; ZT_ERR_DEVICE also when the
 * TMA descriptor encoder is unavailable; ZT_ERR_UNSUPPORTED when the plan's weight-row
 * tiles exceed CUDA's 65535 grid rows (millions of weight rows; checked before any
 * launch).  The *_errors calls are synchronous.
 */
ZT_API int zt_q4_dequant_f16(const uint32_t *qw, const uint16_t *scales, uint16_t *w16, int N, int K, int group,
                             void *stream);
ZT_API size_t zt_q4_gemm_f16w_workspace_bytes(int M, int N, int K);
ZT_API int zt_q4_gemm_f16w(const uint16_t *w16, const uint16_t *x, uint16_t *y, int M, int N, int K,
                           void *workspace, size_t ws_bytes, void *stream);
ZT_API int zt_q4_gemm_f16w_errors(const void *workspace, unsigned int *out);
ZT_API size_t zt_q4_gemm_workspace_bytes(int M, int N, int K);
ZT_API int zt_q4_gemm(const uint32_t *qw, const uint16_t *scales, const uint16_t *x, uint16_t *y, int M, int N,
                      int K, int group, void *workspace, size_t ws_bytes, void *stream);
ZT_API int zt_q4_gemm_errors(const void *workspace, int N, int K, unsigned int *out);

/*
 * Batched fused FFN (Zero-TVM write-up, kernel-fusion section: gate, up and
 * SiLU in one pass) on the prefill reading of the weights: qw / scales hold 2N
 * rows (gate rows 0..N-1, up rows N..2N-1), w16 likewise [2N][K];
 *     y[m][n] = fp16(SiLU(g) * u),  g = sum_k w16[n][k] x[m][k],  u = sum_k w16[N+n][k] x[m][k],
 * g and u in fp32 (tensor-core accumulation), SiLU(g) = g / (1 + e^-g) in fp32.
 * The 2N-wide intermediate never leaves tensor memory.  Workspace: for
 * zt_q4_gemm_gate_up_silu zt_q4_gemm_gate_up_workspace_bytes(M, N, K) bytes (w16,
 * then the error word; read it with zt_q4_gemm_errors(workspace, 2 * N, K, &e));
 * for zt_q4_gemm_f16w_gate_up_silu at least 256 bytes (the error word, read with
 * zt_q4_gemm_f16w_errors).  Shapes, alignment and status codes as for zt_q4_gemm,
 * with 2N in place of N.
 */
ZT_API size_t zt_q4_gemm_gate_up_workspace_bytes(int M, int N, int K);
ZT_API int zt_q4_gemm_gate_up_silu(const uint32_t *qw, const uint16_t *scales, const uint16_t *x, uint16_t *y,
                                   int M, int N, int K, int group, void *workspace, size_t ws_bytes, void *stream);
ZT_API int zt_q4_gemm_f16w_gate_up_silu(const uint16_t *w16, const uint16_t *x, uint16_t *y, int M, int N, int K,
                                        void *workspace, size_t ws_bytes, void *stream);

/*
 * Host-side layout helpers (HOST pointers, synchronous, no CUDA calls).
 * pack:   q uint8 [N][K] codes 0..15  ->  qw uint32 [N][K/8], low nibble first.
 *         A code above 15 is ZT_ERR_INVALID_ARG (qw is then unspecified).
 * unpack: qw [N][K/8] -> q [N][K].
 * K % 8 == 0 and K >= 8 for both.
 */
ZT_API int zt_q4_pack_host(const uint8_t *q, int N, int K, uint32_t *qw);
ZT_API int zt_q4_unpack_host(const uint32_t *qw, int N, int K, uint8_t *q);

/* Static English text for a status code (never NULL). */
ZT_API const char *zt_q4_strerror(int status);

/*
 * Name of the last CUDA runtime error a library call met on the calling host
 * thread (e.g. "cudaErrorInvalidResourceHandle"), or "" if none.  Diagnostics
 * for ZT_ERR_LAUNCH / ZT_ERR_DEVICE; static storage, never NULL.
 */
ZT_API const char *zt_q4_last_cuda_error(void);

/* Library ABI version, (major << 16) | minor.  1.3 added zt_q4_pass_plan; 1.4 its column_blocks; 1.5 its
 * warps_per_cta; 1.6 zt_q4_build_flags and zt_q4_pass_test_cut. */
ZT_API int zt_q4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ZT_Q4_H */
