// zt_q4.cu -- the C ABI of the q4f16 dequantizing GEMV library (see
// include/zt_q4.h for the contract of every entry point).
//
// Host side only: argument checks, launch-shape selection and launches.  Every
// check runs before the first CUDA call, so a rejected call launches nothing.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <climits>
#include <cstdint>
#include <mutex>
#include <unordered_map>

#include "q4_common.cuh"
#include "q4_mma.cuh"
#include "q4_pass.cuh"
#include "q4_gemm_tc.cuh"
#include "zt_q4.h"

namespace {

using namespace zt;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_shapes(int M, int N, int K, int row_mult)
{
    if (M < 1 || M > 16 || N < 1 || K < kGroup || K % kGroup) return ZT_ERR_INVALID_ARG;
    if ((int64_t)N * row_mult > INT_MAX) return ZT_ERR_INVALID_ARG;
    return ZT_OK;
}

struct OccKey {
    const void *fn;
    int dev, threads;
    size_t smem;
    bool operator==(const OccKey &o) const
    {
        return fn == o.fn && dev == o.dev && threads == o.threads && smem == o.smem;
    }
};
struct OccHash {
    size_t operator()(const OccKey &k) const
    {
        return std::hash<const void *>()(k.fn) ^ (size_t)k.dev * 131 ^ (size_t)k.threads * 7919 ^
               k.smem * 104729;
    }
};

// last CUDA error seen by a library call on this host thread (diagnostics only)
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// Launch status: clear a stale non-sticky error left by an earlier, unrelated
// runtime call before launching (so it is not blamed on this launch), then
// read and clear the launch's own error.
void clear_stale_error() { (void)cudaGetLastError(); }

int launch_status()
{
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) return ZT_OK;
    g_last_cuda_error = e;
    return ZT_ERR_LAUNCH;
}

std::mutex g_mu;
std::unordered_map<OccKey, int, OccHash> g_occ;   // resident CTAs per SM, or -1 if unusable
std::unordered_map<int, int> g_sms;               // device -> SM count

std::unordered_map<uint64_t, bool> g_optin;      // (kernel, device) opted in to the max smem

// Resident CTAs per SM for (kernel, block, smem) on the current device.  On
// first use of a kernel on a device its dynamic shared memory limit is raised
// once to the device's opt-in maximum, so every later launch of any size fits.
int resident_ctas(const void *fn, int threads, size_t smem, int &sms)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        g_last_cuda_error = e;
        return -1;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    auto it_s = g_sms.find(dev);
    if (it_s == g_sms.end()) {
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess || n < 1) {
            g_last_cuda_error = e;
            return -1;
        }
        it_s = g_sms.emplace(dev, n).first;
    }
    sms = it_s->second;
    const uint64_t fkey = (uint64_t)(uintptr_t)fn * 64u + (uint64_t)dev;
    if (g_optin.find(fkey) == g_optin.end()) {
        int optin = 0;
        e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        if (e != cudaSuccess) {
            g_last_cuda_error = e;
            (void)cudaGetLastError();
            return -1;
        }
        g_optin.emplace(fkey, true);
    }
    OccKey key{fn, dev, threads, smem};
    auto it = g_occ.find(key);
    if (it != g_occ.end()) return it->second;
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, threads, smem);
    if (e != cudaSuccess) {
        g_last_cuda_error = e;
        (void)cudaGetLastError();
        return -1;
    }
    g_occ.emplace(key, nb > 0 ? nb : -1);
    return nb > 0 ? nb : -1;
}

// shared memory per CTA for 2 and for 1 resident CTA per SM (228 KiB per SM,
// 1 KiB reserved per CTA)
constexpr size_t kSmemTwoPerSm = 113 * 1024;
constexpr size_t kSmemOnePerSm = 227 * 1024;

// How a pass launch stages its activations: warps per CTA, CTAs per SM, ring
// depth, the groups of K per column the activation area holds, and whether
// longer projections go through K windows of that many groups.  A function of
// (M, the list's largest K, the list length) only.
struct PassPlan {
    int mw, cps, stages, g_stage;
    bool win;
    int red;   // WK partial buffer, floats
};

// Whole-K staging when the rings (2..4 stages) and all of x fit: first one CTA
// of 16 warps per SM (with the full WK partial buffer, else the least one),
// then two CTAs of 8, then one of 8; otherwise K windows (a
// multiple of 8 groups, one item's chunk) with 8 warps, as long as fit three
// stages at two CTAs per SM, else one CTA per SM with four stages.  Always
// succeeds for M <= 16 and lists of up to kPassMax projections: the smallest
// window (8 groups) needs 96 KiB.  One CTA of 16 warps beats two of 8 when it
// fits: two CTAs on an SM do not share its issue slots evenly (the older one
// runs ahead), and the kernel ends with the slower one.  Except for a single
// projection of one token: there two 8-warp CTAs per SM leave room on each SM
// for the next call's CTAs to start (programmatic dependent launch) while this
// one drains, and measured faster alone too.  `wide`: 16 warps may be planned.
PassPlan pass_plan(int M, int g_max, int n, int NT, bool wide = true)
{
    const bool one = M == 1;
    if (wide && !(one && n == 1)) {
        // the full partial buffer, else the least one (room for the rings of 16 warps)
        for (const int red : {pass_red_floats(NT, 16, one), pass_red_floats_min(NT, one)}) {
            const size_t fixed = pass_smem_bytes(M, g_max, 0, n, NT, 16, red);
            const size_t per_stage = (size_t)16 * kMStage;
            const int stages =
                kSmemOnePerSm > fixed ? (int)std::min<size_t>(kPassMaxStages, (kSmemOnePerSm - fixed) / per_stage) : 0;
            if (stages >= 2) return PassPlan{16, 1, stages, g_max, false, red};
        }
    }
    const int red8 = pass_red_floats(NT, 8, one);
    const size_t per_stage = (size_t)8 * kMStage;
    for (int cps = 2; cps >= 1; --cps) {
        const size_t budget = cps == 2 ? kSmemTwoPerSm : kSmemOnePerSm;
        const size_t fixed = pass_smem_bytes(M, g_max, 0, n, NT, 8, red8);
        const int stages = budget > fixed ? (int)std::min<size_t>(kPassMaxStages, (budget - fixed) / per_stage) : 0;
        if (stages >= 2) return PassPlan{8, cps, stages, g_max, false, red8};
    }
    for (int cps = 2; cps >= 1; --cps) {
        const size_t budget = cps == 2 ? kSmemTwoPerSm : kSmemOnePerSm;
        const int stages = cps == 2 ? 3 : kPassMaxStages;
        int best = 0;
        for (int gw = kMChunkG; gw < g_max; gw += kMChunkG)
            if (pass_smem_bytes(M, gw, stages, n, NT, 8, red8) <= budget) best = gw;
        if (best > 0) return PassPlan{8, cps, stages, best, true, red8};
    }
    return PassPlan{0, 0, 0, 0, false, 0};
}

// M > 8 runs as two column blocks of ceil(M/2) and floor(M/2) tokens (the
// kernel's colsplit) when the list's longest K would not fit whole at 16
// columns: each CTA of a pair then stages its <= 8 columns whole (or in
// windows twice as long), instead of restaging 16 columns per K window.  The
// pair shares its rows' weights, the second read of them coming from L2.
bool pass_colsplit(int M, int g_max, int n) { return M > 8 && pass_plan(M, g_max, n, 2).win; }

// Launch the tensor-core pass kernel over a.p[0 .. a.n).  `cooperative`:
// some projection waits on earlier ones (all CTAs must be co-resident).
constexpr int kNotResident = 1;   // launch_pass_s: this shape does not reach the wanted residency

template <int NT, int PMAX, int S, bool ONE, bool WIN, int MW>
int launch_pass_s(const PassArgs<PMAX> &a, bool cooperative, cudaStream_t st, int grid, size_t smem, int cps)
{
    const void *fn = reinterpret_cast<const void *>(&q4_pass_kernel<NT, PMAX, S, ONE, WIN, MW>);
    int sms = 0;
    if (resident_ctas(fn, MW * 32, smem, sms) < cps) return kNotResident;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(MW * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (cooperative) {
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    } else {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    clear_stale_error();
    const cudaError_t e = cudaLaunchKernelEx(&cfg, q4_pass_kernel<NT, PMAX, S, ONE, WIN, MW>, a);
    if (e != cudaSuccess) {
        g_last_cuda_error = e;
        (void)cudaGetLastError();
        return ZT_ERR_LAUNCH;
    }
    return ZT_OK;
}

template <int NT, int PMAX, bool ONE, bool WIN, int MW>
int launch_pass_w(const PassArgs<PMAX> &a, bool cooperative, cudaStream_t st, int grid, size_t smem, int cps,
                  int stages)
{
    switch (stages) {
    case 2: return launch_pass_s<NT, PMAX, 2, ONE, WIN, MW>(a, cooperative, st, grid, smem, cps);
    case 3: return launch_pass_s<NT, PMAX, 3, ONE, WIN, MW>(a, cooperative, st, grid, smem, cps);
    default: return launch_pass_s<NT, PMAX, 4, ONE, WIN, MW>(a, cooperative, st, grid, smem, cps);
    }
}

// Launch the tensor-core pass kernel over a.p[0 .. a.n) with the plan of
// pass_plan.  ZT_ERR_DEVICE if the device cannot hold the planned residency.
template <int NT, int PMAX, bool ONE>
int launch_pass(PassArgs<PMAX> &a, bool cooperative, cudaStream_t st, int *grid_out)
{
    int sms = 0;
    if (resident_ctas(reinterpret_cast<const void *>(&q4_pass_kernel<NT, PMAX, 2, ONE, false, 8>), 8 * 32, 0, sms) < 1)
        return ZT_ERR_DEVICE;
    int g_max = 0;
    for (int i = 0; i < a.n; ++i) g_max = std::max(g_max, a.p[i].G);
    // Phases: a new one at every projection that waits.  Each CTA takes a
    // byte-balanced share of each phase's concatenated rows.
    long long rows = 0;      // a CTA with no rows of a list without waits would only idle
    long long off = 0;       // HBM bytes of the projections so far
    a.phases = 0;
    for (int w = 0; w < (PMAX + 31) / 32; ++w) a.lm_bits[w] = 0;
    for (int i = 0; i < a.n; ++i) {
        PassProj &p = a.p[i];
        if (i == 0 || p.wait) a.phbeg[a.phases++] = off;
        a.pphase[i] = a.phases - 1;
        p.row_bytes = (p.K / 2 + (p.K / 16 >> p.gsh)) * ((p.kind == kEpiGateUp || p.kind == kEpiRope) ? 2 : 1);
        a.pbeg[i] = off;
        off += (long long)p.N * p.row_bytes;
        rows += p.N;
        if (p.kind == kEpiLogits) a.lm_bits[i >> 5] |= 1u << (i & 31);
    }
    a.pbeg[a.n] = off;
    a.phbeg[a.phases] = off;
    const int Mc = a.colsplit ? (a.M + 1) / 2 : a.M;   // columns one CTA stages at most
    const long long per_row = a.colsplit ? 2 : 1;
    // the plan, then (if the device holds fewer CTAs of it) the plan without 16-warp CTAs
    for (int attempt = 0; attempt < 2; ++attempt) {
        const PassPlan plan = pass_plan(Mc, g_max, a.n, NT, attempt == 0);
        if (plan.cps == 0) return ZT_ERR_UNSUPPORTED;
        a.g_stage = plan.g_stage;
        a.red_floats = plan.red;
        const size_t smem = pass_smem_bytes(Mc, plan.g_stage, plan.stages, a.n, NT, plan.mw, plan.red);
        // the planned CTAs per SM, or one if the device holds fewer at this shared memory size
        // (with the column split, an even grid: CTAs 2s and 2s + 1 take the same rows)
        for (int cps = plan.cps; cps >= 1; --cps) {
            long long g = std::min<long long>(
                {(long long)sms * cps, cooperative ? (long long)sms * cps : rows * per_row, kMaxCtas});
            if (a.colsplit) g &= ~1LL;
            const int grid = (int)std::max<long long>(per_row, g);
            int rc = ZT_ERR_UNSUPPORTED;
            if (plan.mw == 16)
                rc = launch_pass_w<NT, PMAX, ONE, false, 16>(a, cooperative, st, grid, smem, cps, plan.stages);
            else if (!plan.win)
                rc = launch_pass_w<NT, PMAX, ONE, false, 8>(a, cooperative, st, grid, smem, cps, plan.stages);
            else if constexpr (NT == 1)   // 16 columns that would need windows run as two column blocks instead
                rc = launch_pass_w<NT, PMAX, ONE, true, 8>(a, cooperative, st, grid, smem, cps, plan.stages);
            if (rc == kNotResident) continue;
            if (rc == ZT_OK && grid_out) *grid_out = grid;
            return rc;
        }
    }
    return ZT_ERR_DEVICE;
}

// One projection through the pass kernel (no waits, launched with PDL).
// ws_val: the LM head's per-CTA maxima (the arg-max follows at ws_val +
// kMaxCtas * M), null otherwise.
template <int EPI>
int launch_q4(const uint32_t *qw, const uint16_t *scales, const uint16_t *x, void *out, float *ws_val, int M,
              int N, int K, void *stream, int *grid_out)
{
    PassArgs<1> a;
    a.n = 1;
    a.M = M;
    a.colsplit = pass_colsplit(M, K / kGroup, 1) ? 1 : 0;
    a.counters = nullptr;
    a.error = nullptr;
    a.withhold = -1;
    a.chk_cut = 0;
    PassProj &p = a.p[0];
    p.qw = reinterpret_cast<const uint4 *>(qw);
    p.scales = reinterpret_cast<const __half *>(scales);
    p.x = reinterpret_cast<const __half *>(x);
    p.out = out;
    p.ws_val = ws_val;
    p.N = N;
    p.K = K;
    p.G = K / kGroup;
    p.kind = EPI;
    p.scales_async = (K % 256 == 0) && aligned(scales, 16);
    p.wait = 0;
    p.norm = 0;
    p.res = p.dlt = p.gamma = nullptr;
    p.res_out = p.x_out = nullptr;
    p.eps = 0.f;
    p.ldo = N;
    p.pos = nullptr;
    p.theta = 0.f;
    p.rope_d = 0;
    p.gsh = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (M == 1) return launch_pass<1, 1, true>(a, false, st, grid_out);
    return (M <= 8 || a.colsplit) ? launch_pass<1, 1, false>(a, false, st, grid_out)
                                  : launch_pass<2, 1, false>(a, false, st, grid_out);
}

size_t lmhead_ws_bytes(int M) { return (size_t)kMaxCtas * M * (sizeof(float) + sizeof(int)); }

// Scratch of zt_q4_lmhead_argmax_noalloc: one per device, for the whole life
// of the library.  Sized for the largest LM-head workspace (M = 16).
constexpr size_t kNoAllocScratchBytes = (size_t)kMaxCtas * 16 * (sizeof(float) + sizeof(int));   // 512 KiB
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
std::unordered_map<int, void *> g_noalloc_ptr;   // device -> device address of g_noalloc_scratch

// Device address of the scratch array on the current device, looked up once
// per device (a host-side `g_noalloc_scratch` is only a stand-in, not a device
// address, so it must never be passed to a kernel directly).
void *noalloc_scratch()
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        g_last_cuda_error = e;
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_noalloc_ptr.find(dev);
    if (it != g_noalloc_ptr.end()) return it->second;
    void *ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
        g_last_cuda_error = e;
        (void)cudaGetLastError();
        return nullptr;
    }
    g_noalloc_ptr.emplace(dev, ptr);
    return ptr;
}

// ------------------------------------------------ batched (prefill) GEMM ----
// cuTensorMapEncodeTiled, looked up once through the runtime (no link to the
// driver library needed).
PFN_cuTensorMapEncodeTiled_v12000 tma_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        (void)cudaGetLastError();
    });
    return fn;
}

// fp16 [rows][K] row-major, boxes of 64 k x box_rows rows, 128-byte swizzle,
// out-of-range elements read as zero.
bool tma_map_f16(CUtensorMap *map, const void *base, int K, long long rows, int box_rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tma_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)kTcK, (cuuint32_t)box_rows};   // box_rows <= 256
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int check_gemm_shapes(int M, int N, int K)
{
    if (M < 1 || M > (1 << 22) || N < 1 || K < kGroup || K % kGroup) return ZT_ERR_INVALID_ARG;
    if ((long long)N * K > (1ll << 40)) return ZT_ERR_INVALID_ARG;
    return ZT_OK;
}

int group_shift(int K, int group)
{
    if (group == 0) group = kGroup;
    if (group != 32 && group != 64 && group != 128) return -1;
    if (K % group) return -1;
    return group == 32 ? 0 : group == 64 ? 1 : 2;
}

// Workspace of the GEMM on binary16 weights: the error word (256 bytes
// reserved), then split-K partials fp32 [splits][M][N].  zt_q4_gemm puts the
// w16 weights in front of it.
size_t w16_bytes(int N, int K) { return ((size_t)N * (size_t)K * 2 + 255) & ~(size_t)255; }

// Launch plan, a function of the shape only (computed for the 148 SMs of a
// B200, so the workspace query needs no device).  From 128 tokens on, tokens
// are the A operand and weight rows the B operand (AM x BN = 256 x 256,
// 128 x 256, 128 x 128 or 128 x 64); below 128 tokens weight rows are A (128
// per CTA) and
// the tokens a 64- or 128-wide B tile.  K may be split into s <= 8 parts of
// at least 16 k blocks (fp32 partials, summed in order by a second launch).
// Among these the plan with the least estimated time wins:
//   waves x (MMA cycles of one CTA / ingest efficiency + epilogue + fixed)
//   + the partials' round trip when split,
// where one k block of an AM x BN tile is AM * BN / 64 MMA cycles and the
// ingest efficiency is min(1, 70 / (bytes per MMA cycle the tile needs)),
// 70 bytes per cycle being about what one SM takes in from L2 (measured: the
// 128 x 256 tile needs 96 and keeps the tensor pipe ~60 % busy), and the
// partials' round trip is priced at 24 bytes per cycle per SM.  (A 256 x 128
// tile needs as many bytes per cycle as 128 x 256 but measured slower, so it
// is not offered.)
constexpr int kPlanSms = 148;
struct GemmPlan {
    int am, bn, splits, kb_per;
    bool toka;
};

double plan_cost(int am, int bn, int s, long long M, long long N, long long kb_n, bool toka)
{
    const long long ra = toka ? M : N, rb = toka ? N : M;
    const long long ctas = ((ra + am - 1) / am) * ((rb + bn - 1) / bn) * s;
    const long long waves = (ctas + kPlanSms - 1) / kPlanSms;
    const long long kb_per = (kb_n + s - 1) / s;
    const double need = 8192.0 * (am + bn) / ((double)am * bn);          // bytes per MMA cycle
    const double eff = std::min(1.0, 70.0 / need);
    const double mma = (double)am * bn / 64.0 * kb_per / eff;
    const double epi = (double)am * bn * (s > 1 ? 4 : 2) / 48.0;
    double cost = (double)waves * (mma + epi + 3000.0);
    if (s > 1) cost += 2.0 * s * (double)M * N * 4 / (kPlanSms * 24.0);
    return cost;
}

GemmPlan gemm_plan(int M, int N, int K)
{
    const long long kb_n = (K + kTcK - 1) / kTcK;
    static const int toka_tiles[][2] = {{256, 256}, {128, 256}, {128, 128}, {128, 64}};
    static const int swap_tiles[][2] = {{128, 128}, {128, 64}};
    const bool toka = M >= 128;
    GemmPlan best{128, 64, 1, (int)kb_n, toka};
    double best_cost = 1e300;
    const int n_tiles = toka ? 4 : 2;
    for (int t = 0; t < n_tiles; ++t) {
        const int am = toka ? toka_tiles[t][0] : swap_tiles[t][0];
        const int bn = toka ? toka_tiles[t][1] : swap_tiles[t][1];
        if (!toka && bn == 128 && M <= 64) continue;        // a 64-wide token tile covers M
        for (int sp = 1; sp <= 8; ++sp) {
            if (sp > 1 && kb_n / sp < 16) break;
            const double c = plan_cost(am, bn, sp, M, N, kb_n, toka);
            if (c < best_cost) {
                best_cost = c;
                best = GemmPlan{am, bn, sp, (int)((kb_n + sp - 1) / sp), toka};
            }
        }
    }
    return best;
}

// CUDA caps grid.y (the weight-row tiles when tokens are the A operand, the
// token tiles otherwise) at 65535: beyond that the shape is unsupported.
// Checked on the host before anything is launched.
bool gemm_grid_ok(const GemmPlan &p, int M, int N, bool silu)
{
    const long long b_rows = p.toka ? N : M;
    const long long b_out = silu ? p.bn / 2 : p.bn;
    return (b_rows + b_out - 1) / b_out <= 65535 && p.splits <= 65535;
}

size_t f16w_ws_bytes(int M, int N, int K)
{
    const GemmPlan p = gemm_plan(M, N, K);
    return 256 + (p.splits > 1 ? (size_t)p.splits * M * N * 4 : 0);
}

int launch_dequant(const uint32_t *qw, const uint16_t *scales, uint16_t *w16, int N, int K, int gsh,
                   unsigned int *err, cudaStream_t st)
{
    const void *fn = reinterpret_cast<const void *>(&q4_dequant_f16_kernel);
    int sms = 0;
    const int occ = resident_ctas(fn, 256, 0, sms);
    if (occ < 1) return ZT_ERR_DEVICE;
    const long long want = ((long long)N + 7) / 8;          // 8 warps per block, one row per warp
    const int grid = (int)std::max(1ll, std::min(want, (long long)sms * occ));
    clear_stale_error();
    q4_dequant_f16_kernel<<<grid, 256, 0, st>>>(qw, reinterpret_cast<const __half *>(scales),
                                                  reinterpret_cast<uint4 *>(w16), N, K / 8, gsh, err);
    return launch_status();
}

template <int AM, int BN, bool TOKA, bool SILU = false>
int launch_gemm_tc_cfg(const GemmPlan &p, const uint16_t *w16, const uint16_t *x, uint16_t *y, float *part, int M,
                       int N, int K, unsigned int *err, cudaStream_t st)
{
    using C = TcCfg<AM, BN>;
    const void *fn = reinterpret_cast<const void *>(&q4_gemm_tc_kernel<AM, BN, TOKA, SILU>);
    int sms = 0;
    if (resident_ctas(fn, kTcThreads, C::kSmem, sms) < 1) return ZT_ERR_DEVICE;
    const uint16_t *a = TOKA ? x : w16, *b = TOKA ? w16 : x;
    const int ra = TOKA ? M : N, rb = TOKA ? (SILU ? 2 * N : N) : M;   // rows of the two tensors
    const int b_out = SILU ? BN / 2 : BN;                              // B rows (outputs) per CTA
    const int b_rows = TOKA ? N : M;
    CUtensorMap ma, mb;
    if (!tma_map_f16(&ma, a, K, ra, AM) || !tma_map_f16(&mb, b, K, rb, b_out)) return ZT_ERR_DEVICE;
    const dim3 grid((unsigned)((ra + AM - 1) / AM), (unsigned)((b_rows + b_out - 1) / b_out), (unsigned)p.splits);
    clear_stale_error();
    q4_gemm_tc_kernel<AM, BN, TOKA, SILU><<<grid, kTcThreads, C::kSmem, st>>>(
        ma, mb, reinterpret_cast<__half *>(y), p.splits > 1 ? part : nullptr, M, N, K, p.kb_per, err);
    int rc = launch_status();
    if (rc || p.splits == 1) return rc;
    const long long mn = (long long)M * N;
    const int grid_r = (int)std::max(1ll, std::min((mn / 4 + 255) / 256, (long long)sms * 8));
    q4_splitk_reduce_kernel<<<grid_r, 256, 0, st>>>(part, reinterpret_cast<__half *>(y), mn, p.splits);
    return launch_status();
}

// The fused FFN on binary16 weights [2N][K]: tokens as the A operand (also
// below 128 tokens: the tile's spare rows read zeros), B = BN/2 gate rows and
// their BN/2 up rows, never split (SiLU needs whole sums); tile by the same
// cost estimate over the 2N weight rows.
GemmPlan gate_up_plan(int M, int N, int K)
{
    const long long kb_n = (K + kTcK - 1) / kTcK;
    static const int tiles[][2] = {{256, 256}, {128, 256}, {128, 128}};
    GemmPlan best{128, 128, 1, (int)kb_n, true};
    double best_cost = 1e300;
    for (const auto &t : tiles) {
        if (t[0] == 256 && M < 128) continue;
        const double c = plan_cost(t[0], t[1], 1, M, 2ll * N, kb_n, true);
        if (c < best_cost) {
            best_cost = c;
            best = GemmPlan{t[0], t[1], 1, (int)kb_n, true};
        }
    }
    return best;
}

int launch_gate_up_tc(const uint16_t *w16, const uint16_t *x, uint16_t *y, int M, int N, int K, void *ws,
                      cudaStream_t st)
{
    const GemmPlan p = gate_up_plan(M, N, K);
    unsigned int *err = static_cast<unsigned int *>(ws);
    if (p.am == 256) return launch_gemm_tc_cfg<256, 256, true, true>(p, w16, x, y, nullptr, M, N, K, err, st);
    if (p.bn == 256) return launch_gemm_tc_cfg<128, 256, true, true>(p, w16, x, y, nullptr, M, N, K, err, st);
    return launch_gemm_tc_cfg<128, 128, true, true>(p, w16, x, y, nullptr, M, N, K, err, st);
}

// ws: the GEMM's workspace (error word, then partials), f16w_ws_bytes long.
int launch_gemm_tc(const uint16_t *w16, const uint16_t *x, uint16_t *y, int M, int N, int K, void *ws,
                   cudaStream_t st)
{
    const GemmPlan p = gemm_plan(M, N, K);
    unsigned int *err = static_cast<unsigned int *>(ws);
    float *part = reinterpret_cast<float *>(static_cast<unsigned char *>(ws) + 256);
    if (p.toka) {
        if (p.am == 256) return launch_gemm_tc_cfg<256, 256, true>(p, w16, x, y, part, M, N, K, err, st);
        if (p.bn == 256) return launch_gemm_tc_cfg<128, 256, true>(p, w16, x, y, part, M, N, K, err, st);
        if (p.bn == 128) return launch_gemm_tc_cfg<128, 128, true>(p, w16, x, y, part, M, N, K, err, st);
        return launch_gemm_tc_cfg<128, 64, true>(p, w16, x, y, part, M, N, K, err, st);
    }
    if (p.bn == 128) return launch_gemm_tc_cfg<128, 128, false>(p, w16, x, y, part, M, N, K, err, st);
    return launch_gemm_tc_cfg<128, 64, false>(p, w16, x, y, part, M, N, K, err, st);
}

int read_error_word(const void *p, unsigned int *out)
{
    const cudaError_t e = cudaMemcpy(out, p, sizeof(unsigned int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
        g_last_cuda_error = e;
        (void)cudaGetLastError();
        return ZT_ERR_DEVICE;
    }
    return ZT_OK;
}

}  // namespace

extern "C" {

int zt_q4_version(void) { return (1 << 16) | 6; }

const char *zt_q4_last_cuda_error(void)
{
    return g_last_cuda_error == cudaSuccess ? "" : cudaGetErrorName(g_last_cuda_error);
}

const char *zt_q4_strerror(int status)
{
    switch (status) {
    case ZT_OK: return "success";
    case ZT_ERR_INVALID_ARG: return "invalid argument (null pointer, or M/N/K out of range, or K % 32 != 0)";
    case ZT_ERR_MISALIGNED: return "pointer misaligned (qw and x need 16 bytes, workspace 16, logits/argmax 4, scales/y 2)";
    case ZT_ERR_WORKSPACE: return "workspace smaller than zt_q4_lmhead_workspace_bytes()";
    case ZT_ERR_LAUNCH: return "CUDA kernel launch failed";
    case ZT_ERR_UNSUPPORTED: return "shape is valid but exceeds this build's limits";
    case ZT_ERR_DEVICE: return "no usable CUDA device, or a device attribute query failed";
    default: return "unknown status";
    }
}

int zt_q4_gemv(const uint32_t *qw, const uint16_t *scales, const uint16_t *x, uint16_t *y, int M, int N,
               int K, void *stream)
{
    if (!qw || !scales || !x || !y) return ZT_ERR_INVALID_ARG;
    int rc = check_shapes(M, N, K, 1);
    if (rc) return rc;
    if (!aligned(qw, 16) || !aligned(x, 16) || !aligned(scales, 2) || !aligned(y, 2)) return ZT_ERR_MISALIGNED;
    return launch_q4<kEpiF16>(qw, scales, x, y, nullptr, M, N, K, stream, nullptr);
}

int zt_q4_gate_up_silu(const uint32_t *qw, const uint16_t *scales, const uint16_t *x, uint16_t *y, int M,
                       int N, int K, void *stream)
{
    if (!qw || !scales || !x || !y) return ZT_ERR_INVALID_ARG;
    int rc = check_shapes(M, N, K, 2);
    if (rc) return rc;
    if (!aligned(qw, 16) || !aligned(x, 16) || !aligned(scales, 2) || !aligned(y, 2)) return ZT_ERR_MISALIGNED;
    return launch_q4<kEpiGateUp>(qw, scales, x, y, nullptr, M, N, K, stream, nullptr);
}

size_t zt_q4_lmhead_workspace_bytes(int M, int N, int K)
{
    if (check_shapes(M, N, K, 1) != ZT_OK) return 0;
    return lmhead_ws_bytes(M);
}

int zt_q4_lmhead_argmax(const uint32_t *qw, const uint16_t *scales, const uint16_t *x, float *logits,
                        int32_t *argmax, void *workspace, size_t ws_bytes, int M, int N, int K, void *stream)
{
    if (!qw || !scales || !x || !logits || !argmax || !workspace) return ZT_ERR_INVALID_ARG;
    int rc = check_shapes(M, N, K, 1);
    if (rc) return rc;
    if (!aligned(qw, 16) || !aligned(x, 16) || !aligned(scales, 2) || !aligned(logits, 4) ||
        !aligned(argmax, 4) || !aligned(workspace, 16))
        return ZT_ERR_MISALIGNED;
    if (ws_bytes < lmhead_ws_bytes(M)) return ZT_ERR_WORKSPACE;
    float *ws_val = reinterpret_cast<float *>(workspace);
    int *ws_idx = reinterpret_cast<int *>(ws_val + (size_t)kMaxCtas * M);
    int grid = 0;
    rc = launch_q4<kEpiLogits>(qw, scales, x, logits, ws_val, M, N, K, stream, &grid);
    if (rc) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(M);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    clear_stale_error();
    const cudaError_t e = cudaLaunchKernelEx(&cfg, q4_argmax_reduce_kernel, (const float *)ws_val, (const int *)ws_idx,
                                             grid, M, argmax);
    if (e != cudaSuccess) {
        g_last_cuda_error = e;
        (void)cudaGetLastError();
        return ZT_ERR_LAUNCH;
    }
    return ZT_OK;
}

int zt_q4_lmhead_argmax_noalloc(const uint32_t *qw, const uint16_t *scales, const uint16_t *x, float *logits,
                                int32_t *argmax, int M, int N, int K, void *stream)
{
    if (!qw || !scales || !x || !logits || !argmax) return ZT_ERR_INVALID_ARG;
    const int rc = check_shapes(M, N, K, 1);
    if (rc) return rc;
    if (!aligned(qw, 16) || !aligned(x, 16) || !aligned(scales, 2) || !aligned(logits, 4) || !aligned(argmax, 4))
        return ZT_ERR_MISALIGNED;
    if (lmhead_ws_bytes(M) > kNoAllocScratchBytes) return ZT_ERR_WORKSPACE;
    void *scratch = noalloc_scratch();
    if (!scratch) return ZT_ERR_DEVICE;
    return zt_q4_lmhead_argmax(qw, scales, x, logits, argmax, scratch, kNoAllocScratchBytes, M, N, K, stream);
}

static size_t pass_ws_layout(const zt_q4_proj *projs, int n, int M, size_t *err_off, size_t *lm_off)
{
    const size_t counters = ((size_t)n * 4 + 15) & ~(size_t)15;
    if (err_off) *err_off = counters;
    if (lm_off) *lm_off = counters + 16;
    size_t bytes = counters + 16;
    for (int i = 0; i < n; ++i)
        if (projs[i].kind == ZT_Q4_LM_HEAD) bytes += lmhead_ws_bytes(M);
    return bytes;
}

size_t zt_q4_pass_workspace_bytes(const zt_q4_proj *projs, int n, int M)
{
    if (!projs || n < 1 || n > ZT_Q4_PASS_MAX || M < 1 || M > 16) return 0;
    return pass_ws_layout(projs, n, M, nullptr, nullptr);
}

static int pass_impl(const zt_q4_proj *projs, int n, int M, void *workspace, size_t ws_bytes, void *stream,
                     int withhold, int chk_cut = 0)
{
    if (!projs || !workspace || n < 1 || n > ZT_Q4_PASS_MAX || M < 1 || M > 16) return ZT_ERR_INVALID_ARG;
    bool cooperative = false;
    for (int i = 0; i < n; ++i) {
        const zt_q4_proj &q = projs[i];
        if (!q.qw || !q.scales || !q.out || (!q.x && !q.norm)) return ZT_ERR_INVALID_ARG;
        if (q.kind != ZT_Q4_GEMV && q.kind != ZT_Q4_GATE_UP_SILU && q.kind != ZT_Q4_LM_HEAD) return ZT_ERR_INVALID_ARG;
        if (q.kind == ZT_Q4_LM_HEAD && !q.argmax) return ZT_ERR_INVALID_ARG;
        const int rc = check_shapes(M, q.N, q.K, q.kind == ZT_Q4_GATE_UP_SILU ? 2 : 1);
        if (rc) return rc;
        if (q.norm) {
            const zt_q4_norm &nm = *q.norm;
            if (!nm.residual || !nm.gamma || !(nm.eps >= 0.f) || nm.eps > 3.0e38f) return ZT_ERR_INVALID_ARG;
            if (!aligned(nm.residual, 16) || !aligned(nm.delta, 16) || !aligned(nm.gamma, 16) ||
                !aligned(nm.residual_out, 16) || !aligned(nm.x_out, 16))
                return ZT_ERR_MISALIGNED;
            const uintptr_t bytes = (uintptr_t)M * (uintptr_t)q.K * 2;
            auto overlap = [bytes](const void *a, const void *b) {
                const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
                return a && b && pa < pb + bytes && pb < pa + bytes;
            };
            if (overlap(nm.residual_out, nm.residual) || overlap(nm.residual_out, nm.delta)) return ZT_ERR_INVALID_ARG;
        }
        if (q.ld_out != 0 && q.ld_out < q.N) return ZT_ERR_INVALID_ARG;
        if (q.group != 0 && q.group != 32 && q.group != 64 && q.group != 128) return ZT_ERR_INVALID_ARG;
        if (q.group != 0 && q.K % q.group) return ZT_ERR_INVALID_ARG;
        if (q.rope) {
            const zt_q4_rope &rp = *q.rope;
            if (q.kind != ZT_Q4_GEMV || !rp.pos || rp.head_dim < 2 || rp.head_dim % 2 || q.N % rp.head_dim ||
                !(rp.theta > 0.f) || rp.theta > 3.0e38f)
                return ZT_ERR_INVALID_ARG;
            if (!aligned(rp.pos, 4)) return ZT_ERR_MISALIGNED;
        }
        if (!aligned(q.qw, 16) || !aligned(q.x, 16) || !aligned(q.scales, 2) ||
            !aligned(q.out, q.kind == ZT_Q4_LM_HEAD ? 4 : 2) || (q.argmax && !aligned(q.argmax, 4)))
            return ZT_ERR_MISALIGNED;
        if (i > 0 && q.wait) cooperative = true;
    }
    if (!aligned(workspace, 16)) return ZT_ERR_MISALIGNED;
    size_t err_off = 0, lm_off = 0;
    if (ws_bytes < pass_ws_layout(projs, n, M, &err_off, &lm_off)) return ZT_ERR_WORKSPACE;

    static thread_local PassArgs<kPassMax> a;    // ~32 KB: kept off the stack
    unsigned char *ws = reinterpret_cast<unsigned char *>(workspace);
    a.n = n;
    a.M = M;
    a.counters = cooperative ? reinterpret_cast<unsigned int *>(ws) : nullptr;
    a.error = reinterpret_cast<unsigned int *>(ws + err_off);
    a.withhold = cooperative ? withhold : -1;
    a.chk_cut = chk_cut;
    size_t lm = lm_off;
    for (int i = 0; i < n; ++i) {
        const zt_q4_proj &q = projs[i];
        PassProj &p = a.p[i];
        p.qw = reinterpret_cast<const uint4 *>(q.qw);
        p.scales = reinterpret_cast<const __half *>(q.scales);
        p.x = reinterpret_cast<const __half *>(q.x);
        p.out = q.out;
        p.N = q.N;
        p.K = q.K;
        p.G = q.K / kGroup;
        p.kind = q.kind == ZT_Q4_GEMV ? kEpiF16 : q.kind == ZT_Q4_GATE_UP_SILU ? kEpiGateUp : kEpiLogits;
        p.gsh = q.group == 64 ? 1 : q.group == 128 ? 2 : 0;
        p.scales_async = (q.K % 256 == 0) && aligned(q.scales, 16 >> p.gsh);
        p.wait = (i > 0 && q.wait) ? 1 : 0;
        p.norm = q.norm ? 1 : 0;
        p.res = q.norm ? reinterpret_cast<const __half *>(q.norm->residual) : nullptr;
        p.dlt = q.norm ? reinterpret_cast<const __half *>(q.norm->delta) : nullptr;
        p.gamma = q.norm ? reinterpret_cast<const __half *>(q.norm->gamma) : nullptr;
        p.res_out = q.norm ? reinterpret_cast<__half *>(q.norm->residual_out) : nullptr;
        p.x_out = q.norm ? reinterpret_cast<__half *>(q.norm->x_out) : nullptr;
        p.eps = q.norm ? q.norm->eps : 0.f;
        p.ldo = q.ld_out ? q.ld_out : q.N;
        p.pos = nullptr;
        p.theta = 0.f;
        p.rope_d = 0;
        if (q.rope) {
            p.kind = kEpiRope;
            p.N = q.N / 2;                    // pairs
            p.pos = q.rope->pos;
            p.rope_d = q.rope->head_dim;
            p.theta = q.rope->theta;
        }
        p.ws_val = nullptr;
        if (q.kind == ZT_Q4_LM_HEAD) {
            p.ws_val = reinterpret_cast<float *>(ws + lm);
            lm += lmhead_ws_bytes(M);
        }
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    clear_stale_error();
    // counters + error bits; a list without waits has no counters and can set no error bit, so
    // its kernel clears the error word itself (one launch fewer per call)
    cudaError_t e = cooperative ? cudaMemsetAsync(ws, 0, err_off + 16, st) : cudaSuccess;
    if (e != cudaSuccess) {
        g_last_cuda_error = e;
        (void)cudaGetLastError();
        return ZT_ERR_LAUNCH;
    }
    int g_max = 0;
    for (int i = 0; i < n; ++i) g_max = std::max(g_max, projs[i].K / kGroup);
    a.colsplit = pass_colsplit(M, g_max, n) ? 1 : 0;
    int grid = 0;
    const int rc = M == 1                   ? launch_pass<1, kPassMax, true>(a, cooperative, st, &grid)
                   : (M <= 8 || a.colsplit) ? launch_pass<1, kPassMax, false>(a, cooperative, st, &grid)
                                            : launch_pass<2, kPassMax, false>(a, cooperative, st, &grid);
    if (rc) return rc;
    for (int i = 0; i < n; ++i) {
        if (projs[i].kind != ZT_Q4_LM_HEAD) continue;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(M);
        cfg.blockDim = dim3(256);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, q4_argmax_reduce_kernel, (const float *)a.p[i].ws_val,
                               (const int *)(a.p[i].ws_val + (size_t)kMaxCtas * M), grid, M, projs[i].argmax);
        if (e != cudaSuccess) {
            g_last_cuda_error = e;
            (void)cudaGetLastError();
            return ZT_ERR_LAUNCH;
        }
    }
    return ZT_OK;
}

int zt_q4_pass_plan(int M, int K_max, int n, int *ctas_per_sm, int *stages, int *k_window, int *column_blocks,
                    int *warps_per_cta)
{
    if (!ctas_per_sm || !stages || !k_window || !column_blocks || !warps_per_cta) return ZT_ERR_INVALID_ARG;
    if (M < 1 || M > 16 || n < 1 || n > ZT_Q4_PASS_MAX || K_max < kGroup || K_max % kGroup) return ZT_ERR_INVALID_ARG;
    const bool split = pass_colsplit(M, K_max / kGroup, n);
    const PassPlan plan = pass_plan(split ? (M + 1) / 2 : M, K_max / kGroup, n, (M <= 8 || split) ? 1 : 2);
    if (plan.cps == 0) return ZT_ERR_UNSUPPORTED;
    *ctas_per_sm = plan.cps;
    *stages = plan.stages;
    *k_window = plan.win ? plan.g_stage * kGroup : 0;
    *column_blocks = split ? 2 : 1;
    *warps_per_cta = plan.mw;
    return ZT_OK;
}

int zt_q4_pass(const zt_q4_proj *projs, int n, int M, void *workspace, size_t ws_bytes, void *stream)
{
    return pass_impl(projs, n, M, workspace, ws_bytes, stream, -1);
}

int zt_q4_pass_test_withhold(const zt_q4_proj *projs, int n, int M, void *workspace, size_t ws_bytes, void *stream)
{
    bool waits = false;
    for (int i = 1; projs && i < n && i <= ZT_Q4_PASS_MAX; ++i) waits = waits || projs[i].wait;
    if (!waits) return ZT_ERR_INVALID_ARG;
    return pass_impl(projs, n, M, workspace, ws_bytes, stream, 0);
}

int zt_q4_pass_test_cut(const zt_q4_proj *projs, int n, int M, void *workspace, size_t ws_bytes, void *stream,
                        int rows)
{
    if (!kChecked) return ZT_ERR_UNSUPPORTED;
    if (rows < 1) return ZT_ERR_INVALID_ARG;
    return pass_impl(projs, n, M, workspace, ws_bytes, stream, -1, rows);
}

int zt_q4_build_flags(void) { return kChecked ? ZT_Q4_BUILD_CHECKED : 0; }

int zt_q4_pass_errors(const void *workspace, int n, unsigned int *out)
{
    if (!workspace || !out || n < 1 || n > ZT_Q4_PASS_MAX) return ZT_ERR_INVALID_ARG;
    const size_t err_off = ((size_t)n * 4 + 15) & ~(size_t)15;
    const cudaError_t e = cudaMemcpy(out, reinterpret_cast<const unsigned char *>(workspace) + err_off,
                                     sizeof(unsigned int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
        g_last_cuda_error = e;
        (void)cudaGetLastError();
        return ZT_ERR_DEVICE;
    }
    return ZT_OK;
}

int zt_q4_dequant_f16(const uint32_t *qw, const uint16_t *scales, uint16_t *w16, int N, int K, int group,
                      void *stream)
{
    if (!qw || !scales || !w16) return ZT_ERR_INVALID_ARG;
    if (check_gemm_shapes(1, N, K) != ZT_OK) return ZT_ERR_INVALID_ARG;
    const int gsh = group_shift(K, group);
    if (gsh < 0) return ZT_ERR_INVALID_ARG;
    if (!aligned(qw, 16) || !aligned(w16, 16) || !aligned(scales, 2)) return ZT_ERR_MISALIGNED;
    return launch_dequant(qw, scales, w16, N, K, gsh, nullptr, static_cast<cudaStream_t>(stream));
}

size_t zt_q4_gemm_f16w_workspace_bytes(int M, int N, int K)
{
    if (check_gemm_shapes(M, N, K) != ZT_OK) return 0;
    return f16w_ws_bytes(M, N, K);
}

int zt_q4_gemm_f16w(const uint16_t *w16, const uint16_t *x, uint16_t *y, int M, int N, int K, void *workspace,
                    size_t ws_bytes, void *stream)
{
    if (!w16 || !x || !y || !workspace) return ZT_ERR_INVALID_ARG;
    int rc = check_gemm_shapes(M, N, K);
    if (rc) return rc;
    if (!aligned(w16, 16) || !aligned(x, 16) || !aligned(y, 2) || !aligned(workspace, 16)) return ZT_ERR_MISALIGNED;
    if (ws_bytes < f16w_ws_bytes(M, N, K)) return ZT_ERR_WORKSPACE;
    if (!gemm_grid_ok(gemm_plan(M, N, K), M, N, false)) return ZT_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    clear_stale_error();
    const cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(unsigned int), st);
    if (e != cudaSuccess) {
        g_last_cuda_error = e;
        (void)cudaGetLastError();
        return ZT_ERR_LAUNCH;
    }
    return launch_gemm_tc(w16, x, y, M, N, K, workspace, st);
}

size_t zt_q4_gemm_workspace_bytes(int M, int N, int K)
{
    if (check_gemm_shapes(M, N, K) != ZT_OK) return 0;
    return w16_bytes(N, K) + f16w_ws_bytes(M, N, K);
}

int zt_q4_gemm(const uint32_t *qw, const uint16_t *scales, const uint16_t *x, uint16_t *y, int M, int N, int K,
               int group, void *workspace, size_t ws_bytes, void *stream)
{
    if (!qw || !scales || !x || !y || !workspace) return ZT_ERR_INVALID_ARG;
    int rc = check_gemm_shapes(M, N, K);
    if (rc) return rc;
    const int gsh = group_shift(K, group);
    if (gsh < 0) return ZT_ERR_INVALID_ARG;
    if (!aligned(qw, 16) || !aligned(x, 16) || !aligned(workspace, 16) || !aligned(scales, 2) || !aligned(y, 2))
        return ZT_ERR_MISALIGNED;
    if (ws_bytes < w16_bytes(N, K) + f16w_ws_bytes(M, N, K)) return ZT_ERR_WORKSPACE;
    if (!gemm_grid_ok(gemm_plan(M, N, K), M, N, false)) return ZT_ERR_UNSUPPORTED;
    uint16_t *w16 = static_cast<uint16_t *>(workspace);
    void *gws = static_cast<unsigned char *>(workspace) + w16_bytes(N, K);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = launch_dequant(qw, scales, w16, N, K, gsh, static_cast<unsigned int *>(gws), st);
    if (rc) return rc;
    return launch_gemm_tc(w16, x, y, M, N, K, gws, st);
}

int zt_q4_gemm_f16w_errors(const void *workspace, unsigned int *out)
{
    if (!workspace || !out) return ZT_ERR_INVALID_ARG;
    return read_error_word(workspace, out);
}

int zt_q4_gemm_errors(const void *workspace, int N, int K, unsigned int *out)
{
    if (!workspace || !out || check_gemm_shapes(1, N, K) != ZT_OK) return ZT_ERR_INVALID_ARG;
    return read_error_word(static_cast<const unsigned char *>(workspace) + w16_bytes(N, K), out);
}

size_t zt_q4_gemm_gate_up_workspace_bytes(int M, int N, int K)
{
    if (N > INT_MAX / 2 || check_gemm_shapes(M, 2 * N, K) != ZT_OK) return 0;
    return w16_bytes(2 * N, K) + 256;
}

int zt_q4_gemm_f16w_gate_up_silu(const uint16_t *w16, const uint16_t *x, uint16_t *y, int M, int N, int K,
                                 void *workspace, size_t ws_bytes, void *stream)
{
    if (!w16 || !x || !y || !workspace) return ZT_ERR_INVALID_ARG;
    if (N > INT_MAX / 2) return ZT_ERR_INVALID_ARG;
    int rc = check_gemm_shapes(M, 2 * N, K);
    if (rc) return rc;
    if (!aligned(w16, 16) || !aligned(x, 16) || !aligned(y, 2) || !aligned(workspace, 16)) return ZT_ERR_MISALIGNED;
    if (ws_bytes < 256) return ZT_ERR_WORKSPACE;
    if (!gemm_grid_ok(gate_up_plan(M, N, K), M, N, true)) return ZT_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    clear_stale_error();
    const cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(unsigned int), st);
    if (e != cudaSuccess) {
        g_last_cuda_error = e;
        (void)cudaGetLastError();
        return ZT_ERR_LAUNCH;
    }
    return launch_gate_up_tc(w16, x, y, M, N, K, workspace, st);
}

int zt_q4_gemm_gate_up_silu(const uint32_t *qw, const uint16_t *scales, const uint16_t *x, uint16_t *y, int M,
                            int N, int K, int group, void *workspace, size_t ws_bytes, void *stream)
{
    if (!qw || !scales || !x || !y || !workspace) return ZT_ERR_INVALID_ARG;
    if (N > INT_MAX / 2) return ZT_ERR_INVALID_ARG;
    int rc = check_gemm_shapes(M, 2 * N, K);
    if (rc) return rc;
    const int gsh = group_shift(K, group);
    if (gsh < 0) return ZT_ERR_INVALID_ARG;
    if (!aligned(qw, 16) || !aligned(x, 16) || !aligned(workspace, 16) || !aligned(scales, 2) || !aligned(y, 2))
        return ZT_ERR_MISALIGNED;
    if (ws_bytes < w16_bytes(2 * N, K) + 256) return ZT_ERR_WORKSPACE;
    if (!gemm_grid_ok(gate_up_plan(M, N, K), M, N, true)) return ZT_ERR_UNSUPPORTED;
    uint16_t *w16 = static_cast<uint16_t *>(workspace);
    void *gws = static_cast<unsigned char *>(workspace) + w16_bytes(2 * N, K);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = launch_dequant(qw, scales, w16, 2 * N, K, gsh, static_cast<unsigned int *>(gws), st);
    if (rc) return rc;
    return launch_gate_up_tc(w16, x, y, M, N, K, gws, st);
}

int zt_q4_pack_host(const uint8_t *q, int N, int K, uint32_t *qw)
{
    if (!q || !qw || N < 1 || K < 8 || K % 8) return ZT_ERR_INVALID_ARG;
    const int64_t W = K / 8;
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *src = q + n * (int64_t)K;
        for (int64_t w = 0; w < W; ++w) {
            uint32_t word = 0;
            for (int j = 0; j < 8; ++j) {
                const uint32_t c = src[8 * w + j];
                if (c > 15u) return ZT_ERR_INVALID_ARG;
                word |= c << (4 * j);
            }
            qw[n * W + w] = word;
        }
    }
    return ZT_OK;
}

int zt_q4_unpack_host(const uint32_t *qw, int N, int K, uint8_t *q)
{
    if (!q || !qw || N < 1 || K < 8 || K % 8) return ZT_ERR_INVALID_ARG;
    const int64_t W = K / 8;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t w = 0; w < W; ++w) {
            const uint32_t word = qw[n * W + w];
            for (int j = 0; j < 8; ++j) q[n * (int64_t)K + 8 * w + j] = (uint8_t)((word >> (4 * j)) & 0xFu);
        }
    return ZT_OK;
}

}  // extern "C"
