// q4_pass.cuh -- persistent executor for a list of q4f16 projections (one
// launch for a whole decode weight pass), built on the tensor-core GEMV of
// q4_mma.cuh.
//
// Operation: a sequence of the int4 dequantizing matrix products of the
// Zero-TVM write-up (section "完整的推理流水线": the projections of each of the
// 32 decoder layers, then the f32-output LM head) with the fused FFN of section
// "内核融合".  A single projection is the one-element case; every public entry
// point of the library runs through this kernel.
//
// Why one launch for many projections: each projection streams 5..56 MB,
// i.e. 1..9 us of HBM time, comparable to what a boundary costs (activation
// staging, reductions, tail: ~3 us measured per projection when every CTA
// takes a slice of every projection).  So the list is cut into PHASES at the
// projections that must wait for earlier outputs; the projections inside a
// phase are independent, and their rows, concatenated, are split into one
// contiguous, byte-balanced range per CTA.  A CTA then meets only the two or
// three projection boundaries inside its own range, and its warps' cp.async
// streams run straight from one projection's weights into the next one's --
// across phase boundaries too, since weights never depend on earlier outputs.
//
// Cross-CTA waits: phase k > 0 starts only when every CTA has finished phase
// k - 1 (counters[k-1] counts them).  Such a launch is cooperative (all CTAs
// co-resident) and the wait is bounded: after 2 s the CTA records an error
// bit, stops, lets its own copies land and exits.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

#include "q4_mma.cuh"

namespace zt {

constexpr int kPassMax = 192;                       // projections per launch
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
constexpr unsigned kErrWaitExpired = 1u;
constexpr unsigned kErrBounds = 2u;

// Bounds-checked build (compiled with -DZT_Q4_CHECKED): before every global access whose
// address the kernel computes (weight and scale copies and loads, output and workspace
// stores) and every read of the shared partial buffer, the index is compared with the
// extent of its buffer; an index outside it sets kErrBounds in the error word and the
// access is skipped, so a wrong index shows as an error bit, never as a fault.  The
// default build compiles the comparisons out.
#ifdef ZT_Q4_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif

// weight rows of a projection: gate_up and RoPE projections hold two rows per output
__host__ __device__ constexpr int pass_weight_rows(int kind, int N)
{
    return (kind == kEpiGateUp || kind == kEpiRope) ? 2 * N : N;
}

struct PassProj {
    const uint4 *qw;            // [rows][G] 16-byte chunks
    const __half *scales;       // [rows][G]
    const __half *x;            // [M][K]
    void *out;                  // fp16 [M][ldo] (gemv, gate/up, RoPE) or f32 [M][ldo] (LM head)
    float *ws_val;              // LM head: per-CTA maximum [gridDim.x][M], then the arg-max as int
                                // at ws_val + kMaxCtas * M (pass_ws_idx)
    // residual add + RMSNorm prologue (norm != 0): x = fp16(h * gamma / rms(h)),
    // h = fp16(res + dlt); res_out / x_out receive h / x (the CTA holding row 0)
    const __half *res, *dlt, *gamma;
    __half *res_out, *x_out;
    // RoPE epilogue (kind kEpiRope): pairs (i, i + d/2) of each head of d rows
    // turned by pos[m] * theta^(-2i/d); N counts pairs
    const int *pos;
    int N, K, G, kind;          // kind: kEpiF16 / kEpiGateUp / kEpiLogits / kEpiRope (N: outputs, pairs for RoPE)
    int ldo;                    // elements between output rows
    int row_bytes;              // HBM bytes per output (codes + scales of its weight rows)
    int scales_async;           // scales copied by cp.async (16-byte aligned rows)
    int wait;                   // starts a phase: wait for all earlier projections
    int norm;
    int rope_d;
    int gsh;                    // log2(group / 32): 0, 1, 2 for 32, 64, 128 k per scale
    float eps;
    float theta;
};

__device__ __forceinline__ int *pass_ws_idx(const PassProj &P, int M)
{
    return reinterpret_cast<int *>(P.ws_val + (size_t)kMaxCtas * M);
}

// PMAX bounds the list: 1 for the single-call entry points (a small kernel
// parameter block), kPassMax for zt_q4_pass.
template <int PMAX>
struct PassArgs {
    int n, M, phases;
    int g_stage;                // groups of K per column the activation area holds: the largest G of
                                // the list, or (windowed kernel) the K window of longer projections
    unsigned int *counters;     // [phases - 1], zero at launch (only when phases > 1)
    unsigned int *error;        // error bits
    int withhold;               // test hook: CTA 0 does not count this phase done (-1: none)
    int red_floats;             // size of the WK partial buffer (floats)
    int chk_cut;                // test hook of the checked build: weight rows taken off every projection's
                                // extent, so that the last rows' checks fire (0: none)
    int colsplit;               // M > 8 as two column blocks: CTAs 2s and 2s + 1 take row share s, tokens
                                // 0 .. ceil(M/2) - 1 and the rest (each an M <= 8 problem of 5..8 tokens)
    // What every CTA reads to find its rows, kept apart from p[] in dense arrays: a warp
    // reading one entry per lane then touches a few consecutive constant-cache lines,
    // not one line per lane.
    long long pbeg[PMAX + 1];   // HBM byte offset of projection i's rows in the list; pbeg[n]: the total
    long long phbeg[PMAX + 1];  // HBM byte offset where phase i starts; phbeg[phases]: the total
    int pphase[PMAX];           // phase of projection i
    unsigned lm_bits[(PMAX + 31) / 32];   // bit i: projection i is an LM head
    PassProj p[PMAX];
};

// WK > 1 partial buffer: (tiles x WK) warp tiles of 16 rows x 8 NT columns
// per segment.  The LM head's per-thread maxima reuse it once a segment's
// partial sums have been read.
// Its size in floats is a launch parameter: 128 per warp and n-tile (16-float partials with
// one column: 128 per warp), or, where shared memory is short (16 warps, several columns),
// the least that still holds the LM head's maxima (2 x MW x 8 NT words) with room for some
// K splitting: 1024 per n-tile.
__host__ __device__ constexpr int pass_red_floats(int NT, int MW, bool ONE) { return ONE ? 128 * MW : 128 * MW * NT; }
__host__ __device__ constexpr int pass_red_floats_min(int NT, bool ONE) { return ONE ? 128 * 16 : 1024 * NT; }
static_assert(2 * 16 * 8 * 2 <= pass_red_floats_min(2, false) && 2 * 16 * 8 <= pass_red_floats_min(1, true),
              "LM-head maxima must fit the partial buffer");
constexpr int kPassMaxStages = 4;           // ring depths 2..4 are instantiated

// One projection's rows in one CTA, with the CTA's warp layout for them.
struct PassSeg {
    int p, o_begin, o_end, phase;           // rows [o_begin, o_end) of projection p
    int n_tiles, n_chunks, wkl, rout;       // warp tiles, K chunks, log2 of the K-splitting warps
};

// Shared memory per CTA: rings, permuted activations (n-stride g_stage*64 +
// 32 bytes), C-operand table, WK partials / LM-head maxima, segment list,
// flags, the RMSNorm factors of a windowed segment (16 floats).
__host__ __device__ inline size_t pass_smem_bytes(int M, int g_stage, int stages, int n, int NT, int MW,
                                                   int red_floats)
{
    const size_t ring = (size_t)MW * stages * kMStage + 1024;   // + alignment of the code stages
    // M = 1: the block-diagonal layout (a zero block, 80 bytes per group, one C float per group)
    const size_t xp = M == 1 ? bd_area_bytes(round8(g_stage), MW == 16) : (size_t)M * ((size_t)g_stage * 64 + 32);
    const size_t x7 = M == 1 ? bd_ctable_bytes(round8(g_stage), MW == 16) : (size_t)g_stage * NT * 64;
    return ring + ((xp + 15) & ~(size_t)15) + x7 + (size_t)red_floats * 4 + (size_t)n * sizeof(PassSeg) +
           (MW + 4) * sizeof(int) + 16 * sizeof(float);
}

// Per-segment geometry of one warp.
struct PassGeo {
    int o_begin, o_end, rout, n_tiles, n_chunks, wk, wr_n, my_wk, my_wr, my_tiles, my_chunks;
};

static_assert(kPassMax <= 8 * 32, "one thread per projection builds the segment list");
static_assert(sizeof(PassArgs<kPassMax>) <= 32764, "the list must fit the kernel parameter block");

// log2 of the warps splitting K for a segment: minimise the items of the
// busiest warp (tiles per row-warp x chunks per K-warp), ties -> fewer
// K-warps.  LW: log2 of the CTA's warps.  `bounded`: the whole segment's
// partials meet at once, so the partial buffer bounds them (tiles * WK * the
// floats of one partial <= pass_red_floats); a windowed segment reduces one
// round of at most (warps / WK) tiles at a time.  A partial is 16 rows x 8 NT
// columns, or 16 row sums with a single column (ONE).
template <int LW, bool ONE>
__device__ __forceinline__ int pick_wkl(int n_tiles, int n_chunks, int NT, bool bounded, int red_floats)
{
    constexpr int kPart = ONE ? kMTileRows : kMTileRows * 8;
    int best = 0, best_cost = -1;
#pragma unroll
    for (int wkl = 0; wkl <= LW; ++wkl) {
        const int wk = 1 << wkl;
        if (wk > n_chunks) break;
        if (bounded && wkl > 0 && n_tiles * wk * kPart * (ONE ? 1 : NT) > red_floats) break;
        const int cost = ((n_tiles + ((1 << LW) >> wkl) - 1) >> (LW - wkl)) * ((n_chunks + wk - 1) >> wkl);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = wkl;
        }
    }
    return best;
}

template <int LW>
__device__ __forceinline__ PassGeo pass_geo(const PassSeg &sg, int warp)
{
    PassGeo g;
    g.o_begin = sg.o_begin;
    g.o_end = sg.o_end;
    g.rout = sg.rout;
    g.n_tiles = sg.n_tiles;
    g.n_chunks = sg.n_chunks;
    g.wk = 1 << sg.wkl;
    g.wr_n = (1 << LW) >> sg.wkl;
    g.my_wk = warp & (g.wk - 1);
    g.my_wr = warp >> sg.wkl;
    g.my_tiles = g.my_wr < g.n_tiles ? (g.n_tiles - g.my_wr + g.wr_n - 1) >> (LW - sg.wkl) : 0;
    g.my_chunks = g.my_wk < g.n_chunks ? (g.n_chunks - g.my_wk + g.wk - 1) >> sg.wkl : 0;
    if (g.my_chunks == 0) g.my_tiles = 0;
    return g;
}

// weight row of tile slot r (0..15) of the tile starting at output o0.  Gate/up
// and RoPE tiles hold 8 outputs: slots 0..7 their first rows, 8..15 the
// partner rows (up rows; the second feature of each RoPE pair).
__device__ __forceinline__ int pass_slot_row(int kind, int N, int rope_d, int o_end, int o0, int r, bool &valid)
{
    if (kind == kEpiRope) {
        const int o = min(o0 + (r & 7), N - 1), half = rope_d >> 1;
        valid = o0 + (r & 7) < o_end;
        const int h = o / half, i = o - h * half;
        return h * rope_d + i + (r < 8 ? 0 : half);
    }
    if (kind == kEpiGateUp) {
        const int o = o0 + (r & 7);
        valid = o < o_end;
        return (r < 8 ? 0 : N) + min(o, N - 1);
    }
    const int o = o0 + r;
    valid = o < o_end;
    return min(o, N - 1);
}

// groups in the last chunk this warp reads of a segment (8 unless G % 8 != 0
// and that chunk is the projection's last)
__device__ __forceinline__ int pass_last_kc(const PassGeo &g, int G)
{
    const int c_last = g.my_wk + g.wk * (g.my_chunks - 1);
    return min(kMChunkG, G - c_last * kMChunkG);
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned int *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Wait until *counter >= target; false after kWaitLimitNs.
__device__ __forceinline__ bool wait_counter(const unsigned int *counter, unsigned target)
{
    if (ld_acquire_u32(counter) >= target) return true;
    unsigned long long t0;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t0));
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i) {
            __nanosleep(200);
            if (ld_acquire_u32(counter) >= target) return true;
        }
        unsigned long long t;
        asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
        if (t - t0 > kWaitLimitNs) return false;
    }
}

// Scales of an item for groups of 64 (gsh 1) or 128 (gsh 2) k: the first 4
// (or 2) halves of the slot, each repeated so that half j is block j's scale.
__device__ __forceinline__ uint4 spread_scales(uint4 v, int gsh)
{
    if (gsh == 1)
        return make_uint4(__byte_perm(v.x, 0, 0x1010), __byte_perm(v.x, 0, 0x3232), __byte_perm(v.y, 0, 0x1010),
                          __byte_perm(v.y, 0, 0x3232));
    const uint32_t a = __byte_perm(v.x, 0, 0x1010), b = __byte_perm(v.x, 0, 0x3232);
    return make_uint4(a, a, b, b);
}

// RoPE epilogue of one pair: a, b = the pair's two projections (fp32 sums),
// turned by pos * theta^(-2i/d) in double and rounded once to fp16.  Out of
// line: the double-precision pow / sincos stay out of the hot loop's register
// allocation (inlined, they cost the plain projections ~5 %).
__device__ __noinline__ void rope_store(__half *out, size_t row_off, int pair, int d, float theta, int pos,
                                           float a, float b)
{
    const int half = d >> 1, h = pair / half, i = pair - h * half;
    const double phi = (double)pos * pow((double)theta, -2.0 * i / d);
    double sn, cs;
    sincos(phi, &sn, &cs);
    const int n = h * d + i;
    out[row_off + n] = __double2half((double)a * cs - (double)b * sn);
    out[row_off + n + half] = __double2half((double)b * cs + (double)a * sn);
}

// NT: n-tiles of 8 activation columns (M <= 8 NT); ONE: M == 1, so the mma's
// odd columns are never read and their accumulation is skipped; S: ring depth;
// WIN: projections with more than g_stage groups stage their activations in
// K windows of g_stage groups (a multiple of 8): the CTA walks its tiles in
// rounds of one tile per warp, and each round stages the windows in turn
// while the warps' accumulators carry over (the weight stream's order is the
// same as without windows).
template <int NT, int PMAX, int S, bool ONE, bool WIN, int MW>
__global__ void __launch_bounds__(MW * 32, MW == 16 ? 1 : 2) q4_pass_kernel(const __grid_constant__ PassArgs<PMAX> a)
{
    static_assert(MW == 8 || MW == 16, "8 or 16 warps per CTA");
    constexpr int kMW = MW, kMThreads = MW * 32, LW = MW == 16 ? 4 : 3;
    constexpr bool PAIRED = ONE && MW == 16;   // the paired single-column layout (q4_mma.cuh)
    static_assert(S >= 2 && S <= kPassMaxStages, "ring depth");
    static_assert(!ONE || NT == 1, "one column fits one n-tile");
    extern __shared__ __align__(1024) unsigned char smem[];
    // checked build: false (and the error bit) for an index outside its buffer; else always true
    auto chk = [&](bool in_bounds) -> bool {
        if constexpr (kChecked) {
            if (!in_bounds && a.error) atomicOr(a.error, kErrBounds);
            return in_bounds;
        } else {
            return true;
        }
    };
    // this CTA's tokens (columns) and row share: with the column split, tokens m0 .. m0 + M - 1
    // of the list's Mt (the first ceil(Mt / 2) or the other floor(Mt / 2), so never a single
    // column: the staging helpers take M == 1 for the block-diagonal layout of ONE), and
    // share sb of nsb (two CTAs per share)
    const int Mt = a.M, n = a.n;
    const int cb = a.colsplit ? (int)(blockIdx.x & 1) : 0, m0 = cb * ((Mt + 1) >> 1);
    const int M = a.colsplit ? (cb ? Mt >> 1 : (Mt + 1) >> 1) : Mt;
    const int sb = a.colsplit ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int nsb = a.colsplit ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int qg = lane >> 2, qt = lane & 3;       // mma quad row / thread in quad

    // code stages [kMW][S][2048] start on a 1024-byte boundary (128-byte
    // swizzle), scale stages [kMW][S][256] follow, then the activations
    unsigned char *codes = smem + ((1024u - (smem_u32(smem) & 1023u)) & 1023u);
    unsigned char *ring_c = codes + (size_t)warp * S * kMCodeStage;
    unsigned char *ring_s = codes + (size_t)kMW * S * kMCodeStage + (size_t)warp * S * kMScaleStage;
    unsigned char *xp = codes + (size_t)kMW * S * kMStage;
    const size_t xp_bytes = ONE ? bd_area_bytes(round8(a.g_stage), PAIRED)
                                : ((size_t)M * ((size_t)a.g_stage * 64 + 32) + 15) & ~(size_t)15;
    float *x7 = reinterpret_cast<float *>(xp + xp_bytes);
    float *red = x7 + (ONE ? bd_ctable_bytes(round8(a.g_stage), PAIRED) / 4 : (size_t)a.g_stage * NT * 16);
    float *bvs = red;                                           // LM-head maxima reuse red
    int *bis = reinterpret_cast<int *>(bvs + kMW * 8 * NT);
    PassSeg *segs = reinterpret_cast<PassSeg *>(red + a.red_floats);
    int *wcount = reinterpret_cast<int *>(segs + n);           // [kMW] segments per warp
    volatile int *abort_flag = wcount + kMW;
    float *rn = reinterpret_cast<float *>(wcount + kMW + 4);   // RMSNorm factors of a windowed segment

    pdl_launch_dependents();

    // ---- this CTA's segments: per phase, its byte-balanced share of the
    //      phase's concatenated rows (a row belongs to the CTA whose share
    //      holds the row's first byte).  Thread p looks at projection p. ----
    bool neutral_max = false;   // an LM head this CTA has no rows of: write a neutral partial maximum
    {
        PassSeg mine{};
        bool has = false;
        if (tid < n) {
            const int ph = a.pphase[tid];
            const long long s0 = a.phbeg[ph], len = a.phbeg[ph + 1] - s0;
            const long long lo = s0 + len * sb / nsb, hi = s0 + len * (sb + 1) / nsb;
            const long long beg = a.pbeg[tid], end = a.pbeg[tid + 1];
            if (hi > beg && lo < end) {
                const PassProj &P = a.p[tid];
                const long long rb = P.row_bytes;
                const int o0 = lo > beg ? (int)((lo - beg + rb - 1) / rb) : 0;
                const int o1 = hi < end ? (int)((hi - beg + rb - 1) / rb) : P.N;
                if (o1 > o0) {
                    has = true;
                    mine.p = tid;
                    mine.o_begin = o0;
                    mine.o_end = o1;
                    mine.phase = ph;
                    mine.rout = (P.kind == kEpiGateUp || P.kind == kEpiRope) ? kMTileRows / 2 : kMTileRows;
                    mine.n_tiles = (o1 - o0 + mine.rout - 1) / mine.rout;
                    mine.n_chunks = (P.G + kMChunkG - 1) / kMChunkG;
                    mine.wkl = pick_wkl<LW, ONE>(mine.n_tiles, mine.n_chunks, NT, !(WIN && P.G > a.g_stage), a.red_floats);
                }
            }
            neutral_max = !has && ((a.lm_bits[tid >> 5] >> (tid & 31)) & 1u);
        }
        const unsigned ball = __ballot_sync(0xffffffffu, has);
        if (lane == 0) wcount[warp] = __popc(ball);
        if (tid == 0) *abort_flag = 0;
        if (ONE && tid < (PAIRED ? kBdZero : kBd1Zero) / 16)
            reinterpret_cast<uint4 *>(xp)[tid] = make_uint4(0, 0, 0, 0);   // the zero region
        __syncthreads();
        if (has) {
            int idx = __popc(ball & ((1u << lane) - 1u));
            for (int w = 0; w < warp; ++w) idx += wcount[w];
            segs[idx] = mine;
        }
    }
    int nseg = 0;
#pragma unroll
    for (int w = 0; w < kMW; ++w) nseg += wcount[w];
    __syncthreads();
    const int nphase = a.phases;

    const uint32_t ring_cu = smem_u32(ring_c), ring_su = smem_u32(ring_s);

    // ---------------------------------------------------------- issue side --
    // The warp's items of all segments form one stream (segment, tile,
    // chunk); lane l copies pieces l + 32 i (i < 4) of an item: tile row
    // l / 8 + 4 i, group l % 8 of the chunk.  The stream runs S - 1 items
    // ahead of the math, across segment and phase boundaries (weights never
    // depend on outputs).  Per item it only advances pointers; segment and
    // tile changes recompute them.
    // piece i: row l / 8 + 4 i, chunk pg at swizzled position pg ^ (row & 7);
    // rows + 8 sit 1024 bytes further with the same swizzle
    const int pg = lane & 7, l3 = lane >> 3;
    const uint32_t piece_u0 = ring_cu + l3 * 128 + ((pg ^ l3) << 4);               // rows l3, l3 + 8
    const uint32_t piece_u1 = ring_cu + (l3 + 4) * 128 + ((pg ^ (l3 + 4)) << 4);   // rows l3 + 4, l3 + 12
    const uint32_t scale_u = ring_su + lane * 16;
    int is_s = -1;                  // segment being issued
    int is_gsh = 0;                 // log2(group / 32) of its projection
    int is_tiles = 0;               // tiles left after the current one
    int is_chunks = 0;              // chunks left in the current tile (0: stream ended)
    int is_kc_last = kMChunkG;      // groups of the tile's last chunk
    int is_step = 0;                // uint4 per chunk step (WK chunks of 8 groups)
    int is_sstep = 0;               // scale elements per chunk step
    const uint4 *is_qlo = nullptr, *is_qhi = nullptr;      // checked build: the weight buffer
    const __half *is_slo = nullptr, *is_shi = nullptr;     // and the scale buffer of the segment
    uint32_t is_st = 0;             // ring stage of the next item to issue
    int is_o0 = 0, is_rstep = 0;    // current tile's first output, outputs per tile step
    PassGeo ig{};
    const uint4 *src_w[4];          // the next chunk's source, per piece
    bool ok_w[4];
    const __half *src_s = nullptr;
    bool ok_s = false;
    // the tile's last chunk holds only is_kc_last groups (K % 256 != 0): drop the other pieces
    auto last_chunk = [&]() {
        if (is_kc_last < kMChunkG) {
#pragma unroll
            for (int i = 0; i < 4; ++i) ok_w[i] = ok_w[i] && pg < is_kc_last;
        }
    };
    auto set_tile = [&]() {
        const PassProj &P = a.p[segs[is_s].p];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int row = pass_slot_row(P.kind, P.N, P.rope_d, ig.o_end, is_o0, (lane >> 3) + 4 * i, ok_w[i]);
            src_w[i] = P.qw + (size_t)row * P.G + ig.my_wk * kMChunkG + pg;
        }
        ok_s = false;
        const int row = pass_slot_row(P.kind, P.N, P.rope_d, ig.o_end, is_o0, lane & 15, ok_s);
        ok_s = ok_s && lane < kMTileRows && P.scales_async;
        src_s = P.scales + (size_t)row * (P.G >> P.gsh) + ((ig.my_wk * kMChunkG) >> P.gsh);
        if constexpr (kChecked) {
            const int rows = pass_weight_rows(P.kind, P.N);
            is_qlo = P.qw;
            is_qhi = P.qw + (size_t)max(rows - a.chk_cut, 0) * P.G;
            is_slo = P.scales;
            is_shi = P.scales + (size_t)rows * (P.G >> P.gsh);
        }
        is_gsh = P.gsh;
        is_sstep = is_step >> P.gsh;
        is_chunks = ig.my_chunks;
        if (is_chunks == 1) last_chunk();
    };
    // this warp's next tile: the current segment's next one, else the first one of the next
    // segment that has any for this warp (is_chunks 0: the stream has ended).  One place for
    // every tile change keeps the code small where issue_next is inlined.
    auto advance = [&]() {
        if (is_tiles > 0) {
            --is_tiles;
            is_o0 += is_rstep;
        } else {
            for (;;) {
                if (++is_s >= nseg) {
                    is_chunks = 0;
                    return;
                }
                ig = pass_geo<LW>(segs[is_s], warp);
                if (ig.my_tiles > 0) break;
            }
            is_tiles = ig.my_tiles - 1;
            is_kc_last = pass_last_kc(ig, a.p[segs[is_s].p].G);
            is_step = ig.wk * kMChunkG;
            is_rstep = ig.wr_n * ig.rout;
            is_o0 = ig.o_begin + ig.my_wr * ig.rout;
        }
        set_tile();
    };
    advance();
    auto issue_next = [&]() {
        if (is_chunks > 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (ok_w[i] && chk(src_w[i] >= is_qlo && src_w[i] < is_qhi))
                    cp_async16_u32(((i & 1) ? piece_u1 : piece_u0) + (is_st << 11) + (i >> 1) * 1024, src_w[i]);
            if (ok_s && chk(src_s >= is_slo && src_s + (16 >> (1 + is_gsh)) <= is_shi)) {
                // the item's 8 blocks of 32 share 8, 4 or 2 scales: 16, 8 or 4 bytes per row
                if (is_gsh == 0) cp_async16_u32(scale_u + (is_st << 8), src_s);
                else if (is_gsh == 1) cp_async8_u32(scale_u + (is_st << 8), src_s);
                else cp_async4_u32(scale_u + (is_st << 8), src_s);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) src_w[i] += is_step;
            src_s += is_sstep;
            if (--is_chunks == 0) advance();
            else if (is_chunks == 1) last_chunk();
        }
        cp_async_commit();     // one group per item slot, so wait counts stay uniform
        is_st = (is_st + 1 == (uint32_t)S) ? 0u : is_st + 1;
    };

    // prologue: the first weights stream before the previous kernel has finished
#pragma unroll 1
    for (int j = 0; j < S - 1; ++j) issue_next();
    pdl_wait();
    // a list without waits is launched without clearing its workspace: no wait can expire,
    // so its error word is simply cleared (after the wait: the kernel ahead may be a pass on
    // the same workspace)
    if (!a.counters && a.error && blockIdx.x == 0 && tid == 0) *a.error = 0;
    if (neutral_max) {
        // written only after the wait: the kernel ahead on the stream may be
        // the argmax reduction of an earlier call that reads the same scratch
        const PassProj &P = a.p[tid];
        for (int m = 0; m < Mt && chk(blockIdx.x < (unsigned)kMaxCtas); ++m) {
            P.ws_val[(size_t)blockIdx.x * Mt + m] = -INFINITY;
            pass_ws_idx(P, Mt)[(size_t)blockIdx.x * Mt + m] = 0x7fffffff;
        }
    }

    // row qg's codes: bits 4..6 of this offset hold qg (the stage bases are
    // multiples of 1024 from a 128-aligned array start), so XOR-ing gl * 16
    // gives the swizzled chunk of group gl; row qg + 8 is 1024 bytes on
    const uint32_t wq_o = (uint32_t)(ring_c - smem) + qg * 128 + qt * 4 + (qg << 4);   // + stage * 2048
    const uint32_t sc_o = (uint32_t)(ring_s - smem) + qg * 16;                          // + stage * 256
    const uint32_t x7_o = (uint32_t)(reinterpret_cast<unsigned char *>(x7) - smem) + (ONE && !PAIRED ? qt * 8 : qt * 16);
    // M = 1 (block-diagonal): the mma's 8 columns are the item's 8 groups; lane (qg, qt) holds
    // the codes of groups 2 qt and 2 qt + 1 of rows qg and qg + 8 (16 bytes each), and as its B
    // operand pairs group 2 qt's x (as b0) if its column qg is that group, group 2 qt + 1's (as
    // b1) if it is that one, else zeros: the staged layout gives each pair in one load
    const uint32_t bd_c0 = (uint32_t)(ring_c - smem) + qg * 128 + (((2 * qt) ^ qg) << 4);       // + stage * 2048
    const uint32_t bd_c1 = (uint32_t)(ring_c - smem) + qg * 128 + (((2 * qt + 1) ^ qg) << 4);
    const uint32_t xp_o = (uint32_t)(xp - smem);
    const bool bd_sel0 = qg == 2 * qt, bd_sel1 = qg == 2 * qt + 1;
    // paired layout: one address per lane; plain layout: one per B half (b0 from group 2 qt, b1 from 2 qt + 1)
    const uint32_t bd_b = (bd_sel0 || bd_sel1) ? xp_o + kBdZero + qt * kBdPair + (bd_sel1 ? kBdPair / 2 : 0)
                                               : xp_o + 32 * (qg >> 1);   // + chunk offset if selected
    const uint32_t bd_m = (bd_sel0 || bd_sel1) ? 0xffffffffu : 0u;
    const uint32_t bd_b0 = bd_sel0 ? xp_o + kBd1Zero + 2 * qt * kBd1Group : xp_o;
    const uint32_t bd_b1 = bd_sel1 ? xp_o + kBd1Zero + (2 * qt + 1) * kBd1Group : xp_o;
    const uint32_t bd_m0 = bd_sel0 ? 0xffffffffu : 0u, bd_m1 = bd_sel1 ? 0xffffffffu : 0u;
    uint32_t st = 0;                // ring stage of the next item to compute
    int cs = 0;

    for (int ph = 0; ph < nphase; ++ph) {
        if (ph > 0) {
            if (tid == 0 && !wait_counter(&a.counters[ph - 1], gridDim.x)) {
                atomicOr(a.error, kErrWaitExpired);
                *abort_flag = 1;
            }
            consumer_sync();
            if (*abort_flag) break;
        }
        for (; cs < nseg && segs[cs].phase == ph; ++cs) {
            const PassSeg sgm = segs[cs];
            const PassProj &P = a.p[sgm.p];
            const PassGeo g = pass_geo<LW>(sgm, warp);
            const int G = P.G, N = P.N, kind = P.kind, ldo = P.ldo, rope_d = P.rope_d, gsh = P.gsh;
            const bool sasync = P.scales_async;
            // this CTA's tokens m0 .. m0 + M - 1 of the [Mt][K] inputs and [Mt][ldo] outputs
            const size_t xo = (size_t)m0 * P.K;
            const __half *const px = P.x ? P.x + xo : nullptr;
            const __half *const pres = P.res ? P.res + xo : nullptr;
            const __half *const pdlt = P.dlt ? P.dlt + xo : nullptr;
            __half *const pres_out = P.res_out ? P.res_out + xo : nullptr;
            __half *const px_out = P.x_out ? P.x_out + xo : nullptr;
            const int *const ppos = P.pos ? P.pos + m0 : nullptr;
            void *const out = kind == kEpiLogits ? (void *)(reinterpret_cast<float *>(P.out) + (size_t)m0 * ldo)
                                                 : (void *)(reinterpret_cast<__half *>(P.out) + (size_t)m0 * ldo);
            const bool writer = sgm.o_begin == 0;   // the CTA (of each column block) holding row 0
            // windowed: the segment's activations exceed the staging area (WIN kernels only)
            const bool windowed = WIN && G > a.g_stage;
            if (!windowed) {
                if (P.norm) {
                    stage_x_norm(pres, pdlt, P.gamma, P.eps, writer ? pres_out : nullptr,
                                 writer ? px_out : nullptr, xp, x7, red, M, P.K, G, NT, PAIRED);
                } else {
                    stage_x_mma(px, P.K, xp, x7, M, G, G, NT, PAIRED);
                }
                consumer_sync();
            } else if (P.norm) {
                norm_rows(pres, pdlt, P.eps, writer ? pres_out : nullptr, rn, red, M, P.K);
            }

            const int gs = windowed ? a.g_stage : G;   // groups per staged activation column
            const uint32_t nstride = (uint32_t)gs * 64u + 32u;
            uint32_t xb[NT];   // B-operand column of this lane (columns >= M read column M-1: ignored)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                xb[nt] = (uint32_t)(xp - smem) + (uint32_t)min(qg + 8 * nt, M - 1) * nstride + qt * 16;
            const int kc_last = g.my_tiles > 0 ? pass_last_kc(g, G) : kMChunkG;
            // per chunk: XG bytes of staged x per group, CG bytes of the C table per group
            constexpr uint32_t XG = ONE ? (PAIRED ? kBdGroup : kBd1Group) : 64u,
                               CG = ONE ? (PAIRED ? 8u : 4u) : 64u * NT;
            const uint32_t xstep = (uint32_t)g.wk * kMChunkG * XG, cstep = (uint32_t)g.wk * kMChunkG * CG;

            // The WK partials of tiles [t0, t0 + tn) meet here in a fixed order
            // (tile t's partials sit at local index t - t0 of the buffer), and
            // the epilogue of their outputs runs; best_v / best_i: the LM head's
            // running maxima of this thread (slot 0: column tid % (8 NT)).
            // a warp's partial of a tile: [16 rows][8 NT columns] floats, or (ONE) the 16 row sums
            constexpr int PC = ONE ? 1 : 8 * NT, PART = kMTileRows * PC;
            auto reduce_tiles = [&](auto log_tag, int t0, int tn, float (&best_v)[2 * NT], int (&best_i)[2 * NT]) {
                constexpr bool LOG = decltype(log_tag)::value;
                const int VO = g.rout * PC;                   // (output row, column) pairs per tile
                for (int idx = tid; idx < tn * VO; idx += kMThreads) {
                    const int tt = idx / VO, vo = idx - (idx / VO) * VO;
                    const int r = vo / PC, m = vo - (vo / PC) * PC;
                    const int nn = g.o_begin + (t0 + tt) * g.rout + r;
                    if (nn >= g.o_end || m >= M) continue;
                    if (!chk(nn < N && (size_t)(tt + 1) * g.wk * PART <= (size_t)a.red_floats)) continue;
                    const float *rp = red + (size_t)tt * g.wk * PART;
                    float y = 0.f, u = 0.f;
                    for (int k2 = 0; k2 < g.wk; ++k2) {
                        y += rp[(size_t)k2 * PART + r * PC + m];
                        if (kind == kEpiGateUp || kind == kEpiRope)
                            u += rp[(size_t)k2 * PART + (r + 8) * PC + m];
                    }
                    y *= pow2f(24);
                    if constexpr (LOG) {
                        reinterpret_cast<float *>(out)[(size_t)m * ldo + nn] = y;
                        // thread tid handles m = idx % PC = tid % PC: slot 0 of its table
                        if (better(y, nn, best_v[0], best_i[0])) {
                            best_v[0] = isnan(y) ? -INFINITY : y;
                            best_i[0] = nn;
                        }
                    } else if (kind == kEpiF16) {
                        reinterpret_cast<__half *>(out)[(size_t)m * ldo + nn] = __float2half_rn(y);
                    } else if (kind == kEpiRope) {
                        rope_store(reinterpret_cast<__half *>(out), (size_t)m * ldo, nn, rope_d, P.theta, ppos[m],
                                   y, u * pow2f(24));
                    } else {
                        u *= pow2f(24);
                        const float silu = y / (1.0f + expf(-y));
                        reinterpret_cast<__half *>(out)[(size_t)m * ldo + nn] = __float2half_rn(silu * u);
                    }
                }
            };

            // The segment's tiles; LOG: the LM head's epilogue (f32 logits and
            // running maxima) -- compiled apart so that the other projections'
            // loop does not carry the maxima.  WS: a windowed segment.
            auto run_segment = [&](auto log_tag, auto win_tag) {
                constexpr bool LOG = decltype(log_tag)::value;
                constexpr bool WS = decltype(win_tag)::value;
                float best_v[2 * NT];
                int best_i[2 * NT];
#pragma unroll
                for (int i = 0; i < 2 * NT; ++i) {
                    best_v[i] = -INFINITY;
                    best_i[i] = 0x7fffffff;
                }
                // windowed: rounds of one tile per warp (the same count for all
                // warps: every round stages the windows with the whole CTA)
                const int n_rounds = WS ? (g.n_tiles + g.wr_n - 1) / g.wr_n : g.my_tiles;
                const int n_win = WS ? (G + gs - 1) / gs : 1;
                for (int tl = 0; tl < n_rounds; ++tl) {
                    const bool have = !WS || tl < g.my_tiles;
                    const int t = g.my_wr + g.wr_n * tl;
                    const int o0 = g.o_begin + t * g.rout;
                    float acc[NT][4];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
                    uint32_t xoff = (uint32_t)g.my_wk * kMChunkG * XG;   // B bytes of this warp's first chunk
                    uint32_t coff = (uint32_t)g.my_wk * kMChunkG * CG;   // C-table bytes
                    // single column: this lane's B-operand address, stepped per item by the
                    // chunk step or by 0 (lanes that read the zero region)
                    uint32_t bo = bd_b + (xoff & bd_m);
                    [[maybe_unused]] const uint32_t xs = xstep & bd_m;
                    uint32_t bo0 = bd_b0 + (xoff & bd_m0), bo1 = bd_b1 + (xoff & bd_m1);
                    [[maybe_unused]] const uint32_t xs0 = xstep & bd_m0, xs1 = xstep & bd_m1;
                    int cl = 0;
                    for (int w = 0; w < n_win; ++w) {
                        int cl_end = g.my_chunks;
                        if constexpr (WS) {
                            // stage window w (groups [w gs, w gs + gn)) once every warp is done with w - 1
                            consumer_sync();
                            const int g0 = w * gs, gn = min(gs, G - g0);
                            if (P.norm)
                                stage_x_norm_window(pres, pdlt, P.gamma, (writer && tl == 0) ? px_out : nullptr,
                                                    rn, xp, x7, M, P.K, g0, gn, gs, NT, PAIRED);
                            else
                                stage_x_mma(px + (size_t)g0 * kGroup, P.K, xp, x7, M, gn, gs, NT, PAIRED);
                            consumer_sync();
                            if (w > 0) {   // the area now starts at group w gs
                                xoff -= (uint32_t)gs * XG;
                                coff -= (uint32_t)gs * CG;
                                bo -= ((uint32_t)gs * XG) & bd_m;
                                bo0 -= ((uint32_t)gs * XG) & bd_m0;
                                bo1 -= ((uint32_t)gs * XG) & bd_m1;
                            }
                            // this warp's chunks c = my_wk + wk cl below the window's end
                            const int c_end = (w + 1) * (gs / kMChunkG);
                            cl_end = have ? min(g.my_chunks, (c_end - g.my_wk + g.wk - 1) / g.wk) : 0;
                        }
                        for (; cl < cl_end; ++cl) {
                            cp_async_wait<S - 2>();
                            __syncwarp();
                            const int kc = cl == g.my_chunks - 1 ? kc_last : kMChunkG;
                            if constexpr (ONE) {
                                // Block-diagonal contraction of the item (M = 1): 16 mma steps, step
                                // 4 t + p takes pair p of word t of the lane's four 16-byte chunks
                                // (p: codes {0,4} | {2,6} | 16 {1,5} | 16 {3,7}), so column c of D
                                // sums group c's 32 products; C starts it at -7 X_c 2^-24.
                                const unsigned char *cw = smem + (st << 11);
                                const uint4 qa = *reinterpret_cast<const uint4 *>(cw + bd_c0);          // row qg,     group 2 qt
                                const uint4 qb = *reinterpret_cast<const uint4 *>(cw + bd_c0 + 1024);   // row qg + 8, group 2 qt
                                const uint4 qc = *reinterpret_cast<const uint4 *>(cw + bd_c1);          // row qg,     group 2 qt + 1
                                const uint4 qd = *reinterpret_cast<const uint4 *>(cw + bd_c1 + 1024);   // row qg + 8, group 2 qt + 1
                                // scales of (row qg, qg + 8) x (group 2 qt, 2 qt + 1)
                                float s00, s01, s10, s11;
                                if (sasync) {
                                    const unsigned char *sp = smem + sc_o + (st << 8);
                                    if (gsh == 0) {
                                        const __half2 h0 = *reinterpret_cast<const __half2 *>(sp + 4 * qt);
                                        const __half2 h1 = *reinterpret_cast<const __half2 *>(sp + 128 + 4 * qt);
                                        s00 = __low2float(h0);
                                        s01 = __high2float(h0);
                                        s10 = __low2float(h1);
                                        s11 = __high2float(h1);
                                    } else {
                                        // 64 or 128 k per scale: both groups read the same one
                                        const int off = 2 * ((2 * qt) >> gsh);
                                        s00 = s01 = __half2float(*reinterpret_cast<const __half *>(sp + off));
                                        s10 = s11 = __half2float(*reinterpret_cast<const __half *>(sp + 128 + off));
                                    }
                                } else {
                                    bool v0, v1;
                                    const int c = g.my_wk + g.wk * cl;
                                    const int r0 = pass_slot_row(kind, N, rope_d, g.o_end, o0, qg, v0);
                                    const int r1 = pass_slot_row(kind, N, rope_d, g.o_end, o0, qg + 8, v1);
                                    const __half *p0 = P.scales + (size_t)r0 * (G >> gsh);
                                    const __half *p1 = P.scales + (size_t)r1 * (G >> gsh);
                                    const int b = c * kMChunkG + 2 * qt;
                                    const int wr = pass_weight_rows(kind, N), sr = G >> gsh;
                                    const bool e0 = 2 * qt < kc && chk(r0 >= 0 && r0 < wr && r1 >= 0 && r1 < wr &&
                                                                      (b >> gsh) < sr);
                                    const bool e1 = 2 * qt + 1 < kc && chk(r0 >= 0 && r0 < wr && r1 >= 0 &&
                                                                          r1 < wr && ((b + 1) >> gsh) < sr);
                                    s00 = e0 ? __half2float(p0[b >> gsh]) : 0.f;
                                    s10 = e0 ? __half2float(p1[b >> gsh]) : 0.f;
                                    s01 = e1 ? __half2float(p0[(b + 1) >> gsh]) : 0.f;
                                    s11 = e1 ? __half2float(p1[(b + 1) >> gsh]) : 0.f;
                                }
                                // (a chunk with missing groups, kc < 8, occurs only when K % 256 != 0, and
                                // then scales are never copied asynchronously: the loads above give 0)
                                // two accumulators (the steps of codes {0,4} and 16 {1,5} -> d, of {2,6} and
                                // 16 {3,7} -> e): two chains of 8 dependent mma instead of one of 16
                                float d[4], e[4] = {0.f, 0.f, 0.f, 0.f};
                                if constexpr (PAIRED) {
                                    const float4 cz = *reinterpret_cast<const float4 *>(smem + x7_o + coff);
                                    d[0] = cz.x; d[1] = cz.y; d[2] = cz.z; d[3] = cz.w;
                                } else {
                                    const float2 cz = *reinterpret_cast<const float2 *>(smem + x7_o + coff);
                                    d[0] = cz.x; d[1] = cz.y; d[2] = cz.x; d[3] = cz.y;
                                }
                                const uint32_t wa4[4] = {qa.x, qa.y, qa.z, qa.w}, wb4[4] = {qb.x, qb.y, qb.z, qb.w};
                                const uint32_t wc4[4] = {qc.x, qc.y, qc.z, qc.w}, wd4[4] = {qd.x, qd.y, qd.z, qd.w};
#pragma unroll
                                for (int t4 = 0; t4 < 4; ++t4) {
                                    // (b0, b1) of steps 4 t4 .. 4 t4 + 3: paired, (xa.x, xa.y), (xa.z, xa.w),
                                    // (xb.x, xb.y), (xb.z, xb.w); plain, (xa.x, xb.x), (xa.y, xb.y), ...
                                    uint4 xa, xb;
                                    if constexpr (PAIRED) {
                                        xa = *reinterpret_cast<const uint4 *>(smem + bo + 32 * t4);
                                        xb = *reinterpret_cast<const uint4 *>(smem + bo + 32 * t4 + 16);
                                    } else {
                                        const uint4 x0 = *reinterpret_cast<const uint4 *>(smem + bo0 + 16 * t4);
                                        const uint4 x1 = *reinterpret_cast<const uint4 *>(smem + bo1 + 16 * t4);
                                        xa = make_uint4(x0.x, x1.x, x0.y, x1.y);
                                        xb = make_uint4(x0.z, x1.z, x0.w, x1.w);
                                    }
                                    const uint32_t wa = wa4[t4], wb = wb4[t4], wc = wc4[t4], wd = wd4[t4];
                                    const uint32_t was = wa >> 8, wbs = wb >> 8, wcs = wc >> 8, wds = wd >> 8;
                                    const uint32_t A0[4] = {wa & 0x000F000Fu, wb & 0x000F000Fu, wc & 0x000F000Fu,
                                                            wd & 0x000F000Fu};
                                    mma_16816(d, A0, xa.x, xa.y, d[0], d[1], d[2], d[3]);
                                    const uint32_t A1[4] = {was & 0x000F000Fu, wbs & 0x000F000Fu, wcs & 0x000F000Fu,
                                                            wds & 0x000F000Fu};
                                    mma_16816(e, A1, xa.z, xa.w, e[0], e[1], e[2], e[3]);
                                    const uint32_t A2[4] = {wa & 0x00F000F0u, wb & 0x00F000F0u, wc & 0x00F000F0u,
                                                            wd & 0x00F000F0u};
                                    mma_16816(d, A2, xb.x, xb.y, d[0], d[1], d[2], d[3]);
                                    const uint32_t A3[4] = {was & 0x00F000F0u, wbs & 0x00F000F0u, wcs & 0x00F000F0u,
                                                            wds & 0x00F000F0u};
                                    mma_16816(e, A3, xb.z, xb.w, e[0], e[1], e[2], e[3]);
                                }
                                acc[0][0] = fmaf(d[0] + e[0], s00, acc[0][0]);
                                acc[0][1] = fmaf(d[1] + e[1], s01, acc[0][1]);
                                acc[0][2] = fmaf(d[2] + e[2], s10, acc[0][2]);
                                acc[0][3] = fmaf(d[3] + e[3], s11, acc[0][3]);
                            } else {
                                uint4 sg, sg8;     // scales of rows qg and qg + 8 for the item's 8 groups
                                if (sasync) {
                                    const unsigned char *sp = smem + sc_o + (st << 8);
                                    sg = *reinterpret_cast<const uint4 *>(sp);
                                    sg8 = *reinterpret_cast<const uint4 *>(sp + 8 * 16);
                                    if (gsh) {
                                        // one scale per 32-block: repeat each of the 4 (or 2) scales 2 (or 4) times
                                        sg = spread_scales(sg, gsh);
                                        sg8 = spread_scales(sg8, gsh);
                                    }
                                } else {
                                    bool v0, v1;
                                    const int c = g.my_wk + g.wk * cl;
                                    const int r0 = pass_slot_row(kind, N, rope_d, g.o_end, o0, qg, v0);
                                    const int r1 = pass_slot_row(kind, N, rope_d, g.o_end, o0, qg + 8, v1);
                                    uint32_t u0[4] = {0, 0, 0, 0}, u1[4] = {0, 0, 0, 0};
                                    const unsigned short *p0 = reinterpret_cast<const unsigned short *>(P.scales) +
                                                               (size_t)r0 * (G >> gsh);
                                    const unsigned short *p1 = reinterpret_cast<const unsigned short *>(P.scales) +
                                                               (size_t)r1 * (G >> gsh);
                                    const int wr = pass_weight_rows(kind, N), sr = G >> gsh;
                                    for (int gl = 0; gl < kc; ++gl) {
                                        const int b = (c * kMChunkG + gl) >> gsh;      // the block's scale
                                        if (!chk(r0 >= 0 && r0 < wr && r1 >= 0 && r1 < wr && b < sr)) continue;
                                        u0[gl >> 1] |= (uint32_t)p0[b] << (16 * (gl & 1));
                                        u1[gl >> 1] |= (uint32_t)p1[b] << (16 * (gl & 1));
                                    }
                                    sg = make_uint4(u0[0], u0[1], u0[2], u0[3]);
                                    sg8 = make_uint4(u1[0], u1[1], u1[2], u1[3]);
                                }
                                const uint32_t sgw[4] = {sg.x, sg.y, sg.z, sg.w}, sg8w[4] = {sg8.x, sg8.y, sg8.z, sg8.w};
                                // shared-memory pointers of the item; the unrolled groups add constants
                                const uint32_t wb = wq_o + (st << 11);
                                const unsigned char *cp = smem + x7_o + coff;     // + (gl * NT + nt) * 64, compact: + gl * 16
                                const unsigned char *bp[NT];
    #pragma unroll
                                for (int nt = 0; nt < NT; ++nt) bp[nt] = smem + xb[nt] + xoff;   // + gl * 64
                                auto step = [&](int gl) {
                                    const unsigned char *wa = smem + (wb ^ (uint32_t)(gl << 4));
                                    const uint32_t w0 = *reinterpret_cast<const uint32_t *>(wa);
                                    const uint32_t w1 = *reinterpret_cast<const uint32_t *>(wa + 1024);
                                    const uint32_t w0s = w0 >> 8, w1s = w1 >> 8;
                                    const uint32_t A0[4] = {w0 & 0x000F000Fu, w1 & 0x000F000Fu, w0s & 0x000F000Fu,
                                                            w1s & 0x000F000Fu};
                                    const uint32_t A1[4] = {w0 & 0x00F000F0u, w1 & 0x00F000F0u, w0s & 0x00F000F0u,
                                                            w1s & 0x00F000F0u};
                                    const __half2 sh0 = *reinterpret_cast<const __half2 *>(&sgw[gl >> 1]);
                                    const __half2 sh1 = *reinterpret_cast<const __half2 *>(&sg8w[gl >> 1]);
                                    const float s0 = (gl & 1) ? __high2float(sh0) : __low2float(sh0);
                                    const float s1 = (gl & 1) ? __high2float(sh1) : __low2float(sh1);
    #pragma unroll
                                    for (int nt = 0; nt < NT; ++nt) {
                                        const uint4 bb = *reinterpret_cast<const uint4 *>(bp[nt] + gl * 64);
                                        const uint4 czu =
                                            *reinterpret_cast<const uint4 *>(cp + (ONE ? gl * 16 : (gl * NT + nt) * 64));
                                        float d[4];
                                        mma_16816(d, A0, bb.x, bb.y, __uint_as_float(czu.x), __uint_as_float(czu.y),
                                                  __uint_as_float(czu.z), __uint_as_float(czu.w));
                                        mma_16816(d, A1, bb.z, bb.w, d[0], d[1], d[2], d[3]);
                                        acc[nt][0] = fmaf(d[0], s0, acc[nt][0]);
                                        acc[nt][2] = fmaf(d[2], s1, acc[nt][2]);
                                        if (!ONE) {
                                            acc[nt][1] = fmaf(d[1], s0, acc[nt][1]);
                                            acc[nt][3] = fmaf(d[3], s1, acc[nt][3]);
                                        }
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
                            }
                            // the refill goes to the previous item's stage, which every lane finished
                            // reading before it passed this item's __syncwarp above
                            issue_next();
                            st = (st + 1 == (uint32_t)S) ? 0u : st + 1;
                            xoff += xstep;
                            coff += cstep;
                            if constexpr (PAIRED) bo += xs;
                            else {
                                bo0 += xs0;
                                bo1 += xs1;
                            }
                        }
                    }

                    if constexpr (ONE) {
                        // a row's group partials are spread over the quad: sum them (the
                        // same butterfly on every lane, so the order is fixed) into the
                        // slots the single-column epilogue reads (quad thread 0, column 0)
                        float r0 = acc[0][0] + acc[0][1], r1 = acc[0][2] + acc[0][3];
                        r0 += __shfl_xor_sync(0xffffffffu, r0, 1);
                        r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
                        r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
                        r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
                        acc[0][0] = r0;
                        acc[0][2] = r1;
                        acc[0][1] = acc[0][3] = 0.f;
                    }

                    // ---- tile epilogue ----
                    if (have && g.wk > 1 &&
                        chk(((size_t)(WS ? g.my_wr : t) * g.wk + g.my_wk + 1) * PART <= (size_t)a.red_floats)) {
                        // this warp's partial of tile t; windowed rounds number their tiles
                        // from the round's first (my_wr)
                        float *rp = red + ((size_t)(WS ? g.my_wr : t) * g.wk + g.my_wk) * PART;
                        if constexpr (ONE) {
                            // the quad's row sums (slots 0 and 2 of every lane of the quad)
                            if (qt == 0) {
                                rp[qg] = acc[0][0];
                                rp[qg + 8] = acc[0][2];
                            }
                        } else {
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                rp[qg * 8 * NT + 8 * nt + 2 * qt] = acc[nt][0];
                                rp[qg * 8 * NT + 8 * nt + 2 * qt + 1] = acc[nt][1];
                                rp[(qg + 8) * 8 * NT + 8 * nt + 2 * qt] = acc[nt][2];
                                rp[(qg + 8) * 8 * NT + 8 * nt + 2 * qt + 1] = acc[nt][3];
                            }
                        }
                    } else if (have) {
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int m = 8 * nt + 2 * qt + e;
                                if (m >= M) continue;
                                if (kind == kEpiGateUp) {
                                    const int nn = o0 + qg;
                                    if (nn < g.o_end && chk(nn < N)) {
                                        const float gv = acc[nt][e] * pow2f(24), u = acc[nt][2 + e] * pow2f(24);
                                        const float silu = gv / (1.0f + expf(-gv));
                                        reinterpret_cast<__half *>(out)[(size_t)m * ldo + nn] = __float2half_rn(silu * u);
                                    }
                                } else if (!LOG && kind == kEpiRope) {
                                    const int nn = o0 + qg;
                                    if (nn < g.o_end && chk(nn < N))
                                        rope_store(reinterpret_cast<__half *>(out), (size_t)m * ldo, nn, rope_d, P.theta,
                                                   ppos[m], acc[nt][e] * pow2f(24), acc[nt][2 + e] * pow2f(24));
                                } else {
#pragma unroll
                                    for (int h = 0; h < 2; ++h) {
                                        const int nn = o0 + qg + 8 * h;
                                        if (nn >= g.o_end || !chk(nn < N)) continue;
                                        const float y = acc[nt][2 * h + e] * pow2f(24);
                                        if constexpr (!LOG) {
                                            reinterpret_cast<__half *>(out)[(size_t)m * ldo + nn] = __float2half_rn(y);
                                        } else {
                                            reinterpret_cast<float *>(out)[(size_t)m * ldo + nn] = y;
                                            if (better(y, nn, best_v[2 * nt + e], best_i[2 * nt + e])) {
                                                best_v[2 * nt + e] = isnan(y) ? -INFINITY : y;
                                                best_i[2 * nt + e] = nn;
                                            }
                                        }
                                    }
                                }
                            }
                        }
                    }
                    if constexpr (WS) {
                        if (g.wk > 1) {
                            // this round's WK partials meet before the next round writes the buffer
                            consumer_sync();
                            reduce_tiles(log_tag, tl * g.wr_n, min(g.wr_n, g.n_tiles - tl * g.wr_n), best_v, best_i);
                        }
                    }
                }

                if (!WS && g.wk > 1) {
                    // WK partials of each tile meet here; fixed summation order
                    consumer_sync();
                    reduce_tiles(log_tag, 0, g.n_tiles, best_v, best_i);
                }

                if constexpr (LOG) {
                    // The CTA's (maximum, lowest index) per column m under better()'s total order
                    // (so the reduction order does not matter): within each warp a butterfly over
                    // the lanes that hold the same column, then the warps' results per column.
                    // Column of slot i: with WK > 1 only slot 0, column lane % PC (column 0 in
                    // every lane with ONE); otherwise column 8 (i >> 1) + 2 qt + (i & 1), shared by
                    // the lanes of equal qt.
                    auto comb = [&](float &v, int &ix, int mask) {
                        const float ov = __shfl_xor_sync(0xffffffffu, v, mask);
                        const int oi = __shfl_xor_sync(0xffffffffu, ix, mask);
                        if (better(ov, oi, v, ix)) {
                            v = isnan(ov) ? -INFINITY : ov;
                            ix = oi;
                        }
                    };
                    if (g.wk > 1) {
                        // slot 0 holds column lane % PC (every lane column 0 with ONE)
                        for (int mask = PC; mask < 32; mask <<= 1) comb(best_v[0], best_i[0], mask);
                    } else {
#pragma unroll
                        for (int i = 0; i < 2 * NT; ++i)
#pragma unroll
                            for (int mask = 4; mask < 32; mask <<= 1) comb(best_v[i], best_i[i], mask);
                    }
                    consumer_sync();   // the warp results overwrite the partial buffer
                    if (g.wk > 1) {
                        if (lane < 8 * NT) {
                            bvs[warp * 8 * NT + lane] = best_v[0];
                            bis[warp * 8 * NT + lane] = best_i[0];
                        }
                    } else if (qg == 0) {
#pragma unroll
                        for (int i = 0; i < 2 * NT; ++i) {
                            const int m = 8 * (i >> 1) + 2 * qt + (i & 1);
                            bvs[warp * 8 * NT + m] = best_v[i];
                            bis[warp * 8 * NT + m] = best_i[i];
                        }
                    }
                    consumer_sync();
                    if (!chk(blockIdx.x < (unsigned)kMaxCtas && m0 + M <= Mt)) {
                    } else if (tid < M) {
                        float bv = -INFINITY;
                        int bi = 0x7fffffff;
                        for (int w = 0; w < kMW; ++w) {
                            if (better(bvs[w * 8 * NT + tid], bis[w * 8 * NT + tid], bv, bi)) {
                                bv = bvs[w * 8 * NT + tid];
                                bi = bis[w * 8 * NT + tid];
                            }
                        }
                        P.ws_val[(size_t)blockIdx.x * Mt + m0 + tid] = bv;
                        pass_ws_idx(P, Mt)[(size_t)blockIdx.x * Mt + m0 + tid] = bi;
                    } else if (tid < Mt) {
                        // the Mt - M tokens of the other column block: a neutral partial maximum
                        const int m = (m0 + tid) % Mt;
                        P.ws_val[(size_t)blockIdx.x * Mt + m] = -INFINITY;
                        pass_ws_idx(P, Mt)[(size_t)blockIdx.x * Mt + m] = 0x7fffffff;
                    }
                }
            };
            if constexpr (WIN) {
                if (windowed) {
                    if (kind == kEpiLogits) run_segment(std::true_type{}, std::true_type{});
                    else run_segment(std::false_type{}, std::true_type{});
                } else {
                    if (kind == kEpiLogits) run_segment(std::true_type{}, std::false_type{});
                    else run_segment(std::false_type{}, std::false_type{});
                }
            } else {
                if (kind == kEpiLogits) run_segment(std::true_type{}, std::false_type{});
                else run_segment(std::false_type{}, std::false_type{});
            }
            consumer_sync();   // the activation area and partial buffers are free again
        }
        if (ph + 1 < nphase) {
            // publish this CTA's outputs of the phase, then count it done: every output was
            // written before the CTA barrier that closes each segment, so one fence by the
            // counting thread orders them all before its count
            if (tid == 0 && !(ph == a.withhold && blockIdx.x == 0)) {
                __threadfence();
                atomicAdd(&a.counters[ph], 1u);
            }
        }
    }
    cp_async_wait<0>();
}

}  // namespace zt
