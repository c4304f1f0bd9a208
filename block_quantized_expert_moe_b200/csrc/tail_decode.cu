// The device-planned MoE tail of 1 to 64 tokens in one launch.
//
// The "Qwen3.8-Flash-Next UD-IQ2_XS (L4 fix) for Basalt" model card ("What was
// changed") names the fast decode path a device-planned MoE tail with grouped
// kernels: the per-expert token lists are planned on the GPU, without a host
// round trip, and each selected expert's weights are read once for all of its
// tokens.  Here the whole tail is one persistent kernel, one CTA per SM:
//
//   route     CTA c takes a block of router rows and a block of tokens: logits
//             = Wr x (fp32), its router rows bulk-copied into shared memory
//             before the kernel waits on the previous one of the stream
//             (programmatic dependent launch); the first CTA of each token
//             block also picks each token's power-of-two fp16 scale; then a
//             grid-wide counter barrier
//   plan      every CTA selects the top-k of every token (one warp per token)
//             and builds the same plan in its shared memory: active experts in
//             ascending order (the groups; the shared expert last), each
//             group's tokens in ascending order (its slots), slot of each
//             (token, choice); then writes its share of the fp16 slot rows of
//             x and counts it on each group's readiness counter
//   gate/up   stream-K: the units {group, 128 row pairs, 256 of K} (gate and
//             up rows: two 128-row tensor-core tiles) are cut into equal
//             contiguous ranges, one per CTA; a tile whose units span CTAs is
//             summed from their fp32 pieces, in CTA order, by the last CTA to
//             finish its piece; then h = silu(g) * u (fp16, slot rows) and a
//             count on the group's h counter
//   down      the same over {group, 256 output rows, 256 of K}, each unit's B
//             operand the group's h rows once its counter is full; y per slot
//             (fp32) and a count on the 256-row block's counter
//   combine   CTA c owns output rows [H c / G, H (c + 1) / G) of every token:
//             once every group's y rows of their blocks are in,
//             out[t] = sum_j gate_tj y[slot(t, j)] (+ the shared expert's y),
//             in the layer's order
//
// The tensor-core tile is M = 128 weight rows, N = the group's tokens (padded
// to 16), K = 64 per stage, fp16 x fp16 -> fp32 in tensor memory: the weights
// are expanded from their blocks to fp16 straight into tensor memory (the MMA's
// A operand; one rounding each, exact for the 4-bit codes), the slot rows of x
// (the B operand, shared memory) are exact fp16 after the token's power-of-two
// scale, h is rounded to fp16.  Tensor memory: columns 0-255 two accumulator
// buffers, 256-511 four A stages of 64 columns (two tiles of 32).
//
//   warps 0-3   epilogue: tensor-memory lanes 32w .. 32w + 31 (tile rows)
//   warp 4      MMA issuer (one elected thread)
//   warp 5      raw producer (two bulk copies a unit from the tiled planes)
//   warp 6      B producer: once the group's readiness counter is full, TMA
//               loads (16-row boxes) of the group's slot rows of x or h, one
//               ring slot per slice
//   warps 7-14  expanders: warp 7 + i expands tile i / 4, lanes 32 (warp % 4)
//               .. + 31 (the lanes a warp may store to), both 32-blocks of
//               its row per slice
//
// Every wait is bounded (~1 s): a wait that runs out records MOE_ERR_TIMEOUT,
// raises the CTA's abort flag and the CTA drains what it issued before it
// frees tensor memory and returns.  Counters live in the workspace, zero
// between launches: the last CTA to finish clears the ones the launch used.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "decode_common.cuh"
#include "dequant.cuh"
#include "moe_internal.cuh"
#include "tc_common.cuh"
#include "tma_maps.cuh"

namespace moe {

namespace {

using namespace tc;

constexpr int kTlEpiWarps = 4, kTlMmaWarp = 4, kTlRawWarp = 5, kTlBWarp = 6, kTlDeqWarp0 = 7, kTlDeqWarps = 8;
constexpr int kTlWarps = kTlDeqWarp0 + kTlDeqWarps;  // 15
constexpr int kTlThreads = 32 * kTlWarps;
constexpr int kTlWriters = 32 * (kTlEpiWarps + kTlDeqWarps);  // the warps that write the x slot rows
constexpr int kTlMaxRaw = 4, kTlMaxB = 8;
constexpr int kTlTmemCols = 512;          // two accumulator buffers of 128 columns, then the A stages
constexpr int kTlAcc = 256;               // first tensor-memory column of the A stages
constexpr int kTlAStageCols = 64;         // a stage: the unit's two 128-row tiles x 64 fp16 of K (32 columns each)
constexpr int kTlNA = 4;                  // A stages (the rest of tensor memory)
constexpr long long kTlSpin = 1ll << 31;  // clocks

__host__ __device__ inline int tl_cdiv(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline int tl_al16(int v) { return (v + 15) & ~15; }

// One raw stage: the unit's 256 rows (two 128-row tiles) x K = 256, each tile's
// block of the pack's tiled copy as one bulk copy lands it: codes (128-byte
// rows in the 128-byte swizzle; Q8_0 two 16 KB halves), scales (16 bytes a
// row; Q5_1 32 in the 32-byte swizzle) and Q5_1 fifth bits (32, same swizzle).
template <int FMT>
struct TlRaw {
    static constexpr int kCodes = 128 * 128 * (FMT == MOE_FMT_Q8_0 ? 2 : 1);
    static constexpr int kScales = 128 * (FMT == MOE_FMT_Q5_1 ? 32 : 16);
    static constexpr int kQh = FMT == MOE_FMT_Q5_1 ? 128 * 32 : 0;
    static constexpr int kTile = kCodes + kScales + kQh;  // = tl_block_bytes(FMT)
    static constexpr int kStage = 2 * kTile;
    __device__ static int codes(int t) { return t * kTile; }
    __device__ static int scales(int t) { return t * kTile + kCodes; }
    __device__ static int qh(int t) { return t * kTile + kCodes + kScales; }
};

__host__ __device__ inline int tl_raw_bytes(int fmt)
{
    switch (fmt) {
    case MOE_FMT_Q8_0: return TlRaw<MOE_FMT_Q8_0>::kStage;
    case MOE_FMT_Q5_1: return TlRaw<MOE_FMT_Q5_1>::kStage;
    case MOE_FMT_IQ4_NL: return TlRaw<MOE_FMT_IQ4_NL>::kStage;
    default: return TlRaw<MOE_FMT_NVFP4>::kStage;
    }
}

// Word offsets of the workspace counters (unsigned, zero between launches).
struct TlCtr {
    int bar, ticket, gu_tile, dn_tile, grp_x, grp_h, rb, total;
};
__host__ __device__ inline TlCtr tl_ctr(int E, int H, int I)
{
    TlCtr c;
    c.bar = 0;
    c.ticket = 1;
    c.gu_tile = 4;
    c.dn_tile = c.gu_tile + (E + 1) * (I / 128);
    c.grp_x = c.dn_tile + (E + 1) * (H / 256);
    c.grp_h = c.grp_x + (E + 1);
    c.rb = c.grp_h + (E + 1);
    c.total = c.rb + H / 256;
    return c;
}

// The launch's plan in shared memory (after the rings), the same in every CTA.
struct TlPlanLayout {
    int xscale, sel_e, sel_g, slot_of, grp_e, grp_n, grp_off, slot_tok, total;
};
__host__ __device__ inline TlPlanLayout tl_plan_layout(int T, int k, int E)
{
    TlPlanLayout L;
    const int tk = T * k, ng = E + 1, slots = T * (k + 1);
    int o = 0;
    L.xscale = o;   o = tl_al16(o + 4 * T);
    L.sel_e = o;    o = tl_al16(o + 2 * tk);
    L.sel_g = o;    o = tl_al16(o + 4 * tk);
    L.slot_of = o;  o = tl_al16(o + 2 * tk);
    L.grp_e = o;    o = tl_al16(o + 2 * ng);
    L.grp_n = o;    o = tl_al16(o + 2 * ng);
    L.grp_off = o;  o = tl_al16(o + 4 * ng);
    L.slot_tok = o; o = tl_al16(o + 2 * slots);
    L.total = o;
    return L;
}

// Routing geometry: token blocks of at most rt tokens, row blocks over the rest
// of the grid.
struct TlRoute {
    int rt, ntb, nrb;
};
__host__ __device__ inline TlRoute tl_route(int T, int E, int G, int xbytes)
{
    TlRoute r;
    r.rt = min(T, xbytes == 2 ? 16 : 8);
    r.ntb = tl_cdiv(T, r.rt);
    r.nrb = max(1, min(E, G / r.ntb));
    return r;
}

// Bytes of the routing and planning scratch (overlaid on the rings).
__host__ __device__ inline int tl_scratch_bytes(int T, int H, int E, int G, int xbytes)
{
    const TlRoute r = tl_route(T, E, G, xbytes);
    const int rows = tl_cdiv(E, r.nrb);
    const int gemv = tl_al16(rows * H * 2) + r.rt * H * 4 + rows * 8 * r.rt * 4;  // router rows, x, partial dots
    const int nsw = min(kTlWarps, T);
    const int sel = nsw * (E * 4 + 512);
    const int plan = tl_al16((E + 1) * 4) + E * 8 + E * 4;  // counts, token masks, own {flag, tokens}
    return max(gemv, max(sel, plan));
}

struct TailArgs {
    const void *x;
    int x_dtype;
    const uint16_t *wr;
    int T, H, E, I, k, has_shared;
    int eb, ee;                  // routed experts [eb, ee) are in the pack, at slots e - eb
    CodeTable tab_gu, tab_dn;
    const float *ts_gu, *ts_dn;  // NVFP4 per-pack-slot matrix scales
    const uint8_t *tl_gu, *tl_dn;  // the projections' tiled copies (DevProj::tl)
    int64_t tl_gu_stride, tl_dn_stride;
    float *logits;               // [T x E]
    float *slot_scale;           // [slots] 2^s: the slot's row of x was scaled by 2^-s into fp16
    __half *xg;                  // [slots x H] fp16 slot rows of x
    __half *h;                   // [slots x I]
    float *y;                    // [slots x H]
    float *part;                 // [2 phases][G][2 pieces][n16max x 256] fp32 partial tiles
    unsigned *ctr;               // counters (TlCtr)
    int32_t *err;
    float *out;                  // [T x H]
    int32_t *idx_out;            // routing readback, written by CTA 0
    float *gate_out;
    int32_t *cnt_out;
    int nr, na, nb;              // ring depths: raw stages, A stages (tensor memory), B slots
    int raw_stride, bslot, n16max;  // a B slot: n16max rows of 128 bytes
    int rings;                   // bytes of the rings (the plan follows)
    long long *stamps;           // profiling only: grid events {2^62 - first, last} at words 10..19
};

struct Ring {
    int s = 0, u = 0;
    __device__ __forceinline__ void next(int n)
    {
        if (++s == n) {
            s = 0;
            ++u;
        }
    }
};

__device__ __forceinline__ const uint8_t *raw_code(const uint8_t *box0, int bx, int r, int c)
{
    return box0 + bx * 16384 + r * 128 + ((c ^ (r & 7)) << 4);
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Tensor memory: one thread's 16 consecutive 32-bit columns of its lane (the warp's 32 lanes at once).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                 "%13, %14, %15, %16};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
                 "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// f16 x f16 -> f32 MMA with A in tensor memory (M = 128: row m in lane m, K packed two
// fp16 per 32-bit column), B a shared-memory descriptor.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void grid_event(long long *st, int ev)
{
    if (!st || threadIdx.x != 0) return;
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    atomicMax(st + 10 + 2 * ev, (1ll << 62) - (long long)t);
    atomicMax(st + 11 + 2 * ev, (long long)t);
}

// Profiling only: CTA 0's SM clock at step i (words 0..9 of the forward's stamps).
__device__ __forceinline__ void cta0_clock(long long *st, int i)
{
    if (st && blockIdx.x == 0 && threadIdx.x == 0) st[i] = clock64();
}

__device__ __forceinline__ unsigned ld_acq(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded wait on an mbarrier phase that backs off between tests: for warps
// whose wait is not on the critical path (epilogue, producers), so that their
// polling does not take issue slots from the expanding warps.
__device__ __forceinline__ bool mbar_wait_idle(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kTlSpin) return false;
        __nanosleep(128);
    }
    return true;
}

// Spin (bounded) until *p >= target; false if the wait ran out.
__device__ __forceinline__ bool wait_count(const unsigned *p, unsigned target)
{
    if (ld_acq(p) >= target) return true;
    const long long t0 = clock64();
    while (ld_acq(p) < target) {
        if (clock64() - t0 > kTlSpin) return false;
        __nanosleep(32);
    }
    return true;
}

// Named barrier of the four epilogue warps.
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// The CTA whose contiguous range [U c / G, U (c + 1) / G) holds unit u.
__device__ __forceinline__ int cta_of(int u, int U, int G) { return (int)(((long long)G * (u + 1) - 1) / U); }
__device__ __forceinline__ int range_lo(int U, int c, int G) { return (int)((long long)U * c / G); }

// Number of CTAs whose ranges hold any of units [u0, u0 + n) (ranges are
// contiguous and ascending; CTAs with empty ranges hold none).
__device__ __forceinline__ int owners(int u0, int n, int U, int G)
{
    int cnt = 0, prev = -1;
    for (int u = u0; u < u0 + n; ++u) {
        const int cu = cta_of(u, U, G);
        cnt += cu != prev;
        prev = cu;
    }
    return cnt;
}

// Exclusive scan of n ints in shared memory v (n <= 4 * blockDim), in place;
// returns the total.  tmp: 32 ints of scratch.
__device__ int block_scan(int *v, int n, int *tmp)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int i0 = 4 * tid;
    int e[4], s = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        e[j] = i0 + j < n ? v[i0 + j] : 0;
        s += e[j];
    }
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? tmp[lane] : 0, wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < nw) tmp[lane] = wi - w;
        if (lane == 31) tmp[31] = wi;
    }
    __syncthreads();
    int base = tmp[warp] + incl - s;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (i0 + j < n) v[i0 + j] = base;
        base += e[j];
    }
    const int total = tmp[31];
    __syncthreads();
    return total;
}

// A unit of one phase (0 gate/up, 1 down) and the segment of this CTA it is in.
struct Unit {
    int g, b, kc;        // group, tile within the group, K chunk
    int tile;            // tile index within the phase
    bool first, last;    // first / last unit of this CTA's piece of the tile
};

struct Geo {
    int KC[2], NB[2], U[2], lo[2], hi[2];
};

__device__ __forceinline__ Unit unit_at(const Geo &q, int p, int u)
{
    Unit x;
    x.tile = u / q.KC[p];
    x.kc = u - x.tile * q.KC[p];
    x.g = x.tile / q.NB[p];
    x.b = x.tile - x.g * q.NB[p];
    const int t0 = x.tile * q.KC[p];
    x.first = u == max(q.lo[p], t0);
    x.last = u + 1 == min(q.hi[p], t0 + q.KC[p]);
    return x;
}

// The piece CTA c wrote for tile t of phase p: 0 if t is the tile its range
// starts in, else 1 (the range's last tile).
__device__ __forceinline__ float *piece(const TailArgs &a, const Geo &q, int p, int c, int t, int G)
{
    const int first_tile = range_lo(q.U[p], c, G) / q.KC[p];
    const int which = first_tile == t ? 0 : 1;
    return a.part + (((size_t)p * G + c) * 2 + which) * (size_t)a.n16max * 256;
}

// A unit's raw stage: two bulk copies, one per tile (128-row blocks rb0, rb1,
// K chunk kc of expert slot ex), from the pack's tiled copy.
template <int FMT>
__device__ __forceinline__ void raw_load(uint8_t *st, const uint8_t *tl, int64_t tl_stride, int KC, uint64_t *bar,
                                         int kc, int rb0, int rb1, int ex)
{
    using RL = TlRaw<FMT>;
    mbar_arrive_expect_tx(bar, (uint32_t)RL::kStage);
    const uint8_t *base = tl + (int64_t)ex * tl_stride;
    bulk_g2s(st, base + ((int64_t)rb0 * KC + kc) * RL::kTile, (uint32_t)RL::kTile, bar);
    bulk_g2s(st + RL::kTile, base + ((int64_t)rb1 * KC + kc) * RL::kTile, (uint32_t)RL::kTile, bar);
}

// The raw bytes of one slice of one row for one expanding thread: both 32-blocks
// (codes, scale word, Q5_1 fifth bits), loaded from the raw stage a slice
// ahead of their expansion.
template <int FMT>
struct SliceRaw {
    uint32_t q[2][FMT == MOE_FMT_Q8_0 ? 8 : 4];
    uint32_t s[2], h[2];
};

template <int FMT>
__device__ __forceinline__ void load_slice(const uint8_t *st, int r, int tile, int d, SliceRaw<FMT> &R)
{
    using RL = TlRaw<FMT>;
    const uint8_t *cq = st + RL::codes(tile), *cs = st + RL::scales(tile), *ch = st + RL::qh(tile);
#pragma unroll
    for (int bsel = 0; bsel < 2; ++bsel) {
        const int blk = 2 * d + bsel;
        if constexpr (FMT == MOE_FMT_Q8_0) {
            const uint4 x0 = *reinterpret_cast<const uint4 *>(raw_code(cq, blk >> 2, r, (2 * blk) & 7));
            const uint4 x1 = *reinterpret_cast<const uint4 *>(raw_code(cq, blk >> 2, r, ((2 * blk) & 7) + 1));
            R.q[bsel][0] = x0.x; R.q[bsel][1] = x0.y; R.q[bsel][2] = x0.z; R.q[bsel][3] = x0.w;
            R.q[bsel][4] = x1.x; R.q[bsel][5] = x1.y; R.q[bsel][6] = x1.z; R.q[bsel][7] = x1.w;
        } else {
            const uint4 x0 = *reinterpret_cast<const uint4 *>(raw_code(cq, 0, r, blk));
            R.q[bsel][0] = x0.x; R.q[bsel][1] = x0.y; R.q[bsel][2] = x0.z; R.q[bsel][3] = x0.w;
        }
        if constexpr (FMT == MOE_FMT_Q5_1) {
            const int gsw = (r >> 2) & 1;  // 32-byte swizzle: 16-byte chunk ^ ((r / 4) % 2)
            const int o = r * 32 + ((((blk * 4) >> 4) ^ gsw) << 4) + ((blk * 4) & 15);
            R.s[bsel] = *reinterpret_cast<const uint32_t *>(cs + o);
            R.h[bsel] = *reinterpret_cast<const uint32_t *>(ch + o);
        } else {
            R.s[bsel] = *reinterpret_cast<const uint16_t *>(cs + r * 16 + blk * 2);
            R.h[bsel] = 0;
        }
    }
}

// fp16 of both blocks of the thread's row into its tensor-memory lane: block
// bsel of the slice at columns col + 16 bsel .. + 15 (two fp16 of K per column,
// in K order), the layout the MMA reads A from.
template <int FMT>
__device__ __forceinline__ void store_slice(const SliceRaw<FMT> &R, uint32_t taddr, const CodeTable &tab)
{
#pragma unroll
    for (int bsel = 0; bsel < 2; ++bsel) {
        uint4 o4[4];
        dq::blk_f16<FMT>(R.q[bsel], R.s[bsel], R.h[bsel], tab, o4);
        const uint32_t w[16] = {o4[0].x, o4[0].y, o4[0].z, o4[0].w, o4[1].x, o4[1].y, o4[1].z, o4[1].w,
                                o4[2].x, o4[2].y, o4[2].z, o4[2].w, o4[3].x, o4[3].y, o4[3].z, o4[3].w};
        tmem_st16(taddr + 16 * bsel, w);
    }
}

// The expanding warps' walk over their rings, kept across the two phases.
struct ExpState {
    Ring ra, rr;  // A stages (tensor memory), raw stages
};

// Everything the expanding warps read of the kernel's state.
struct ExpCtx {
    const TailArgs *a;
    const Geo *q;
    const uint8_t *raw;
    uint32_t tmem;  // the CTA's tensor memory
    uint64_t *rf, *re, *fa, *ae;
    volatile int *abort_flag;
    int c, lane, warp;
};

// One phase (0 gate/up, FMT = the gate/up format; 1 down) of the expanding
// warps; false when a wait ran out or the CTA aborted.  Expanding warp w
// (0 .. 7) expands tile w / 4, rows 32 (warp % 4) .. + 31 (the tensor-memory
// lanes its warp may write), one row per lane, into the A stage in tensor
// memory; the next slice's raw bytes are loaded before the current slice's
// expansion.
template <int FMT>
__device__ bool expand_phase(const ExpCtx &x, int p, ExpState &es, const CodeTable &tab)
{
    const TailArgs &a = *x.a;
    const Geo &q = *x.q;
    const int r = 32 * (x.warp & 3) + x.lane, tile = (x.warp - kTlDeqWarp0) >> 2;
    // this thread's lane and tile in an A stage (the stage's columns are added per slice)
    const uint32_t t_row = x.tmem + ((uint32_t)(32 * (x.warp & 3)) << 16) + kTlAcc + tile * 32;
    for (int u = q.lo[p]; u < q.hi[p]; ++u, es.rr.next(a.nr)) {
        if (*x.abort_flag) return false;
        if (!mbar_wait(&x.rf[es.rr.s], es.rr.u & 1)) {
            *x.abort_flag = 1;
            return false;
        }
        if (a.stamps && x.c == 0 && x.warp == kTlDeqWarp0 && x.lane == 0) {  // profiling: CTA 0's first units
            const int ui = (p == 0 ? u - q.lo[0] : q.hi[0] - q.lo[0] + u - q.lo[1]);
            if (ui < 4) a.stamps[24 + ui] = clock64();
        }
        const uint8_t *st = x.raw + es.rr.s * a.raw_stride;
        SliceRaw<FMT> R;
        load_slice<FMT>(st, r, tile, 0, R);
#pragma unroll 1
        for (int d = 0; d < 4; ++d, es.ra.next(a.na)) {
            SliceRaw<FMT> Rn;
            if (d < 3) load_slice<FMT>(st, r, tile, d + 1, Rn);
            if (es.ra.u > 0 && !__all_sync(0xffffffffu, mbar_wait(&x.ae[es.ra.s], (es.ra.u - 1) & 1))) {
                *x.abort_flag = 1;
                return false;
            }
            tc_fence_after_sync();  // the MMAs that read this stage are complete
            store_slice<FMT>(R, t_row + es.ra.s * kTlAStageCols, tab);
            tmem_wait_st();
            tc_fence_before_sync();
            __syncwarp();
            if (x.lane == 0) mbar_arrive(&x.fa[es.ra.s]);
            if (d < 3) R = Rn;
        }
        __syncwarp();
        if (x.lane == 0) mbar_arrive(&x.re[es.rr.s]);
    }
    return true;
}

__host__ __device__ constexpr uint32_t tl_idesc(int N)
{
    // kind::f16: f16 x f16 -> f32, both K-major, M = 128
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

template <int FG, int FD>
__global__ void __launch_bounds__(kTlThreads, 1)
    tail_kernel(const __grid_constant__ CUtensorMap mXg, const __grid_constant__ CUtensorMap mH, const TailArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t rf_bar[kTlMaxRaw], re_bar[kTlMaxRaw], fa_bar[kTlNA], ae_bar[kTlNA],
        fb_bar[kTlMaxB], be_bar[kTlMaxB], accf_bar[2], acce_bar[2], dr_bar, wr_bar;
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;
    __shared__ volatile int s_epi_abort;  // the four epilogue warps leave together
    __shared__ int s_misc[8];  // [0] groups, [1] slots, [3] epilogue: last arrival
    __shared__ int s_tmp[32];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int G = gridDim.x, c = blockIdx.x;
    const int T = a.T, H = a.H, E = a.E, I = a.I, k = a.k;
    const TlCtr C = tl_ctr(E, H, I);
    const TlPlanLayout PL = tl_plan_layout(T, k, E);
    uint8_t *plan = smem + a.rings;
    int16_t *p_sel_e = reinterpret_cast<int16_t *>(plan + PL.sel_e);
    float *p_sel_g = reinterpret_cast<float *>(plan + PL.sel_g);
    int16_t *p_slot_of = reinterpret_cast<int16_t *>(plan + PL.slot_of);
    int16_t *p_grp_e = reinterpret_cast<int16_t *>(plan + PL.grp_e);
    int16_t *p_grp_n = reinterpret_cast<int16_t *>(plan + PL.grp_n);
    int *p_grp_off = reinterpret_cast<int *>(plan + PL.grp_off);
    int16_t *p_slot_tok = reinterpret_cast<int16_t *>(plan + PL.slot_tok);
    const int xbytes = a.x_dtype == MOE_DT_BF16 ? 2 : 4;
    const TlRoute R = tl_route(T, E, G, xbytes);
    const int tb = c % R.ntb, rb = c / R.ntb;
    const bool router_cta = rb < R.nrb;
    const int t0 = tb * R.rt, tn = min(R.rt, T - t0);
    const int e0 = router_cta ? E * rb / R.nrb : 0, e1 = router_cta ? E * (rb + 1) / R.nrb : 0;
    const int rows_max = tl_cdiv(E, R.nrb);
    uint16_t *sWr = reinterpret_cast<uint16_t *>(smem);
    float *sX = reinterpret_cast<float *>(smem + tl_al16(rows_max * H * 2));

    if (warp == kTlMmaWarp) {
        tmem_alloc(&tmem_base, kTlTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < a.na; ++s) {
            mbar_init(&fa_bar[s], kTlDeqWarps);
            mbar_init(&ae_bar[s], 1);
        }
        for (int s = 0; s < a.nb; ++s) {
            mbar_init(&fb_bar[s], 1);
            mbar_init(&be_bar[s], 1);
        }
        for (int s = 0; s < a.nr; ++s) {
            mbar_init(&rf_bar[s], 1);
            mbar_init(&re_bar[s], kTlDeqWarps);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&accf_bar[s], 1);
            mbar_init(&acce_bar[s], kTlEpiWarps);
        }
        mbar_init(&dr_bar, 1);
        mbar_init(&wr_bar, 1);
        abort_flag = 0;
        s_epi_abort = 0;
        s_misc[0] = s_misc[1] = s_misc[2] = s_misc[3] = 0;
        fence_mbar_init();
        // router rows: independent of the previous kernel, requested before waiting on it
        if (router_cta && e1 > e0) {
            mbar_arrive_expect_tx(&wr_bar, (uint32_t)((e1 - e0) * H * 2));
            bulk_g2s(sWr, a.wr + (size_t)e0 * H, (uint32_t)((e1 - e0) * H * 2), &wr_bar);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_base;
    grid_event(a.stamps, 0);
    cta0_clock(a.stamps, 0);
    asm volatile("griddepcontrol.wait;" ::: "memory");  // x, out and the workspace are ours from here

    // ---- route: logits of rows [e0, e1) for tokens [t0, t0 + tn) ------------------------
    if (router_cta) {
        // x as fp32 in shared memory: each thread's 16-byte loads all in flight first
        const int cpr = H / 8, nch = tn * cpr;
        for (int i0 = 0; i0 < nch; i0 += 8 * kTlThreads) {
            uint4 q[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = i0 + j * kTlThreads + tid;
                if (i < nch) {
                    const int t = i / cpr, ch = i - t * cpr;
                    q[j] = a.x_dtype == MOE_DT_BF16
                               ? __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(a.x) +
                                                                       (size_t)(t0 + t) * H) + ch)
                               : __ldg(reinterpret_cast<const uint4 *>(static_cast<const float *>(a.x) +
                                                                       (size_t)(t0 + t) * H) + ch * 2);
                }
            }
            uint4 q2[8];  // fp32 x: the second half of each 8-value chunk
            if (a.x_dtype != MOE_DT_BF16) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int i = i0 + j * kTlThreads + tid;
                    if (i < nch) {
                        const int t = i / cpr, ch = i - t * cpr;
                        q2[j] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const float *>(a.x) +
                                                                      (size_t)(t0 + t) * H) + ch * 2 + 1);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = i0 + j * kTlThreads + tid;
                if (i < nch) {
                    const int t = i / cpr, ch = i - t * cpr;
                    float4 *d = reinterpret_cast<float4 *>(sX + (size_t)t * H + ch * 8);
                    if (a.x_dtype == MOE_DT_BF16) {
                        d[0] = make_float4(__uint_as_float(q[j].x << 16), __uint_as_float(q[j].x & 0xFFFF0000u),
                                           __uint_as_float(q[j].y << 16), __uint_as_float(q[j].y & 0xFFFF0000u));
                        d[1] = make_float4(__uint_as_float(q[j].z << 16), __uint_as_float(q[j].z & 0xFFFF0000u),
                                           __uint_as_float(q[j].w << 16), __uint_as_float(q[j].w & 0xFFFF0000u));
                    } else {
                        d[0] = make_float4(__uint_as_float(q[j].x), __uint_as_float(q[j].y),
                                           __uint_as_float(q[j].z), __uint_as_float(q[j].w));
                        d[1] = make_float4(__uint_as_float(q2[j].x), __uint_as_float(q2[j].y),
                                           __uint_as_float(q2[j].z), __uint_as_float(q2[j].w));
                    }
                }
            }
        }
        __syncthreads();
        bool ok = e1 <= e0 || mbar_wait(&wr_bar, 0);
        if (!ok && lane == 0) {
            abort_flag = 1;
            atomicExch(a.err, (int)MOE_ERR_TIMEOUT);
        }
        // router rows x K parts over the warps: warp w takes (row, K part) items
        // w, w + 23, ...; lane l 8 consecutive weights of each 256; each item's
        // partial dot products per token go to shared memory and are summed in
        // K-part order
        const int rows = e1 - e0, H256 = H / 256;
        int kparts = 1;
        while (kparts * 2 <= H256 && rows * kparts * 2 <= kTlWarps && H256 % (kparts * 2) == 0) kparts *= 2;
        const int klen = H / kparts;
        float *part = sX + (size_t)R.rt * H;  // [rows][kparts][rt]
        for (int item = warp; ok && item < rows * kparts; item += kTlWarps) {
            const int row = item / kparts, kp = item - row * kparts;
            const uint16_t *wrow = sWr + (size_t)row * H;
            for (int tq = 0; tq < tn; tq += 8) {
                float acc[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) acc[t] = 0.f;
                for (int k0 = kp * klen + lane * 8; k0 < (kp + 1) * klen; k0 += 256) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(wrow + k0);
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                    float wf[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        wf[2 * j] = __uint_as_float(ww[j] << 16);
                        wf[2 * j + 1] = __uint_as_float(ww[j] & 0xFFFF0000u);
                    }
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        if (tq + t < tn) {
                            const float *xr = sX + (size_t)(tq + t) * H + k0;
                            const float4 x0 = *reinterpret_cast<const float4 *>(xr);
                            const float4 x1 = *reinterpret_cast<const float4 *>(xr + 4);
                            float s2 = acc[t];
                            s2 = fmaf(wf[0], x0.x, s2); s2 = fmaf(wf[1], x0.y, s2);
                            s2 = fmaf(wf[2], x0.z, s2); s2 = fmaf(wf[3], x0.w, s2);
                            s2 = fmaf(wf[4], x1.x, s2); s2 = fmaf(wf[5], x1.y, s2);
                            s2 = fmaf(wf[6], x1.z, s2); s2 = fmaf(wf[7], x1.w, s2);
                            acc[t] = s2;
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    if (tq + t < tn) {
                        float s2 = acc[t];
#pragma unroll
                        for (int o = 16; o >= 1; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
                        if (lane == 0) part[((size_t)row * kparts + kp) * R.rt + tq + t] = s2;
                    }
                }
            }
        }
        __syncthreads();
        for (int i = tid; ok && i < rows * tn; i += kTlThreads) {
            const int row = i / tn, t = i - row * tn;
            float l = 0.f;
            for (int kp = 0; kp < kparts; ++kp) l += part[((size_t)row * kparts + kp) * R.rt + t];
            a.logits[(size_t)(t0 + t) * E + e0 + row] = l;
        }
    }
    // ---- grid barrier: every logit written ------------------------------------------------
    __syncthreads();
    grid_event(a.stamps, 1);
    cta0_clock(a.stamps, 1);
    if (tid == 0) {
        __threadfence();
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(a.ctr + C.bar) : "memory");
        if (!wait_count(a.ctr + C.bar, (unsigned)G)) {
            abort_flag = 1;
            atomicExch(a.err, (int)MOE_ERR_TIMEOUT);
        }
    }
    __syncthreads();
    const bool run = !abort_flag;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    cta0_clock(a.stamps, 2);

    // ---- plan: top-k of every token, then groups and slots --------------------------------
    if (run) {
        const int nsw = min(kTlWarps, T);
        if (warp < nsw) {
            float *row = reinterpret_cast<float *>(smem) + (size_t)warp * E;
            unsigned *cand = reinterpret_cast<unsigned *>(smem + (size_t)nsw * E * 4) + warp * 128;
            for (int t = warp; t < T; t += nsw) {
                // every load of the lane in flight before the stores (one L2 round trip)
                if (E <= 512) stage_logits<16>(a.logits + (size_t)t * E, row, E, lane);
                else stage_logits<32>(a.logits + (size_t)t * E, row, E, lane);
                __syncwarp();
                int my_e;
                float my_g;
                if (E <= 512) topk_threshold<16>(row, E, k, my_e, my_g, cand);
                else topk_threshold<32>(row, E, k, my_e, my_g, cand);
                if (lane < k) {
                    p_sel_e[t * k + lane] = (int16_t)my_e;
                    p_sel_g[t * k + lane] = my_g;
                    if (c == 0) {
                        a.idx_out[t * k + lane] = my_e;
                        a.gate_out[t * k + lane] = my_g;
                    }
                }
                __syncwarp();
            }
        }
        __syncthreads();
        cta0_clock(a.stamps, 3);
        // counts and 64-bit token masks per expert
        int *cnt = reinterpret_cast<int *>(smem);
        unsigned *mask = reinterpret_cast<unsigned *>(smem + tl_al16((E + 1) * 4));
        for (int e = tid; e <= E; e += kTlThreads) cnt[e] = 0;
        for (int e = tid; e < 2 * E; e += kTlThreads) mask[e] = 0u;
        __syncthreads();
        for (int i = tid; i < T * k; i += kTlThreads) {
            const int e = p_sel_e[i], t = i / k;
            if (e < a.eb || e >= a.ee) continue;  // another pack's expert (expert parallelism)
            atomicAdd(&cnt[e], 1);
            atomicOr(&mask[2 * e + (t >> 5)], 1u << (t & 31));
        }
        __syncthreads();
        // groups: active experts in ascending order; packed scan of {flag, tokens}
        for (int e = tid; e < E; e += kTlThreads) {
            const int n = cnt[e];
            if (c == 0) a.cnt_out[e] = n;
            cnt[e] = n ? (1 << 16) | n : 0;
        }
        if (c == 0 && tid == 0) a.cnt_out[E] = a.has_shared ? T : 0;
        __syncthreads();
        // entries hold {flag, tokens} of expert e; after the scan, the groups and
        // slots before it
        {
            // save each expert's own {flag, tokens} before the in-place scan overwrites it
            int *own = reinterpret_cast<int *>(smem + tl_al16((E + 1) * 4) + E * 8);
            for (int e = tid; e < E; e += kTlThreads) own[e] = cnt[e];
            __syncthreads();
            const int total = block_scan(cnt, E, s_tmp);
            const int n_routed = total >> 16, routed_slots = total & 0xFFFF;
            for (int e = tid; e < E; e += kTlThreads) {
                const int v = own[e];
                if (v) {
                    const int g = cnt[e] >> 16;
                    p_grp_e[g] = (int16_t)(e - a.eb);  // the expert's slot in the pack
                    p_grp_n[g] = (int16_t)(v & 0xFFFF);
                    p_grp_off[g] = cnt[e] & 0xFFFF;
                }
            }
            if (tid == 0) {
                int ng = n_routed;
                if (a.has_shared) {
                    p_grp_e[ng] = (int16_t)(a.ee - a.eb);
                    p_grp_n[ng] = (int16_t)T;
                    p_grp_off[ng] = routed_slots;
                    ++ng;
                }
                s_misc[0] = ng;
                s_misc[1] = routed_slots + (a.has_shared ? T : 0);
            }
            __syncthreads();
            // slot of each (token, choice): the expert's first slot + earlier tokens of it
            for (int i = tid; i < T * k; i += kTlThreads) {
                const int e = p_sel_e[i], t = i / k;
                if (e < a.eb || e >= a.ee) {
                    p_slot_of[i] = -1;  // not this pack's: no slot, no share of the output
                    continue;
                }
                const unsigned long long m =
                    (unsigned long long)mask[2 * e] | ((unsigned long long)mask[2 * e + 1] << 32);
                const int slot = (cnt[e] & 0xFFFF) + __popcll(m & ((1ull << t) - 1ull));
                p_slot_of[i] = (int16_t)slot;
                p_slot_tok[slot] = (int16_t)t;
            }
            if (a.has_shared)
                for (int t = tid; t < T; t += kTlThreads) p_slot_tok[routed_slots + t] = (int16_t)t;
        }
        __syncthreads();
        cta0_clock(a.stamps, 4);
    }
    __syncthreads();
    grid_event(a.stamps, 2);
    cta0_clock(a.stamps, 5);

    // ---- gate/up and down units -------------------------------------------------------
    const int ng = s_misc[0];
    Geo q;
    q.KC[0] = H / 256;
    q.NB[0] = I / 128;
    q.KC[1] = I / 256;
    q.NB[1] = H / 256;
    for (int p = 0; p < 2; ++p) {
        q.U[p] = ng * q.NB[p] * q.KC[p];
        q.lo[p] = range_lo(q.U[p], c, G);
        q.hi[p] = range_lo(q.U[p], c + 1, G);
    }
    uint8_t *raw = smem, *bring = smem + a.nr * a.raw_stride;
    int raw_issued = 0, b_issued = 0;

    // ---- this CTA's share of the fp16 slot rows of x (slots [s0, s1)), by the
    // epilogue and expanding warps while the raw producer and the MMA issuer
    // start: the row's largest magnitude picks the power of two 2^s that keeps
    // it below 2^15 (x stays exact in fp16), the row is written times 2^-s and
    // 2^s kept per slot; then one count on the readiness counter of each group
    // met
    if (run && (warp < kTlEpiWarps || warp >= kTlDeqWarp0)) {
        const int wt = warp < kTlEpiWarps ? tid : tid - 32 * (kTlDeqWarp0 - kTlEpiWarps);
        const int wwarp = wt >> 5;
        const int S = s_misc[1];
        const int s0 = (int)((long long)S * c / G), s1 = (int)((long long)S * (c + 1) / G);
        const int cpr = H / 8;  // 8-value chunks per row
        auto load8 = [&](int t, int ch, float *v) {
            if (a.x_dtype == MOE_DT_BF16) {
                const uint4 q4 =
                    __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(a.x) + (size_t)t * H) + ch);
                const uint32_t w4[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    v[2 * i] = __uint_as_float(w4[i] << 16);
                    v[2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
                }
            } else {
                const float4 *pf = reinterpret_cast<const float4 *>(static_cast<const float *>(a.x) + (size_t)t * H) +
                                   2 * ch;
                const float4 x0 = __ldg(pf), x1 = __ldg(pf + 1);
                v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
                v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
            }
        };
        for (int sl = s0; sl < s1; ++sl) {
            const int t = p_slot_tok[sl];
            unsigned mx = 0u;
            for (int ch = wt; ch < cpr; ch += kTlWriters) {
                float v[8];
                load8(t, ch, v);
#pragma unroll
                for (int i = 0; i < 8; ++i) mx = max(mx, __float_as_uint(fabsf(v[i])));
            }
            mx = __reduce_max_sync(0xffffffffu, mx);
            if ((wt & 31) == 0) s_tmp[wwarp] = (int)mx;
            asm volatile("bar.sync 2, %0;" ::"n"(kTlWriters) : "memory");
#pragma unroll 1
            for (int w2 = 0; w2 < kTlWriters / 32; ++w2) mx = max(mx, (unsigned)s_tmp[w2]);
            asm volatile("bar.sync 2, %0;" ::"n"(kTlWriters) : "memory");  // s_tmp is reused by the next slot
            const int ex = (int)((mx >> 23) & 0xFFu) - 127;  // exponent of max |x| (inf / NaN: unscaled)
            const int sh = (ex >= 15 && ex < 128) ? ex - 14 : 0;
            const float down = __uint_as_float((uint32_t)(127 - sh) << 23);
            if (wt == 0) a.slot_scale[sl] = __uint_as_float((uint32_t)(127 + sh) << 23);
            for (int ch = wt; ch < cpr; ch += kTlWriters) {  // second pass: the row again, from L1 / L2
                float v[8];
                load8(t, ch, v);
                uint4 o;
                o.x = dq::pack_f16x2(v[0] * down, v[1] * down);
                o.y = dq::pack_f16x2(v[2] * down, v[3] * down);
                o.z = dq::pack_f16x2(v[4] * down, v[5] * down);
                o.w = dq::pack_f16x2(v[6] * down, v[7] * down);
                reinterpret_cast<uint4 *>(a.xg + (size_t)sl * H)[ch] = o;
            }
        }
        asm volatile("bar.sync 2, %0;" ::"n"(kTlWriters) : "memory");
        if (wt == 0 && s1 > s0) {
            __threadfence();
            for (int g = 0; g < ng; ++g) {  // groups whose slot range meets [s0, s1)
                const int o = p_grp_off[g], n = p_grp_n[g];
                if (o < s1 && o + n > s0) atomicAdd(a.ctr + C.grp_x + g, 1u);
            }
        }
    }

    if (run && warp == kTlRawWarp) {
        if (lane == 0) {
            Ring rr;
            for (int p = 0; p < 2 && !abort_flag; ++p)
                for (int u = q.lo[p]; u < q.hi[p] && !abort_flag; ++u, rr.next(a.nr)) {
                    const Unit x = unit_at(q, p, u);
                    if (rr.u > 0 && !mbar_wait_idle(&re_bar[rr.s], (rr.u - 1) & 1)) {
                        abort_flag = 1;
                        break;
                    }
                    uint8_t *st = raw + rr.s * a.raw_stride;
                    const int ex = p_grp_e[x.g];
                    if (p == 0)  // gate rows block b and up rows block I / 128 + b
                        raw_load<FG>(st, a.tl_gu, a.tl_gu_stride, q.KC[0], &rf_bar[rr.s], x.kc, x.b, I / 128 + x.b, ex);
                    else  // output rows blocks 2b and 2b + 1
                        raw_load<FD>(st, a.tl_dn, a.tl_dn_stride, q.KC[1], &rf_bar[rr.s], x.kc, 2 * x.b, 2 * x.b + 1, ex);
                }
            raw_issued = rr.u * a.nr + rr.s;
        }
    } else if (run && warp == kTlBWarp) {
        if (lane == 0) {
            prefetch_tmap(&mXg);
            prefetch_tmap(&mH);
            Ring rb;
            int ready_g = -1, ready_p = -1;
            for (int p = 0; p < 2 && !abort_flag; ++p)
                for (int u = q.lo[p]; u < q.hi[p] && !abort_flag; ++u) {
                    const Unit x = unit_at(q, p, u);
                    const int n = p_grp_n[x.g], off = p_grp_off[x.g], n16 = (n + 15) >> 4;
                    if (x.g != ready_g || p != ready_p) {
                        // gate/up: the group's x slot rows written by the CTAs that own
                        // them; down: all of the group's h tiles finished.  The rows were
                        // written with generic stores: the acquire of the full count, then
                        // a proxy fence, before the TMA reads them
                        const unsigned *cp = a.ctr + (p == 0 ? C.grp_x : C.grp_h) + x.g;
                        if (!wait_count(cp, p == 0 ? (unsigned)owners(off, n, s_misc[1], G) : (unsigned)q.NB[0])) {
                            abort_flag = 1;
                            atomicExch(a.err, (int)MOE_ERR_TIMEOUT);
                            break;
                        }
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                        ready_g = x.g;
                        ready_p = p;
                    }
                    for (int sl = 0; sl < 4; ++sl, rb.next(a.nb)) {
                        if (rb.u > 0 && !mbar_wait_idle(&be_bar[rb.s], (rb.u - 1) & 1)) {
                            abort_flag = 1;
                            break;
                        }
                        uint8_t *b_s = bring + rb.s * a.bslot;
                        mbar_arrive_expect_tx(&fb_bar[rb.s], (uint32_t)n16 * 2048u);
                        for (int jj = 0; jj < n16; ++jj)
                            tma_load_2d(b_s + jj * 2048, p == 0 ? &mXg : &mH, &fb_bar[rb.s], x.kc * 256 + sl * 64,
                                        off + 16 * jj);
                    }
                }
            b_issued = rb.u * a.nb + rb.s;
        }
    } else if (run && warp == kTlMmaWarp) {
        if (lane == 0) {
            Ring ra, rbm;
            int seg = 0;
            for (int p = 0; p < 2 && !abort_flag; ++p)
                for (int u = q.lo[p]; u < q.hi[p] && !abort_flag; ++u) {
                    const Unit x = unit_at(q, p, u);
                    const int ab = seg & 1;
                    if (x.first && seg >= 2 && !mbar_wait(&acce_bar[ab], ((seg >> 1) - 1) & 1)) {
                        abort_flag = 1;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t idesc = tl_idesc((p_grp_n[x.g] + 15) & ~15);
                    for (int sl = 0; sl < 4; ++sl, ra.next(a.na), rbm.next(a.nb)) {
                        if (!mbar_wait(&fa_bar[ra.s], ra.u & 1) || !mbar_wait(&fb_bar[rbm.s], rbm.u & 1)) {
                            abort_flag = 1;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint32_t a_t = tmem + kTlAcc + ra.s * kTlAStageCols;
                        const uint64_t bd = desc_kmajor_sw128(bring + rbm.s * a.bslot);
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_f16_ts(tmem + ab * 128 + hh * 64, a_t + hh * 32 + kk * 8, bd + 2 * kk, idesc,
                                           !(x.first && sl == 0 && kk == 0));
                        }
                        mma_commit(&ae_bar[ra.s]);
                        mma_commit(&be_bar[rbm.s]);
                    }
                    if (a.stamps && c == 0) {  // profiling: CTA 0's first units, MMAs issued
                        const int ui = (p == 0 ? u - q.lo[0] : q.hi[0] - q.lo[0] + u - q.lo[1]);
                        if (ui < 4) a.stamps[28 + ui] = clock64();
                    }
                    if (x.last) {
                        mma_commit(&accf_bar[ab]);
                        ++seg;
                    }
                }
        }
    } else if (run && warp >= kTlDeqWarp0) {
        ExpCtx xc;
        xc.a = &a;
        xc.q = &q;
        xc.raw = raw;
        xc.tmem = tmem;
        xc.rf = rf_bar;
        xc.re = re_bar;
        xc.fa = fa_bar;
        xc.ae = ae_bar;
        xc.abort_flag = &abort_flag;
        xc.c = c;
        xc.lane = lane;
        xc.warp = warp;
        ExpState es;
        if (expand_phase<FG>(xc, 0, es, a.tab_gu)) expand_phase<FD>(xc, 1, es, a.tab_dn);
        tmem_wait_st();  // no store into tensor memory outlives the loop (abort included)
    } else if (run && warp < kTlEpiWarps) {
        // ---- epilogue: one tensor-memory lane (tile row) per thread --------------------
        const int r = warp * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
        int seg = 0;
        bool range_ok = true;
        for (int p = 0; p < 2; ++p)
            for (int u = q.lo[p]; u < q.hi[p]; ++u) {
                const Unit x = unit_at(q, p, u);
                if (!x.last) continue;
                const int ab = seg & 1;
                const bool w_ok = mbar_wait_idle(&accf_bar[ab], (seg >> 1) & 1);
                tc_fence_after_sync();
                // one decision for all four warps (they share named barriers): each
                // raises the vote before the barrier, all read it after; every later
                // iteration passes a barrier before the next vote is raised
                if (!__all_sync(0xffffffffu, w_ok) || __any_sync(0xffffffffu, abort_flag != 0)) s_epi_abort = 1;
                epi_sync();
                if (s_epi_abort) {
                    if (r == 0) {
                        abort_flag = 1;
                        atomicExch(a.err, (int)MOE_ERR_TIMEOUT);
                    }
                    p = 2;
                    break;
                }
                ++seg;
                const int n = p_grp_n[x.g], off = p_grp_off[x.g], n16 = (n + 15) >> 4;
                const int t0u = x.tile * q.KC[p];
                // the whole tile in this CTA: straight from tensor memory; else this
                // CTA's piece goes out and the CTA that finishes the tile's last piece
                // sums them in CTA order
                const bool whole = t0u >= q.lo[p] && t0u + q.KC[p] <= q.hi[p];
                const uint32_t tb0 = tl + ab * 128;
                float *pc = whole ? nullptr : piece(a, q, p, c, x.tile, G);
                bool finalize = whole;
                if (!whole) {
                    for (int c0 = 0; c0 < n16; ++c0) {
                        float v0[16], v1[16];
                        tmem_ld16(tb0 + c0 * 16, v0);
                        tmem_ld16(tb0 + 64 + c0 * 16, v1);
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (c0 * 16 + j < n) {
                                pc[(size_t)(c0 * 16 + j) * 256 + r] = v0[j];
                                pc[(size_t)(c0 * 16 + j) * 256 + 128 + r] = v1[j];
                            }
                    }
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acce_bar[ab]);
                    // the four warps' piece stores, then one release by the leader (the
                    // named barrier orders them before its fence)
                    epi_sync();
                    if (r == 0) {
                        __threadfence();
                        const unsigned prev = atomicAdd(a.ctr + (p == 0 ? C.gu_tile : C.dn_tile) + x.tile, 1u);
                        s_misc[3] = prev + 1 == (unsigned)owners(t0u, q.KC[p], q.U[p], G);
                        __threadfence();
                    }
                    epi_sync();
                    finalize = s_misc[3] != 0;
                    epi_sync();
                    if (!finalize) continue;
                }
                const int e = p_grp_e[x.g];
                const float hts = (p == 0 ? FG : FD) == MOE_FMT_NVFP4 ? 0.5f * __ldg((p == 0 ? a.ts_gu : a.ts_dn) + e)
                                                                        : 1.f;
                // the slot scales came with the x rows the B producer waited for: an
                // acquire of the group's (full) readiness count orders their reads
                if (p == 0) (void)ld_acq(a.ctr + C.grp_x + x.g);
                for (int c0 = 0; c0 < n16; ++c0) {
                    float v0[16], v1[16], ssc[16];
                    if (p == 0) {  // the slots' scales, requested with the pieces
#pragma unroll
                        for (int j = 0; j < 16; ++j) ssc[j] = c0 * 16 + j < n ? __ldcg(a.slot_scale + off + c0 * 16 + j) : 0.f;
                    }
                    if (whole) {
                        tmem_ld16(tb0 + c0 * 16, v0);
                        tmem_ld16(tb0 + 64 + c0 * 16, v1);
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) v0[j] = v1[j] = 0.f;
                        // the owners of the tile's units in CTA order, two at a time: both
                        // pieces requested before either is added (the sum keeps CTA order)
                        int uu = t0u, prev = -1;
                        auto next_owner = [&]() {
                            while (uu < t0u + q.KC[p]) {
                                const int cu = cta_of(uu++, q.U[p], G);
                                if (cu != prev) {
                                    prev = cu;
                                    return cu;
                                }
                            }
                            return -1;
                        };
                        for (int oa = next_owner(); oa >= 0; oa = next_owner()) {
                            const int ob = next_owner();
                            const float *pa = piece(a, q, p, oa, x.tile, G);
                            const float *pb = ob >= 0 ? piece(a, q, p, ob, x.tile, G) : pa;
                            float a0[16], a1[16], b0[16], b1[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const bool in = c0 * 16 + j < n;
                                const size_t o = (size_t)(c0 * 16 + j) * 256 + r;
                                a0[j] = in ? __ldcg(pa + o) : 0.f;
                                a1[j] = in ? __ldcg(pa + o + 128) : 0.f;
                                b0[j] = in && ob >= 0 ? __ldcg(pb + o) : 0.f;
                                b1[j] = in && ob >= 0 ? __ldcg(pb + o + 128) : 0.f;
                            }
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                v0[j] += a0[j];
                                v1[j] += a1[j];
                            }
                            if (ob < 0) break;
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                v0[j] += b0[j];
                                v1[j] += b1[j];
                            }
                        }
                    }
                    if (p == 0) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int jj = c0 * 16 + j;
                            if (jj < n) {
                                const int slot = off + jj;
                                const float sc = ssc[j] * hts;
                                const float gv = v0[j] * sc, uv = v1[j] * sc;
                                const float hv = gv / (1.f + expf(-gv)) * uv;
                                range_ok = range_ok && fabsf(hv) <= 65504.f;
                                a.h[(size_t)slot * I + x.b * 128 + r] = __float2half_rn(hv);
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int jj = c0 * 16 + j;
                            if (jj < n) {
                                float *yr = a.y + (size_t)(off + jj) * H + x.b * 256 + r;
                                yr[0] = v0[j] * hts;
                                yr[128] = v1[j] * hts;
                            }
                        }
                    }
                }
                if (whole) {
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acce_bar[ab]);
                }
                epi_sync();
                if (r == 0) {
                    __threadfence();  // the four warps' h / y stores, released by the leader
                    if (p == 0) {
                        atomicAdd(a.ctr + C.grp_h + x.g, 1u);
                    } else {
                        atomicAdd(a.ctr + C.rb + x.b, 1u);  // one more group's y rows of this block are in
                    }
                }
            }
        if (!__all_sync(0xffffffffu, range_ok) && lane == 0) atomicExch(a.err, (int)MOE_ERR_RANGE);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (abort_flag) {  // block-uniform after the barrier: drain what was issued, then release
        if (tid == 0 && router_cta && e1 > e0) mbar_wait(&wr_bar, 0);  // the router rows' bulk copy
        if (lane == 0 && warp == kTlRawWarp) drain_ring(rf_bar, a.nr, raw_issued);
        if (lane == 0 && warp == kTlBWarp) drain_ring(fb_bar, a.nb, b_issued);
        if (lane == 0 && warp == kTlMmaWarp) drain_mma(&dr_bar);
        if (tid == 0) atomicExch(a.err, (int)MOE_ERR_TIMEOUT);
        tc_fence_before_sync();
        __syncthreads();
    }
    grid_event(a.stamps, 3);
    cta0_clock(a.stamps, 6);
    // ---- combine: rows [H c / G, H (c + 1) / G) of every token, once every group's
    // y rows of their 256-row blocks are in: out[t] = sum_j gate_tj y[slot(t, j)]
    // (+ the shared expert's y), in the layer's order ------------------------------------
    if (!abort_flag) {
        const int has = a.has_shared, routed_slots = s_misc[1] - (has ? T : 0);
        const int r0 = (int)((long long)H * c / G), r1 = (int)((long long)H * (c + 1) / G), nrow = r1 - r0;
        if (ng > 0 && nrow > 0 && tid == 0) {
            for (int b = r0 / 256; b <= (r1 - 1) / 256; ++b)
                if (!wait_count(a.ctr + C.rb + b, (unsigned)ng)) {
                    abort_flag = 1;
                    atomicExch(a.err, (int)MOE_ERR_TIMEOUT);
                    break;
                }
        }
        __syncthreads();
        if (!abort_flag && nrow > 0) {
            for (int i = tid; i < T * nrow; i += kTlThreads) {
                const int t = i / nrow, row = r0 + (i - t * nrow);
                float o = 0.f;
                if (ng > 0) {  // else no expert of this pack was selected and it has no shared expert: a zero share
                    float yv[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {  // every gather in flight before the sum
                        const int sl = j < k ? p_slot_of[t * k + j] : -1;
                        yv[j] = sl >= 0 ? __ldcg(a.y + (size_t)sl * H + row) : 0.f;
                    }
                    const float ys = has ? __ldcg(a.y + (size_t)(routed_slots + t) * H + row) : 0.f;
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (j < k && p_slot_of[t * k + j] >= 0) o += p_sel_g[t * k + j] * yv[j];
                    if (has) o += ys;
                }
                a.out[(size_t)t * H + row] = o;
            }
        }
    }
    __syncthreads();
    grid_event(a.stamps, 4);
    cta0_clock(a.stamps, 7);
    // ---- the last CTA to finish clears the counters this launch used --------------------
    if (tid == 0) {
        __threadfence();
        s_tmp[0] = atomicAdd(a.ctr + C.ticket, 1u) == (unsigned)G - 1u;
    }
    __syncthreads();
    if (s_tmp[0]) {
        __threadfence();
        if (__ldcg(a.err) != 0) {
            // a CTA gave up somewhere: every counter, whatever the plan reached
            for (int i = tid; i < C.total; i += kTlThreads)
                if (i != C.ticket) a.ctr[i] = 0u;
        } else {
            for (int i = tid; i < ng * q.NB[0]; i += kTlThreads) a.ctr[C.gu_tile + i] = 0u;
            for (int i = tid; i < ng * q.NB[1]; i += kTlThreads) a.ctr[C.dn_tile + i] = 0u;
            for (int i = tid; i < ng; i += kTlThreads) {
                a.ctr[C.grp_x + i] = 0u;
                a.ctr[C.grp_h + i] = 0u;
            }
            for (int i = tid; i < H / 256; i += kTlThreads) a.ctr[C.rb + i] = 0u;
            if (tid == 0) a.ctr[C.bar] = 0u;
        }
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            a.ctr[C.ticket] = 0u;
        }
    }
    if (warp == kTlMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTlTmemCols);
    }
}

using TlKernel = void (*)(const CUtensorMap, const CUtensorMap, const TailArgs);

template <int FG>
TlKernel tl_pick_dn(int fd)
{
    switch (fd) {
    case MOE_FMT_Q8_0: return tail_kernel<FG, MOE_FMT_Q8_0>;
    case MOE_FMT_Q5_1: return tail_kernel<FG, MOE_FMT_Q5_1>;
    case MOE_FMT_IQ4_NL: return tail_kernel<FG, MOE_FMT_IQ4_NL>;
    default: return tail_kernel<FG, MOE_FMT_NVFP4>;
    }
}

TlKernel tl_pick(int fg, int fd)
{
    switch (fg) {
    case MOE_FMT_Q8_0: return tl_pick_dn<MOE_FMT_Q8_0>(fd);
    case MOE_FMT_Q5_1: return tl_pick_dn<MOE_FMT_Q5_1>(fd);
    case MOE_FMT_IQ4_NL: return tl_pick_dn<MOE_FMT_IQ4_NL>(fd);
    default: return tl_pick_dn<MOE_FMT_NVFP4>(fd);
    }
}

constexpr int kTlSmemMax = 225 * 1024;  // dynamic shared memory per CTA (the static part comes on top)

}  // namespace

int tail_counter_words(int E, int H, int I) { return tl_ctr(E, H, I).total; }

size_t tail_part_floats(int grid, int max_tokens) { return (size_t)2 * grid * 2 * 256 * ((std::min(max_tokens, 64) + 15) & ~15); }

bool tail_plan(const TailPlanIn &in, TailLaunch *out)
{
    if (in.T < 1 || in.T > kDecodeTcMaxN || in.max_tokens < in.T || in.k > 16 || in.E > 1024 || in.E > 4 * kTlThreads) return false;
    if (in.H % 256 || in.I % 256 || in.H > 16384 || in.I > 16384) return false;
    const int xbytes = in.x_dtype == MOE_DT_BF16 ? 2 : 4;
    const int n16max = (std::min(in.max_tokens, 64) + 15) & ~15;
    const TlPlanLayout PL = tl_plan_layout(in.T, in.k, in.E);
    const int raw = std::max(tl_raw_bytes(in.fmt_gu), tl_raw_bytes(in.fmt_dn));
    const int bslot = n16max * 128;  // a multiple of 2048
    const int budget = kTlSmemMax - 1024 - PL.total;
    // the A stages live in tensor memory (kTlNA of them); shared memory holds
    // the raw stages and the B slots: two raw stages and four slots at least,
    // then more of each, in turn, while they fit
    int nr = 2, nb = 4;
    const int na = kTlNA;
    auto rings = [&] { return nr * raw + nb * bslot; };
    if (rings() > budget) return false;
    bool grown = true;
    while (grown) {
        grown = false;
        if (nr < kTlMaxRaw && rings() + raw <= budget) { ++nr; grown = true; }
        if (nb < kTlMaxB && rings() + bslot <= budget) { ++nb; grown = true; }
    }
    // the routing and planning scratch is overlaid on the rings: the region is the larger of the two
    const int region = std::max(rings(), tl_scratch_bytes(in.T, in.H, in.E, in.grid, xbytes));
    if (region > budget) return false;
    out->nr = nr;
    out->na = na;
    out->nb = nb;
    out->raw_stride = raw;
    out->bslot = bslot;
    out->n16max = n16max;
    out->rings = region;
    out->smem = (size_t)1024 + region + PL.total;
    return true;
}

cudaError_t tail_set_attributes()
{
    const int fmts[4] = {MOE_FMT_Q8_0, MOE_FMT_Q5_1, MOE_FMT_IQ4_NL, MOE_FMT_NVFP4};
    for (int fg : fmts)
        for (int fd : fmts) {
            const cudaError_t e =
                cudaFuncSetAttribute(tl_pick(fg, fd), cudaFuncAttributeMaxDynamicSharedMemorySize, kTlSmemMax);
            if (e != cudaSuccess) return e;
        }
    return cudaSuccess;
}

int tail_blocks_per_sm(int fmt_gu, int fmt_dn, size_t smem)
{
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, tl_pick(fmt_gu, fmt_dn), kTlThreads, smem) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

cudaError_t launch_tail(const TailCall &t, const TailLaunch &L, int grid, int pdl, cudaStream_t s)
{
    TailArgs a{};
    a.x = t.x;
    a.x_dtype = t.x_dtype;
    a.wr = t.wr;
    a.T = t.T;
    a.H = t.H;
    a.E = t.E;
    a.I = t.I;
    a.k = t.k;
    a.has_shared = t.has_shared;
    a.eb = t.eb;
    a.ee = t.ee;
    a.tab_gu = t.tab_gu;
    a.tab_dn = t.tab_dn;
    a.ts_gu = t.gu->ts;
    a.ts_dn = t.dn->ts;
    a.tl_gu = t.gu->tl;
    a.tl_dn = t.dn->tl;
    a.tl_gu_stride = t.gu->tl_stride;
    a.tl_dn_stride = t.dn->tl_stride;
    a.logits = t.ws->logits;
    a.slot_scale = t.ws->slot_scale;
    a.xg = reinterpret_cast<__half *>(t.ws->xg);
    a.h = reinterpret_cast<__half *>(t.ws->h);
    a.y = t.ws->y;
    a.part = t.ws->tail_part;
    a.ctr = t.ws->tail_ctr;
    a.err = t.ws->err;
    a.out = t.out;
    a.idx_out = t.ws->idx;
    a.gate_out = t.ws->gate;
    a.cnt_out = t.ws->cnt;
    a.nr = L.nr;
    a.na = L.na;
    a.nb = L.nb;
    a.raw_stride = L.raw_stride;
    a.bslot = L.bslot;
    a.n16max = L.n16max;
    a.rings = L.rings;
    a.stamps = t.stamps;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kTlThreads);
    cfg.dynamicSmemBytes = L.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (pdl) {
        // CTAs wait on one another (grid barrier, counters): one CTA per SM and
        // grid = SMs, all resident once the previous kernel's CTAs have left
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
    } else {
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const DecodeTcMaps &m = *t.maps;
    return cudaLaunchKernelEx(&cfg, tl_pick(t.gu->fmt, t.dn->fmt), m.xg, m.h, a);
}

}  // namespace moe
