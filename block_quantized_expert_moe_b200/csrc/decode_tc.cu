// Grouped decode of 2 to 64 tokens on the tensor cores.
//
// The "Qwen3.8-Flash-Next UD-IQ2_XS (L4 fix) for Basalt" model card ("What was
// changed") runs the MoE tail as grouped expert kernels over block-quantised
// weights, each expert's weights read once for all of its tokens.  With a few
// tokens per expert that is a GEMM with a tiny N: here the weight rows are the
// M side of tcgen05.mma (128 rows of one expert per tile), the expert's tokens
// the N side (padded to a multiple of 16, at most 64), and K the reduction.
// The weights are expanded from their blocks to fp16 in shared memory once per
// tile, however many tokens the expert has; the products accumulate in fp32
// in tensor memory.  fp16 keeps 11 significant bits: the weights (d times a
// code of at most 7 bits, or an NVFP4 code times its E4M3 scale, exact) lose at
// most 2^-12 relatively, x is exact (bf16 has 8) once scaled by a power of two
// below 2^15 per token, h loses 2^-12.
//
//   gather    one CTA per token: x[t] into the fp16 rows of its k routed
//             slots and of its shared-expert slot (the plan's slot order: every
//             expert's slots contiguous), times 2^-s with s the smallest
//             exponent that brings max |x[t]| below 2^15; the slot's 2^s beside
//   gate/up   tile = {group, 128 row pairs}: A = 128 gate rows and 128 up rows
//             (two accumulators), B = the group's x slot rows; epilogue
//             h = silu(g) * u per (row, slot), written fp16 for the down tiles
//   down      tile = {group, 128 output rows}: A = 128 down rows, B = the
//             group's h slot rows; epilogue y[slot] (fp32), which the combine
//             kernel sums per token in the layer's order (gate-weighted), so
//             the output does not depend on the order tiles finish in
//
//   warps 0-3   epilogue (tensor-memory lanes 32w .. 32w + 31 = tile rows)
//   warp 4      TMA producer of the B tiles (16-row boxes, 128-byte swizzle)
//   warp 5      MMA issuer (one elected thread)
//   warp 6      TMA producer of the raw weight tiles (codes, scales, fifth
//               bits; K = 256 of every tile row per stage)
//   warps 7-22  dequantisers: each thread expands one 32-block of one tile
//               row per slice into the fp16 A tile
//
// Every mbarrier wait is bounded; a wait that runs out records MOE_ERR_TIMEOUT
// and the CTA stops issuing work.  An h outside the fp16 range records
// MOE_ERR_RANGE (MOE_PATH_GROUPED computes such layers in fp32).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "dequant.cuh"
#include "moe_internal.cuh"
#include "tc_common.cuh"
#include "tma_maps.cuh"

namespace moe {

namespace {

using namespace tc;

constexpr int kDtEpiWarps = 4;
constexpr int kDtBWarp = 4, kDtMmaWarp = 5, kDtRawWarp = 6, kDtDeqWarp0 = 7, kDtDeqWarps = 16;
constexpr int kDtThreads = 32 * (kDtDeqWarp0 + kDtDeqWarps);  // 23 warps
constexpr int kDtMaxAStages = 4, kDtMaxRawStages = 4, kDtMaxBSlots = 8;
constexpr size_t kDtSmemBudget = 225 * 1024;  // dynamic shared memory per CTA
constexpr int kDtA = 128 * 128;                  // 128 rows x 64 fp16 of K
constexpr int kDtTmemCols = 128;                 // gate accumulator at column 0, up at 64

// One raw stage holds K = 256 (four MMA slices) of every A tile's rows, as the
// TMA boxes land: codes (128-byte rows, 128-byte swizzle; Q8_0 two boxes),
// scales (16 bytes a row; Q5_1 32, 32-byte swizzle) and Q5_1 fifth bits (32).
template <int FMT, int TILES>
struct RawLayout {
    static constexpr int kCodeBoxes = FMT == MOE_FMT_Q8_0 ? 2 : 1;
    static constexpr int kCodes = kCodeBoxes * 128 * 128;  // per tile
    static constexpr int kScW = FMT == MOE_FMT_Q5_1 ? 32 : 16;
    static constexpr int kScales = 128 * kScW;
    static constexpr int kQh = FMT == MOE_FMT_Q5_1 ? 128 * 32 : 0;
    static constexpr int kStage = TILES * (kCodes + kScales + kQh);
    static constexpr int kA = TILES * kDtA;  // one A stage: the expanded fp16 tiles of a 64-wide slice
    __device__ static int codes(int t) { return t * kCodes; }
    __device__ static int scales(int t) { return TILES * kCodes + t * kScales; }
    __device__ static int qh(int t) { return TILES * (kCodes + kScales) + t * kQh; }
};

struct DtArgs {
    const int4 *groups;        // {expert slot, first slot, tokens, -}
    const int32_t *n_groups;
    int NB;                    // 128-row tiles per group
    int K;                     // reduction length (a multiple of 256)
    // shared memory: nr raw stages | na A stages | nbs B slots of bslot bytes
    // (the group's padded token rows x 64 fp16), at a_off and b_off
    int nr, na, nbs, bslot, a_off, b_off;
    CodeTable tab;
    const float *ts;           // NVFP4 per-expert scale
    int up_off;                // gate/up: row offset of the up rows (= I)
    const float *slot_scale;   // gate/up: 2^s of the slot's x
    __half *h;                 // gate/up output [slots x I]
    int I;
    float *y;                  // down output [slots x H]
    int H;
    int32_t *err;
};

__host__ __device__ constexpr uint32_t idesc_f16(int M, int N)
{
    // kind::f16: f16 x f16 -> f32, both K-major (formats 0 = f16)
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Position in a ring of n buffers: slot s, and u = how many times the ring has
// wrapped (the parity of an mbarrier phase); advanced without a division.
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

// Address in a raw stage of the 16-byte code chunk c (0..7) of row r in box bx
// (128-byte rows, chunk swizzled by r % 8).
__device__ __forceinline__ const uint8_t *raw_code(const uint8_t *box0, int bx, int r, int c)
{
    return box0 + bx * 16384 + r * 128 + ((c ^ (r & 7)) << 4);
}

template <bool GATEUP, int FMT>
__global__ void __launch_bounds__(kDtThreads, 1)
    dtc_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmQ,
               const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmH, const DtArgs g)
{
    constexpr int TILES = GATEUP ? 2 : 1;
    using RL = RawLayout<FMT, TILES>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t fa_bar[kDtMaxAStages], ae_bar[kDtMaxAStages], fb_bar[kDtMaxBSlots],
        be_bar[kDtMaxBSlots];
    __shared__ __align__(8) uint64_t rf_bar[kDtMaxRawStages], re_bar[kDtMaxRawStages], accf_bar, acce_bar, dr_bar;
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NR = g.nr, NA = g.na, NBS = g.nbs;
    uint8_t *raw = smem, *atile = smem + g.a_off, *btile = smem + g.b_off;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tasks = *g.n_groups * g.NB;
    const int KT = g.K / 64, KR = g.K / 256;  // MMA slices and raw stages per task
    int raw_issued = 0, b_issued = 0;         // stages the two TMA producers armed

    if (warp == kDtMmaWarp) {
        tmem_alloc(&tmem_base, kDtTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NA; ++s) {
            mbar_init(&fa_bar[s], GATEUP ? kDtDeqWarps : kDtDeqWarps / 2);
            mbar_init(&ae_bar[s], 1);
        }
        for (int s = 0; s < NBS; ++s) {
            mbar_init(&fb_bar[s], 1);
            mbar_init(&be_bar[s], 1);
        }
        for (int s = 0; s < NR; ++s) {
            mbar_init(&rf_bar[s], 1);
            mbar_init(&re_bar[s], kDtDeqWarps);
        }
        mbar_init(&accf_bar, 1);
        mbar_init(&acce_bar, kDtEpiWarps);
        mbar_init(&dr_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_base;

    if (warp == kDtRawWarp) {  // ---- raw weight tiles: 256 of K of every tile row per stage
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmS);
            if (FMT == MOE_FMT_Q5_1) prefetch_tmap(&tmH);
            Ring rr;
            for (int task = blockIdx.x; task < n_tasks && !abort_flag; task += gridDim.x) {
                const int4 gr = g.groups[task / g.NB];
                const int b = task % g.NB;
                for (int j = 0; j < KR; ++j, rr.next(NR)) {
                    const int s = rr.s, u = rr.u;
                    if (u > 0 && !mbar_wait(&re_bar[s], (u - 1) & 1)) {
                        abort_flag = 1;
                        break;
                    }
                    uint8_t *st = raw + s * RL::kStage;
                    mbar_arrive_expect_tx(&rf_bar[s], (uint32_t)RL::kStage);
#pragma unroll
                    for (int t = 0; t < TILES; ++t) {
                        const int row0 = (t ? g.up_off : 0) + b * 128;
#pragma unroll
                        for (int bx = 0; bx < RL::kCodeBoxes; ++bx)
                            tma_load_3d(st + RL::codes(t) + bx * 16384, &tmQ, &rf_bar[s],
                                        (j * RL::kCodeBoxes + bx) * 128, row0, gr.x);
                        tma_load_3d(st + RL::scales(t), &tmS, &rf_bar[s], j * RL::kScW, row0, gr.x);
                        if (FMT == MOE_FMT_Q5_1) tma_load_3d(st + RL::qh(t), &tmH, &rf_bar[s], j * 32, row0, gr.x);
                    }
                }
            }
            raw_issued = rr.u * NR + rr.s;
        }
    } else if (warp == kDtBWarp) {  // ---- B tiles: the group's slot rows, 16 at a time
        if (lane == 0) {
            prefetch_tmap(&tmB);
            Ring rb;
            for (int task = blockIdx.x; task < n_tasks && !abort_flag; task += gridDim.x) {
                const int4 gr = g.groups[task / g.NB];
                const int n16 = (gr.z + 15) >> 4;
                for (int kt = 0; kt < KT; ++kt, rb.next(NBS)) {
                    const int s = rb.s, u = rb.u;
                    if (u > 0 && !mbar_wait(&be_bar[s], (u - 1) & 1)) {
                        abort_flag = 1;
                        break;
                    }
                    uint8_t *b_s = btile + s * g.bslot;
                    mbar_arrive_expect_tx(&fb_bar[s], (uint32_t)n16 * 2048u);
                    for (int jj = 0; jj < n16; ++jj)
                        tma_load_2d(b_s + jj * 2048, &tmB, &fb_bar[s], kt * 64, gr.y + 16 * jj);
                }
            }
            b_issued = rb.u * NBS + rb.s;
        }
    } else if (warp == kDtMmaWarp) {  // ---- MMA issuer
        if (lane == 0) {
            Ring ra, rb;
            int tcount = 0;
            for (int task = blockIdx.x; task < n_tasks && !abort_flag; task += gridDim.x, ++tcount) {
                const int4 gr = g.groups[task / g.NB];
                const uint32_t idesc = idesc_f16(128, (gr.z + 15) & ~15);
                if (tcount > 0 && !mbar_wait(&acce_bar, (tcount - 1) & 1)) {
                    abort_flag = 1;
                    break;
                }
                tc_fence_after_sync();
                for (int kt = 0; kt < KT; ++kt, ra.next(NA), rb.next(NBS)) {
                    const int sa = ra.s, ua = ra.u, sb = rb.s, ub = rb.u;
                    if (!mbar_wait(&fa_bar[sa], ua & 1) || !mbar_wait(&fb_bar[sb], ub & 1)) {
                        abort_flag = 1;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint8_t *a_s = atile + sa * RL::kA;
                    const uint64_t bd = desc_kmajor_sw128(btile + sb * g.bslot);
#pragma unroll
                    for (int hh = 0; hh < TILES; ++hh) {
                        const uint64_t ad = desc_kmajor_sw128(a_s + hh * kDtA);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_f16(tmem + hh * 64, ad + 2 * kk, bd + 2 * kk, idesc, (kt | kk) != 0);
                    }
                    mma_commit(&ae_bar[sa]);
                    mma_commit(&be_bar[sb]);
                }
                mma_commit(&accf_bar);
            }
        }
    } else if (warp >= kDtDeqWarp0) {  // ---- dequantisers: raw blocks -> fp16 A tiles
        // thread n expands one 32-block of one row per slice: gate/up row n % 128
        // of tile (n / 128) % 2, block n / 256 of every slice; down row n % 128,
        // block (n / 128) % 2 of the slices of parity n / 256 (a slice of down is
        // half the rows' work of gate/up)
        const int n = threadIdx.x - 32 * kDtDeqWarp0;
        const int r = n & 127;
        const int tile = GATEUP ? (n >> 7) & 1 : 0;
        const int bsel = GATEUP ? n >> 8 : (n >> 7) & 1;
        const int par = GATEUP ? -1 : n >> 8;
        Ring ra, rr;
        bool ok = true;
        for (int task = blockIdx.x; task < n_tasks && ok && !abort_flag; task += gridDim.x) {
            for (int j = 0; j < KR && ok; ++j, rr.next(NR)) {
                const int rs = rr.s, ru = rr.u;
                if (!mbar_wait(&rf_bar[rs], ru & 1)) {
                    abort_flag = 1;
                    ok = false;
                    break;
                }
                const uint8_t *st = raw + rs * RL::kStage;
                const uint8_t *cq = st + RL::codes(tile), *cs = st + RL::scales(tile), *ch = st + RL::qh(tile);
#pragma unroll 1
                for (int d = 0; d < 4; ++d, ra.next(NA)) {
                    const int s = ra.s, u = ra.u;
                    if (!GATEUP && (d & 1) != par) continue;  // the other half of the warps' slice
                    if (u > 0) {
                        bool w = true;
                        if (lane == 0) w = mbar_wait(&ae_bar[s], (u - 1) & 1);
                        if (!__shfl_sync(0xffffffffu, w, 0)) {
                            abort_flag = 1;
                            ok = false;
                            break;
                        }
                    }
                    uint8_t *a_row = atile + s * RL::kA + tile * kDtA + (r >> 3) * 1024 + (r & 7) * 128;
                    {
                        const int blk = 2 * d + bsel;  // block of the raw stage (0..7)
                        uint32_t qw[8];
                        if constexpr (FMT == MOE_FMT_Q8_0) {
                            const uint4 a = *reinterpret_cast<const uint4 *>(raw_code(cq, blk >> 2, r, (2 * blk) & 7));
                            const uint4 b2 = *reinterpret_cast<const uint4 *>(raw_code(cq, blk >> 2, r, ((2 * blk) & 7) + 1));
                            qw[0] = a.x; qw[1] = a.y; qw[2] = a.z; qw[3] = a.w;
                            qw[4] = b2.x; qw[5] = b2.y; qw[6] = b2.z; qw[7] = b2.w;
                        } else {
                            const uint4 a = *reinterpret_cast<const uint4 *>(raw_code(cq, 0, r, blk));
                            qw[0] = a.x; qw[1] = a.y; qw[2] = a.z; qw[3] = a.w;
                        }
                        uint32_t sc, hb = 0;
                        if constexpr (FMT == MOE_FMT_Q5_1) {
                            const int gsw = (r >> 2) & 1;  // 32-byte swizzle: 16-byte chunk ^ ((r / 4) % 2)
                            const int o = r * 32 + ((((blk * 4) >> 4) ^ gsw) << 4) + ((blk * 4) & 15);
                            sc = *reinterpret_cast<const uint32_t *>(cs + o);
                            hb = *reinterpret_cast<const uint32_t *>(ch + o);
                        } else {
                            sc = *reinterpret_cast<const uint16_t *>(cs + r * 16 + blk * 2);
                        }
                        uint4 o4[4];
                        dq::blk_f16<FMT>(qw, sc, hb, g.tab, o4);
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {  // chunk c: elements 8c .. 8c+7 of the slice
                            const int c = 4 * bsel + cc;
                            *reinterpret_cast<uint4 *>(a_row + ((c ^ (r & 7)) << 4)) = o4[cc];
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&fa_bar[s]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&re_bar[rs]);  // this warp is done with the raw stage
            }
        }
    } else if (warp < kDtEpiWarps) {  // ---- epilogue, warps 0-3: thread = tile row
        int tcount = 0;
        bool range_ok = true;
        for (int task = blockIdx.x; task < n_tasks; task += gridDim.x, ++tcount) {
            const bool w_ok = mbar_wait(&accf_bar, tcount & 1);
            tc_fence_after_sync();
            // the warp leaves together (its tensor-memory loads are warp-wide)
            if (!__all_sync(0xffffffffu, w_ok) || __any_sync(0xffffffffu, abort_flag != 0)) {
                if (lane == 0) {
                    abort_flag = 1;
                    atomicExch(g.err, (int)MOE_ERR_TIMEOUT);
                }
                break;
            }
            const int4 gr = g.groups[task / g.NB];
            const int b = task % g.NB;
            const int r = warp * 32 + lane;
            const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
            const float hts = FMT == MOE_FMT_NVFP4 ? 0.5f * __ldg(g.ts + gr.x) : 1.f;
            for (int c0 = 0; c0 < gr.z; c0 += 16) {  // warp-uniform
                float v0[16];
                tmem_ld16(tl + c0, v0);
                if (GATEUP) {
                    float v1[16];
                    tmem_ld16(tl + 64 + c0, v1);
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const int c = c0 + jj;
                        if (c < gr.z) {
                            const int slot = gr.y + c;
                            const float sc = __ldg(g.slot_scale + slot) * hts;
                            const float gv = v0[jj] * sc, uv = v1[jj] * sc;
                            const float hv = gv / (1.f + expf(-gv)) * uv;
                            range_ok = range_ok && fabsf(hv) <= 65504.f;
                            g.h[(size_t)slot * g.I + b * 128 + r] = __float2half_rn(hv);
                        }
                    }
                } else {
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const int c = c0 + jj;
                        if (c < gr.z) g.y[(size_t)(gr.y + c) * g.H + b * 128 + r] = v0[jj] * hts;
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce_bar);
        }
        if (GATEUP && !__all_sync(0xffffffffu, range_ok) && lane == 0) atomicExch(g.err, (int)MOE_ERR_RANGE);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (abort_flag) {  // block-uniform after the barrier: drain what was issued, then release
        if (lane == 0 && warp == kDtRawWarp) drain_ring(rf_bar, NR, raw_issued);
        if (lane == 0 && warp == kDtBWarp) drain_ring(fb_bar, NBS, b_issued);
        if (lane == 0 && warp == kDtMmaWarp) drain_mma(&dr_bar);
        if (threadIdx.x == 0) atomicExch(g.err, (int)MOE_ERR_TIMEOUT);
        tc_fence_before_sync();
        __syncthreads();
    }
    if (warp == kDtMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kDtTmemCols);
    }
}

// One CTA per token: x[t] scaled by 2^-s into the fp16 rows of its slots, and
// the slots' 2^s.  Every thread loads its 16-byte chunks first (at most
// kGatherChunks, H <= 16384), so the row arrives in one memory round trip.
constexpr int kGatherChunks = 8;

__global__ void __launch_bounds__(256) dtc_gather_kernel(const void *x, int x_dtype, int T, int H, int k,
                                                         int has_shared, const int32_t *slot_pos, __half *xg,
                                                         float *slot_scale)
{
    __shared__ unsigned s_max[8];
    const int t = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool bf = x_dtype == MOE_DT_BF16;
    const int nch = H / 8;  // chunks of 8 elements
    float v[kGatherChunks][8];
    unsigned mx = 0u;  // bits of max |x|: non-negative floats order as unsigned
#pragma unroll
    for (int i = 0; i < kGatherChunks; ++i) {
        const int c = threadIdx.x + 256 * i;
        if (c < nch) {
            if (bf) {
                const uint4 q = __ldg(reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(x) + (size_t)t * H) + c);
                const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    v[i][2 * j] = __uint_as_float(w[j] << 16);
                    v[i][2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
                }
            } else {
                const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(x) + (size_t)t * H) + 2 * c;
                const float4 a = __ldg(p), b = __ldg(p + 1);
                v[i][0] = a.x; v[i][1] = a.y; v[i][2] = a.z; v[i][3] = a.w;
                v[i][4] = b.x; v[i][5] = b.y; v[i][6] = b.z; v[i][7] = b.w;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kGatherChunks; ++i)
        if (threadIdx.x + 256 * i < nch)
#pragma unroll
            for (int j = 0; j < 8; ++j) mx = max(mx, __float_as_uint(fabsf(v[i][j])));
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) s_max[warp] = mx;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < 8; ++w) mx = max(mx, s_max[w]);
    const int ex = (int)((mx >> 23) & 0xFFu) - 127;  // exponent of max |x| (inf / NaN: left unscaled)
    const int sh = (ex >= 15 && ex < 128) ? ex - 14 : 0;
    const float down = __uint_as_float((uint32_t)(127 - sh) << 23), up = __uint_as_float((uint32_t)(127 + sh) << 23);
    const int nd = k + (has_shared ? 1 : 0);
#pragma unroll
    for (int i = 0; i < kGatherChunks; ++i) {
        const int c = threadIdx.x + 256 * i;
        if (c < nch) {
            uint4 o;
            o.x = dq::pack_f16x2(v[i][0] * down, v[i][1] * down);
            o.y = dq::pack_f16x2(v[i][2] * down, v[i][3] * down);
            o.z = dq::pack_f16x2(v[i][4] * down, v[i][5] * down);
            o.w = dq::pack_f16x2(v[i][6] * down, v[i][7] * down);
#pragma unroll 1
            for (int j = 0; j < nd; ++j) {
                const int slot = j < k ? __ldg(slot_pos + (size_t)t * k + j) : T * k + t;
                reinterpret_cast<uint4 *>(xg + (size_t)slot * H)[c] = o;
            }
        }
    }
    for (int j = threadIdx.x; j < nd; j += 256)
        slot_scale[j < k ? __ldg(slot_pos + (size_t)t * k + j) : T * k + t] = up;
}

using DtKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap, const DtArgs);

template <bool GATEUP>
DtKernel dt_pick(int fmt)
{
    switch (fmt) {
    case MOE_FMT_Q8_0: return dtc_kernel<GATEUP, MOE_FMT_Q8_0>;
    case MOE_FMT_Q5_1: return dtc_kernel<GATEUP, MOE_FMT_Q5_1>;
    case MOE_FMT_IQ4_NL: return dtc_kernel<GATEUP, MOE_FMT_IQ4_NL>;
    case MOE_FMT_NVFP4: return dtc_kernel<GATEUP, MOE_FMT_NVFP4>;
    default: return nullptr;
    }
}

// Shared-memory plan of one launch: two of each ring at least, then up to four
// A stages (each slice is a round trip between the expanding warps and the MMA
// issuer), up to eight B slots (B rows come from L2), up to four raw stages
// (from HBM), as far as 225 KB allow.
struct DtLayout {
    int nr, na, nbs, bslot;
    size_t raw, a, total;
};

template <int FMT>
DtLayout dt_layout_fmt(bool gateup, int nmax)
{
    DtLayout L;
    L.raw = gateup ? RawLayout<FMT, 2>::kStage : RawLayout<FMT, 1>::kStage;
    L.a = gateup ? RawLayout<FMT, 2>::kA : RawLayout<FMT, 1>::kA;
    L.bslot = nmax * 128;
    L.nr = L.na = L.nbs = 2;
    auto total = [&] { return 1024 + L.nr * L.raw + L.na * L.a + (size_t)L.nbs * L.bslot; };
    while (L.na < kDtMaxAStages && total() + L.a <= kDtSmemBudget) ++L.na;
    while (L.nbs < kDtMaxBSlots && total() + L.bslot <= kDtSmemBudget) ++L.nbs;
    while (L.nr < kDtMaxRawStages && total() + L.raw <= kDtSmemBudget) ++L.nr;
    L.total = total();
    return L;
}

DtLayout dt_layout(bool gateup, int fmt, int nmax)
{
    switch (fmt) {
    case MOE_FMT_Q8_0: return dt_layout_fmt<MOE_FMT_Q8_0>(gateup, nmax);
    case MOE_FMT_Q5_1: return dt_layout_fmt<MOE_FMT_Q5_1>(gateup, nmax);
    case MOE_FMT_IQ4_NL: return dt_layout_fmt<MOE_FMT_IQ4_NL>(gateup, nmax);
    default: return dt_layout_fmt<MOE_FMT_NVFP4>(gateup, nmax);
    }
}

// 3-D [slots x rows x row_bytes] byte map of one plane, (w x 128 x 1) boxes.
bool dt_plane_map(CUtensorMap *m, const uint8_t *base, int slots, int rows, int row_bytes, int64_t stride, int w)
{
    tmaps::EncodeTiledFn f = tmaps::encode_fn();
    if (!f || !base || row_bytes < w || row_bytes % 16 || stride % 16) return false;
    cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)rows, (cuuint64_t)slots};
    cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)stride};
    cuuint32_t box[3] = {(cuuint32_t)w, 128, 1};
    cuuint32_t es[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw = w == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : w == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                            : CU_TENSOR_MAP_SWIZZLE_NONE;
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool dt_proj_maps(CUtensorMap (&m)[3], const DevProj &w, int slots)
{
    if (!dt_plane_map(&m[0], w.qs, slots, w.rows, w.qs_row, w.qs_stride, 128)) return false;
    if (!dt_plane_map(&m[1], w.sr, slots, w.rows, w.sr_row, w.sr_stride, w.fmt == MOE_FMT_Q5_1 ? 32 : 16)) return false;
    if (w.fmt == MOE_FMT_Q5_1) return dt_plane_map(&m[2], w.qh, slots, w.rows, w.qh_row, w.qh_stride, 32);
    m[2] = m[1];
    return true;
}

}  // namespace

bool decode_tc_supported(const DevProj &gu, const DevProj &dn, int H, int I, int max_tokens, int max_top_k)
{
    if (!gu.f16_ok || !dn.f16_ok || !gu.sr || !dn.sr) return false;
    if (H % 256 || I % 256) return false;  // 128-row tiles; K in raw stages of 256
    if (max_tokens < 1 || H > 16384) return false;  // (the staged launches run 2-64 tokens, the tail 1-64)
    // the slot rows the B maps cover must fit 32-bit TMA coordinates
    return (int64_t)max_tokens * (max_top_k + 1) < (1ll << 30);
}

cudaError_t decode_tc_set_attributes()
{
    const int fmts[4] = {MOE_FMT_Q8_0, MOE_FMT_Q5_1, MOE_FMT_IQ4_NL, MOE_FMT_NVFP4};
    for (int f : fmts)
        for (int gu = 0; gu < 2; ++gu) {
            const cudaError_t e = cudaFuncSetAttribute(gu ? dt_pick<true>(f) : dt_pick<false>(f),
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)kDtSmemBudget);
            if (e != cudaSuccess) return e;
        }
    return cudaSuccess;
}

bool decode_tc_maps(DecodeTcMaps *m, const DevProj &gu, const DevProj &dn, int n_experts, const void *xg,
                    const void *h16, int slots, int H, int I)
{
    // fp16 rows: the bf16 map builder moves the same 2-byte elements
    return tmaps::make_map_bf16(&m->xg, xg, slots, H, 16) && tmaps::make_map_bf16(&m->h, h16, slots, I, 16) &&
           dt_proj_maps(m->gu, gu, n_experts) && dt_proj_maps(m->dn, dn, n_experts);
}

cudaError_t launch_decode_tc_gather(const void *x, int x_dtype, int T, int H, int k, int has_shared,
                                    const int32_t *slot_pos, void *xg, float *slot_scale, cudaStream_t s)
{
    dtc_gather_kernel<<<T, 256, 0, s>>>(x, x_dtype, T, H, k, has_shared, slot_pos,
                                        static_cast<__half *>(xg), slot_scale);
    return cudaGetLastError();
}

cudaError_t launch_decode_tc(const DecodeTcMaps &m, bool gateup, const DevProj &w, const int4 *groups,
                             const int32_t *n_groups, int H, int I, const CodeTable &tab, const float *slot_scale,
                             void *h16, float *y, int32_t *err, int max_tokens, int grid, cudaStream_t s)
{
    const int nmax = (std::min(std::max(max_tokens, 1), kDecodeTcMaxN) + 15) & ~15;
    const DtLayout L = dt_layout(gateup, w.fmt, nmax);
    if (L.total > kDtSmemBudget) return cudaErrorInvalidValue;
    DtArgs a{};
    a.nr = L.nr;
    a.na = L.na;
    a.nbs = L.nbs;
    a.bslot = L.bslot;
    a.a_off = (int)(L.nr * L.raw);
    a.b_off = (int)(L.nr * L.raw + L.na * L.a);
    a.groups = groups;
    a.n_groups = n_groups;
    a.NB = gateup ? I / 128 : H / 128;
    a.K = gateup ? H : I;
    a.tab = tab;
    a.ts = w.ts;
    a.err = err;
    a.up_off = gateup ? I : 0;
    a.slot_scale = slot_scale;
    a.h = static_cast<__half *>(h16);
    a.I = I;
    a.y = y;
    a.H = H;
    DtKernel kfn = gateup ? dt_pick<true>(w.fmt) : dt_pick<false>(w.fmt);
    if (!kfn) return cudaErrorInvalidValue;
    const CUtensorMap *pm = gateup ? m.gu : m.dn;
    kfn<<<grid, kDtThreads, L.total, s>>>(gateup ? m.xg : m.h, pm[0], pm[1], pm[2], a);
    return cudaGetLastError();
}

}  // namespace moe
