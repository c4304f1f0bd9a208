// Tensor-core prefill for Q8_0, IQ4_NL, Q5_1 (and NVFP4) experts: the weight blocks are
// dequantised to bf16 in shared memory and multiplied with tcgen05.mma
// kind::f16.  One kernel instance per format (the two projections may differ);
// only the dequantiser warps depend on it.
//
// The same padded slot space as the NVFP4 prefill (every 128-row M tile
// belongs to one expert).  A CTA tile is up to two consecutive M tiles of one
// expert (256 rows) by 256 weight rows: each dequantised weight stage then feeds
// two 128 x 256 MMAs, halving the dequantisation work per multiply-add, and the
// two f32 accumulators fill the 512 tensor-memory columns.
//
//   warps 0-7    epilogue (warps q and q + 4 read accumulator lanes 32q..32q+31
//                and split the columns)
//   warp 8       TMA producer of the activation tiles (bf16, 128-byte swizzle)
//   warp 9       MMA issuer (one elected thread)
//   warps 10-17  dequantisers: thread n owns weight row n of the stage; it
//                loads the row's two 32-weight blocks (Q8_0: 64 int8 codes and
//                two fp16 scales; IQ4_NL: 32 code bytes looked up in the pack's
//                table; Q5_1: 32 code bytes, fifth bits, {d, m}) with the next
//                stage's already in flight, converts to bf16 and stores
//                the eight 16-byte chunks at their 128-byte-swizzle positions,
//                then makes them visible to the tensor core (fence.proxy.async)
//
//   gate/up  A = x rows gathered into slot order (bf16); B rows 0..127 the gate
//            rows n0..n0+127, rows 128..255 the up rows I+n0..;
//            epilogue h = silu(d_g) * d_u, stored bf16 for the down GEMM
//   down     A = h (bf16); B = D_e rows n0..n0+255;
//            epilogue out[token] += gate * d (fp32 vector reductions)
// All mbarrier waits are bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "moe_internal.cuh"
#include "dequant.cuh"
#include "quant_dot.cuh"
#include "tc_common.cuh"
#include "tma_maps.cuh"

namespace moe {

namespace {

using namespace tc;
using namespace tmaps;

constexpr int kQ8EpiWarps = 8;
constexpr int kQ8TmaWarp = kQ8EpiWarps, kQ8MmaWarp = kQ8EpiWarps + 1, kQ8DeqWarp0 = kQ8EpiWarps + 2;
constexpr int kQ8Threads = 32 * (kQ8DeqWarp0 + 8);  // 18 warps
constexpr int kQ8Stages = 3;
constexpr int kQ8A = 128 * 128;  // one 128-row half: 128 rows x 64 bf16
constexpr int kQ8B = 256 * 128;  // 256 weight rows x 64 bf16
constexpr int kQ8Stage = 2 * kQ8A + kQ8B;
constexpr size_t kQ8Smem = (size_t)kQ8Stages * kQ8Stage + 1024;

struct Q8GemmArgs {
    const int4 *ptiles;        // {expert, first padded row, halves (1|2), 0}
    const int32_t *n_ptiles;
    int NT;                    // weight-row tiles of 256 (gate/up: I/128 pairs of 128)
    int K;                     // reduction length
    const uint8_t *qs;         // codes plane: Q8_0 K bytes per row (stored +128), 4-bit K/2
    int64_t qs_stride;
    int qs_row;
    const uint8_t *sc;         // row-major scales: fp16 d per 32 (Q5_1: {d, m}; NVFP4: two E4M3)
    int64_t sc_stride;
    int sc_row;
    const uint8_t *qh;         // Q5_1 fifth bits, u32 per 32
    int64_t qh_stride;
    int qh_row;
    CodeTable tab;             // IQ4_NL / NVFP4 table (biased bytes; the pack's code positions)
    const float *ts;           // NVFP4: per-expert matrix scale (the table holds twice E2M1)
    int up_off;                // gate/up: row offset of U (= I); down: 0
    const int32_t *perm_tok;
    const float *row_gate;
    __nv_bfloat16 *h;          // gate/up output [rows x I] bf16
    int I;
    float *out;                // down output [T x H]
    int H;
    int32_t *err;
};

template <bool GATEUP, int FMT>
__global__ void __launch_bounds__(kQ8Threads, 1)
    dq_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const Q8GemmArgs g)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t fa_bar[kQ8Stages], fb_bar[kQ8Stages], empty_bar[kQ8Stages], accf_bar, acce_bar,
        dr_bar;
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = *g.n_ptiles * g.NT;
    const int KT = g.K / 64;
    int tma_issued = 0;  // stages the activation producer armed

    if (warp == kQ8MmaWarp) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kQ8Stages; ++s) {
            mbar_init(&fa_bar[s], 1);
            mbar_init(&fb_bar[s], 8);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&accf_bar, 1);
        mbar_init(&acce_bar, kQ8EpiWarps);
        mbar_init(&dr_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_base;

    if (warp == kQ8TmaWarp) {  // ---- activation producer
        if (lane == 0) {
            prefetch_tmap(&tmA);
            int it = 0;
            for (int tile = blockIdx.x; tile < n_tiles && !abort_flag; tile += gridDim.x) {
                const int4 pt = g.ptiles[tile / g.NT];
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % kQ8Stages, u = it / kQ8Stages;
                    if (u > 0 && !mbar_wait(&empty_bar[s], (u - 1) & 1)) {
                        abort_flag = 1;
                        break;
                    }
                    uint8_t *a_s = smem + s * kQ8Stage;
                    mbar_arrive_expect_tx(&fa_bar[s], pt.z * kQ8A);
                    tma_load_2d(a_s, &tmA, &fa_bar[s], kt * 64, pt.y);
                    if (pt.z == 2) tma_load_2d(a_s + kQ8A, &tmA, &fa_bar[s], kt * 64, pt.y + 128);
                }
            }
            tma_issued = it;
        }
    } else if (warp == kQ8MmaWarp) {  // ---- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, 256);
            int it = 0, tcount = 0;
            for (int tile = blockIdx.x; tile < n_tiles && !abort_flag; tile += gridDim.x, ++tcount) {
                const int nh = g.ptiles[tile / g.NT].z;
                if (tcount > 0 && !mbar_wait(&acce_bar, (tcount - 1) & 1)) {
                    abort_flag = 1;
                    break;
                }
                tc_fence_after_sync();
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % kQ8Stages, u = it / kQ8Stages;
                    if (!mbar_wait(&fa_bar[s], u & 1) || !mbar_wait(&fb_bar[s], u & 1)) {
                        abort_flag = 1;
                        break;
                    }
                    tc_fence_after_sync();
                    uint8_t *a_s = smem + s * kQ8Stage, *b_s = a_s + 2 * kQ8A;
                    const uint64_t bd = desc_kmajor_sw128(b_s);
                    for (int hh = 0; hh < nh; ++hh) {
                        const uint64_t ad = desc_kmajor_sw128(a_s + hh * kQ8A);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_f16(tmem + hh * 256, ad + 2 * kk, bd + 2 * kk, idesc, (kt | kk) != 0);
                    }
                    mma_commit(&empty_bar[s]);
                }
                mma_commit(&accf_bar);
            }
        }
    } else if (warp >= kQ8DeqWarp0) {  // ---- weight dequantisers: thread n owns weight row n
        const int n = threadIdx.x - 32 * kQ8DeqWarp0;
        int it = 0;
        for (int tile = blockIdx.x; tile < n_tiles && !abort_flag; tile += gridDim.x) {
            const int mt = tile / g.NT, nt = tile % g.NT;
            const int e = g.ptiles[mt].x;
            const int row = GATEUP ? (n < 128 ? nt * 128 + n : g.up_off + nt * 128 + (n - 128)) : nt * 256 + n;
            const uint8_t *qrow = g.qs + (int64_t)e * g.qs_stride + (int64_t)row * g.qs_row;
            const uint8_t *srow = g.sc + (int64_t)e * g.sc_stride + (int64_t)row * g.sc_row;
            const uint8_t *hrow = FMT == MOE_FMT_Q5_1 ? g.qh + (int64_t)e * g.qh_stride + (int64_t)row * g.qh_row : nullptr;
            // the 64-wide K slice kt = blocks 2 kt, 2 kt + 1; the next slice's loads
            // are in flight while this one is converted
            dq::Blk<FMT> cur[2] = {dq::load_blk<FMT>(qrow, srow, hrow, 0), dq::load_blk<FMT>(qrow, srow, hrow, 1)};
            for (int kt = 0; kt < KT; ++kt, ++it) {
                const int s = it % kQ8Stages, u = it / kQ8Stages;
                dq::Blk<FMT> nxt[2] = {cur[0], cur[1]};
                if (kt + 1 < KT) {
                    nxt[0] = dq::load_blk<FMT>(qrow, srow, hrow, 2 * kt + 2);
                    nxt[1] = dq::load_blk<FMT>(qrow, srow, hrow, 2 * kt + 3);
                }
                if (u > 0) {
                    bool ok = true;
                    if (lane == 0) ok = mbar_wait(&empty_bar[s], (u - 1) & 1);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) {
                        abort_flag = 1;
                        break;
                    }
                }
                uint8_t *b_row = smem + s * kQ8Stage + 2 * kQ8A + (n >> 3) * 1024 + (n & 7) * 128;
#pragma unroll
                for (int blk = 0; blk < 2; ++blk) {
                    float v[32];
                    dq::blk_values<FMT>(cur[blk], g.tab, v);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {  // chunk c = 4 blk + cc: k = 8c .. 8c+7
                        const int c = 4 * blk + cc;
                        uint4 o;
                        o.x = dq::pack_bf16x2(v[8 * cc], v[8 * cc + 1]);
                        o.y = dq::pack_bf16x2(v[8 * cc + 2], v[8 * cc + 3]);
                        o.z = dq::pack_bf16x2(v[8 * cc + 4], v[8 * cc + 5]);
                        o.w = dq::pack_bf16x2(v[8 * cc + 6], v[8 * cc + 7]);
                        *reinterpret_cast<uint4 *>(b_row + ((c ^ (n & 7)) << 4)) = o;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&fb_bar[s]);
                cur[0] = nxt[0];
                cur[1] = nxt[1];
            }
        }
    } else {  // ---- epilogue, warps 0-7
        int tcount = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tcount) {
            const bool ok = mbar_wait(&accf_bar, tcount & 1);
            tc_fence_after_sync();
            if (!ok || abort_flag) {
                abort_flag = 1;
                if (threadIdx.x == 0) atomicExch(g.err, (int)MOE_ERR_TIMEOUT);
                break;
            }
            const int mt = tile / g.NT, nt = tile % g.NT;
            const int4 pt = g.ptiles[mt];
            const int quarter = warp & 3, part = warp >> 2;
            // NVFP4 codes were expanded as twice their E2M1 value; the expert's fp32
            // scale and the 1/2 apply to its accumulators
            const float hts = FMT == MOE_FMT_NVFP4 ? 0.5f * __ldg(g.ts + pt.x) : 1.f;
            for (int hh = 0; hh < pt.z; ++hh) {
                const int row = pt.y + hh * 128 + quarter * 32 + lane;
                const int tok = g.perm_tok[row];
                const uint32_t tl = tmem + hh * 256 + ((uint32_t)(quarter * 32) << 16);
                if (GATEUP) {
#pragma unroll 1
                    for (int c = part * 64; c < part * 64 + 64; c += 16) {
                        float vg[16], vu[16];
                        tmem_ld16(tl + c, vg);
                        tmem_ld16(tl + 128 + c, vu);
                        if (tok >= 0) {
                            uint32_t o[8];
#pragma unroll
                            for (int i = 0; i < 16; i += 2) {
                                const float a0 = vg[i] * hts, a1 = vg[i + 1] * hts;
                                // silu with the fast exponential (well inside the prefill tolerance)
                                o[i / 2] = dq::pack_bf16x2(a0 * __frcp_rn(1.f + __expf(-a0)) * (vu[i] * hts),
                                                       a1 * __frcp_rn(1.f + __expf(-a1)) * (vu[i + 1] * hts));
                            }
                            uint4 *dst = reinterpret_cast<uint4 *>(g.h + (size_t)row * g.I + nt * 128 + c);
                            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
                        }
                    }
                } else {
                    const float gt = tok >= 0 ? g.row_gate[row] * hts : 0.f;
#pragma unroll 1
                    for (int c = part * 128; c < part * 128 + 128; c += 16) {
                        float v[16];
                        tmem_ld16(tl + c, v);
                        if (tok >= 0) {
                            float *dst = g.out + (size_t)tok * g.H + nt * 256 + c;
#pragma unroll
                            for (int i = 0; i < 16; i += 4)
                                asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + i),
                                             "f"(v[i] * gt), "f"(v[i + 1] * gt), "f"(v[i + 2] * gt), "f"(v[i + 3] * gt)
                                             : "memory");
                        }
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce_bar);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (abort_flag) {  // block-uniform after the barrier: drain what was issued, then release
        if (warp == kQ8TmaWarp && lane == 0) drain_ring(fa_bar, kQ8Stages, tma_issued);
        if (warp == kQ8MmaWarp && lane == 0) drain_mma(&dr_bar);
        if (threadIdx.x == 0) atomicExch(g.err, (int)MOE_ERR_TIMEOUT);
        tc_fence_before_sync();
        __syncthreads();
    }
    if (warp == kQ8MmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// One warp per token: copy x[t] (bf16) into its k routed slot rows (and the
// shared slot) of the padded slot space.
__global__ void __launch_bounds__(256) gather_scatter_kernel(const uint16_t *x, int T, int H, int k, int E,
                                                             int has_shared, const int32_t *idx, const float *gate,
                                                             const int32_t *pad_off, int32_t *fill, uint16_t *xp,
                                                             int32_t *perm_tok, float *row_gate, int32_t *slot_pos,
                                                             int max_rows)
{
    __shared__ int s_pos[8][33];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int t = blockIdx.x * 8 + wib;
    if (t >= T) return;
    const int nd = k + (has_shared ? 1 : 0);
    for (int j = 0; j < nd; ++j) {
        int pos = 0;
        if (lane == 0) {
            const int e = j < k ? idx[(size_t)t * k + j] : E;
            pos = pad_off[e] + atomicAdd(&fill[e], 1);
            if (pos >= max_rows) pos = -1;
            s_pos[wib][j] = pos;
            if (pos >= 0) {
                perm_tok[pos] = t;
                row_gate[pos] = j < k ? gate[(size_t)t * k + j] : 1.f;
                if (j < k) slot_pos[(size_t)t * k + j] = pos;
            }
        }
    }
    __syncwarp();
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
    for (int c = lane; c < H / 8; c += 32) {
        const uint4 v = __ldg(src + c);
        for (int j = 0; j < nd; ++j) {
            const int pos = s_pos[wib][j];
            if (pos >= 0) reinterpret_cast<uint4 *>(xp + (size_t)pos * H)[c] = v;
        }
    }
}



using DqKernel = void (*)(const CUtensorMap, const Q8GemmArgs);

DqKernel dq_pick(bool gateup, int fmt)
{
    switch (fmt) {
    case MOE_FMT_Q8_0: return gateup ? dq_grouped_gemm_kernel<true, MOE_FMT_Q8_0> : dq_grouped_gemm_kernel<false, MOE_FMT_Q8_0>;
    case MOE_FMT_IQ4_NL:
        return gateup ? dq_grouped_gemm_kernel<true, MOE_FMT_IQ4_NL> : dq_grouped_gemm_kernel<false, MOE_FMT_IQ4_NL>;
    case MOE_FMT_Q5_1: return gateup ? dq_grouped_gemm_kernel<true, MOE_FMT_Q5_1> : dq_grouped_gemm_kernel<false, MOE_FMT_Q5_1>;
    case MOE_FMT_NVFP4:
        return gateup ? dq_grouped_gemm_kernel<true, MOE_FMT_NVFP4> : dq_grouped_gemm_kernel<false, MOE_FMT_NVFP4>;
    default: return nullptr;
    }
}

bool dq_fmt(int f, bool nvfp4)
{
    return f == MOE_FMT_Q8_0 || f == MOE_FMT_IQ4_NL || f == MOE_FMT_Q5_1 || (nvfp4 && f == MOE_FMT_NVFP4);
}

}  // namespace

bool prefill_q8_supported(int fmt_gu, int fmt_dn, int H, int I, int E, int k, bool nvfp4)
{
    return dq_fmt(fmt_gu, nvfp4) && dq_fmt(fmt_dn, nvfp4) && H % 256 == 0 && I % 256 == 0 && E <= 1023 && k <= 32;
}

cudaError_t prefill_q8_set_attributes()
{
    const int fmts[4] = {MOE_FMT_Q8_0, MOE_FMT_IQ4_NL, MOE_FMT_Q5_1, MOE_FMT_NVFP4};
    for (int f : fmts)
        for (int gu = 0; gu < 2; ++gu) {
            const cudaError_t e =
                cudaFuncSetAttribute(dq_pick(gu != 0, f), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kQ8Smem);
            if (e != cudaSuccess) return e;
        }
    return cudaSuccess;
}

cudaError_t prefill_q8_forward(const PrefillNvArgs &a, cudaStream_t s)
{
    const int H = a.H, I = a.I, E = a.E, k = a.k, T = a.T;
    const PrefillWorkspace &w = *a.ws;
    cudaError_t e;
    if ((e = cudaMemsetAsync(w.cnt, 0, sizeof(int32_t) * (E + 1), s)) != cudaSuccess) return e;
    if ((e = prefill_route(a.x, a.wr, T, H, E, k, w.logits, w.idx, w.gate, w.cnt, a.err, s)) != cudaSuccess) return e;
    if ((e = prefill_plan_launch(w, E, T, a.has_shared, a.err, s)) != cudaSuccess) return e;
    uint16_t *xp = reinterpret_cast<uint16_t *>(w.a_q);  // bf16 slot rows, sized for the dequantising path
    gather_scatter_kernel<<<(T + 7) / 8, 256, 0, s>>>(reinterpret_cast<const uint16_t *>(a.x), T, H, k, E,
                                                       a.has_shared, w.idx, w.gate, w.pad_off, w.fill, xp, w.perm_tok,
                                                       w.row_gate, w.slot_pos, w.max_rows);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    CUtensorMap ma;
    if (!make_map_bf16(&ma, xp, w.max_rows, H, 128)) return cudaErrorInvalidValue;
    Q8GemmArgs g{};
    g.ptiles = w.ptiles;
    g.n_ptiles = w.n_ptiles;
    g.NT = I / 128;
    g.K = H;
    g.qs = a.gu->qs;
    g.qs_stride = a.gu->qs_stride;
    g.qs_row = a.gu->qs_row;
    g.sc = a.gu->sr;  // scales row by row (for NVFP4 its row-major copy)
    g.sc_stride = a.gu->sr_stride;
    g.sc_row = a.gu->sr_row;
    g.ts = a.gu->ts;
    g.qh = a.gu->qh;
    g.qh_stride = a.gu->qh_stride;
    g.qh_row = a.gu->qh_row;
    g.tab = a.tab_gu;
    g.up_off = I;
    g.perm_tok = w.perm_tok;
    g.row_gate = w.row_gate;
    g.h = reinterpret_cast<__nv_bfloat16 *>(w.h);
    g.I = I;
    g.out = a.out;
    g.H = H;
    g.err = a.err;
    DqKernel kgu = dq_pick(true, a.gu->fmt), kdn = dq_pick(false, a.dn->fmt);
    if (!kgu || !kdn) return cudaErrorInvalidValue;
    kgu<<<a.num_sms, kQ8Threads, kQ8Smem, s>>>(ma, g);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.out, 0, sizeof(float) * (size_t)T * H, s)) != cudaSuccess) return e;
    CUtensorMap mh;
    if (!make_map_bf16(&mh, w.h, w.max_rows, I, 128)) return cudaErrorInvalidValue;
    Q8GemmArgs d = g;
    d.NT = H / 256;
    d.K = I;
    d.qs = a.dn->qs;
    d.qs_stride = a.dn->qs_stride;
    d.qs_row = a.dn->qs_row;
    d.sc = a.dn->sr;
    d.sc_stride = a.dn->sr_stride;
    d.sc_row = a.dn->sr_row;
    d.ts = a.dn->ts;
    d.qh = a.dn->qh;
    d.qh_stride = a.dn->qh_stride;
    d.qh_row = a.dn->qh_row;
    d.tab = a.tab_dn;
    d.up_off = 0;
    kdn<<<a.num_sms, kQ8Threads, kQ8Smem, s>>>(mh, d);
    return cudaGetLastError();
}

// ---- diagnostic: the block decoders on rows of a packed projection ---------------
// One thread per 32-block: kind 0 writes the fp16 expansion of the tensor-core
// decode (dq::blk_f16), kind 1 the fp32 values of the bf16-dequantising
// prefill's decoder (dq::blk_values) before their bf16 rounding; NVFP4 values
// are twice E2M1 x E4M3, the matrix scale left to the callers' epilogues.
template <int FMT>
__global__ void debug_dequant_kernel(DevProj w, CodeTable tab, int slot, int row0, int nrows, int kind, void *out)
{
    const int nb = w.cols / 32;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nrows * nb) return;
    const int r = i / nb, b = i - r * nb, row = row0 + r;
    const uint8_t *qrow = w.qs + (int64_t)slot * w.qs_stride + (int64_t)row * w.qs_row;
    const uint8_t *srow = w.sr + (int64_t)slot * w.sr_stride + (int64_t)row * w.sr_row;
    const uint8_t *hrow = w.qh ? w.qh + (int64_t)slot * w.qh_stride + (int64_t)row * w.qh_row : nullptr;
    const dq::Blk<FMT> blk = dq::load_blk<FMT>(qrow, srow, hrow, b);
    if (kind == 0) {
        uint32_t q[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] = j < (FMT == MOE_FMT_Q8_0 ? 8 : 4) ? (&blk.q[0].x)[j] : 0u;
        uint4 o4[4];
        dq::blk_f16<FMT>(q, blk.s, blk.h, tab, o4);
        uint4 *o = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + ((size_t)r * w.cols + b * 32));
#pragma unroll
        for (int c = 0; c < 4; ++c) o[c] = o4[c];
    } else {
        float v[32];
        dq::blk_values<FMT>(blk, tab, v);
        float *o = static_cast<float *>(out) + ((size_t)r * w.cols + b * 32);
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = v[j];
    }
}

cudaError_t debug_dequant(const DevProj &w, const CodeTable &tab, int slot, int row0, int nrows, int kind, void *out,
                          cudaStream_t s)
{
    const int n = nrows * (w.cols / 32), grid = (n + 255) / 256;
    switch (w.fmt) {
    case MOE_FMT_Q8_0: debug_dequant_kernel<MOE_FMT_Q8_0><<<grid, 256, 0, s>>>(w, tab, slot, row0, nrows, kind, out); break;
    case MOE_FMT_Q5_1: debug_dequant_kernel<MOE_FMT_Q5_1><<<grid, 256, 0, s>>>(w, tab, slot, row0, nrows, kind, out); break;
    case MOE_FMT_IQ4_NL:
        debug_dequant_kernel<MOE_FMT_IQ4_NL><<<grid, 256, 0, s>>>(w, tab, slot, row0, nrows, kind, out);
        break;
    case MOE_FMT_NVFP4:
        debug_dequant_kernel<MOE_FMT_NVFP4><<<grid, 256, 0, s>>>(w, tab, slot, row0, nrows, kind, out);
        break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace moe
