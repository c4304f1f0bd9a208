// Tensor-core prefill (sm_100a tcgen05): the router as a bf16 GEMM, top-k over
// its logits, and the routing plan for large token batches.
//
// Prefill runs many tokens through the layer at once (the pages report prefill
// speeds of thousands of tokens per second on long prompts: llms-full.txt,
// "Prefill speed, tokens per second, by prompt length"), so the contractions
// become GEMMs and belong on the tensor cores.  The router GEMM here:
//
//   logits[T x E] (f32) = X[T x H] (bf16) . Wr[E x H]^T (bf16)
//
// one 128 x BN output tile per CTA; warp 4 streams 64-wide K slices of both
// operands with TMA (128-byte swizzle) into a ring of STAGES shared-memory
// stages, warp 5 issues tcgen05.mma (kind::f16, M 128, N BN, K 16 per
// instruction) into a tensor-memory accumulator and commits each stage back to
// the producer, and warps 0-3 read the accumulator (one row per thread) once
// the last MMA has committed.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <mutex>

#include "decode_common.cuh"
#include "moe_internal.cuh"
#include "tc_common.cuh"
#include "tma_maps.cuh"

namespace moe {

namespace {

using namespace tc;
using namespace tmaps;

constexpr int kGemmThreads = 192;  // warps 0-3 epilogue, 4 TMA, 5 MMA
constexpr int kBM = 128, kBK = 64;

struct GemmArgs {
    int M, N, K;
    float *C;
    int ldc;
    int32_t *err;
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_tn_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const GemmArgs g)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES], acc_bar;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    constexpr int A_BYTES = kBM * kBK * 2, B_BYTES = BN * kBK * 2, STAGE = A_BYTES + B_BYTES;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kBM, n0 = blockIdx.y * BN;
    const int KT = (g.K + kBK - 1) / kBK;
    int tma_issued = 0;  // stages the TMA producer armed

    if (warp == 5) {
        tmem_alloc(&tmem_base, BN);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&acc_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_base;

    if (warp == 4) {
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES, u = kt / STAGES;
                if (u > 0 && !mbar_wait(&empty_bar[s], (u - 1) & 1)) {
                    abort_flag = 1;
                    break;
                }
                uint8_t *a_s = smem + s * STAGE, *b_s = a_s + A_BYTES;
                mbar_arrive_expect_tx(&full_bar[s], STAGE);
                tma_load_2d(a_s, &tmA, &full_bar[s], kt * kBK, m0);
                tma_load_2d(b_s, &tmB, &full_bar[s], kt * kBK, n0);
                tma_issued = kt + 1;
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(kBM, BN);
            int issued = 0;
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES, u = kt / STAGES;
                if (!mbar_wait(&full_bar[s], u & 1)) {
                    abort_flag = 1;
                    break;
                }
                tc_fence_after_sync();
                uint8_t *a_s = smem + s * STAGE, *b_s = a_s + A_BYTES;
                const uint64_t ad = desc_kmajor_sw128(a_s), bd = desc_kmajor_sw128(b_s);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)  // 16 bf16 = 32 bytes = 2 descriptor units
                    mma_f16(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kt | kk) != 0);
                mma_commit(&empty_bar[s]);
                ++issued;
            }
            (void)issued;
            mma_commit(&acc_bar);  // also covers the abort case: arrives when issued MMAs finish
        }
    } else {
        const bool ok = mbar_wait(&acc_bar, 0);
        tc_fence_after_sync();
        if (ok && !abort_flag) {
            const int row = warp * 32 + lane;
            const int m = m0 + row;
#pragma unroll 1
            for (int c = 0; c < BN; c += 16) {
                float v[16];
                tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c, v);
                if (m < g.M) {
                    float *dst = g.C + (size_t)m * g.ldc + n0 + c;
                    if (n0 + c + 16 <= g.N) {
#pragma unroll
                        for (int i = 0; i < 16; i += 4)
                            *reinterpret_cast<float4 *>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                    } else {
                        for (int i = 0; i < 16; ++i)
                            if (n0 + c + i < g.N) dst[i] = v[i];
                    }
                }
            }
        } else {
            abort_flag = 1;
            if (threadIdx.x == 0) atomicExch(g.err, (int)MOE_ERR_TIMEOUT);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (abort_flag) {  // block-uniform after the barrier: drain what was issued, then release
        if (warp == 4 && lane == 0) drain_ring(full_bar, STAGES, tma_issued);
        if (warp == 5 && lane == 0) mbar_wait(&acc_bar, 0);  // committed after the last MMA this thread issued
        if (threadIdx.x == 0) atomicExch(g.err, (int)MOE_ERR_TIMEOUT);
        tc_fence_before_sync();
        __syncthreads();
    }
    if (warp == 5) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, BN);
    }
}

// ---- top-k over a logits matrix: one warp per token --------------------------------
__global__ void __launch_bounds__(256) topk_rows_kernel(const float *logits, int T, int E, int k, int32_t *idx,
                                                        float *gate, int32_t *cnt)
{
    extern __shared__ float topk_smem[];
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    if (k <= 32 && E <= 1024) {
        // the token's logits into shared memory, then the one-pass threshold selection
        float *row = topk_smem + (size_t)(threadIdx.x >> 5) * (E + 128);
        if (E <= 512) stage_logits<16>(logits + (size_t)t * E, row, E, lane);
        else stage_logits<32>(logits + (size_t)t * E, row, E, lane);
        __syncwarp();
        int me;
        float mg;
        if (E <= 512) topk_threshold<16>(row, E, k, me, mg, reinterpret_cast<unsigned *>(row + E));
        else topk_threshold<32>(row, E, k, me, mg, reinterpret_cast<unsigned *>(row + E));
        if (lane < k) {
            idx[(size_t)t * k + lane] = me;
            gate[(size_t)t * k + lane] = mg;
            if (cnt) atomicAdd(&cnt[me], 1);
        }
        return;
    }
    float v[32];
    uint32_t taken = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int e = lane + 32 * i;
        if (e < E) v[i] = __ldg(logits + (size_t)t * E + e);
        else { v[i] = -INFINITY; taken |= 1u << i; }
    }
    float vmax = 0.f, den = 0.f, myv = 0.f;
    int myi = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = INT_MAX;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (!((taken >> i) & 1u) && (bi == INT_MAX || v[i] > bv)) {
                bv = v[i];
                bi = lane + 32 * i;
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (oi != INT_MAX && (bi == INT_MAX || ov > bv || (ov == bv && oi < bi))) {
                bv = ov;
                bi = oi;
            }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (j == 0) vmax = bv;
        den += expf(bv - vmax);
        if (lane == (j & 31)) {
            myv = bv;
            myi = bi;
        }
        if ((j & 31) == 31 || j == k - 1) {
            // flush this group of up to 32 selections (gates need the final den: done below)
            const int jb = j & ~31;
            if (lane <= (j & 31)) {
                idx[(size_t)t * k + jb + lane] = myi;
                gate[(size_t)t * k + jb + lane] = myv;
                if (cnt) atomicAdd(&cnt[myi], 1);
            }
        }
    }
    __syncwarp();
    for (int j = lane; j < k; j += 32) gate[(size_t)t * k + j] = expf(gate[(size_t)t * k + j] - vmax) / den;
}

constexpr int kRouterBN = 256, kRouterStages = 4;
constexpr size_t kRouterSmem = (size_t)kRouterStages * (kBM * kBK * 2 + kRouterBN * kBK * 2) + 1024;

}  // namespace

cudaError_t prefill_set_attributes()
{
    return cudaFuncSetAttribute(gemm_bf16_tn_kernel<kRouterBN, kRouterStages>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRouterSmem);
}

// logits = x . Wr^T on the tensor cores (x bf16), then top-k per token.
// cnt (E ints, zeroed by the caller) receives per-expert counts when non-null.
cudaError_t prefill_route(const void *x_bf16, const uint16_t *wr, int T, int H, int E, int k, float *logits,
                          int32_t *idx, float *gate, int32_t *cnt, int32_t *err, cudaStream_t s)
{
    CUtensorMap ma, mb;
    if (!make_map_bf16(&ma, x_bf16, T, H, kBM) || !make_map_bf16(&mb, wr, E, H, kRouterBN))
        return cudaErrorInvalidValue;
    GemmArgs g{T, E, H, logits, E, err};
    dim3 grid((T + kBM - 1) / kBM, (E + kRouterBN - 1) / kRouterBN);
    gemm_bf16_tn_kernel<kRouterBN, kRouterStages><<<grid, kGemmThreads, kRouterSmem, s>>>(ma, mb, g);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    topk_rows_kernel<<<(T + 7) / 8, 256, (size_t)8 * (E + 128) * sizeof(float), s>>>(logits, T, E, k, idx, gate, cnt);
    return cudaGetLastError();
}

namespace {

// ======================================================================================
// Grouped NVFP4 expert GEMMs of the prefill (native block-scaled FP4 MMA)
//
// The routed slots of each expert are laid out in a padded slot space: expert
// e owns rows [pad_off[e], pad_off[e] + ceil(cnt[e]/128)*128), so every
// 128-row M tile belongs to one expert and starts on a 128-row boundary of the
// activation and scale arrays.  Activations enter as NVFP4 with a per-row fp32
// scale (the reading of the prefill's activation quantisation: amax/(6*448)
// per token, E4M3 scale per 16, E2M1 codes, round to nearest even, saturating).
//
//   gate/up tile  D[128 x 256] = A_q[128 x H] . [G_e rows n0..n0+127 ; U_e rows
//                 I+n0..I+n0+127]^T  (block-scaled, f32 in tensor memory);
//                 epilogue h = silu(d_g * s_row * s_e) * (d_u * s_row * s_e)
//   down tile     D[128 x 256] = H_q[128 x I] . D_e[rows n0..n0+255]^T;
//                 epilogue out[token] += gate * d * s_row * s_e (fp32 vector
//                 reductions into the output, which starts at zero)
//
// Warp roles as in the router GEMM; per 256-wide K stage the producer brings
// A (16 KB), B (32 KB) and their 512-byte scale atoms, and the MMA thread
// copies the scale atoms of each 64-wide K step into tensor memory
// (tcgen05.cp 32x128b.warpx4: 32 rows x 16 bytes, replicated to the four lane
// quarters) before the MMA that reads them.
// ======================================================================================

constexpr int kNvStages = 3;
constexpr int kNvStageA = 128 * 128, kNvStageB = 256 * 128;  // bytes (256 fp4 per row)
constexpr int kNvSfA = 4 * 512, kNvSfB = 2 * 4 * 512;       // four K steps
constexpr int kNvStage = kNvStageA + kNvStageB + kNvSfA + kNvSfB;
constexpr size_t kNvSmem = (size_t)kNvStages * kNvStage + 1024;
constexpr uint32_t kNvTmemCols = 512;  // accumulator 256 + scales 48 (+ unused)
constexpr int kNvEpiWarps = 16;         // warps 0-15: epilogue (four per TMEM lane quarter)
constexpr int kNvEpiParts = kNvEpiWarps / 4;
constexpr int kNvTmaWarp = kNvEpiWarps, kNvMmaWarp = kNvEpiWarps + 1;
constexpr int kNvThreads = 32 * (kNvEpiWarps + 2);

struct NvGemmArgs {
    const int2 *tiles;        // M tiles: {expert, first padded row}
    const int32_t *n_tiles;   // device count of M tiles
    int NT;                   // N tiles per M tile
    int K;                    // reduction length (elements)
    int ksteps_a;             // 64-wide K steps of the activations
    const uint8_t *sfa;       // activation scales, block-scale layout over padded rows
    const uint8_t *sfb;       // weight scales (plane base), per expert stride sfb_stride
    int64_t sfb_stride;
    int ksteps_b;
    int b_rows_gate_off;      // gate/up: row offset of U inside the stacked matrix (= I)
    const float *ts;          // per-expert fp32 matrix scale
    const float *row_scale;   // per padded row fp32 scale of the activations
    const int32_t *perm_tok;  // padded row -> token (-1 for padding rows)
    const float *row_gate;    // padded row -> gate (down epilogue)
    float *h;                 // gate/up output [padded rows x I]
    int I;
    float *out;               // down output [T x H]
    int H;
    int32_t *err;
};

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

template <bool GATEUP>
__global__ void __launch_bounds__(kNvThreads, 1)
    nvfp4_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                              const NvGemmArgs g)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kNvStages], empty_bar[kNvStages], accf_bar, acce_bar, dr_bar;
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = *g.n_tiles * g.NT;
    const int KT = g.K / 256;  // stages per tile
    int tma_issued = 0;        // stages the TMA producer armed

    if (warp == kNvMmaWarp) {
        tmem_alloc(&tmem_base, kNvTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kNvStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&accf_bar, 1);
        mbar_init(&acce_bar, kNvEpiWarps);
        mbar_init(&dr_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_base;
    const uint32_t t_acc = tmem, t_sfa = tmem + 256, t_sfb = tmem + 256 + 16;

    if (warp == kNvTmaWarp) {
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            int it = 0;
            for (int tile = blockIdx.x; tile < n_tiles && !abort_flag; tile += gridDim.x) {
                const int mt = tile / g.NT, nt = tile % g.NT;
                const int2 td = g.tiles[mt];
                const int e = td.x, r0 = td.y;
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % kNvStages, u = it / kNvStages;
                    if (u > 0 && !mbar_wait(&empty_bar[s], (u - 1) & 1)) {
                        abort_flag = 1;
                        break;
                    }
                    uint8_t *a_s = smem + s * kNvStage, *b_s = a_s + kNvStageA, *sfa_s = b_s + kNvStageB;
                    uint8_t *sfb_s = sfa_s + kNvSfA;
                    mbar_arrive_expect_tx(&full_bar[s], kNvStage);
                    tma_load_2d(a_s, &tmA, &full_bar[s], kt * 128, r0);
                    // activation scales: K steps 4kt..4kt+3 of the 128-row block at r0
                    bulk_load(sfa_s, g.sfa + ((int64_t)(r0 >> 7) * g.ksteps_a + kt * 4) * 512, kNvSfA, &full_bar[s]);
                    const uint8_t *sfb_e = g.sfb + (int64_t)e * g.sfb_stride;
                    if (GATEUP) {
                        const int ng = nt * 128, nu = g.b_rows_gate_off + nt * 128;
                        tma_load_3d(b_s, &tmB, &full_bar[s], kt * 128, ng, e);
                        tma_load_3d(b_s + 128 * 128, &tmB, &full_bar[s], kt * 128, nu, e);
                        bulk_load(sfb_s, sfb_e + ((int64_t)(ng >> 7) * g.ksteps_b + kt * 4) * 512, 2048, &full_bar[s]);
                        bulk_load(sfb_s + 2048, sfb_e + ((int64_t)(nu >> 7) * g.ksteps_b + kt * 4) * 512, 2048,
                                  &full_bar[s]);
                    } else {
                        const int n0 = nt * 256;
                        tma_load_3d(b_s, &tmB, &full_bar[s], kt * 128, n0, e);
                        bulk_load(sfb_s, sfb_e + ((int64_t)(n0 >> 7) * g.ksteps_b + kt * 4) * 512, 2048, &full_bar[s]);
                        bulk_load(sfb_s + 2048, sfb_e + ((int64_t)((n0 >> 7) + 1) * g.ksteps_b + kt * 4) * 512, 2048,
                                  &full_bar[s]);
                    }
                }
            }
            tma_issued = it;
        }
    } else if (warp == kNvMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_nvf4(128, 256);
            int it = 0, tcount = 0;
            for (int tile = blockIdx.x; tile < n_tiles && !abort_flag; tile += gridDim.x, ++tcount) {
                if (tcount > 0 && !mbar_wait(&acce_bar, (tcount - 1) & 1)) {  // epilogue drained the accumulator
                    abort_flag = 1;
                    break;
                }
                tc_fence_after_sync();
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % kNvStages, u = it / kNvStages;
                    if (!mbar_wait(&full_bar[s], u & 1)) {
                        abort_flag = 1;
                        break;
                    }
                    tc_fence_after_sync();
                    uint8_t *a_s = smem + s * kNvStage, *b_s = a_s + kNvStageA, *sfa_s = b_s + kNvStageB;
                    uint8_t *sfb_s = sfa_s + kNvSfA;
                    const uint64_t ad = desc_kmajor_sw128(a_s), bd = desc_kmajor_sw128(b_s);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        tmem_cp_32x128b_warpx4(t_sfa + ks * 4, desc_plain(sfa_s + ks * 512, 128, 128));
                        tmem_cp_32x128b_warpx4(t_sfb + ks * 8, desc_plain(sfb_s + ks * 512, 128, 128));
                        tmem_cp_32x128b_warpx4(t_sfb + ks * 8 + 4, desc_plain(sfb_s + 2048 + ks * 512, 128, 128));
                        // 64 fp4 = 32 bytes = 2 descriptor units per K step
                        mma_nvf4(t_acc, ad + 2 * ks, bd + 2 * ks, idesc, t_sfa + ks * 4, t_sfb + ks * 8, (kt | ks) != 0);
                    }
                    mma_commit(&empty_bar[s]);
                }
                mma_commit(&accf_bar);
            }
        }
    } else {
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
            const int2 td = g.tiles[mt];
            // warps q, q + 4, ... read TMEM lanes 32 q .. 32 q + 31 and split the columns
            const int quarter = warp & 3, part = warp >> 2;
            const int e = td.x, row = td.y + quarter * 32 + lane;
            const int tok = g.perm_tok[row];
            const float sc = g.row_scale[row] * g.ts[e];
            const uint32_t tl = t_acc + ((uint32_t)(quarter * 32) << 16);
            if (GATEUP) {
#pragma unroll 1
                for (int c = part * (128 / kNvEpiParts); c < (part + 1) * (128 / kNvEpiParts); c += 16) {
                    float vg[16], vu[16];
                    tmem_ld16(tl + c, vg);
                    tmem_ld16(tl + 128 + c, vu);
                    if (tok >= 0) {
                        float *dst = g.h + (size_t)row * g.I + nt * 128 + c;
#pragma unroll
                        for (int i = 0; i < 16; i += 4) {
                            float o[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float a = vg[i + q] * sc, b = vu[i + q] * sc;
                                // silu with the fast exponential (ex2-based; well inside the prefill tolerance)
                                o[q] = a * __frcp_rn(1.f + __expf(-a)) * b;
                            }
                            *reinterpret_cast<float4 *>(dst + i) = make_float4(o[0], o[1], o[2], o[3]);
                        }
                    }
                }
            } else {
                const float gsc = tok >= 0 ? sc * g.row_gate[row] : 0.f;
#pragma unroll 1
                for (int c = part * (256 / kNvEpiParts); c < (part + 1) * (256 / kNvEpiParts); c += 16) {
                    float v[16];
                    tmem_ld16(tl + c, v);
                    if (tok >= 0) {
                        float *dst = g.out + (size_t)tok * g.H + nt * 256 + c;
#pragma unroll
                        for (int i = 0; i < 16; i += 4)
                            red_add_v4(dst + i, v[i] * gsc, v[i + 1] * gsc, v[i + 2] * gsc, v[i + 3] * gsc);
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
        if (warp == kNvTmaWarp && lane == 0) drain_ring(full_bar, kNvStages, tma_issued);
        if (warp == kNvMmaWarp && lane == 0) drain_mma(&dr_bar);
        if (threadIdx.x == 0) atomicExch(g.err, (int)MOE_ERR_TIMEOUT);
        tc_fence_before_sync();
        __syncthreads();
    }
    if (warp == kNvMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kNvTmemCols);
    }
}

// ---- plan of the padded slot space (one CTA) ----------------------------------------
// cnt[0..E) counted by top-k, cnt[E] = T when there is a shared expert.
__global__ void __launch_bounds__(1024) prefill_plan_kernel(int32_t *cnt, int E, int T, int has_shared,
                                                            int32_t *pad_off, int32_t *fill, int2 *tiles,
                                                            int32_t *n_tiles, int32_t *total_rows_out,
                                                            int32_t *perm_tok, int max_rows, int32_t *err,
                                                            int4 *ptiles, int32_t *n_ptiles)
{
    __shared__ int s_pad[1025], s_nt[1025], s_np[1025], s_tmp[33];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = E + 1;
    if (tid == 0) cnt[E] = has_shared ? T : 0;
    __syncthreads();
    for (int e = tid; e < n; e += 1024) {
        const int c = cnt[e];
        s_pad[e] = (c + 127) / 128 * 128;
        s_nt[e] = (c + 127) / 128;
        s_np[e] = (c + 255) / 256;  // pairs of 128-row tiles
        fill[e] = 0;
    }
    __syncthreads();
    // two exclusive scans over n <= 1025 entries (thread i owns entry i; entry 1024 by thread 0's tail)
    for (int which = 0; which < 3; ++which) {
        int *v = which == 0 ? s_pad : which == 1 ? s_nt : s_np;
        const int x = tid < n ? v[tid] : 0;
        int incl = x;
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        if (lane == 31) s_tmp[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int w = s_tmp[lane];
            int wi = w;
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += u;
            }
            s_tmp[lane] = wi - w;
            if (lane == 31) s_tmp[32] = wi;
        }
        __syncthreads();
        const int excl = s_tmp[warp] + incl - x;
        const int total1024 = s_tmp[32];
        __syncthreads();
        if (tid < n && tid < 1024) v[tid] = excl;
        if (n > 1024 && tid == 0) v[1024] = total1024;  // entry 1024 follows all others
        __syncthreads();
    }
    const int last = n - 1;
    const int total_rows = s_pad[last] + (cnt[last] + 127) / 128 * 128;
    const int total_tiles = s_nt[last] + (cnt[last] + 127) / 128;
    const int total_pairs = s_np[last] + (cnt[last] + 255) / 256;
    if (total_rows > max_rows) {
        if (tid == 0) {
            atomicExch(err, (int)MOE_ERR_DEVICE);
            *n_tiles = 0;
            *total_rows_out = 0;
            if (n_ptiles) *n_ptiles = 0;
        }
        return;
    }
    for (int e = tid; e < n; e += 1024) {
        const int c = cnt[e], base = s_pad[e], tb = s_nt[e];
        pad_off[e] = base;
        for (int i = 0; i * 128 < c; ++i) tiles[tb + i] = make_int2(e, base + i * 128);
        if (ptiles) {
            const int nt = (c + 127) / 128;
            for (int i = 0; 2 * i < nt; ++i)
                ptiles[s_np[e] + i] = make_int4(e, base + i * 256, min(2, nt - 2 * i), 0);
        }
        for (int r = c; r < (c + 127) / 128 * 128; ++r) perm_tok[base + r] = -1;  // padding rows
    }
    if (tid == 0) {
        *n_tiles = total_tiles;
        *total_rows_out = total_rows;
        if (n_ptiles) *n_ptiles = total_pairs;
    }
}

// NVFP4 rounding of 64 consecutive values held 2 per lane-register pair:
// codes (32 bytes) and the 4 block scales of one 64-wide K step.
__device__ __forceinline__ uint32_t e4m3_rn_sat(float v)  // v >= 0
{
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.f), "f"(v));
    return r & 0xFFu;
}

// eight values -> eight E2M1 codes, element 2i in the low nibble of byte i
__device__ __forceinline__ uint32_t e2m1x8(float v0, float v1, float v2, float v3, float v4, float v5, float v6,
                                           float v7)
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
    return r;
}

__device__ __forceinline__ float e4m3_val(uint32_t b)
{
    return __uint_as_float((b & 0x7Fu) << 20) * 1.329227995784916e36f;  // 2^120
}

// Quantise 64 values (v[0..63]) of one K step with the row scale s (> 0):
// writes 32 code bytes to dst_codes and the 4 E4M3 scales to dst_sf.
__device__ __forceinline__ void quant_step(const float (&v)[64], float s, uint8_t *dst_codes, uint8_t *dst_sf)
{
    uint32_t sfw = 0;
    uint32_t cw[8];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        float bmax = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(v[b * 16 + i]));
        const uint32_t sb = s > 0.f ? e4m3_rn_sat(bmax / (6.f * s)) : 0u;
        sfw |= sb << (8 * b);
        const float sbv = e4m3_val(sb);
        const float den = s * sbv;
#pragma unroll
        for (int i = 0; i < 16; i += 8) {
            const float *p = v + b * 16 + i;
            cw[b * 2 + i / 8] = sbv > 0.f ? e2m1x8(p[0] / den, p[1] / den, p[2] / den, p[3] / den, p[4] / den,
                                                   p[5] / den, p[6] / den, p[7] / den)
                                          : 0u;
        }
    }
    uint4 *d = reinterpret_cast<uint4 *>(dst_codes);
    d[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    d[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    *reinterpret_cast<uint32_t *>(dst_sf) = sfw;
}

// One warp per token: quantise x[t] (bf16) to NVFP4 with its own scale and
// write it to the token's k routed slots (and the shared slot).
__global__ void __launch_bounds__(256) quant_scatter_kernel(const uint16_t *x, int T, int H, int k, int E,
                                                            int has_shared, const int32_t *idx, const float *gate,
                                                            const int32_t *pad_off, int32_t *fill, uint8_t *a_q,
                                                            uint8_t *sfa, int ksteps, float *row_scale,
                                                            int32_t *perm_tok, float *row_gate, int32_t *slot_pos,
                                                            int max_rows)
{
    __shared__ int s_pos[8][33];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int t = blockIdx.x * 8 + wib;
    if (t >= T) return;
    const uint16_t *xr = x + (size_t)t * H;
    float amax = 0.f;
    for (int c = lane * 8; c < H; c += 256) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(xr + c));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[i] << 16)), fabsf(__uint_as_float(w[i] & 0xFFFF0000u))));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = amax / (6.f * 448.f);
    // destination rows: k routed slots (+ shared)
    const int nd = k + (has_shared ? 1 : 0);
    for (int j = 0; j < nd; ++j) {
        int pos = 0;
        if (lane == 0) {
            const int e = j < k ? idx[(size_t)t * k + j] : E;
            pos = pad_off[e] + atomicAdd(&fill[e], 1);
            if (pos >= max_rows) pos = -1;  // only if the plan failed (its error is already set)
        }
        pos = __shfl_sync(0xffffffffu, pos, 0);
        if (lane == 0) s_pos[wib][j] = pos;
        if (pos < 0) continue;
        if (lane == 0) {
            row_scale[pos] = s;
            perm_tok[pos] = t;
            row_gate[pos] = j < k ? gate[(size_t)t * k + j] : 1.f;
            if (j < k) slot_pos[(size_t)t * k + j] = pos;
        }
    }
    __syncwarp();
    for (int st = lane; st < ksteps; st += 32) {  // one 64-wide K step per lane
        float v[64];
#pragma unroll
        for (int i = 0; i < 64; i += 8) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(xr + st * 64 + i));
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                v[i + 2 * q] = __uint_as_float(w[q] << 16);
                v[i + 2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
            }
        }
        uint4 codes[2];
        uint32_t sfw;
        quant_step(v, s, reinterpret_cast<uint8_t *>(codes), reinterpret_cast<uint8_t *>(&sfw));
        for (int j = 0; j < nd; ++j) {
            const int pos = s_pos[wib][j];
            if (pos < 0) continue;
            uint4 *dst = reinterpret_cast<uint4 *>(a_q + (size_t)pos * (H / 2) + st * 32);
            dst[0] = codes[0];
            dst[1] = codes[1];
            *reinterpret_cast<uint32_t *>(sfa + sf_offset(pos, st, 0, ksteps)) = sfw;
        }
    }
}

// One warp per padded row: quantise h (fp32) of real rows to NVFP4 with a
// per-row scale (the activation of the down GEMM).
// Row quantisation of h for the down GEMM: one warp per row, one lane per
// 16-value block (the same per-block rule as quant_step, so every code and
// scale is bit-identical to it); I/16 blocks per row, 32 at I = 512.
__global__ void __launch_bounds__(256) quant_rows_kernel(const float *h, int rows_cap, const int32_t *n_rows_dev,
                                                         int I, const int32_t *perm_tok, uint8_t *h_q, uint8_t *sfh,
                                                         int ksteps, float *row_scale)
{
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= rows_cap || r >= *n_rows_dev) return;
    if (perm_tok[r] < 0) return;
    const float *hr = h + (size_t)r * I;
    const int nb = I >> 4;
    float amax = 0.f;
    for (int b = lane; b < nb; b += 32) {
        const float4 *p = reinterpret_cast<const float4 *>(hr + b * 16);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = __ldcg(p + q);
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = amax / (6.f * 448.f);
    if (lane == 0) row_scale[r] = s;
    for (int b = lane; b < nb; b += 32) {
        float v[16];
        const float4 *p = reinterpret_cast<const float4 *>(hr + b * 16);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 w = __ldcg(p + q);
            v[4 * q] = w.x;
            v[4 * q + 1] = w.y;
            v[4 * q + 2] = w.z;
            v[4 * q + 3] = w.w;
        }
        float bmax = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
        const uint32_t sb = s > 0.f ? e4m3_rn_sat(bmax / (6.f * s)) : 0u;
        const float sbv = e4m3_val(sb);
        const float den = s * sbv;
        uint2 cw = make_uint2(0u, 0u);
        if (sbv > 0.f) {
            cw.x = e2m1x8(v[0] / den, v[1] / den, v[2] / den, v[3] / den, v[4] / den, v[5] / den, v[6] / den,
                          v[7] / den);
            cw.y = e2m1x8(v[8] / den, v[9] / den, v[10] / den, v[11] / den, v[12] / den, v[13] / den, v[14] / den,
                          v[15] / den);
        }
        *reinterpret_cast<uint2 *>(h_q + (size_t)r * (I / 2) + b * 8) = cw;
        sfh[sf_offset(r, b >> 2, b & 3, ksteps)] = (uint8_t)sb;
    }
}

// Diagnostic: the prefill's activation quantisers on plain rows.  x_bf16 rows
// go through quant_scatter_kernel (the gate/up activations: row t routed to a
// one-token "expert" t, so it lands at padded row t), fp32 rows through
// quant_rows_kernel (the down activations); codes come out row-major, scales
// in the block-scale layout (sf_offset) of rows rounded up to 128.
__global__ void debug_iota_kernel(int32_t *idx, int32_t *pad_off, int32_t *fill, int32_t *perm_tok, int32_t *n_rows,
                                  int rows)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= rows; i += gridDim.x * blockDim.x) {
        if (i < rows) {
            idx[i] = i;
            perm_tok[i] = i;
        }
        pad_off[i] = i;
        fill[i] = 0;
        if (i == 0) *n_rows = rows;
    }
}

}  // namespace

cudaError_t debug_act_quant(const void *x, bool bf16, int rows, int cols, uint8_t *codes, uint8_t *sf_atoms,
                            float *row_scale, int32_t *scratch, cudaStream_t s)
{
    // scratch: idx, pad_off, fill, perm_tok [rows + 1 each], gate, row_gate,
    // slot_pos [rows each], n_rows and an unused error word
    int32_t *idx = scratch, *pad_off = idx + rows + 1, *fill = pad_off + rows + 1, *perm_tok = fill + rows + 1;
    float *gate = reinterpret_cast<float *>(perm_tok + rows + 1), *row_gate = gate + rows;
    int32_t *slot_pos = reinterpret_cast<int32_t *>(row_gate + rows), *n_rows = slot_pos + rows;
    debug_iota_kernel<<<(rows + 256) / 256, 256, 0, s>>>(idx, pad_off, fill, perm_tok, n_rows, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (bf16) {
        quant_scatter_kernel<<<(rows + 7) / 8, 256, 0, s>>>(static_cast<const uint16_t *>(x), rows, cols, 1, rows, 0,
                                                             idx, gate, pad_off, fill, codes, sf_atoms, cols / 64,
                                                             row_scale, perm_tok, row_gate, slot_pos, rows);
    } else {
        quant_rows_kernel<<<(rows + 7) / 8, 256, 0, s>>>(static_cast<const float *>(x), rows, n_rows, cols, perm_tok,
                                                          codes, sf_atoms, cols / 64, row_scale);
    }
    return cudaGetLastError();
}

cudaError_t prefill_plan_launch(const PrefillWorkspace &w, int E, int T, int has_shared, int32_t *err, cudaStream_t s)
{
    prefill_plan_kernel<<<1, 1024, 0, s>>>(w.cnt, E, T, has_shared, w.pad_off, w.fill, w.tiles, w.n_tiles,
                                           w.total_rows, w.perm_tok, w.max_rows, err, w.ptiles, w.n_ptiles);
    return cudaGetLastError();
}

cudaError_t prefill_nvfp4_set_attributes()
{
    cudaError_t e = cudaFuncSetAttribute(nvfp4_grouped_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kNvSmem);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(nvfp4_grouped_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kNvSmem);
}

bool prefill_nvfp4_supported(int H, int I, int E, int k)
{
    return H % 256 == 0 && I % 256 == 0 && E <= 1023 && k <= 32;
}

cudaError_t prefill_nvfp4_forward(const PrefillNvArgs &a, cudaStream_t s)
{
    const int H = a.H, I = a.I, E = a.E, k = a.k, T = a.T;
    const PrefillWorkspace &w = *a.ws;
    cudaError_t e;
    if ((e = cudaMemsetAsync(w.cnt, 0, sizeof(int32_t) * (E + 1), s)) != cudaSuccess) return e;
    if ((e = prefill_route(a.x, a.wr, T, H, E, k, w.logits, w.idx, w.gate, w.cnt, a.err, s)) != cudaSuccess) return e;
    prefill_plan_kernel<<<1, 1024, 0, s>>>(w.cnt, E, T, a.has_shared, w.pad_off, w.fill, w.tiles, w.n_tiles,
                                           w.total_rows, w.perm_tok, w.max_rows, a.err, nullptr, nullptr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int ks_h = H / 64, ks_i = I / 64;
    quant_scatter_kernel<<<(T + 7) / 8, 256, 0, s>>>(reinterpret_cast<const uint16_t *>(a.x), T, H, k, E,
                                                      a.has_shared, w.idx, w.gate, w.pad_off, w.fill, w.a_q, w.sfa,
                                                      ks_h, w.row_scale_x, w.perm_tok, w.row_gate, w.slot_pos,
                                                      w.max_rows);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    CUtensorMap ma, mb;
    if (!make_map_u8_2d(&ma, w.a_q, w.max_rows, H / 2, 128) ||
        !make_map_u8_3d(&mb, a.gu->qs, E + (a.has_shared ? 1 : 0), 2 * I, H / 2, a.gu->qs_stride, 128))
        return cudaErrorInvalidValue;
    NvGemmArgs g{};
    g.tiles = w.tiles;
    g.n_tiles = w.n_tiles;
    g.NT = I / 128;
    g.K = H;
    g.ksteps_a = ks_h;
    g.sfa = w.sfa;
    g.sfb = a.gu->sc;
    g.sfb_stride = a.gu->sc_stride;
    g.ksteps_b = a.gu->ksteps;
    g.b_rows_gate_off = I;
    g.ts = a.gu->ts;
    g.row_scale = w.row_scale_x;
    g.perm_tok = w.perm_tok;
    g.row_gate = w.row_gate;
    g.h = w.h;
    g.I = I;
    g.out = a.out;
    g.H = H;
    g.err = a.err;
    nvfp4_grouped_gemm_kernel<true><<<a.num_sms, kNvThreads, kNvSmem, s>>>(ma, mb, g);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    quant_rows_kernel<<<(w.max_rows + 7) / 8, 256, 0, s>>>(w.h, w.max_rows, w.total_rows, I, w.perm_tok, w.h_q,
                                                           w.sfh, ks_i, w.row_scale_h);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.out, 0, sizeof(float) * (size_t)T * H, s)) != cudaSuccess) return e;
    CUtensorMap ma2, mb2;
    if (!make_map_u8_2d(&ma2, w.h_q, w.max_rows, I / 2, 128) ||
        !make_map_u8_3d(&mb2, a.dn->qs, E + (a.has_shared ? 1 : 0), H, I / 2, a.dn->qs_stride, 256))
        return cudaErrorInvalidValue;
    NvGemmArgs d = g;
    d.NT = H / 256;
    d.K = I;
    d.ksteps_a = ks_i;
    d.sfa = w.sfh;
    d.sfb = a.dn->sc;
    d.sfb_stride = a.dn->sc_stride;
    d.ksteps_b = a.dn->ksteps;
    d.ts = a.dn->ts;
    d.row_scale = w.row_scale_h;
    nvfp4_grouped_gemm_kernel<false><<<a.num_sms, kNvThreads, kNvSmem, s>>>(ma2, mb2, d);
    return cudaGetLastError();
}

}  // namespace moe
