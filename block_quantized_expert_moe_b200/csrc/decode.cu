// Grouped decode matvecs over block-quantised experts, and the combine.
//
// The "Qwen3.8-Flash-Next UD-IQ2_XS (L4 fix) for Basalt" model card, section
// "What was changed", names the decode fast path "device-planned tail +
// grouped kernels" and lists the expert formats those kernels read: IQ4_NL,
// NVFP4, Q5_1, Q8_0 (and Q2_0, whose layout the pages do not give).  Decode
// reads every selected expert's weights from memory, so the kernels are
// built to stream each expert's blocks once, whatever the number of tokens
// routed to it:
//
//   * work group = {expert, up to TT of its tokens}; the plan lists the groups
//   * a task = one output row (down) or one gate/up row pair (gate/up) of a
//     group; tasks are split evenly across a persistent grid, CTA c taking the
//     contiguous range [N*c/G, N*(c+1)/G)
//   * the CTA stages the group's TT activation rows in shared memory as fp32
//     (16-byte chunks XOR-swizzled per 32-weight unit, so the 8 lanes of a
//     quarter-warp hit 8 different bank groups)
//   * each lane owns whole 32-weight units of the row: one 16-byte
//     non-allocating load of codes (32 bytes for Q8_0) and the unit's scale;
//     codes are decoded in registers and multiplied against every token of
//     the group, so the weights are read once per group
//   * per-unit partial sums are scaled once per block (d * sum q x, plus
//     m * sum x for Q5_1), accumulated in fp32, and reduced across the row's
//     lanes with shuffles; the gate/up kernel writes h = silu(G x) * (U x)
//
// Decoding in registers:
//   * 4-bit codes (IQ4_NL, NVFP4): a 16-entry byte table held in 4 registers;
//     eight nibbles are looked up with four byte permutes (entries 0-7 and 8-15
//     in separate halves) and a per-byte select mask built from each nibble's
//     top bit by a sign-replicating permute.  NVFP4 uses the fixed table
//     2*e2m1 (integers -12..12), its block scale E4M3 decoded by placing the
//     7 bits in an fp32 exponent/mantissa and scaling by 2^120, times s/2.
//   * a table byte b (stored as value + 128) becomes a float by writing it in
//     the low mantissa byte of 2^23 and subtracting 2^23 + 128 (exact).
//   * Q5_1: the fifth bits of four elements are spread into their bytes with
//     one multiply (bit i -> bit 8i + 4).
#include <cuda_fp16.h>

#include "quant_dot.cuh"

namespace moe {

namespace {

using namespace qd;

// Stage the group's activation rows as fp32 into shared memory, chunk c of
// unit u at position u*8 + (c ^ (u & 7)); for Q5_1 also the per-unit sums.
template <int FMT, bool GATEUP, int TT>
__device__ __forceinline__ void stage_group(const MatvecArgs &a, float4 *xs4, float *xsum, int slot0,
                                            int ntok, int K, int NU)
{
    const int nc = K >> 2;
    for (int i = threadIdx.x; i < ntok * nc; i += kThreads) {
        const int t = i / nc, c = i - t * nc;
        float4 v;
        if constexpr (GATEUP) {
            const int tok = __ldg(a.perm_tok + slot0 + t);
            if (a.x_dtype == MOE_DT_BF16) {
                const uint2 b = __ldg(reinterpret_cast<const uint2 *>(
                    reinterpret_cast<const uint16_t *>(a.x) + (size_t)tok * K + c * 4));
                v = make_float4(bf16lo(b.x), bf16hi(b.x), bf16lo(b.y), bf16hi(b.y));
            } else {
                v = __ldg(reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.x) +
                                                           (size_t)tok * K + c * 4));
            }
        } else {
            v = __ldcg(reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.x) +
                                                        (size_t)(slot0 + t) * K + c * 4));
        }
        const int u = c >> 3, j = c & 7;
        xs4[t * nc + u * 8 + (j ^ (u & 7))] = v;
    }
    if constexpr (FMT == MOE_FMT_Q5_1) {
        __syncthreads();
        for (int i = threadIdx.x; i < ntok * NU; i += kThreads) {
            const int t = i / NU, u = i - t * NU;
            const float4 *p = xs4 + t * nc + u * 8;
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 q = p[j];
                s += q.x;
                s += q.y;
                s += q.z;
                s += q.w;
            }
            xsum[t * NU + u] = s;
        }
    }
}

template <int TT>
__device__ __forceinline__ void reduce_lanes(float (&v)[TT], int lpr)
{
#pragma unroll
    for (int t = 0; t < TT; ++t) {
        float s = v[t];
        for (int o = lpr >> 1; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        v[t] = s;
    }
}

template <int FMT, bool GATEUP, int TT>
__global__ void __launch_bounds__(kThreads, 1) matvec_kernel(const MatvecArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    float4 *xs4 = reinterpret_cast<float4 *>(smem);
    const int K = a.w.cols;
    const int NU = K >> 5;
    const int nc = K >> 2;
    float *xsum = reinterpret_cast<float *>(smem) + (size_t)TT * K;
    const int LPR = NU >= 32 ? 32 : NU >= 16 ? 16 : NU >= 8 ? 8 : NU >= 4 ? 4 : NU >= 2 ? 2 : 1;
    const int RPW = 32 / LPR;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane / LPR, sl = lane - sub * LPR;
    const int rows = a.rows_out;
    const int tpg = (rows + RPW - 1) / RPW;  // tasks per group
    const long long total = (long long)__ldg(a.n_groups) * tpg;
    long long task = total * blockIdx.x / gridDim.x;
    const long long tend = total * (blockIdx.x + 1) / gridDim.x;
    while (task < tend) {
        const int g = (int)(task / tpg);
        const long long gend = min(tend, (long long)(g + 1) * tpg);
        const int4 gd = __ldg(a.groups + g);
        const int e = gd.x, slot0 = gd.y, ntok = gd.z;
        float half_ts = 0.5f;
        if constexpr (FMT == MOE_FMT_NVFP4) half_ts = 0.5f * __ldg(a.w.ts + e);
        __syncthreads();
        stage_group<FMT, GATEUP, TT>(a, xs4, xsum, slot0, ntok, K, NU);
        __syncthreads();
        for (long long tk = task + warp; tk < gend; tk += kThreads / 32) {
            const int r = (int)(tk - (long long)g * tpg) * RPW + sub;
            const bool valid = r < rows;
            const int rr = valid ? r : rows - 1;
            float acc0[TT], acc1[TT];
            int xoff[TT], xsoff[TT];
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                acc0[t] = 0.f;
                acc1[t] = 0.f;
                xoff[t] = t * nc;
                xsoff[t] = t * NU;
            }
            for (int u = sl; u < NU; u += 2 * LPR) {
                const int u2 = u + LPR;
                const bool has2 = u2 < NU;
                Raw g0 = load_unit<FMT>(a.w, e, rr, u);
                Raw g1 = has2 ? load_unit<FMT>(a.w, e, rr, u2) : g0;
                Raw v0, v1;
                if constexpr (GATEUP) {
                    v0 = load_unit<FMT>(a.w, e, rows + rr, u);
                    v1 = has2 ? load_unit<FMT>(a.w, e, rows + rr, u2) : v0;
                }
                unit_dot<FMT, TT>(g0, u, xs4, xsum, xoff, xsoff, ntok, a.tab, half_ts, acc0);
                if constexpr (GATEUP) unit_dot<FMT, TT>(v0, u, xs4, xsum, xoff, xsoff, ntok, a.tab, half_ts, acc1);
                if (has2) {
                    unit_dot<FMT, TT>(g1, u2, xs4, xsum, xoff, xsoff, ntok, a.tab, half_ts, acc0);
                    if constexpr (GATEUP) unit_dot<FMT, TT>(v1, u2, xs4, xsum, xoff, xsoff, ntok, a.tab, half_ts, acc1);
                }
            }
            reduce_lanes<TT>(acc0, LPR);
            if constexpr (GATEUP) reduce_lanes<TT>(acc1, LPR);
            if (valid) {
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    if (t < ntok && (t % LPR) == sl) {
                        float v = acc0[t];
                        if constexpr (GATEUP) v = v / (1.f + expf(-v)) * acc1[t];
                        a.out[(size_t)(slot0 + t) * a.out_stride + r] = v;
                    }
                }
            }
        }
        task = gend;
    }
}

__global__ void __launch_bounds__(kThreads) combine_kernel(const CombineArgs a)
{
    const int t = blockIdx.y;
    const int H4 = a.H >> 2;
    const int *sp = a.slot_pos + (size_t)t * a.k;
    const float *gt = a.gate + (size_t)t * a.k;
    for (int c = blockIdx.x * kThreads + threadIdx.x; c < H4; c += gridDim.x * kThreads) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < a.k; ++j) {
            const float g = __ldg(gt + j);
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.y + (size_t)__ldg(sp + j) * a.H) + c);
            acc.x = fmaf(g, v.x, acc.x);
            acc.y = fmaf(g, v.y, acc.y);
            acc.z = fmaf(g, v.z, acc.z);
            acc.w = fmaf(g, v.w, acc.w);
        }
        if (a.has_shared) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.y + (size_t)(a.T * a.k + t) * a.H) + c);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        reinterpret_cast<float4 *>(a.out + (size_t)t * a.H)[c] = acc;
    }
}

// Dense-batched combine: out[t] = sum over active experts a of dgate[a*T+t] *
// y[a*T+t] (the shared expert's gate is 1), in expert order.
__global__ void __launch_bounds__(kThreads) combine_dense_kernel(const float *y, const float *dgate,
                                                                 const int32_t *n_rows, int T, int H, float *out)
{
    const int t = blockIdx.y;
    const int H4 = H >> 2;
    const int n_act = __ldg(n_rows) / T;
    for (int c = blockIdx.x * kThreads + threadIdx.x; c < H4; c += gridDim.x * kThreads) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int a = 0; a < n_act; ++a) {
            const float g = __ldcg(dgate + (size_t)a * T + t);
            if (g == 0.f) continue;
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(y + ((size_t)a * T + t) * H) + c);
            acc.x = fmaf(g, v.x, acc.x);
            acc.y = fmaf(g, v.y, acc.y);
            acc.z = fmaf(g, v.z, acc.z);
            acc.w = fmaf(g, v.w, acc.w);
        }
        reinterpret_cast<float4 *>(out + (size_t)t * H)[c] = acc;
    }
}

using KernelFn = void (*)(MatvecArgs);

template <int FMT>
KernelFn pick_fmt(bool gateup, int tt)
{
    if (gateup) return tt == 1 ? matvec_kernel<FMT, true, 1> : matvec_kernel<FMT, true, 8>;
    return tt == 1 ? matvec_kernel<FMT, false, 1> : matvec_kernel<FMT, false, 8>;
}

KernelFn pick(int fmt, bool gateup, int tt)
{
    switch (fmt) {
    case MOE_FMT_Q8_0: return pick_fmt<MOE_FMT_Q8_0>(gateup, tt);
    case MOE_FMT_Q5_1: return pick_fmt<MOE_FMT_Q5_1>(gateup, tt);
    case MOE_FMT_IQ4_NL: return pick_fmt<MOE_FMT_IQ4_NL>(gateup, tt);
    case MOE_FMT_NVFP4: return pick_fmt<MOE_FMT_NVFP4>(gateup, tt);
    default: return nullptr;
    }
}

}  // namespace

size_t matvec_smem_bytes(const MatvecArgs &a, bool gateup, int tt)
{
    (void)gateup;
    const int K = a.w.cols;
    size_t b = (size_t)tt * K * sizeof(float);
    if (a.w.fmt == MOE_FMT_Q5_1) b += (size_t)tt * (K / 32) * sizeof(float);
    return b;
}

cudaError_t matvec_set_attributes()
{
    const int fmts[4] = {MOE_FMT_Q8_0, MOE_FMT_Q5_1, MOE_FMT_IQ4_NL, MOE_FMT_NVFP4};
    for (int f : fmts)
        for (int gu = 0; gu < 2; ++gu)
            for (int tt : {1, 8}) {
                cudaError_t e = cudaFuncSetAttribute(pick(f, gu != 0, tt),
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
                if (e != cudaSuccess) return e;
            }
    return cudaSuccess;
}

int matvec_grid(const MatvecArgs &a, bool gateup, int tt, int num_sms)
{
    int per_sm = 0;
    KernelFn f = pick(a.w.fmt, gateup, tt);
    if (!f || cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, f, kThreads,
                                                            matvec_smem_bytes(a, gateup, tt)) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    return per_sm * num_sms;
}

cudaError_t launch_matvec(const MatvecArgs &a, bool gateup, int tt, int grid, cudaStream_t s)
{
    KernelFn f = pick(a.w.fmt, gateup, tt);
    if (!f) return cudaErrorInvalidValue;
    f<<<grid, kThreads, matvec_smem_bytes(a, gateup, tt), s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_combine_dense(const float *y, const float *dgate, const int32_t *n_rows, int T, int H,
                                 float *out, cudaStream_t s)
{
    dim3 grid((H / 4 + kThreads - 1) / kThreads, T);
    combine_dense_kernel<<<grid, kThreads, 0, s>>>(y, dgate, n_rows, T, H, out);
    return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s)
{
    const int H4 = a.H >> 2;
    dim3 grid((H4 + kThreads - 1) / kThreads, a.T);
    combine_kernel<<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
