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

#include "moe_internal.cuh"

namespace moe {

namespace {

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// byte i of r, stored as value + 128, as a float
__device__ __forceinline__ float sbyte(uint32_t r, int i)
{
    return __uint_as_float(prmt(r, 0x4B000000u, 0x7650u + i)) - 8388736.f;
}

// unsigned byte i of r as a float
__device__ __forceinline__ float ubyte(uint32_t r, int i)
{
    return __uint_as_float(prmt(r, 0x4B000000u, 0x7650u + i)) - 8388608.f;
}

// Table lookup of the 8 nibbles of w: byte n of o0 is t[nibble n], byte n of
// o1 is t[nibble 4+n].
__device__ __forceinline__ void lut16(uint32_t w, const uint32_t (&t)[4], uint32_t &o0, uint32_t &o1)
{
    const uint32_t w4 = w << 4, wx = w ^ 0x88888888u;
    const uint32_t m0 = prmt(w4, w, 0xD9C8u);  // 0xFF where nibble n >= 8 (n = 0..3)
    const uint32_t m1 = prmt(w4, w, 0xFBEAu);  // same for nibbles 4..7
    const uint32_t l0 = prmt(t[0], t[1], w), h0 = prmt(t[2], t[3], wx);
    const uint32_t l1 = prmt(t[0], t[1], w >> 16), h1 = prmt(t[2], t[3], wx >> 16);
    o0 = (l0 & ~m0) | (h0 & m0);
    o1 = (l1 & ~m1) | (h1 & m1);
}

__device__ __forceinline__ uint4 ld_stream16(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ld_stream4(const void *p)
{
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ld_stream2(const void *p)
{
    unsigned short r;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float e4m3_pos(uint32_t b)  // b in [0, 0x7E]
{
    return __uint_as_float((b & 0x7Fu) << 20) * 1.329227995784916e36f;  // 2^120
}

// One 32-weight unit of one row: codes and scale words.
struct Raw {
    uint4 q0, q1;  // q1 only for Q8_0
    uint32_t s;    // fp16 d | {fp16 d, fp16 m} | two E4M3 scales
    uint32_t h;    // Q5_1 fifth bits
};

template <int FMT>
__device__ __forceinline__ Raw load_unit(const DevProj &w, int e, int row, int u)
{
    Raw r;
    const uint8_t *qs = w.qs + (int64_t)e * w.qs_stride + (int64_t)row * w.qs_row;
    const uint8_t *sc = w.sc + (int64_t)e * w.sc_stride + (int64_t)row * w.sc_row;
    if constexpr (FMT == MOE_FMT_Q8_0) {
        r.q0 = ld_stream16(qs + u * 32);
        r.q1 = ld_stream16(qs + u * 32 + 16);
        r.s = ld_stream2(sc + u * 2);
        r.h = 0;
    } else {
        r.q0 = ld_stream16(qs + u * 16);
        r.q1 = make_uint4(0, 0, 0, 0);
        if constexpr (FMT == MOE_FMT_Q5_1) {
            r.s = ld_stream4(sc + u * 4);
            r.h = ld_stream4(w.qh + (int64_t)e * w.qh_stride + (int64_t)row * w.qh_row + u * 4);
        } else {
            r.s = ld_stream2(sc + u * 2);
            r.h = 0;
        }
    }
    return r;
}

// acc[t] += (unit u of this row) . x_t for the group's tokens
template <int FMT, int TT>
__device__ __forceinline__ void unit_dot(const Raw &r, int u, const float4 *xs4, const float *xsum,
                                         int nc, int NU, int ntok, const uint32_t (&tab)[4],
                                         float half_ts, float (&acc)[TT])
{
    const float4 *xu = xs4 + u * 8;
    const int sw = u & 7;
    if constexpr (FMT == MOE_FMT_Q8_0) {
        const float d = __half2float(__ushort_as_half((unsigned short)r.s));
        const uint32_t qw[8] = {r.q0.x, r.q0.y, r.q0.z, r.q0.w, r.q1.x, r.q1.y, r.q1.z, r.q1.w};
        float p[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) p[t] = 0.f;
#pragma unroll
        for (int wi = 0; wi < 8; ++wi) {
            const float v0 = sbyte(qw[wi], 0), v1 = sbyte(qw[wi], 1);
            const float v2 = sbyte(qw[wi], 2), v3 = sbyte(qw[wi], 3);
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                if (t < ntok) {
                    const float4 x = xu[t * nc + (wi ^ sw)];
                    float s = p[t];
                    s = fmaf(v0, x.x, s); s = fmaf(v1, x.y, s);
                    s = fmaf(v2, x.z, s); s = fmaf(v3, x.w, s);
                    p[t] = s;
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT; ++t) acc[t] = fmaf(d, p[t], acc[t]);
    } else if constexpr (FMT == MOE_FMT_IQ4_NL) {
        const float d = __half2float(__ushort_as_half((unsigned short)r.s));
        const uint32_t qw[4] = {r.q0.x, r.q0.y, r.q0.z, r.q0.w};
        float p[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) p[t] = 0.f;
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            uint32_t o0, o1;
            lut16(qw[wi], tab, o0, o1);
            // o0 = [elem 4wi, elem 16+4wi, elem 4wi+1, elem 17+4wi], o1 likewise +2
            const float a0 = sbyte(o0, 0), b0 = sbyte(o0, 1), a1 = sbyte(o0, 2), b1 = sbyte(o0, 3);
            const float a2 = sbyte(o1, 0), b2 = sbyte(o1, 1), a3 = sbyte(o1, 2), b3 = sbyte(o1, 3);
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                if (t < ntok) {
                    const float4 xa = xu[t * nc + (wi ^ sw)];
                    const float4 xb = xu[t * nc + ((wi + 4) ^ sw)];
                    float s = p[t];
                    s = fmaf(a0, xa.x, s); s = fmaf(b0, xb.x, s);
                    s = fmaf(a1, xa.y, s); s = fmaf(b1, xb.y, s);
                    s = fmaf(a2, xa.z, s); s = fmaf(b2, xb.z, s);
                    s = fmaf(a3, xa.w, s); s = fmaf(b3, xb.w, s);
                    p[t] = s;
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT; ++t) acc[t] = fmaf(d, p[t], acc[t]);
    } else if constexpr (FMT == MOE_FMT_Q5_1) {
        const __half2 dm = *reinterpret_cast<const __half2 *>(&r.s);
        const float d = __low2float(dm), m = __high2float(dm);
        const uint32_t qw[4] = {r.q0.x, r.q0.y, r.q0.z, r.q0.w};
        float p[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) p[t] = 0.f;
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            const uint32_t hl = (((r.h >> (4 * wi)) & 0xFu) * 0x02040810u) & 0x10101010u;
            const uint32_t hh = (((r.h >> (16 + 4 * wi)) & 0xFu) * 0x02040810u) & 0x10101010u;
            const uint32_t lo = (qw[wi] & 0x0F0F0F0Fu) | hl;
            const uint32_t hi = ((qw[wi] >> 4) & 0x0F0F0F0Fu) | hh;
            const float a0 = ubyte(lo, 0), a1 = ubyte(lo, 1), a2 = ubyte(lo, 2), a3 = ubyte(lo, 3);
            const float b0 = ubyte(hi, 0), b1 = ubyte(hi, 1), b2 = ubyte(hi, 2), b3 = ubyte(hi, 3);
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                if (t < ntok) {
                    const float4 xa = xu[t * nc + (wi ^ sw)];
                    const float4 xb = xu[t * nc + ((wi + 4) ^ sw)];
                    float s = p[t];
                    s = fmaf(a0, xa.x, s); s = fmaf(a1, xa.y, s);
                    s = fmaf(a2, xa.z, s); s = fmaf(a3, xa.w, s);
                    s = fmaf(b0, xb.x, s); s = fmaf(b1, xb.y, s);
                    s = fmaf(b2, xb.z, s); s = fmaf(b3, xb.w, s);
                    p[t] = s;
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            if (t < ntok) acc[t] = fmaf(m, xsum[t * NU + u], fmaf(d, p[t], acc[t]));
        }
    } else {  // NVFP4: two 16-weight blocks per unit
        const float s0 = e4m3_pos(r.s & 0xFFu) * half_ts;
        const float s1 = e4m3_pos((r.s >> 8) & 0xFFu) * half_ts;
        const uint32_t qw[4] = {r.q0.x, r.q0.y, r.q0.z, r.q0.w};
        float p0[TT], p1[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) { p0[t] = 0.f; p1[t] = 0.f; }
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            uint32_t o0, o1;
            lut16(qw[wi], tab, o0, o1);  // elements 8wi .. 8wi+7 in order
            const float v0 = sbyte(o0, 0), v1 = sbyte(o0, 1), v2 = sbyte(o0, 2), v3 = sbyte(o0, 3);
            const float v4 = sbyte(o1, 0), v5 = sbyte(o1, 1), v6 = sbyte(o1, 2), v7 = sbyte(o1, 3);
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                if (t < ntok) {
                    const float4 xa = xu[t * nc + ((2 * wi) ^ sw)];
                    const float4 xb = xu[t * nc + ((2 * wi + 1) ^ sw)];
                    float s = wi < 2 ? p0[t] : p1[t];
                    s = fmaf(v0, xa.x, s); s = fmaf(v1, xa.y, s);
                    s = fmaf(v2, xa.z, s); s = fmaf(v3, xa.w, s);
                    s = fmaf(v4, xb.x, s); s = fmaf(v5, xb.y, s);
                    s = fmaf(v6, xb.z, s); s = fmaf(v7, xb.w, s);
                    if (wi < 2) p0[t] = s; else p1[t] = s;
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT; ++t) acc[t] = fmaf(s1, p1[t], fmaf(s0, p0[t], acc[t]));
    }
}

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
__global__ void __launch_bounds__(kThreads) matvec_kernel(const MatvecArgs a)
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
#pragma unroll
            for (int t = 0; t < TT; ++t) { acc0[t] = 0.f; acc1[t] = 0.f; }
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
                unit_dot<FMT, TT>(g0, u, xs4, xsum, nc, NU, ntok, a.tab, half_ts, acc0);
                if constexpr (GATEUP) unit_dot<FMT, TT>(v0, u, xs4, xsum, nc, NU, ntok, a.tab, half_ts, acc1);
                if (has2) {
                    unit_dot<FMT, TT>(g1, u2, xs4, xsum, nc, NU, ntok, a.tab, half_ts, acc0);
                    if constexpr (GATEUP) unit_dot<FMT, TT>(v1, u2, xs4, xsum, nc, NU, ntok, a.tab, half_ts, acc1);
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

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s)
{
    const int H4 = a.H >> 2;
    dim3 grid((H4 + kThreads - 1) / kThreads, a.T);
    combine_kernel<<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
