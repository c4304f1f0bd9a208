// Device helpers shared by the decode kernels: streaming loads, register
// decoding of the four block formats and the per-unit dot product against
// activations staged in shared memory (see decode.cu for the design).
#pragma once

#include <cuda_fp16.h>

#include "moe_internal.cuh"

namespace moe {
namespace qd {

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
        } else if constexpr (FMT == MOE_FMT_NVFP4) {
            // the unit's two block scales: K step u/2, scales 2(u%2), 2(u%2)+1
            r.s = ld_stream2(w.sc + (int64_t)e * w.sc_stride + sf_offset(row, u >> 1, (u & 1) * 2, w.ksteps));
            r.h = 0;
        } else {
            r.s = ld_stream2(sc + u * 2);
            r.h = 0;
        }
    }
    return r;
}

// acc[t] += (unit u of this row) . x_t for the group's tokens
// x row of group token t starts at xs4 + xoff[t] (float4 units); for Q5_1 its
// per-unit sums at xsum + xsoff[t].
template <int FMT, int TT>
__device__ __forceinline__ void unit_dot(const Raw &r, int u, const float4 *xs4, const float *xsum,
                                         const int (&xoff)[TT], const int (&xsoff)[TT], int ntok,
                                         const uint32_t (&tab)[4], float half_ts, float (&acc)[TT])
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
                    const float4 x = xu[xoff[t] + (wi ^ sw)];
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
                    const float4 xa = xu[xoff[t] + (wi ^ sw)];
                    const float4 xb = xu[xoff[t] + ((wi + 4) ^ sw)];
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
                    const float4 xa = xu[xoff[t] + (wi ^ sw)];
                    const float4 xb = xu[xoff[t] + ((wi + 4) ^ sw)];
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
            if (t < ntok) acc[t] = fmaf(m, xsum[xsoff[t] + u], fmaf(d, p[t], acc[t]));
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
                    const float4 xa = xu[xoff[t] + ((2 * wi) ^ sw)];
                    const float4 xb = xu[xoff[t] + ((2 * wi + 1) ^ sw)];
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


}  // namespace qd
}  // namespace moe
