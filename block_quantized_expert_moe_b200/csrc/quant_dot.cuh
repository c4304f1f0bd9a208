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

// The code table (CodeTable, moe_internal.cuh) holds entry value + bias in
// bytes; in xor mode positions i and i+8 have equal top bits and t[2..3] hold
// the high half pre-XORed with the sign-replicated low half, so a lookup of
// eight nibbles is four byte permutes and two XORs; otherwise a per-byte select
// mask built from each nibble's top bit merges the two halves.
// byte n of o0 = entry[nibble n], byte n of o1 = entry[nibble 4+n], n = 0..3
__device__ __forceinline__ void lut16(uint32_t w, const CodeTable &ct, uint32_t &o0, uint32_t &o1)
{
    const uint32_t wx = w ^ 0x88888888u;
    const uint32_t l0 = prmt(ct.t[0], ct.t[1], w), h0 = prmt(ct.t[2], ct.t[3], wx);
    const uint32_t l1 = prmt(ct.t[0], ct.t[1], w >> 16), h1 = prmt(ct.t[2], ct.t[3], wx >> 16);
    if (ct.xor_mode) {
        o0 = l0 ^ h0;
        o1 = l1 ^ h1;
    } else {
        const uint32_t w4 = w << 4;
        const uint32_t m0 = prmt(w4, w, 0xD9C8u);  // 0xFF where nibble n >= 8 (n = 0..3)
        const uint32_t m1 = prmt(w4, w, 0xFBEAu);  // same for nibbles 4..7
        o0 = (l0 & ~m0) | (h0 & m0);
        o1 = (l1 & ~m1) | (h1 & m1);
    }
}

// ---- packed fp32 pairs (f32x2 arithmetic of sm_100) ----------------------------
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 sub2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// bytes i and j of r (each value + bias) as a float pair: write them into the
// low mantissa byte of 2^23 and subtract 2^23 + bias (exact)
__device__ __forceinline__ float2 bytes2(uint32_t r, int i, int j, float magic)
{
    const float a = __uint_as_float(prmt(r, 0x4B000000u, 0x7650u + i));
    const float b = __uint_as_float(prmt(r, 0x4B000000u, 0x7650u + j));
    return sub2(make_float2(a, b), make_float2(magic, magic));
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
// One of the four steps of a 32-weight unit: four weight pairs, the first two
// against x chunk ca (.xy, .zw), the last two against chunk cb.
//   Q8_0    step s = words 2s, 2s+1 (elements 8s..8s+7), chunks 2s, 2s+1
//   IQ4_NL  step s = word s: low nibbles elements 4s..4s+3 (chunk s), high
//           nibbles elements 16+4s.. (chunk s+4)
//   Q5_1    as IQ4_NL, fifth bits spread from qh with one multiply
//   NVFP4   step s = word s, elements 8s..8s+7 (chunks 2s, 2s+1); steps 0-1 are
//           the unit's first 16-block, 2-3 its second
template <int FMT>
__device__ __forceinline__ void decode_step(const Raw &r, int s, const CodeTable &ct, float2 &a0, float2 &a1,
                                            float2 &b0, float2 &b1, int &ca, int &cb)
{
    const uint32_t qw[8] = {r.q0.x, r.q0.y, r.q0.z, r.q0.w, r.q1.x, r.q1.y, r.q1.z, r.q1.w};
    if constexpr (FMT == MOE_FMT_Q8_0) {
        const uint32_t w0 = qw[2 * s], w1 = qw[2 * s + 1];
        a0 = bytes2(w0, 0, 1, 8388736.f);
        a1 = bytes2(w0, 2, 3, 8388736.f);
        b0 = bytes2(w1, 0, 1, 8388736.f);
        b1 = bytes2(w1, 2, 3, 8388736.f);
        ca = 2 * s;
        cb = 2 * s + 1;
    } else if constexpr (FMT == MOE_FMT_IQ4_NL) {
        uint32_t o0, o1;
        lut16(qw[s], ct, o0, o1);  // o0 = [lo0, hi0, lo1, hi1], o1 = [lo2, hi2, lo3, hi3]
        a0 = bytes2(o0, 0, 2, ct.magic);
        a1 = bytes2(o1, 0, 2, ct.magic);
        b0 = bytes2(o0, 1, 3, ct.magic);
        b1 = bytes2(o1, 1, 3, ct.magic);
        ca = s;
        cb = s + 4;
    } else if constexpr (FMT == MOE_FMT_Q5_1) {
        const uint32_t hl = (((r.h >> (4 * s)) & 0xFu) * 0x02040810u) & 0x10101010u;
        const uint32_t hh = (((r.h >> (16 + 4 * s)) & 0xFu) * 0x02040810u) & 0x10101010u;
        const uint32_t lo = (qw[s] & 0x0F0F0F0Fu) | hl;
        const uint32_t hi = ((qw[s] >> 4) & 0x0F0F0F0Fu) | hh;
        a0 = bytes2(lo, 0, 1, 8388608.f);
        a1 = bytes2(lo, 2, 3, 8388608.f);
        b0 = bytes2(hi, 0, 1, 8388608.f);
        b1 = bytes2(hi, 2, 3, 8388608.f);
        ca = s;
        cb = s + 4;
    } else {
        uint32_t o0, o1;
        lut16(qw[s], ct, o0, o1);  // elements 8s .. 8s+7 in order
        a0 = bytes2(o0, 0, 1, ct.magic);
        a1 = bytes2(o0, 2, 3, ct.magic);
        b0 = bytes2(o1, 0, 1, ct.magic);
        b1 = bytes2(o1, 2, 3, ct.magic);
        ca = 2 * s;
        cb = 2 * s + 1;
    }
}

__device__ __forceinline__ float2 lo2(float4 v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(float4 v) { return make_float2(v.z, v.w); }

// Scale the unit's per-block partial sums (pairs) into the running sum.
template <int FMT>
__device__ __forceinline__ float unit_scale(const Raw &r, float2 p0, float2 p1, float xs, float half_ts, float acc)
{
    if constexpr (FMT == MOE_FMT_Q8_0 || FMT == MOE_FMT_IQ4_NL) {
        const float d = __half2float(__ushort_as_half((unsigned short)r.s));
        return fmaf(d, (p0.x + p0.y) + (p1.x + p1.y), acc);
    } else if constexpr (FMT == MOE_FMT_Q5_1) {
        const __half2 dm = *reinterpret_cast<const __half2 *>(&r.s);
        return fmaf(__high2float(dm), xs, fmaf(__low2float(dm), (p0.x + p0.y) + (p1.x + p1.y), acc));
    } else {
        const float s0 = e4m3_pos(r.s & 0xFFu) * half_ts;
        const float s1 = e4m3_pos((r.s >> 8) & 0xFFu) * half_ts;
        return fmaf(s1, p1.x + p1.y, fmaf(s0, p0.x + p0.y, acc));
    }
}

// acc[t] += (unit u of this row) . x_t for the group's tokens.  The x row of
// group token t starts at xs4 + xoff[t] (float4 units, 16-byte chunk j of unit
// u at u*8 + (j ^ (u & 7))); for Q5_1 its per-unit sums at xsum + xsoff[t].
// Products accumulate in fp32 pairs (f32x2 FMA); each block's partial sum is
// scaled once.
template <int FMT, int TT>
__device__ __forceinline__ void unit_dot(const Raw &r, int u, const float4 *xs4, const float *xsum,
                                         const int (&xoff)[TT], const int (&xsoff)[TT], int ntok,
                                         const CodeTable &ct, float half_ts, float (&acc)[TT])
{
    const float4 *xu = xs4 + u * 8;
    const int sw = u & 7;
    float2 p0[TT], p1[TT];  // NVFP4: p0 first 16-block, p1 second; others: split by step parity
#pragma unroll
    for (int t = 0; t < TT; ++t) {
        p0[t] = make_float2(0.f, 0.f);
        p1[t] = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        float2 a0, a1, b0, b1;
        int ca, cb;
        decode_step<FMT>(r, s, ct, a0, a1, b0, b1, ca, cb);
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            if (t < ntok) {
                const float4 xa = xu[xoff[t] + (ca ^ sw)];
                const float4 xb = xu[xoff[t] + (cb ^ sw)];
                const bool first = FMT == MOE_FMT_NVFP4 ? s < 2 : (s & 1) == 0;
                float2 q = first ? p0[t] : p1[t];
                q = fma2(a0, lo2(xa), q);
                q = fma2(a1, hi2(xa), q);
                q = fma2(b0, lo2(xb), q);
                q = fma2(b1, hi2(xb), q);
                if (first) p0[t] = q; else p1[t] = q;
            }
        }
    }
#pragma unroll
    for (int t = 0; t < TT; ++t) {
        if (t < ntok) {
            const float xs = FMT == MOE_FMT_Q5_1 ? xsum[xsoff[t] + u] : 0.f;
            acc[t] = unit_scale<FMT>(r, p0[t], p1[t], xs, half_ts, acc[t]);
        }
    }
}

// Single token with the unit's 32 x values in registers (natural element order).
template <int FMT>
__device__ __forceinline__ float unit_dot_reg(const Raw &r, const float4 (&xr)[8], float xs, const CodeTable &ct,
                                              float half_ts, float acc)
{
    float2 p0 = make_float2(0.f, 0.f), p1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        float2 a0, a1, b0, b1;
        int ca, cb;
        decode_step<FMT>(r, s, ct, a0, a1, b0, b1, ca, cb);
        const bool first = FMT == MOE_FMT_NVFP4 ? s < 2 : (s & 1) == 0;
        float2 q = first ? p0 : p1;
        q = fma2(a0, lo2(xr[ca]), q);
        q = fma2(a1, hi2(xr[ca]), q);
        q = fma2(b0, lo2(xr[cb]), q);
        q = fma2(b1, hi2(xr[cb]), q);
        if (first) p0 = q; else p1 = q;
    }
    return unit_scale<FMT>(r, p0, p1, xs, half_ts, acc);
}

}  // namespace qd
}  // namespace moe
