// Weight blocks to real values for the tensor-core kernels that dequantise in
// shared memory: one 32-weight block of one row at a time, loaded from the
// pack's planes (codes, scales, fifth bits) and expanded to 32 floats in
// element order.  Used by the dequantising prefill GEMM (bf16 operands) and by
// the tensor-core decode GEMM (fp16 operands, blk_f16: no fp32 step).
//
//   Q8_0    w = d q           q int8 (stored + 128), d fp16 per 32
//   IQ4_NL  w = d t[c]        c 4-bit (element j < 16: low nibble of byte j,
//                             j >= 16: high nibble of byte j - 16), t the
//                             pack's code table, d fp16 per 32
//   Q5_1    w = d q + m       q = nibble | fifth bit << 4 (nibble order as
//                             IQ4_NL), {d, m} fp16 per 32
//   NVFP4   w = t[c] s / 2    c E2M1 codes in element order (two per byte, low
//                             nibble first), t the code table (twice the E2M1
//                             value), s the E4M3 scale of each 16; the expert's
//                             fp32 scale is left to the caller's epilogue
#pragma once

#include <cuda_fp16.h>

#include "moe_internal.cuh"
#include "quant_dot.cuh"

namespace moe {
namespace dq {

__device__ __forceinline__ float byte_f(uint32_t w, int i)  // biased int8 -> float
{
    return __uint_as_float(qd::prmt(w, 0x4B000000u, 0x7650u + i)) - 8388736.f;
}

__device__ __forceinline__ float half_bits(uint32_t b) { return __half2float(__ushort_as_half((unsigned short)b)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// One 32-weight block of one row, as loaded.
template <int FMT>
struct Blk {
    uint4 q[FMT == MOE_FMT_Q8_0 ? 2 : 1];  // codes
    uint32_t s;                            // Q8_0 / IQ4_NL: fp16 d; Q5_1: {d, m}; NVFP4: two E4M3 bytes
    uint32_t h;                            // Q5_1 fifth bits
};

// Block b (weights 32 b .. 32 b + 31) of a row whose planes start at qrow,
// srow (row-major scales) and hrow (Q5_1 only).
template <int FMT>
__device__ __forceinline__ Blk<FMT> load_blk(const uint8_t *qrow, const uint8_t *srow, const uint8_t *hrow, int b)
{
    Blk<FMT> r;
    r.h = 0;
    if constexpr (FMT == MOE_FMT_Q8_0) {
        r.q[0] = __ldg(reinterpret_cast<const uint4 *>(qrow + b * 32));
        r.q[1] = __ldg(reinterpret_cast<const uint4 *>(qrow + b * 32) + 1);
    } else {
        r.q[0] = __ldg(reinterpret_cast<const uint4 *>(qrow + b * 16));
    }
    if constexpr (FMT == MOE_FMT_Q5_1) {
        r.s = __ldg(reinterpret_cast<const uint32_t *>(srow + b * 4));
        r.h = __ldg(reinterpret_cast<const uint32_t *>(hrow + b * 4));
    } else {
        r.s = __ldg(reinterpret_cast<const uint16_t *>(srow + b * 2));
    }
    return r;
}

// The 32 weights of a block, in element order.
template <int FMT>
__device__ __forceinline__ void blk_values(const Blk<FMT> &r, const CodeTable &ct, float (&v)[32])
{
    if constexpr (FMT == MOE_FMT_Q8_0) {
        const float d = half_bits(r.s);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w = (&r.q[0].x)[i];
#pragma unroll
            for (int b = 0; b < 4; ++b) v[4 * i + b] = byte_f(w, b) * d;
        }
    } else if constexpr (FMT == MOE_FMT_IQ4_NL) {
        const float d = half_bits(r.s);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            uint32_t o0, o1;
            qd::lut16((&r.q[0].x)[s], ct, o0, o1);  // o0 = [lo0 hi0 lo1 hi1], o1 = [lo2 hi2 lo3 hi3] of bytes 4s..
            const uint32_t oo[2] = {o0, o1};
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t o = oo[b >> 1];
                const float lo = __uint_as_float(qd::prmt(o, 0x4B000000u, 0x7650u + 2 * (b & 1))) - ct.magic;
                const float hi = __uint_as_float(qd::prmt(o, 0x4B000000u, 0x7650u + 2 * (b & 1) + 1)) - ct.magic;
                v[4 * s + b] = lo * d;
                v[16 + 4 * s + b] = hi * d;
            }
        }
    } else if constexpr (FMT == MOE_FMT_Q5_1) {
        const float d = half_bits(r.s & 0xFFFFu), m = half_bits(r.s >> 16);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint32_t byte = ((&r.q[0].x)[j >> 2] >> (8 * (j & 3))) & 0xFFu;
            const uint32_t lo = (byte & 0xFu) | (((r.h >> j) & 1u) << 4);
            const uint32_t hi = (byte >> 4) | (((r.h >> (j + 16)) & 1u) << 4);
            v[j] = fmaf(d, (float)lo, m);
            v[16 + j] = fmaf(d, (float)hi, m);
        }
    } else {  // NVFP4: words s = 0..3 hold elements 8s .. 8s + 7
        const float s0 = qd::e4m3_pos(r.s & 0xFFu), s1 = qd::e4m3_pos((r.s >> 8) & 0xFFu);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            uint32_t o0, o1;
            qd::lut16((&r.q[0].x)[s], ct, o0, o1);  // o0 = elements 8s .. 8s+3, o1 = 8s+4 .. 8s+7
            const float sc = s < 2 ? s0 : s1;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                v[8 * s + b] = (__uint_as_float(qd::prmt(o0, 0x4B000000u, 0x7650u + b)) - ct.magic) * sc;
                v[8 * s + 4 + b] = (__uint_as_float(qd::prmt(o1, 0x4B000000u, 0x7650u + b)) - ct.magic) * sc;
            }
        }
    }
}

// ---- straight to fp16 (the tensor-core decode path) --------------------------
// A biased byte b is the fp16 number 1024 + b once 0x64 is put above it; two
// of them make an f16x2 with one byte permute.  sel picks the two bytes of w.
__device__ __forceinline__ uint32_t f16pair(uint32_t w, uint32_t sel) { return qd::prmt(w, 0x64646464u, sel); }
constexpr uint32_t kSelB01 = 0x4140u, kSelB23 = 0x4342u, kSelB02 = 0x4240u, kSelB13 = 0x4341u;

__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t f16_bits(float f) { return __half_as_ushort(__float2half_rn(f)); }
__device__ __forceinline__ uint32_t dup16(uint32_t h) { return (h & 0xFFFFu) * 0x10001u; }

// The 32 weights of a block as four 16-byte chunks of fp16 (chunk i: elements
// 8i .. 8i + 7), from its codes (q: 16 bytes, Q8_0 32), its scale word s and
// its fifth bits hb (Q5_1).  Codes become exact small integers in fp16 (1024 +
// biased byte, minus 1024 + bias); one multiply (Q5_1: one fused multiply-add
// with m) by the block scale then rounds each weight once.
template <int FMT>
__device__ __forceinline__ void blk_f16(const uint32_t *q, uint32_t s, uint32_t hb, const CodeTable &ct, uint4 (&o)[4])
{
    uint32_t w[16];  // element pairs (2j, 2j + 1)
    if constexpr (FMT == MOE_FMT_Q8_0) {
        const uint32_t d2 = dup16(s), b2 = 0x64806480u;  // 1024 + 128
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            w[2 * i] = hmul2(hsub2(f16pair(q[i], kSelB01), b2), d2);
            w[2 * i + 1] = hmul2(hsub2(f16pair(q[i], kSelB23), b2), d2);
        }
    } else if constexpr (FMT == MOE_FMT_IQ4_NL || FMT == MOE_FMT_NVFP4) {
        // bias of the table bytes: magic = 2^23 + bias
        const uint32_t b2 = dup16(f16_bits(1024.f + (ct.magic - 8388608.f)));
        uint32_t d2a, d2b;  // scales of elements 0-15 and 16-31
        if constexpr (FMT == MOE_FMT_IQ4_NL) {
            d2a = d2b = dup16(s);
        } else {
            d2a = dup16(f16_bits(qd::e4m3_pos(s & 0xFFu)));
            d2b = dup16(f16_bits(qd::e4m3_pos((s >> 8) & 0xFFu)));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t o0, o1;
            qd::lut16(q[j], ct, o0, o1);
            if constexpr (FMT == MOE_FMT_IQ4_NL) {
                // word j: bytes 4j .. 4j+3; o0 = [lo0 hi0 lo1 hi1], o1 = [lo2 hi2 lo3 hi3]
                // low nibbles are elements 4j .., high nibbles 16 + 4j ..
                w[2 * j] = hmul2(hsub2(f16pair(o0, kSelB02), b2), d2a);          // elements 4j, 4j+1
                w[2 * j + 1] = hmul2(hsub2(f16pair(o1, kSelB02), b2), d2a);      // 4j+2, 4j+3
                w[8 + 2 * j] = hmul2(hsub2(f16pair(o0, kSelB13), b2), d2b);      // 16+4j, 16+4j+1
                w[8 + 2 * j + 1] = hmul2(hsub2(f16pair(o1, kSelB13), b2), d2b);  // 16+4j+2, 16+4j+3
            } else {
                // word j: elements 8j .. 8j+7 in order; o0 = the first four
                const uint32_t d2 = j < 2 ? d2a : d2b;
                w[4 * j] = hmul2(hsub2(f16pair(o0, kSelB01), b2), d2);
                w[4 * j + 1] = hmul2(hsub2(f16pair(o0, kSelB23), b2), d2);
                w[4 * j + 2] = hmul2(hsub2(f16pair(o1, kSelB01), b2), d2);
                w[4 * j + 3] = hmul2(hsub2(f16pair(o1, kSelB23), b2), d2);
            }
        }
    } else {  // Q5_1: w = d q + m, q = nibble | fifth bit << 4
        const uint32_t d2 = dup16(s), m2 = dup16(s >> 16), k2 = 0x64006400u;  // 1024
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t hl = (((hb >> (4 * j)) & 0xFu) * 0x02040810u) & 0x10101010u;
            const uint32_t hh = (((hb >> (16 + 4 * j)) & 0xFu) * 0x02040810u) & 0x10101010u;
            const uint32_t lo = (q[j] & 0x0F0F0F0Fu) | hl;          // elements 4j .. 4j+3
            const uint32_t hi = ((q[j] >> 4) & 0x0F0F0F0Fu) | hh;   // elements 16+4j ..
            w[2 * j] = hfma2(hsub2(f16pair(lo, kSelB01), k2), d2, m2);
            w[2 * j + 1] = hfma2(hsub2(f16pair(lo, kSelB23), k2), d2, m2);
            w[8 + 2 * j] = hfma2(hsub2(f16pair(hi, kSelB01), k2), d2, m2);
            w[8 + 2 * j + 1] = hfma2(hsub2(f16pair(hi, kSelB23), k2), d2, m2);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

}  // namespace dq
}  // namespace moe
