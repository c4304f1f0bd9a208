// Grouped decode matvecs for batches of tokens, fed by TMA into shared memory.
//
// The "Qwen3.8-Flash-Next UD-IQ2_XS (L4 fix) for Basalt" model card ("What was
// changed") runs the MoE tail as grouped kernels over block-quantised experts,
// each expert's weights read once for all the tokens routed to it.  With
// several tokens per expert the multiply-adds (tokens x weights) outweigh the
// decoding, so this kernel gives every lane a whole ROW: the tokens' x values
// are then the same for the 32 lanes of a warp (shared-memory broadcast, one
// wavefront per load whatever the lane count) and each weight is decoded once
// and used for every token of the group.
//
//   task      a work group of the plan {expert, first slot, <= 8 tokens} times
//             a block of 32 weight rows: gate/up = 16 row pairs (gate rows in
//             lanes 0-15, the matching up rows in lanes 16-31), down = 32 rows
//   split     tasks in plan order, cut into one contiguous range per CTA by
//             cost (4 + tokens per task: decoding ~ four tokens' multiply-adds)
//   producer  one warp: for each task, one TMA tile load per 128-byte column
//             segment of every plane of the block's rows (codes, scales, fifth
//             bits) into a ring of stages, 128/64/32-byte swizzled so that 32
//             lanes reading the same unit of 32 different rows hit distinct
//             banks; full/empty mbarriers per stage
//   consumers 8 warps: all work on the same stage, each on 1/8 of the row's
//             32-weight units; per-token partial sums go through shared memory
//             and warp t finishes token t (SwiGLU for gate/up: lane j pairs
//             with lane j + 16)
//   x         the group's tokens (gate/up: rows of the layer input picked by
//             the plan; down: h rows of the group's slots) staged as fp32 when
//             the group changes
//
// Waits are bounded (~1 s); a time-out records MOE_ERR_TIMEOUT in the error
// word and the CTA drains what it has issued before returning.
#include "quant_dot.cuh"
#include "tc_common.cuh"
#include "tma_maps.cuh"

namespace moe {

namespace {

using namespace qd;
using namespace tc;

constexpr int kSgConsumers = 8;                    // consumer warps
constexpr int kSgThreads = 32 * (kSgConsumers + 1);  // + producer warp
constexpr int kSgTT = 8;                           // tokens per work group (the plan's cap)
constexpr int kSgMaxStages = 8;
constexpr int kSgMaxGroups = 2048;                 // groups whose costs fit the CTA's prefix table
constexpr int kSgSmemLimit = 220 * 1024;

struct SgPlane {
    int row_bytes;  // bytes of one row of this plane
    int w;          // TMA box width in bytes (= swizzle span): 128, 64, 32 or 16
    int off;        // byte offset of the plane in a stage
};

struct SgArgs {
    const int4 *groups;       // {expert slot, first slot, tokens, -}
    const int32_t *n_groups;
    const int32_t *perm_tok;  // gate/up: slot -> token row of x
    const void *x;            // gate/up: layer input [T x K]; down: h [slots x K] fp32
    int x_dtype;
    float *out;               // gate/up: h [slots x I]; down: y [slots x H]
    int out_stride;
    int K;                    // reduction length (weights per row)
    int rows_out;             // gate/up: I (row pairs); down: H
    int gateup;
    int fmt;
    const float *ts;          // NVFP4 per-expert scale
    CodeTable tab;
    SgPlane pl[3];            // codes, scales, fifth bits (row_bytes 0 if absent)
    int stage_bytes;          // stage stride (planes 1024-byte aligned)
    int tx_bytes;             // bytes the TMA loads of one stage deliver
    int n_stages;
    int32_t *err;
};

// swizzle of row r within a box `w` bytes wide (TMA 128/64/32-byte modes)
__device__ __forceinline__ int sg_swz(int r, int w)
{
    return w == 128 ? (r & 7) : w == 64 ? ((r >> 1) & 3) : w == 32 ? ((r >> 2) & 1) : 0;
}

// byte `off` of row r of a plane laid out as [segment][32 rows][w bytes]
__device__ __forceinline__ const uint8_t *sg_at(const uint8_t *plane, int w, int r, int off)
{
    const int seg = off / w, in = off - seg * w;
    return plane + seg * (32 * w) + r * w + ((((in >> 4) ^ sg_swz(r, w)) << 4) | (in & 15));
}

// One lane's view of one plane of the stage: its row's base and swizzle.
struct SgRow {
    const uint8_t *base;  // plane + r * w
    int lw;               // log2(w)
    int segs;             // bytes between 32-row segments (32 * w)
    int swz;
    __device__ __forceinline__ const uint8_t *at(int off) const
    {
        const int in = off & ((1 << lw) - 1);
        return base + (off >> lw) * segs + ((((in >> 4) ^ swz) << 4) | (in & 15));
    }
};

__device__ __forceinline__ SgRow sg_row(const uint8_t *stage, const SgPlane &p, int r)
{
    SgRow v;
    v.lw = p.w == 128 ? 7 : p.w == 64 ? 6 : p.w == 32 ? 5 : 4;
    v.base = stage + p.off + r * p.w;
    v.segs = 32 * p.w;
    v.swz = sg_swz(r, p.w);
    return v;
}

template <int FMT>
__device__ __forceinline__ Raw sg_unit_row(const SgRow &q, const SgRow &s, const SgRow &h, int u)
{
    Raw raw;
    raw.h = 0;
    raw.q1 = make_uint4(0, 0, 0, 0);
    if constexpr (FMT == MOE_FMT_Q8_0) {
        raw.q0 = *reinterpret_cast<const uint4 *>(q.at(u * 32));
        raw.q1 = *reinterpret_cast<const uint4 *>(q.at(u * 32 + 16));
        raw.s = *reinterpret_cast<const uint16_t *>(s.at(u * 2));
    } else {
        raw.q0 = *reinterpret_cast<const uint4 *>(q.at(u * 16));
        if constexpr (FMT == MOE_FMT_Q5_1) {
            raw.s = *reinterpret_cast<const uint32_t *>(s.at(u * 4));
            raw.h = *reinterpret_cast<const uint32_t *>(h.at(u * 4));
        } else {
            raw.s = *reinterpret_cast<const uint16_t *>(s.at(u * 2));
        }
    }
    return raw;
}

// This warp's share [u0, u1) of the units of row `lane`, for exactly NT tokens.
template <int FMT, int NT>
__device__ __forceinline__ void sg_rows(const SgArgs &a, const uint8_t *stage, int lane, int u0, int u1,
                                        const float4 *xs4, const float *xsum, int nc, int NU, float half_ts,
                                        float (&acc)[kSgTT])
{
    const SgRow rq = sg_row(stage, a.pl[0], lane), rs = sg_row(stage, a.pl[1], lane),
                rh = sg_row(stage, a.pl[2], lane);
#pragma unroll 1
    for (int u = u0; u < u1; ++u) {
        const Raw raw = sg_unit_row<FMT>(rq, rs, rh, u);
        float2 p0[NT], p1[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            p0[t] = make_float2(0.f, 0.f);
            p1[t] = make_float2(0.f, 0.f);
        }
        const float4 *xu = xs4 + u * 8;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            float2 w0, w1, w2, w3;
            int ca, cb;
            decode_step<FMT>(raw, s, a.tab, w0, w1, w2, w3, ca, cb);
            const bool first = FMT == MOE_FMT_NVFP4 ? s < 2 : (s & 1) == 0;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const float4 xa = xu[t * nc + ca], xb = xu[t * nc + cb];
                float2 q = first ? p0[t] : p1[t];
                q = fma2(w0, lo2(xa), q);
                q = fma2(w1, hi2(xa), q);
                q = fma2(w2, lo2(xb), q);
                q = fma2(w3, hi2(xb), q);
                if (first) p0[t] = q;
                else p1[t] = q;
            }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t)
            acc[t] = unit_scale<FMT>(raw, p0[t], p1[t], FMT == MOE_FMT_Q5_1 ? xsum[t * NU + u] : 0.f, half_ts, acc[t]);
    }
}

template <int FMT>
__device__ __forceinline__ Raw sg_unit(const SgArgs &a, const uint8_t *stage, int r, int u)
{
    Raw raw;
    raw.h = 0;
    raw.q1 = make_uint4(0, 0, 0, 0);
    const uint8_t *q = stage + a.pl[0].off, *s = stage + a.pl[1].off;
    if constexpr (FMT == MOE_FMT_Q8_0) {
        raw.q0 = *reinterpret_cast<const uint4 *>(sg_at(q, a.pl[0].w, r, u * 32));
        raw.q1 = *reinterpret_cast<const uint4 *>(sg_at(q, a.pl[0].w, r, u * 32 + 16));
        raw.s = *reinterpret_cast<const uint16_t *>(sg_at(s, a.pl[1].w, r, u * 2));
    } else {
        raw.q0 = *reinterpret_cast<const uint4 *>(sg_at(q, a.pl[0].w, r, u * 16));
        if constexpr (FMT == MOE_FMT_Q5_1) {
            raw.s = *reinterpret_cast<const uint32_t *>(sg_at(s, a.pl[1].w, r, u * 4));
            raw.h = *reinterpret_cast<const uint32_t *>(sg_at(stage + a.pl[2].off, a.pl[2].w, r, u * 4));
        } else {
            raw.s = *reinterpret_cast<const uint16_t *>(sg_at(s, a.pl[1].w, r, u * 2));
        }
    }
    return raw;
}

__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// Task t of the CTA's cost range -> (group, block).  cum[g] = cost of groups < g.
__device__ __forceinline__ void sg_locate(const int *cum, int ng, int bpg, long long pos, int &g, int &b)
{
    int lo = 0, hi = ng;  // largest g with cum[g] * bpg <= pos
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((long long)cum[mid] * bpg <= pos) lo = mid;
        else hi = mid;
    }
    g = lo;
    const long long w = (long long)(cum[lo + 1] - cum[lo]);  // per-block cost of group lo
    b = (int)((pos - (long long)cum[lo] * bpg + w - 1) / w);
    if (b >= bpg) {
        ++g;
        b = 0;
    }
}

template <int FMT>
__global__ void __launch_bounds__(kSgThreads, 1)
    sgm_kernel(const __grid_constant__ CUtensorMap m0, const __grid_constant__ CUtensorMap m1,
               const __grid_constant__ CUtensorMap m2, const SgArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int K = a.K, NU = K >> 5, nc = K >> 2;
    const int NS = a.n_stages;
    const int bpg = a.gateup ? a.rows_out / 16 : a.rows_out / 32;  // blocks per group
    // shared memory: stages | x [8][K] fp32 | xsum [8][NU] | red [2][8 warps][8 tok][32] | cum | bars
    uint8_t *stages = smem;
    float4 *xs4 = reinterpret_cast<float4 *>(smem + (size_t)NS * a.stage_bytes);
    float *xsum = reinterpret_cast<float *>(xs4 + (size_t)kSgTT * nc);
    float *red = xsum + kSgTT * NU;
    int *cum = reinterpret_cast<int *>(red + 2 * kSgConsumers * kSgTT * 32);
    uint64_t *full = reinterpret_cast<uint64_t *>(cum + kSgMaxGroups + 2);
    uint64_t *empty = full + kSgMaxStages;
    __shared__ int s_range[3];  // first group, first block, task count
    __shared__ volatile int s_fail;  // a wait ran out: everyone skips the rest, keeping the barriers

    const int ng = min(*a.n_groups, kSgMaxGroups);
    // cost prefix over groups (every CTA redundantly; ng is at most a few hundred)
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < ng; base += 32) {
            const int g = base + lane;
            const int v = g < ng ? 4 + __ldg(&a.groups[g].z) : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            if (g < ng) cum[g] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            cum[ng] = carry;
            const long long C = (long long)carry * bpg;
            const long long s0 = C * blockIdx.x / gridDim.x, s1 = C * (blockIdx.x + 1) / gridDim.x;
            int g0 = ng, b0 = 0, g1 = ng, b1 = 0;
            if (ng > 0 && s0 < C) sg_locate(cum, ng, bpg, s0, g0, b0);
            if (ng > 0 && s1 < C) sg_locate(cum, ng, bpg, s1, g1, b1);
            s_range[0] = g0;
            s_range[1] = b0;
            s_range[2] = (g1 - g0) * bpg + (b1 - b0);
            s_fail = 0;
            for (int i = 0; i < NS; ++i) {
                mbar_init(full + i, 1);
                mbar_init(empty + i, kSgConsumers);
            }
            fence_mbar_init();
        }
    }
    __syncthreads();
    const int g_first = s_range[0], b_first = s_range[1], ntask = s_range[2];
    if (ntask <= 0) return;

    if (warp == kSgConsumers) {
        // ---- producer ------------------------------------------------------------
        if (lane == 0) {
            prefetch_tmap(&m0);
            prefetch_tmap(&m1);
            if (a.pl[2].row_bytes) prefetch_tmap(&m2);
            int g = g_first, b = b_first, issued = 0;
            for (int i = 0; i < ntask; ++i) {
                const int st = i % NS;
                if (i >= NS && (s_fail || !mbar_wait(empty + st, ((i / NS) - 1) & 1))) {
                    atomicExch(a.err, (int)MOE_ERR_TIMEOUT);
                    s_fail = 1;
                    break;
                }
                const int ex = __ldg(&a.groups[g].x);
                uint8_t *dst = stages + (size_t)st * a.stage_bytes;
                mbar_arrive_expect_tx(full + st, (uint32_t)a.tx_bytes);
                ++issued;
                const CUtensorMap *maps[3] = {&m0, &m1, &m2};
                for (int p = 0; p < 3; ++p) {
                    const SgPlane &pl = a.pl[p];
                    if (!pl.row_bytes) continue;
                    for (int seg = 0; seg < pl.row_bytes / pl.w; ++seg) {
                        uint8_t *d = dst + pl.off + seg * 32 * pl.w;
                        if (a.gateup) {  // 16 gate rows, then the 16 matching up rows
                            tma_load_3d(d, maps[p], full + st, seg * pl.w, b * 16, ex);
                            tma_load_3d(d + 16 * pl.w, maps[p], full + st, seg * pl.w, a.rows_out + b * 16, ex);
                        } else {
                            tma_load_3d(d, maps[p], full + st, seg * pl.w, b * 32, ex);
                        }
                    }
                }
                if (++b == bpg) {
                    b = 0;
                    ++g;
                }
            }
            // after a failure, wait (bounded) for the loads still in flight
            if (s_fail)
                for (int i = max(0, issued - NS); i < issued; ++i) mbar_wait(full + i % NS, (i / NS) & 1);
        }
        return;
    }

    // ---- consumers ---------------------------------------------------------------
    const int cw = warp;  // 0..7
    const int u0 = NU * cw / kSgConsumers, u1 = NU * (cw + 1) / kSgConsumers;
    int g = g_first, b = b_first, cur_g = -1, ntok = 0, slot0 = 0;
    float half_ts = 0.5f;
    for (int i = 0; i < ntask; ++i) {
        const int st = i % NS;
        if (g != cur_g) {  // stage the group's tokens as fp32
            const int4 gd = __ldg(&a.groups[g]);
            slot0 = gd.y;
            ntok = gd.z;
            if (FMT == MOE_FMT_NVFP4) half_ts = 0.5f * __ldg(a.ts + gd.x);
            named_sync(1, 32 * kSgConsumers);  // everyone is done with the previous x
            // four independent loads in flight per thread per round
            const int n4 = s_fail ? 0 : ntok * nc;
            constexpr int CT = 32 * kSgConsumers;
            for (int j0 = threadIdx.x; j0 < n4; j0 += 4 * CT) {
                float4 v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int j = j0 + q * CT;
                    if (j < n4) {
                        const int t = j / nc, c = j - t * nc;
                        if (a.gateup) {
                            const int tok = __ldg(a.perm_tok + slot0 + t);
                            if (a.x_dtype == MOE_DT_BF16) {
                                const uint2 w2 = __ldg(reinterpret_cast<const uint2 *>(
                                    reinterpret_cast<const uint16_t *>(a.x) + (size_t)tok * K + c * 4));
                                v[q] = make_float4(bf16lo(w2.x), bf16hi(w2.x), bf16lo(w2.y), bf16hi(w2.y));
                            } else {
                                v[q] = __ldg(reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.x) +
                                                                              (size_t)tok * K) + c);
                            }
                        } else {
                            v[q] = __ldcg(reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.x) +
                                                                           (size_t)(slot0 + t) * K) + c);
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (j0 + q * CT < n4) xs4[j0 + q * CT] = v[q];
            }
            if (FMT == MOE_FMT_Q5_1) {
                named_sync(1, 32 * kSgConsumers);
                for (int j = threadIdx.x; j < ntok * NU; j += 32 * kSgConsumers) {
                    const float4 *p = xs4 + j * 8;  // unit j % NU of token j / NU
                    float sacc = 0.f;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 v = p[q];
                        sacc += v.x;
                        sacc += v.y;
                        sacc += v.z;
                        sacc += v.w;
                    }
                    xsum[j] = sacc;
                }
            }
            named_sync(1, 32 * kSgConsumers);
            cur_g = g;
        }
        // a failed wait never skips a named barrier: the remaining tasks are
        // walked without work, so every warp keeps the same barrier sequence
        bool ok = !s_fail;
        if (ok && !mbar_wait(full + st, (i / NS) & 1)) {
            atomicExch(a.err, (int)MOE_ERR_TIMEOUT);
            s_fail = 1;
            ok = false;
        }
        const uint8_t *stage = stages + (size_t)st * a.stage_bytes;
        // lane = row of the block; this warp's share of the row's units
        float acc[kSgTT];
#pragma unroll
        for (int t = 0; t < kSgTT; ++t) acc[t] = 0.f;
        if (ok) {
            switch (ntok) {
            case 1: sg_rows<FMT, 1>(a, stage, lane, u0, u1, xs4, xsum, nc, NU, half_ts, acc); break;
            case 2: sg_rows<FMT, 2>(a, stage, lane, u0, u1, xs4, xsum, nc, NU, half_ts, acc); break;
            case 3: sg_rows<FMT, 3>(a, stage, lane, u0, u1, xs4, xsum, nc, NU, half_ts, acc); break;
            case 4: sg_rows<FMT, 4>(a, stage, lane, u0, u1, xs4, xsum, nc, NU, half_ts, acc); break;
            case 5: sg_rows<FMT, 5>(a, stage, lane, u0, u1, xs4, xsum, nc, NU, half_ts, acc); break;
            case 6: sg_rows<FMT, 6>(a, stage, lane, u0, u1, xs4, xsum, nc, NU, half_ts, acc); break;
            case 7: sg_rows<FMT, 7>(a, stage, lane, u0, u1, xs4, xsum, nc, NU, half_ts, acc); break;
            default: sg_rows<FMT, 8>(a, stage, lane, u0, u1, xs4, xsum, nc, NU, half_ts, acc); break;
            }
        }
        // the stage is free once every consumer warp has read it
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + st);
        float *rb = red + (size_t)(i & 1) * kSgConsumers * kSgTT * 32;
#pragma unroll
        for (int t = 0; t < kSgTT; ++t)
            if (t < ntok) rb[(cw * kSgTT + t) * 32 + lane] = acc[t];
        named_sync(2 + (i & 1), 32 * kSgConsumers);
        if (cw < ntok) {  // warp t finishes token t
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kSgConsumers; ++w) v += rb[(w * kSgTT + cw) * 32 + lane];
            const int slot = slot0 + cw;
            if (a.gateup) {
                const float up = __shfl_down_sync(0xffffffffu, v, 16);
                if (lane < 16) a.out[(size_t)slot * a.out_stride + b * 16 + lane] = v / (1.f + expf(-v)) * up;
            } else {
                a.out[(size_t)slot * a.out_stride + b * 32 + lane] = v;
            }
        }
        if (++b == bpg) {
            b = 0;
            ++g;
        }
    }
}

using SgKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const SgArgs);

SgKernel sg_pick(int fmt)
{
    switch (fmt) {
    case MOE_FMT_Q8_0: return sgm_kernel<MOE_FMT_Q8_0>;
    case MOE_FMT_Q5_1: return sgm_kernel<MOE_FMT_Q5_1>;
    case MOE_FMT_IQ4_NL: return sgm_kernel<MOE_FMT_IQ4_NL>;
    default: return sgm_kernel<MOE_FMT_NVFP4>;
    }
}

int sg_box_width(int row_bytes)
{
    if (row_bytes >= 128) return row_bytes % 128 == 0 ? 128 : 0;
    return (row_bytes == 64 || row_bytes == 32 || row_bytes == 16) ? row_bytes : 0;
}

CUtensorMapSwizzle sg_swizzle(int w)
{
    return w == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
           : w == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
           : w == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                     : CU_TENSOR_MAP_SWIZZLE_NONE;
}

bool sg_map(CUtensorMap *m, const uint8_t *base, int slots, int rows, int row_bytes, int64_t stride, int w,
            int box_rows)
{
    tmaps::EncodeTiledFn f = tmaps::encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)rows, (cuuint64_t)slots};
    cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)stride};
    cuuint32_t box[3] = {(cuuint32_t)w, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sg_swizzle(w), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Tensor maps and stage layout of one projection for the streamed grouped matvec.
int sgm_max_groups() { return kSgMaxGroups; }

bool sgm_prepare(const DevProj &w, int n_slots, bool gateup, SgmProj *out)
{
    SgmProj s{};
    const uint8_t *bases[3] = {w.qs, w.sr, w.qh};
    const int rowb[3] = {w.qs_row, w.sr_row, w.qh_row};
    const int64_t strides[3] = {w.qs_stride, w.sr_stride, w.qh_stride};
    int off = 0;
    for (int p = 0; p < 3; ++p) {
        s.row_bytes[p] = rowb[p];
        if (!rowb[p]) continue;
        if (!bases[p]) return false;
        const int bw = sg_box_width(rowb[p]);
        if (!bw || strides[p] % 16) return false;
        s.w[p] = bw;
        s.off[p] = off;
        off += ((32 * rowb[p] + 1023) / 1024) * 1024;  // keep every plane 1024-byte aligned
        if (!sg_map(&s.map[p], bases[p], n_slots, w.rows, rowb[p], strides[p], bw, gateup ? 16 : 32)) return false;
    }
    if (!rowb[2]) s.map[2] = s.map[0];
    s.stage_bytes = off;
    s.tx_bytes = 32 * (rowb[0] + rowb[1] + rowb[2]);
    s.fmt = w.fmt;
    s.ok = 1;
    *out = s;
    return true;
}

size_t sgm_smem_bytes(const SgmProj &p, int K, int n_stages)
{
    const size_t fixed = (size_t)kSgTT * K * 4 + (size_t)kSgTT * (K / 32) * 4 +
                         (size_t)2 * kSgConsumers * kSgTT * 32 * 4 + (size_t)(kSgMaxGroups + 2) * 4 +
                         (size_t)2 * kSgMaxStages * 8;
    return 1024 + (size_t)n_stages * p.stage_bytes + fixed;
}

int sgm_stages(const SgmProj &p, int K)
{
    int ns = kSgMaxStages;
    while (ns >= 2 && sgm_smem_bytes(p, K, ns) > (size_t)kSgSmemLimit) --ns;
    return ns >= 2 ? ns : 0;
}

cudaError_t sgm_set_attributes()
{
    const int fmts[4] = {MOE_FMT_Q8_0, MOE_FMT_Q5_1, MOE_FMT_IQ4_NL, MOE_FMT_NVFP4};
    for (int f : fmts) {
        const cudaError_t e = cudaFuncSetAttribute(sg_pick(f), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   kSgSmemLimit);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_sgm(const SgmProj &p, const DevProj &w, const int4 *groups, const int32_t *n_groups,
                       const int32_t *perm_tok, const void *x, int x_dtype, float *out, int out_stride, int rows_out,
                       bool gateup, const CodeTable &tab, int32_t *err, int grid, cudaStream_t s)
{
    SgArgs a{};
    a.groups = groups;
    a.n_groups = n_groups;
    a.perm_tok = perm_tok;
    a.x = x;
    a.x_dtype = x_dtype;
    a.out = out;
    a.out_stride = out_stride;
    a.K = w.cols;
    a.rows_out = rows_out;
    a.gateup = gateup ? 1 : 0;
    a.fmt = w.fmt;
    a.ts = w.ts;
    a.tab = tab;
    for (int q = 0; q < 3; ++q) a.pl[q] = SgPlane{p.row_bytes[q], p.w[q], p.off[q]};
    a.stage_bytes = p.stage_bytes;
    a.tx_bytes = p.tx_bytes;
    a.n_stages = sgm_stages(p, w.cols);
    a.err = err;
    if (a.n_stages < 2) return cudaErrorInvalidValue;
    sg_pick(w.fmt)<<<grid, kSgThreads, sgm_smem_bytes(p, w.cols, a.n_stages), s>>>(p.map[0], p.map[1], p.map[2], a);
    return cudaGetLastError();
}

}  // namespace moe
