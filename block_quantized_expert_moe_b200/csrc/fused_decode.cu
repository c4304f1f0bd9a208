// The decode layer in one cooperative launch, for batches of at most 8 tokens
// (decode and speculative-verify): router, top-k, plan, grouped gate/up +
// SwiGLU, down and combine, separated by grid-wide barriers instead of kernel
// boundaries.
//
// This is the B200 form of the "device-planned MoE tail + grouped kernels" that
// the "Qwen3.8-Flash-Next UD-IQ2_XS (L4 fix) for Basalt" model card ("What
// was changed") describes: at one to eight tokens the layer reads ~24 MB of
// expert weights, a few microseconds of HBM time, so four kernel launches and
// their dependent prologues would cost more than the bytes.  Phases:
//
//   stage   every CTA converts the T token vectors to fp32 in shared memory
//   P1      router logits; warp w of the grid owns experts w, w + W, ...
//   sync
//   P2      every CTA redoes top-k and the plan for all tokens in its own shared
//           memory (cheap at T <= 8, and it saves a grid barrier): selected
//           experts and gates, per-expert counts and slot offsets, slot order
//           by token (bit masks), one work group per active expert plus the
//           shared expert's group; CTA 0 also writes the routing for readback
//   P3      gate/up + SwiGLU: tasks (group, row pair) split in contiguous
//           ranges over the CTAs; h goes to a workspace row per slot
//   sync
//   P4      rowsplit: each CTA stages every slot's h and owns a range of output
//           rows; for each row it streams the down rows of every active expert
//           and accumulates gate * (D_e h) per token in expert order, so the
//           combine needs no second pass;  otherwise: down rows per slot into
//           y, a barrier, then the combine in j order.
//
// The barriers are sense-reversing arrive/wait counters in global memory; the
// launch is cooperative, so all CTAs are resident, and every wait gives up
// after ~2 s, records MOE_ERR_TIMEOUT and returns.
#include <algorithm>
#include <climits>

#include "decode_common.cuh"
#include "quant_dot.cuh"

namespace moe {

namespace {

using namespace qd;

__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Bulk-prefetch [p, p + bytes) into L2 in 64 KiB pieces, piece i by CTA i mod G.
__device__ void prefetch_span(const uint8_t *p, int64_t bytes, int &turn)
{
    for (int64_t o = 0; o < bytes; o += 65536) {
        if ((turn++ % (int)gridDim.x) == (int)blockIdx.x && threadIdx.x == 0) {
            const int64_t n = (bytes - o < 65536 ? bytes - o : 65536) & ~15ll;
            if (n > 0) prefetch_l2(p + o, (uint32_t)n);
        }
    }
}

struct Plan {
    int *sel_e;        // [T*k] selected experts, descending logit
    float *sel_g;      // [T*k] gates
    int *cnt;          // [E+1]
    int *off;          // [E+1]
    int *gidx;         // [E+1]
    unsigned *mask;    // [E] token bit mask
    int *perm_tok;     // [slots]
    float *slot_gate;  // [slots]
    int *slot_of;      // [T*k]
    int4 *groups;      // [E+1]
    int *scan_tmp;     // [64]
    int *n_groups;     // [1]
};

template <int FT>
__device__ int block_scan_excl(int *v, int n, int *tmp)
{
    // n <= 2 * FT
    constexpr int NW = FT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int a0 = 2 * tid < n ? v[2 * tid] : 0;
    const int a1 = 2 * tid + 1 < n ? v[2 * tid + 1] : 0;
    const int s = a0 + a1;
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < NW ? tmp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += u;
        }
        if (lane < NW) tmp[lane] = wi - w;
        if (lane == NW - 1) tmp[NW] = wi;
    }
    __syncthreads();
    const int base = tmp[warp] + incl - s;
    if (2 * tid < n) v[2 * tid] = base;
    if (2 * tid + 1 < n) v[2 * tid + 1] = base + a0;
    const int total = tmp[NW];
    __syncthreads();
    return total;
}

// ---- stage: the T token vectors as fp32, unit-swizzled like the matvecs ----
template <int FT>
__device__ void stage_tokens(const FusedArgs &a, float4 *xs4, float *xsum, bool want_sums)
{
    const int H = a.H, nc = H >> 2, NU = H >> 5;
    for (int i = threadIdx.x; i < a.T * nc; i += FT) {
        const int t = i / nc, c = i - t * nc;
        float4 v;
        if (a.x_dtype == MOE_DT_BF16) {
            const uint2 b = __ldg(reinterpret_cast<const uint2 *>(reinterpret_cast<const uint16_t *>(a.x) +
                                                                  (size_t)t * H + c * 4));
            v = make_float4(bf16lo(b.x), bf16hi(b.x), bf16lo(b.y), bf16hi(b.y));
        } else {
            v = __ldg(reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.x) + (size_t)t * H + c * 4));
        }
        const int u = c >> 3, j = c & 7;
        xs4[t * nc + u * 8 + (j ^ (u & 7))] = v;
    }
    if (want_sums) {
        __syncthreads();
        for (int i = threadIdx.x; i < a.T * NU; i += FT) {
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

// ---- P1: router logits -------------------------------------------------------
template <int FT, int TT>
__device__ void phase_router(const FusedArgs &a, const float4 *xs4)
{
    constexpr int NW = FT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = a.H, nc = H >> 2, NU = H >> 5;
    const int gw = blockIdx.x * NW + warp, GW = gridDim.x * NW;
    for (int e = gw; e < a.E; e += GW) {
        const uint16_t *row = a.wr + (size_t)e * H;
        float acc[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) acc[t] = 0.f;
        for (int u0 = lane; u0 < NU; u0 += 64) {
            uint4 w[2][4];
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const int u = u0 + 32 * s;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    w[s][q] = u < NU ? ld_stream16(row + u * 32 + q * 8) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const int u = u0 + 32 * s;
                if (u >= NU) break;
                const float4 *xu = xs4 + u * 8;
                const int sw = u & 7;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 v = w[s][q];
#pragma unroll
                    for (int t = 0; t < TT; ++t) {
                        if (t < a.T) {
                            const float4 x0 = xu[t * nc + ((2 * q) ^ sw)];
                            const float4 x1 = xu[t * nc + ((2 * q + 1) ^ sw)];
                            float r = acc[t];
                            r = fmaf(bf16lo(v.x), x0.x, r); r = fmaf(bf16hi(v.x), x0.y, r);
                            r = fmaf(bf16lo(v.y), x0.z, r); r = fmaf(bf16hi(v.y), x0.w, r);
                            r = fmaf(bf16lo(v.z), x1.x, r); r = fmaf(bf16hi(v.z), x1.y, r);
                            r = fmaf(bf16lo(v.w), x1.z, r); r = fmaf(bf16hi(v.w), x1.w, r);
                            acc[t] = r;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            float v = acc[t];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && t < a.T) a.logits[(size_t)t * a.E + e] = v;
        }
    }
}

// ---- P2: top-k and the plan, in this CTA's shared memory ----------------------
template <int FT>
__device__ void phase_plan(const FusedArgs &a, const Plan &pl)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = a.E, k = a.k, T = a.T;
    if (warp < T) warp_topk(a, warp, pl.sel_e, pl.sel_g);
    for (int e = threadIdx.x; e < E; e += FT) {
        pl.cnt[e] = 0;
        pl.mask[e] = 0u;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < T * k; i += FT) {
        const int e = pl.sel_e[i];
        atomicAdd(&pl.cnt[e], 1);
        atomicOr(&pl.mask[e], 1u << (i / k));
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += FT) {
        pl.off[e] = pl.cnt[e];
        pl.gidx[e] = pl.cnt[e] > 0 ? 1 : 0;
    }
    __syncthreads();
    block_scan_excl<FT>(pl.off, E, pl.scan_tmp);
    const int routed = block_scan_excl<FT>(pl.gidx, E, pl.scan_tmp);
    for (int e = threadIdx.x; e < E; e += FT)
        if (pl.cnt[e] > 0) pl.groups[pl.gidx[e]] = make_int4(e, pl.off[e], pl.cnt[e], 0);
    for (int i = threadIdx.x; i < T * k; i += FT) {
        const int t = i / k, e = pl.sel_e[i];
        const int pos = pl.off[e] + __popc(pl.mask[e] & ((1u << t) - 1u));
        pl.perm_tok[pos] = t;
        pl.slot_gate[pos] = pl.sel_g[i];
        pl.slot_of[i] = pos;
    }
    if (threadIdx.x < T && a.has_shared) {
        pl.perm_tok[T * k + threadIdx.x] = threadIdx.x;
        pl.slot_gate[T * k + threadIdx.x] = 1.f;
    }
    if (threadIdx.x == 0) {
        if (a.has_shared) pl.groups[routed] = make_int4(E, T * k, T, 0);
        *pl.n_groups = routed + (a.has_shared ? 1 : 0);
    }
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i < T * k; i += FT) {
            a.idx_out[i] = pl.sel_e[i];
            a.gate_out[i] = pl.sel_g[i];
        }
        for (int e = threadIdx.x; e <= E; e += FT) a.cnt_out[e] = e < E ? pl.cnt[e] : (a.has_shared ? T : 0);
    }
    __syncthreads();
}

// Plan of a single token: the k experts in ascending id order, one slot and one
// group each, the shared expert's group last.  Warp 0 only; no block scans.
template <int FT>
__device__ void phase_plan_t1(const FusedArgs &a, const Plan &pl)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int k = a.k, E = a.E;
    if (warp == 0) {
        warp_topk(a, 0, pl.sel_e, pl.sel_g);
        const int me = lane < k ? pl.sel_e[lane] : INT_MAX;
        int rank = 0;
        for (int i = 0; i < k; ++i) rank += __shfl_sync(0xffffffffu, me, i) < me;
        if (lane < k) {
            pl.groups[rank] = make_int4(me, rank, 1, 0);
            pl.perm_tok[rank] = 0;
            pl.slot_gate[rank] = pl.sel_g[lane];
            pl.slot_of[lane] = rank;
        }
        if (lane == 0) {
            if (a.has_shared) {
                pl.groups[k] = make_int4(E, k, 1, 0);
                pl.perm_tok[k] = 0;
                pl.slot_gate[k] = 1.f;
            }
            *pl.n_groups = k + (a.has_shared ? 1 : 0);
        }
    }
    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e <= E; e += FT) a.cnt_out[e] = e < E ? 0 : (a.has_shared ? 1 : 0);
        __syncthreads();
        if (warp == 0 && lane < k) {
            a.idx_out[lane] = pl.sel_e[lane];
            a.gate_out[lane] = pl.sel_g[lane];
            a.cnt_out[pl.sel_e[lane]] = 1;
        }
    }
    __syncthreads();
}

// ---- P3: gate/up + SwiGLU over (group, row pair) tasks -------------------------
template <int FMT, int FT, int TT>
__device__ void phase_gateup(const FusedArgs &a, const Plan &pl, const float4 *xs4, const float *xsum)
{
    constexpr int NW = FT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const DevProj &w = a.gu;
    const int K = a.H, nc = K >> 2, NU = K >> 5;
    const int LPR = lanes_per_row(NU), RPW = 32 / LPR;
    const int sub = lane / LPR, sl = lane - sub * LPR;
    const int rows = a.I;
    const int tpg = (rows + RPW - 1) / RPW;
    const int ng = *pl.n_groups;
    const long long total = (long long)ng * tpg;
    const long long t0 = total * blockIdx.x / gridDim.x, t1 = total * (blockIdx.x + 1) / gridDim.x;
    if constexpr (TT == 1) {
        if (NU <= 2 * LPR) {  // one token: this lane's x units live in registers for every task
            const int u = sl, u2 = sl + LPR;
            const bool has2 = u2 < NU;
            float4 xr0[8], xr1[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                xr0[j] = u < NU ? xs4[u * 8 + (j ^ (u & 7))] : make_float4(0.f, 0.f, 0.f, 0.f);
                xr1[j] = has2 ? xs4[u2 * 8 + (j ^ (u2 & 7))] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            const float xs0 = FMT == MOE_FMT_Q5_1 && u < NU ? xsum[u] : 0.f;
            const float xs1 = FMT == MOE_FMT_Q5_1 && has2 ? xsum[u2] : 0.f;
            // one task of look-ahead: the next task's code loads are in flight
            // while this one is decoded
            auto task_of = [&](long long tk, int &e, int &rr, int &r, int &slot0) {
                const int g = (int)(tk / tpg);
                r = (int)(tk - (long long)g * tpg) * RPW + sub;
                rr = r < rows ? r : rows - 1;
                const int4 gd = pl.groups[g];
                e = gd.x;
                slot0 = gd.y;
            };
            Raw c0, c1, c2, c3;  // gate u, up u, gate u2, up u2 of the current task
            int ce = 0, crr = 0, cr = rows, cslot = 0;
            long long tk = t0 + warp;
            if (tk < t1) {
                task_of(tk, ce, crr, cr, cslot);
                if (u < NU) {
                    c0 = load_unit<FMT>(w, ce, crr, u);
                    c1 = load_unit<FMT>(w, ce, rows + crr, u);
                    if (has2) {
                        c2 = load_unit<FMT>(w, ce, crr, u2);
                        c3 = load_unit<FMT>(w, ce, rows + crr, u2);
                    }
                }
            }
            for (; tk < t1; tk += NW) {
                const long long tn = tk + NW;
                Raw n0, n1, n2, n3;
                int ne = 0, nrr = 0, nr = rows, nslot = 0;
                if (tn < t1) {
                    task_of(tn, ne, nrr, nr, nslot);
                    if (u < NU) {
                        n0 = load_unit<FMT>(w, ne, nrr, u);
                        n1 = load_unit<FMT>(w, ne, rows + nrr, u);
                        if (has2) {
                            n2 = load_unit<FMT>(w, ne, nrr, u2);
                            n3 = load_unit<FMT>(w, ne, rows + nrr, u2);
                        }
                    }
                }
                const float half_ts = FMT == MOE_FMT_NVFP4 ? 0.5f * __ldg(w.ts + ce) : 0.5f;
                float s0 = 0.f, s1 = 0.f;
                if (u < NU) {
                    s0 = unit_dot_reg<FMT>(c0, xr0, xs0, a.tab_gu, half_ts, s0);
                    s1 = unit_dot_reg<FMT>(c1, xr0, xs0, a.tab_gu, half_ts, s1);
                    if (has2) {
                        s0 = unit_dot_reg<FMT>(c2, xr1, xs1, a.tab_gu, half_ts, s0);
                        s1 = unit_dot_reg<FMT>(c3, xr1, xs1, a.tab_gu, half_ts, s1);
                    }
                }
                for (int o = LPR >> 1; o >= 1; o >>= 1) {
                    s0 += __shfl_xor_sync(0xffffffffu, s0, o);
                    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
                }
                if (cr < rows && sl == 0) a.h[(size_t)cslot * a.I + cr] = s0 / (1.f + expf(-s0)) * s1;
                c0 = n0;
                c1 = n1;
                c2 = n2;
                c3 = n3;
                ce = ne;
                crr = nrr;
                cr = nr;
                cslot = nslot;
            }
            return;
        }
    }
    for (long long tk = t0 + warp; tk < t1; tk += NW) {
        const int g = (int)(tk / tpg);
        const int r = (int)(tk - (long long)g * tpg) * RPW + sub;
        const bool valid = r < rows;
        const int rr = valid ? r : rows - 1;
        const int4 gd = pl.groups[g];
        const int e = gd.x, slot0 = gd.y, ntok = gd.z;
        int xoff[TT], xsoff[TT];
        float acc0[TT], acc1[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            const int tok = t < ntok ? pl.perm_tok[slot0 + t] : 0;
            xoff[t] = tok * nc;
            xsoff[t] = tok * NU;
            acc0[t] = 0.f;
            acc1[t] = 0.f;
        }
        const float half_ts = FMT == MOE_FMT_NVFP4 ? 0.5f * __ldg(w.ts + e) : 0.5f;
        for (int u = sl; u < NU; u += 2 * LPR) {
            const int u2 = u + LPR;
            const bool has2 = u2 < NU;
            const Raw g0 = load_unit<FMT>(w, e, rr, u);
            const Raw v0 = load_unit<FMT>(w, e, rows + rr, u);
            Raw g1 = g0, v1 = v0;
            if (has2) {
                g1 = load_unit<FMT>(w, e, rr, u2);
                v1 = load_unit<FMT>(w, e, rows + rr, u2);
            }
            unit_dot<FMT, TT>(g0, u, xs4, xsum, xoff, xsoff, ntok, a.tab_gu, half_ts, acc0);
            unit_dot<FMT, TT>(v0, u, xs4, xsum, xoff, xsoff, ntok, a.tab_gu, half_ts, acc1);
            if (has2) {
                unit_dot<FMT, TT>(g1, u2, xs4, xsum, xoff, xsoff, ntok, a.tab_gu, half_ts, acc0);
                unit_dot<FMT, TT>(v1, u2, xs4, xsum, xoff, xsoff, ntok, a.tab_gu, half_ts, acc1);
            }
        }
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            float s0 = acc0[t], s1 = acc1[t];
            for (int o = LPR >> 1; o >= 1; o >>= 1) {
                s0 += __shfl_xor_sync(0xffffffffu, s0, o);
                s1 += __shfl_xor_sync(0xffffffffu, s1, o);
            }
            if (valid && t < ntok && (t % LPR) == sl)
                a.h[(size_t)(slot0 + t) * a.I + r] = s0 / (1.f + expf(-s0)) * s1;
        }
    }
}

// ---- P4 (rowsplit): down rows of every active expert, gated, per output row ----
template <int FMT, int FT, int TT>
__device__ void phase_down_rows(const FusedArgs &a, const Plan &pl, float4 *hs4, float *hsum)
{
    constexpr int NW = FT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const DevProj &w = a.dn;
    const int K = a.I, nc = K >> 2, NU = K >> 5;
    const int ng = *pl.n_groups;
    const int slots = a.T * a.k + (a.has_shared ? a.T : 0);
    for (int i = threadIdx.x; i < slots * nc; i += FT) {
        const int s = i / nc, c = i - s * nc;
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.h + (size_t)s * K) + c);
        const int u = c >> 3, j = c & 7;
        hs4[s * nc + u * 8 + (j ^ (u & 7))] = v;
    }
    if (FMT == MOE_FMT_Q5_1) {
        __syncthreads();
        for (int i = threadIdx.x; i < slots * NU; i += FT) {
            const int s = i / NU, u = i - s * NU;
            const float4 *p = hs4 + s * nc + u * 8;
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 q = p[j];
                acc += q.x;
                acc += q.y;
                acc += q.z;
                acc += q.w;
            }
            hsum[s * NU + u] = acc;
        }
    }
    __syncthreads();
    const int LPR = lanes_per_row(NU), RPW = 32 / LPR;
    const int sub = lane / LPR, sl = lane - sub * LPR;
    const int rows = a.H;
    const int ntask = (rows + RPW - 1) / RPW;
    const int t0 = (int)((long long)ntask * blockIdx.x / gridDim.x);
    const int t1 = (int)((long long)ntask * (blockIdx.x + 1) / gridDim.x);
    for (int tk = t0 + warp; tk < t1; tk += NW) {
        const int r = tk * RPW + sub;
        const bool valid = r < rows;
        const int rr = valid ? r : rows - 1;
        float acc[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) acc[t] = 0.f;
        // GB groups at a time: their code loads are issued together
        constexpr int GB = 4;
        for (int g0 = 0; g0 < ng; g0 += GB) {
            for (int u = sl; u < NU; u += LPR) {
                Raw d[GB];
#pragma unroll
                for (int b = 0; b < GB; ++b)
                    if (g0 + b < ng) d[b] = load_unit<FMT>(w, pl.groups[g0 + b].x, rr, u);
#pragma unroll
                for (int b = 0; b < GB; ++b) {
                    if (g0 + b >= ng) break;
                    const int4 gd = pl.groups[g0 + b];
                    const int e = gd.x, slot0 = gd.y, ntok = gd.z;
                    const float half_ts = FMT == MOE_FMT_NVFP4 ? 0.5f * __ldg(w.ts + e) : 0.5f;
                    int xoff[TT], xsoff[TT];
                    float part[TT];
#pragma unroll
                    for (int t = 0; t < TT; ++t) {
                        xoff[t] = (slot0 + t) * nc;
                        xsoff[t] = (slot0 + t) * NU;
                        part[t] = 0.f;
                    }
                    unit_dot<FMT, TT>(d[b], u, hs4, hsum, xoff, xsoff, ntok, a.tab_dn, half_ts, part);
#pragma unroll
                    for (int t = 0; t < TT; ++t) {
                        if (t < ntok) {
                            const int tok = pl.perm_tok[slot0 + t];
                            const float gsl = pl.slot_gate[slot0 + t];
#pragma unroll
                            for (int q = 0; q < TT; ++q)
                                if (q == tok) acc[q] = fmaf(gsl, part[t], acc[q]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            float s = acc[t];
            for (int o = LPR >> 1; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (valid && t < a.T && (t % LPR) == sl) a.out[(size_t)t * a.H + r] = s;
        }
    }
}

// ---- P4 (slots): down rows per slot into y ---------------------------------------
template <int FMT, int FT, int TT>
__device__ void phase_down_slots(const FusedArgs &a, const Plan &pl, float4 *hs4, float *hsum)
{
    constexpr int NW = FT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const DevProj &w = a.dn;
    const int K = a.I, nc = K >> 2, NU = K >> 5;
    const int LPR = lanes_per_row(NU), RPW = 32 / LPR;
    const int sub = lane / LPR, sl = lane - sub * LPR;
    const int rows = a.H;
    const int tpg = (rows + RPW - 1) / RPW;
    const int ng = *pl.n_groups;
    const long long total = (long long)ng * tpg;
    long long task = total * blockIdx.x / gridDim.x;
    const long long tend = total * (blockIdx.x + 1) / gridDim.x;
    while (task < tend) {
        const int g = (int)(task / tpg);
        const long long gend = min(tend, (long long)(g + 1) * tpg);
        const int4 gd = pl.groups[g];
        const int e = gd.x, slot0 = gd.y, ntok = gd.z;
        __syncthreads();
        for (int i = threadIdx.x; i < ntok * nc; i += FT) {
            const int t = i / nc, c = i - t * nc;
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.h + (size_t)(slot0 + t) * K) + c);
            const int u = c >> 3, j = c & 7;
            hs4[t * nc + u * 8 + (j ^ (u & 7))] = v;
        }
        if (FMT == MOE_FMT_Q5_1) {
            __syncthreads();
            for (int i = threadIdx.x; i < ntok * NU; i += FT) {
                const int t = i / NU, u = i - t * NU;
                const float4 *p = hs4 + t * nc + u * 8;
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 q = p[j];
                    acc += q.x;
                    acc += q.y;
                    acc += q.z;
                    acc += q.w;
                }
                hsum[t * NU + u] = acc;
            }
        }
        __syncthreads();
        const float half_ts = FMT == MOE_FMT_NVFP4 ? 0.5f * __ldg(w.ts + e) : 0.5f;
        for (long long tk = task + warp; tk < gend; tk += NW) {
            const int r = (int)(tk - (long long)g * tpg) * RPW + sub;
            const bool valid = r < rows;
            const int rr = valid ? r : rows - 1;
            int xoff[TT], xsoff[TT];
            float acc[TT];
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                xoff[t] = t * nc;
                xsoff[t] = t * NU;
                acc[t] = 0.f;
            }
            for (int u = sl; u < NU; u += LPR) {
                const Raw d0 = load_unit<FMT>(w, e, rr, u);
                unit_dot<FMT, TT>(d0, u, hs4, hsum, xoff, xsoff, ntok, a.tab_dn, half_ts, acc);
            }
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                float s = acc[t];
                for (int o = LPR >> 1; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                if (valid && t < ntok && (t % LPR) == sl) a.y[(size_t)(slot0 + t) * a.H + r] = s;
            }
        }
        task = gend;
    }
}

// ---- P5 (slots mode): out[t] = sum_j g_j y[slot(t,j)] (+ y_shared) ------------------
template <int FT>
__device__ void phase_combine(const FusedArgs &a, const Plan &pl)
{
    const int H4 = a.H >> 2;
    const int n = a.T * H4;
    for (int i = blockIdx.x * FT + threadIdx.x; i < n; i += gridDim.x * FT) {
        const int t = i / H4, c = i - t * H4;
        float4 v[kFusedMaxK + 1];
        float g[kFusedMaxK + 1];
#pragma unroll
        for (int j = 0; j < kFusedMaxK; ++j) {
            if (j < a.k) {
                const int s = pl.slot_of[t * a.k + j];
                g[j] = pl.sel_g[t * a.k + j];
                v[j] = __ldcg(reinterpret_cast<const float4 *>(a.y + (size_t)s * a.H) + c);
            }
        }
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < kFusedMaxK; ++j) {
            if (j < a.k) {
                acc.x = fmaf(g[j], v[j].x, acc.x);
                acc.y = fmaf(g[j], v[j].y, acc.y);
                acc.z = fmaf(g[j], v[j].z, acc.z);
                acc.w = fmaf(g[j], v[j].w, acc.w);
            }
        }
        if (a.has_shared) {
            const float4 s = __ldcg(reinterpret_cast<const float4 *>(a.y + (size_t)(a.T * a.k + t) * a.H) + c);
            acc.x += s.x;
            acc.y += s.y;
            acc.z += s.z;
            acc.w += s.w;
        }
        reinterpret_cast<float4 *>(a.out + (size_t)t * a.H)[c] = acc;
    }
}

// ---- shared-memory layout (host and device agree on it) -------------------------
struct FusedLayout {
    size_t xs, xsum, sel_e, sel_g, cnt, off, gidx, mask, perm, sgate, slot_of, groups, scan, ng, hs, hsum,
        total;
};

__host__ __device__ inline size_t align16(size_t v) { return (v + 15) & ~(size_t)15; }

__host__ __device__ inline FusedLayout fused_layout(int T, int H, int I, int E, int k, int has_shared,
                                                    int rowsplit, int tt)
{
    FusedLayout L;
    const size_t slots = (size_t)T * k + (has_shared ? T : 0);
    size_t o = 0;
    L.xs = o;      o = align16(o + (size_t)T * H * 4);
    L.xsum = o;    o = align16(o + (size_t)T * (H / 32) * 4);
    L.sel_e = o;   o = align16(o + (size_t)T * k * 4);
    L.sel_g = o;   o = align16(o + (size_t)T * k * 4);
    L.cnt = o;     o = align16(o + (size_t)(E + 1) * 4);
    L.off = o;     o = align16(o + (size_t)(E + 1) * 4);
    L.gidx = o;    o = align16(o + (size_t)(E + 1) * 4);
    L.mask = o;    o = align16(o + (size_t)E * 4);
    L.perm = o;    o = align16(o + slots * 4);
    L.sgate = o;   o = align16(o + slots * 4);
    L.slot_of = o; o = align16(o + (size_t)T * k * 4);
    L.groups = o;  o = align16(o + (size_t)(E + 2) * 16);
    L.scan = o;    o = align16(o + 64 * 4);
    L.ng = o;      o = align16(o + 16);
    const size_t hrows = rowsplit ? slots : (size_t)tt;
    L.hs = o;      o = align16(o + hrows * I * 4);
    L.hsum = o;    o = align16(o + hrows * (I / 32) * 4);
    L.total = o;
    return L;
}

template <int FMT, int FT, int TT>
__device__ __forceinline__ void run_gateup(const FusedArgs &a, const Plan &pl, const float4 *xs4, const float *xsum)
{
    phase_gateup<FMT, FT, TT>(a, pl, xs4, xsum);
}

template <int FT, int TT>
__global__ void __launch_bounds__(FT, 1) fused_decode_kernel(const FusedArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const FusedLayout L = fused_layout(a.T, a.H, a.I, a.E, a.k, a.has_shared, a.rowsplit, TT);
    float4 *xs4 = reinterpret_cast<float4 *>(smem + L.xs);
    float *xsum = reinterpret_cast<float *>(smem + L.xsum);
    float4 *hs4 = reinterpret_cast<float4 *>(smem + L.hs);
    float *hsum = reinterpret_cast<float *>(smem + L.hsum);
    Plan pl;
    pl.sel_e = reinterpret_cast<int *>(smem + L.sel_e);
    pl.sel_g = reinterpret_cast<float *>(smem + L.sel_g);
    pl.cnt = reinterpret_cast<int *>(smem + L.cnt);
    pl.off = reinterpret_cast<int *>(smem + L.off);
    pl.gidx = reinterpret_cast<int *>(smem + L.gidx);
    pl.mask = reinterpret_cast<unsigned *>(smem + L.mask);
    pl.perm_tok = reinterpret_cast<int *>(smem + L.perm);
    pl.slot_gate = reinterpret_cast<float *>(smem + L.sgate);
    pl.slot_of = reinterpret_cast<int *>(smem + L.slot_of);
    pl.groups = reinterpret_cast<int4 *>(smem + L.groups);
    pl.scan_tmp = reinterpret_cast<int *>(smem + L.scan);
    pl.n_groups = reinterpret_cast<int *>(smem + L.ng);

    if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[0] = clock64();
    // the shared expert's weights do not depend on routing: start them into L2
    if (a.has_shared) {
        int turn = 0;
        const DevProj &g = a.gu, &d = a.dn;
        const int S = a.E;
        prefetch_span(g.qs + (int64_t)S * g.qs_stride, (int64_t)g.rows * g.qs_row, turn);
        prefetch_span(g.sc + (int64_t)S * g.sc_stride, g.sc_stride, turn);
        if (g.qh_row) prefetch_span(g.qh + (int64_t)S * g.qh_stride, (int64_t)g.rows * g.qh_row, turn);
        prefetch_span(d.qs + (int64_t)S * d.qs_stride, (int64_t)d.rows * d.qs_row, turn);
        prefetch_span(d.sc + (int64_t)S * d.sc_stride, d.sc_stride, turn);
        if (d.qh_row) prefetch_span(d.qh + (int64_t)S * d.qh_stride, (int64_t)d.rows * d.qh_row, turn);
    }
    stage_tokens<FT>(a, xs4, xsum, a.gu.fmt == MOE_FMT_Q5_1);
    __syncthreads();
    if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[1] = clock64();
    phase_router<FT, TT>(a, xs4);
    if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[2] = clock64();
    if (!grid_sync(a.bar, a.err)) return;
    if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[3] = clock64();
    if (a.T == 1) phase_plan_t1<FT>(a, pl);
    else phase_plan<FT>(a, pl);
    if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[4] = clock64();

    if (a.rowsplit) {  // start this CTA's down rows into L2 while gate/up runs
        const int NU = a.I >> 5;
        const int LPR = lanes_per_row(NU), RPW = 32 / LPR;
        const int ntask = (a.H + RPW - 1) / RPW;
        const int r0 = (int)((long long)ntask * blockIdx.x / gridDim.x) * RPW;
        const int r1 = min(a.H, (int)((long long)ntask * (blockIdx.x + 1) / gridDim.x) * RPW);
        const DevProj &d = a.dn;
        const int ng = *pl.n_groups;
        if (r1 > r0) {
            for (int i = threadIdx.x; i < ng * 3; i += FT) {
                const int e = pl.groups[i / 3].x, which = i % 3;
                if (which == 0)
                    prefetch_l2(d.qs + (int64_t)e * d.qs_stride + (int64_t)r0 * d.qs_row, (uint32_t)((r1 - r0) * d.qs_row));
                else if (which == 1 && ((r1 - r0) * d.sc_row) % 16 == 0 && (r0 * d.sc_row) % 16 == 0)
                    prefetch_l2(d.sc + (int64_t)e * d.sc_stride + (int64_t)r0 * d.sc_row, (uint32_t)((r1 - r0) * d.sc_row));
                else if (which == 2 && d.qh_row && ((r1 - r0) * d.qh_row) % 16 == 0 && (r0 * d.qh_row) % 16 == 0)
                    prefetch_l2(d.qh + (int64_t)e * d.qh_stride + (int64_t)r0 * d.qh_row, (uint32_t)((r1 - r0) * d.qh_row));
            }
        }
    }

    switch (a.gu.fmt) {
    case MOE_FMT_Q8_0: run_gateup<MOE_FMT_Q8_0, FT, TT>(a, pl, xs4, xsum); break;
    case MOE_FMT_Q5_1: run_gateup<MOE_FMT_Q5_1, FT, TT>(a, pl, xs4, xsum); break;
    case MOE_FMT_IQ4_NL: run_gateup<MOE_FMT_IQ4_NL, FT, TT>(a, pl, xs4, xsum); break;
    default: run_gateup<MOE_FMT_NVFP4, FT, TT>(a, pl, xs4, xsum); break;
    }
    if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[5] = clock64();
    if (!grid_sync(a.bar, a.err)) return;
    if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[6] = clock64();
    if (a.rowsplit) {
        switch (a.dn.fmt) {
        case MOE_FMT_Q8_0: phase_down_rows<MOE_FMT_Q8_0, FT, TT>(a, pl, hs4, hsum); break;
        case MOE_FMT_Q5_1: phase_down_rows<MOE_FMT_Q5_1, FT, TT>(a, pl, hs4, hsum); break;
        case MOE_FMT_IQ4_NL: phase_down_rows<MOE_FMT_IQ4_NL, FT, TT>(a, pl, hs4, hsum); break;
        default: phase_down_rows<MOE_FMT_NVFP4, FT, TT>(a, pl, hs4, hsum); break;
        }
    if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[7] = clock64();
    } else {
        switch (a.dn.fmt) {
        case MOE_FMT_Q8_0: phase_down_slots<MOE_FMT_Q8_0, FT, TT>(a, pl, hs4, hsum); break;
        case MOE_FMT_Q5_1: phase_down_slots<MOE_FMT_Q5_1, FT, TT>(a, pl, hs4, hsum); break;
        case MOE_FMT_IQ4_NL: phase_down_slots<MOE_FMT_IQ4_NL, FT, TT>(a, pl, hs4, hsum); break;
        default: phase_down_slots<MOE_FMT_NVFP4, FT, TT>(a, pl, hs4, hsum); break;
        }
        if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[7] = clock64();
        if (!grid_sync(a.bar, a.err)) return;
        if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[8] = clock64();
        phase_combine<FT>(a, pl);
    }
    if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[9] = clock64();
}

constexpr int kFT1 = 384;  // threads per CTA, one-token kernel
constexpr int kFT8 = 256;  // threads per CTA, up-to-8-token kernel

}  // namespace

size_t fused_smem_bytes(const FusedArgs &a, int tt, int rowsplit)
{
    return fused_layout(a.T, a.H, a.I, a.E, a.k, a.has_shared, rowsplit, tt).total;
}

cudaError_t fused_set_attributes()
{
    cudaError_t e = cudaFuncSetAttribute(fused_decode_kernel<kFT1, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         220 * 1024);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(fused_decode_kernel<kFT8, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                220 * 1024);
}

int fused_grid(int tt, size_t smem, int num_sms)
{
    int per_sm = 0;
    cudaError_t e = tt == 1 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused_decode_kernel<kFT1, 1>, kFT1, smem)
                            : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused_decode_kernel<kFT8, 8>, kFT8, smem);
    if (e != cudaSuccess || per_sm < 1) return 0;
    return std::min(per_sm, 2) * num_sms;
}

cudaError_t launch_fused(const FusedArgs &a, int tt, int grid, size_t smem, cudaStream_t s)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(tt == 1 ? kFT1 : kFT8);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (tt == 1) return cudaLaunchKernelEx(&cfg, fused_decode_kernel<kFT1, 1>, a);
    return cudaLaunchKernelEx(&cfg, fused_decode_kernel<kFT8, 8>, a);
}

}  // namespace moe
