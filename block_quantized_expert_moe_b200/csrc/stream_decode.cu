// The single-token decode layer in one launch, fed by bulk asynchronous copies.
//
// The "Qwen3.8-Flash-Next UD-IQ2_XS (L4 fix) for Basalt" model card ("What was
// changed") plans the MoE tail on the device and runs grouped expert kernels.
// At one token that tail reads ~24 MB (router, ten routed experts, the shared
// expert): a few microseconds of HBM time, split by three data dependences
// (x -> every expert's logit -> top-k -> every selected expert's h -> out).
// Time goes to latency, so this kernel splits the work statically over one CTA
// per SM and has every CTA put all of its weight bytes in flight as soon as
// their addresses are known: cp.async.bulk copies into its own shared memory,
// each item completing on its own mbarrier.
//
//   prologue  this CTA's router rows, and its share of the shared expert
//             (gate/up row pairs and down rows), which do not depend on the
//             routing; issued before waiting on the previous kernel of the
//             stream (programmatic dependent launch), so they overlap its tail
//   router    logits of this CTA's rows -> global; hand-over
//   top-k     every CTA's warp 0 selects the k experts from all logits; then
//             each warp issues some of the routed experts' copies (gate/up row
//             pairs and down rows)
//   gate/up   h = silu(G x) * (U x) for this CTA's row pairs as their chunk
//             lands; h -> global, written in the unit-swizzled order the down
//             phase reads; hand-over
//   down      this CTA owns a range of output rows; every group's down rows
//             for them are already in shared memory (they streamed in during
//             gate/up): out[r] = sum_g gate_g (D_g h_g)[r], in fixed group order
//
// A hand-over is a grid-wide counter barrier (each CTA arrives with one
// release-add; one thread per CTA polls) followed by one bulk copy of the whole
// buffer into shared memory.  Measured on B200, polling the published words
// from every warp of the grid costs more than this: 148 SMs reading the same
// few lines through L2 contend for them.  The last CTA to finish resets the
// counters for the next launch.
//
// Groups: the k routed experts in selection order (descending logit), then the
// shared expert, so the combine sums them in the order of the layer's
// definition.  Row pair p of the concatenated gate/up space [0, ng * I)
// belongs to CTA floor(p * G / (ng * I)); the shared expert's pairs are known
// before routing.  A CTA's range is cut into chunks (at most ~8, split at
// group boundaries), each landing on its own mbarrier.
//
// Code that runs once per launch pays for its instruction fetches, so the
// per-unit work is written as small loops rather than unrolled bodies.
//
// Every wait is bounded: a barrier or an mbarrier that does not complete within
// ~1 s records MOE_ERR_TIMEOUT in the workspace's error word, and the CTA waits
// (again bounded) for the copies it issued before it returns.
#include "decode_common.cuh"
#include "quant_dot.cuh"
#include "tc_common.cuh"

namespace moe {

namespace {

using namespace qd;
using tc::mbar_arrive_expect_tx;
using tc::mbar_init;
using tc::mbar_wait;
using tc::smem_u32;

constexpr int kS1Threads = 512;
constexpr int kS1Warps = kS1Threads / 32;
constexpr int kS1MaxSeg = 12;  // gate/up chunks per CTA
constexpr int kS1SmemLimit = 225 * 1024;  // dynamic; the kernel's static shared memory comes on top
constexpr int kS1MaxGroups = kFusedMaxK + 1;
constexpr int kS1BarRouter = 0;
constexpr int kS1BarSeg = 1;                      // + segment
constexpr int kS1BarDown = kS1BarSeg + kS1MaxSeg;  // + group
constexpr int kS1BarLogits = kS1BarDown + kS1MaxGroups;  // grid hand-overs
constexpr int kS1BarH = kS1BarLogits + 1;
constexpr int kS1NumBars = kS1BarH + 1;  // 32: one bit each in the armed mask
constexpr long long kS1PollLimit = 1ll << 31;     // clocks

__host__ __device__ inline size_t s1_al16(size_t v) { return (v + 15) & ~(size_t)15; }
__host__ __device__ inline int s1_cdiv(int a, int b) { return (a + b - 1) / b; }  // 32-bit: shapes are small

// Shared-memory layout; host and device compute it from the same arguments.
struct S1Layout {
    int ng;       // groups: k routed + shared
    int rr;       // router rows per CTA (at most)
    int gp;       // gate/up row pairs per CTA (at most)
    int dr;       // down (output) rows per CTA (at most)
    int gu_pair;  // bytes of one gate/up row pair: gate and up rows of every plane
    int dn_row;   // bytes of one down row
    size_t bars, meta, x, xsum, gu, dn, part, h, hsum, total;
};

__host__ __device__ inline S1Layout s1_layout(const FusedArgs &a, int G)
{
    S1Layout L;
    L.ng = a.k + (a.has_shared ? 1 : 0);
    L.rr = s1_cdiv(a.E, G);
    L.gp = s1_cdiv(L.ng * a.I, G);
    L.dr = s1_cdiv(a.H, G);
    L.gu_pair = 2 * (a.gu.qs_row + a.gu.sr_row + a.gu.qh_row);
    L.dn_row = a.dn.qs_row + a.dn.sr_row + a.dn.qh_row;
    size_t o = 0;
    L.bars = o;  o = s1_al16(o + kS1NumBars * 8);
    L.meta = o;  o = s1_al16(o + 4 * (2 * kS1MaxGroups + 8 + 2 * 32 + 2 * 32) + sizeof(int) * 5 * kS1MaxSeg + 512 + 512);
    L.x = o;     o = s1_al16(o + (size_t)a.H * 4);
    L.xsum = o;  o = s1_al16(o + (size_t)(a.H / 32) * 4);
    L.gu = o;    o = s1_al16(o + (size_t)L.gp * L.gu_pair);
    L.dn = o;    o = s1_al16(o + (size_t)L.ng * L.dr * L.dn_row);
    L.part = o;  o = s1_al16(o + (size_t)L.ng * L.dr * 4);
    // h is staged after gate/up, in the space of the router rows
    L.h = o;
    size_t hb = s1_al16((size_t)L.ng * a.I * 4);
    L.hsum = o + hb;
    hb += s1_al16((size_t)L.ng * (a.I / 32) * 4);
    size_t rb = s1_al16((size_t)L.rr * a.H * 2);  // router rows, then the logits
    if (s1_al16((size_t)a.E * 4) > rb) rb = s1_al16((size_t)a.E * 4);
    o += hb > rb ? hb : rb;
    L.total = o;
    return L;
}

// A chunk of this CTA's gate/up row pairs: one expert, at most `chp` pairs,
// landing on its own mbarrier so compute starts with the first chunk.
struct Seg {
    int g;     // group
    int a;     // first row pair within the expert
    int n;     // row pairs
    int q0;    // first pair within this CTA's range
    int off;   // byte offset in the gate/up region
};

// Pairs per chunk: the CTA's range in at most 8 pieces (plus group boundaries).
__host__ __device__ inline int s1_chunk_pairs(int gp) { return gp / 8 + 1 > 4 ? gp / 8 + 1 : 4; }

__device__ __forceinline__ int s1_segments(int p0, int p1, int I, int pair_bytes, int chp, Seg *seg)
{
    int ns = 0, off = 0;
    for (int p = p0; p < p1 && ns < kS1MaxSeg;) {
        const int g = p / I, a = p - g * I;
        const int n = min(min(p1 - p, I - a), chp);
        seg[ns] = Seg{g, a, n, p - p0, off};
        ++ns;
        off += n * pair_bytes;
        p += n;
    }
    return ns;
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Profiling only: global-timer time of grid event ev (0 start, 1 router rows
// published, 2 routed copies issued, 3 gate/up done, 4 end) folded into the
// first/last pair of the forward's stamps.
__device__ __forceinline__ void grid_event(long long *st, int ev)
{
    if (!st || threadIdx.x != 0) return;
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    atomicMax(st + 10 + 2 * ev, (1ll << 62) - (long long)t);
    atomicMax(st + 11 + 2 * ev, (long long)t);
}

// Grid hand-over of a buffer every CTA has written its part of: the CTA
// arrives on counter `cnt`; thread 0 waits (bounded) until all G have, then
// copies the whole buffer into shared memory with one bulk copy, which every
// thread waits for.  One poller per CTA and one copy request stream keep the
// L2 lines of the buffer from being hammered by every warp of the grid.
__device__ __forceinline__ bool s1_exchange(unsigned *cnt, const void *src, void *dst, uint32_t bytes, uint64_t *bar, int32_t *err,
                            int *flags, int armbit)
{
    __syncthreads();  // this CTA's part is written
    if (threadIdx.x == 0) {
        __threadfence();
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(cnt) : "memory");
        const long long t0 = clock64();
        unsigned v;
        bool ok = true;
        for (;;) {
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
            if (v >= gridDim.x) break;
            if (clock64() - t0 > kS1PollLimit) {
                ok = false;
                break;
            }
        }
        if (ok) {
            asm volatile("fence.proxy.async.global;" ::: "memory");  // generic writes before the async-proxy read
            mbar_arrive_expect_tx(bar, bytes);
            bulk_g2s(dst, src, bytes, bar);
            atomicOr(flags + 1, (int)(1u << armbit));
        } else {
            atomicExch(err, (int)MOE_ERR_TIMEOUT);
            flags[0] = 1;
            tc::mbar_arrive(bar);  // release the waiters without data
        }
    }
    if (mbar_wait(bar, 0)) return flags[0] == 0;
    atomicExch(err, (int)MOE_ERR_TIMEOUT);
    flags[0] = 1;
    return false;
}

// Where the copies read from: both projections' planes, gathered once per CTA
// into shared memory so the (not inlined) issuing code takes one pointer.
struct S1Src {
    const uint8_t *q[2], *s[2], *h[2];  // [0] gate/up, [1] down
    int64_t qstr[2], sstr[2], hstr[2];  // bytes per expert
    int qrow[2], srow[2], hrow[2];      // bytes per row
    int I;
};

// Rows [r, r + n) of gate and of up (rows I + r ...) of expert ex, every plane,
// into dst as [gate qs][up qs][gate scales][up scales][gate qh][up qh].
__device__ __forceinline__ void issue_gateup(const S1Src *c, uint8_t *dst, int ex, int r, int n, int pair_bytes,
                                             uint64_t *bar)
{
    mbar_arrive_expect_tx(bar, (uint32_t)(n * pair_bytes));
    const uint8_t *qs = c->q[0] + (int64_t)ex * c->qstr[0], *sr = c->s[0] + (int64_t)ex * c->sstr[0];
    const int qr = c->qrow[0], sw = c->srow[0], hr = c->hrow[0], I = c->I;
    const uint32_t nq = (uint32_t)(n * qr), ns = (uint32_t)(n * sw);
    bulk_g2s(dst, qs + (int64_t)r * qr, nq, bar);
    bulk_g2s(dst + nq, qs + (int64_t)(I + r) * qr, nq, bar);
    dst += 2 * nq;
    bulk_g2s(dst, sr + (int64_t)r * sw, ns, bar);
    bulk_g2s(dst + ns, sr + (int64_t)(I + r) * sw, ns, bar);
    dst += 2 * ns;
    if (hr) {
        const uint8_t *qh = c->h[0] + (int64_t)ex * c->hstr[0];
        const uint32_t nh = (uint32_t)(n * hr);
        bulk_g2s(dst, qh + (int64_t)r * hr, nh, bar);
        bulk_g2s(dst + nh, qh + (int64_t)(I + r) * hr, nh, bar);
    }
}

// Down rows [r0, r0 + n) of expert ex as [qs][scales][qh].
__device__ __forceinline__ void issue_down(const S1Src *c, uint8_t *dst, int ex, int r0, int n, int row_bytes,
                                           uint64_t *bar)
{
    mbar_arrive_expect_tx(bar, (uint32_t)(n * row_bytes));
    const uint32_t nq = (uint32_t)(n * c->qrow[1]), ns = (uint32_t)(n * c->srow[1]);
    bulk_g2s(dst, c->q[1] + (int64_t)ex * c->qstr[1] + (int64_t)r0 * c->qrow[1], nq, bar);
    bulk_g2s(dst + nq, c->s[1] + (int64_t)ex * c->sstr[1] + (int64_t)r0 * c->srow[1], ns, bar);
    if (c->hrow[1])
        bulk_g2s(dst + nq + ns, c->h[1] + (int64_t)ex * c->hstr[1] + (int64_t)r0 * c->hrow[1],
                 (uint32_t)(n * c->hrow[1]), bar);
}

// Copy item `it` of this CTA: gate/up chunks first, then one down item per
// group.  Issued only if its group is the shared expert (routed = false, before
// the routing is known) or a routed one (routed = true); the barrier it arms is
// recorded in *armed.
__device__ __noinline__ void issue_item(const S1Src *src, const S1Layout *L, uint8_t *smem, const Seg *seg, int nseg,
                                        int it, bool routed, int k, const int *grp_e, int r0, int nd, int *armed)
{
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L->bars);
    if (it < nseg) {
        const Seg &sg = seg[it];
        if (routed ? sg.g >= k : sg.g != k) return;
        issue_gateup(src, smem + L->gu + sg.off, grp_e[sg.g], sg.a, sg.n, L->gu_pair, bars + kS1BarSeg + it);
        atomicOr(armed, (int)(1u << (kS1BarSeg + it)));
    } else {
        const int g = it - nseg;
        if (nd <= 0 || (routed ? g >= k : g != k)) return;
        issue_down(src, smem + L->dn + (size_t)g * L->dr * L->dn_row, grp_e[g], r0, nd, L->dn_row,
                   bars + kS1BarDown + g);
        atomicOr(armed, (int)(1u << (kS1BarDown + g)));
    }
}

// One 32-weight unit of a row staged in shared memory (planes as issued above).
template <int FMT>
__device__ __forceinline__ Raw lds_unit(const uint8_t *q, const uint8_t *s, const uint8_t *h, int u)
{
    Raw r;
    r.h = 0;
    r.q1 = make_uint4(0, 0, 0, 0);
    if constexpr (FMT == MOE_FMT_Q8_0) {
        r.q0 = *reinterpret_cast<const uint4 *>(q + u * 32);
        r.q1 = *reinterpret_cast<const uint4 *>(q + u * 32 + 16);
        r.s = *reinterpret_cast<const uint16_t *>(s + u * 2);
    } else {
        r.q0 = *reinterpret_cast<const uint4 *>(q + u * 16);
        if constexpr (FMT == MOE_FMT_Q5_1) {
            r.s = *reinterpret_cast<const uint32_t *>(s + u * 4);
            r.h = *reinterpret_cast<const uint32_t *>(h + u * 4);
        } else {
            r.s = *reinterpret_cast<const uint16_t *>(s + u * 2);  // NVFP4: the unit's two E4M3 scales
        }
    }
    return r;
}

// Bounded wait of the calling thread on an mbarrier's first phase; on time-out
// records the error and returns false.
__device__ __forceinline__ bool s1_wait(uint64_t *bar, int32_t *err, int *fail)
{
    if (mbar_wait(bar, 0)) return true;
    atomicExch(err, (int)MOE_ERR_TIMEOUT);
    *fail = 1;
    return false;
}

// ---- gate/up over this CTA's row pairs -------------------------------------------
// LPR lanes per pair (RPW pairs per warp at a time), lane sl owning units sl,
// sl + LPR, ...; one compact loop body per (pair, unit): the unit's 32 x values
// from shared memory, then the gate and the up dot products.  The body is
// small and shared by every iteration, so it stays in the instruction cache.
template <int FMT>
__device__ __forceinline__ void s1_gateup(const FusedArgs &a, const S1Layout &L, uint8_t *smem, const Seg *seg, int nseg,
                          int npairs, const float4 *xs4, const float *xsum, const int *grp_e, int *fail)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const DevProj &w = a.gu;
    const int NU = a.H >> 5;
    const int LPR = lanes_per_row(NU), RPW = 32 / LPR;
    const int sub = lane / LPR, sl = lane - sub * LPR;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
    // each lane owns at most two units of x (H <= 64 * lanes per row): keep them in registers
    const bool xreg = NU <= 2 * LPR;
    const int u = sl, u2 = sl + LPR;
    const bool has1 = u < NU, has2 = u2 < NU;
    float4 xr0[8], xr1[8];
    float xs0 = 0.f, xs1 = 0.f;
    if (xreg) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            xr0[j] = has1 ? xs4[u * 8 + (j ^ (u & 7))] : make_float4(0.f, 0.f, 0.f, 0.f);
            xr1[j] = has2 ? xs4[u2 * 8 + (j ^ (u2 & 7))] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (FMT == MOE_FMT_Q5_1) {
            xs0 = has1 ? xsum[u] : 0.f;
            xs1 = has2 ? xsum[u2] : 0.f;
        }
    }
#pragma unroll 1
    for (int base = warp * RPW; base < npairs; base += kS1Warps * RPW) {
        const int q = base + sub;
        const bool valid = q < npairs;
        const int qq = valid ? q : npairs - 1;
        int s = 0;
        while (s + 1 < nseg && qq >= seg[s + 1].q0) ++s;
        const Seg sg = seg[s];
        const bool ok = s1_wait(bars + kS1BarSeg + s, a.err, fail);
        if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0 && base == 0) a.stamps[29] = clock64();
        const int i = qq - sg.q0, n = sg.n;
        const uint8_t *b = smem + L.gu + sg.off;
        const uint8_t *gq = b + (size_t)i * w.qs_row, *uq = gq + (size_t)n * w.qs_row;
        const uint8_t *gs = b + (size_t)2 * n * w.qs_row + (size_t)i * w.sr_row, *us = gs + (size_t)n * w.sr_row;
        const uint8_t *gh = b + (size_t)2 * n * (w.qs_row + w.sr_row) + (size_t)i * w.qh_row,
                      *uh = gh + (size_t)n * w.qh_row;
        const float half_ts = FMT == MOE_FMT_NVFP4 ? 0.5f * __ldg(w.ts + grp_e[sg.g]) : 0.5f;
        float s0 = 0.f, s1 = 0.f;
        if (ok && xreg) {
            // all four unit loads of the pair first, then four independent dot products
            const Raw g0 = lds_unit<FMT>(gq, gs, gh, u), u0r = lds_unit<FMT>(uq, us, uh, u);
            Raw g1 = g0, u1r = u0r;
            if (has2) {
                g1 = lds_unit<FMT>(gq, gs, gh, u2);
                u1r = lds_unit<FMT>(uq, us, uh, u2);
            }
            if (has1) {
                s0 = unit_dot_reg<FMT>(g0, xr0, xs0, a.tab_gu, half_ts, s0);
                s1 = unit_dot_reg<FMT>(u0r, xr0, xs0, a.tab_gu, half_ts, s1);
            }
            if (has2) {
                s0 = unit_dot_reg<FMT>(g1, xr1, xs1, a.tab_gu, half_ts, s0);
                s1 = unit_dot_reg<FMT>(u1r, xr1, xs1, a.tab_gu, half_ts, s1);
            }
        } else if (ok) {
#pragma unroll 1
            for (int v = sl; v < NU; v += LPR) {
                float4 xr[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) xr[j] = xs4[v * 8 + (j ^ (v & 7))];
                const float xs = FMT == MOE_FMT_Q5_1 ? xsum[v] : 0.f;
                s0 = unit_dot_reg<FMT>(lds_unit<FMT>(gq, gs, gh, v), xr, xs, a.tab_gu, half_ts, s0);
                s1 = unit_dot_reg<FMT>(lds_unit<FMT>(uq, us, uh, v), xr, xs, a.tab_gu, half_ts, s1);
            }
        }
        for (int o = LPR >> 1; o >= 1; o >>= 1) {
            s0 += __shfl_xor_sync(0xffffffffu, s0, o);
            s1 += __shfl_xor_sync(0xffffffffu, s1, o);
        }
        if (valid && sl == 0) {
            // h row of group g, element j = pair index, stored unit-swizzled (chunk
            // (j / 4) % 8 of unit j / 32 at chunk ((j / 4) ^ (j / 32)) % 8) so the
            // consumers' bulk copy lands it in the layout their loads want
            const int j = sg.a + i;
            a.h[(size_t)sg.g * a.I + (j & ~31) + ((((j >> 2) & 7) ^ ((j >> 5) & 7)) << 2) + (j & 3)] =
                s0 / (1.f + expf(-s0)) * s1;
        }
    }
}

// ---- Q5_1 down: per-unit sums of every group's h (staged, unit-swizzled) -----------
__device__ __forceinline__ void s1_h_sums(const S1Layout &L, uint8_t *smem, int I)
{
    const int NU = I >> 5;
    const float4 *hs4 = reinterpret_cast<const float4 *>(smem + L.h);
    float *hsum = reinterpret_cast<float *>(smem + L.hsum);
#pragma unroll 1
    for (int i = threadIdx.x; i < L.ng * NU; i += kS1Threads) {
        const float4 *p = hs4 + i * 8;  // unit i of the concatenation
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 v = p[j];
            acc += v.x;
            acc += v.y;
            acc += v.z;
            acc += v.w;
        }
        hsum[i] = acc;
    }
    __syncthreads();
}

// ---- down + combine over this CTA's output rows -----------------------------------
// Row-dots (group g, output row i) are dealt round-robin: step s of the CTA is
// row-dots s*RPW .. s*RPW + RPW - 1 (LPR lanes each), warp w takes steps w,
// w + W, ... two at a time so two independent decode chains are in flight; each
// step reads its group's h unit (one per lane) and writes gate_g * (D_g h_g)[i]
// to part[g][i], summed over g in the layer's order at the end.
template <int FMT>
__device__ __forceinline__ float s1_row_dot(const FusedArgs &a, const S1Layout &L, const uint8_t *smem, int nd,
                                            int rd, int sl, int LPR, int NU, float half_ts_base, const int *grp_e,
                                            const uint64_t *bars, int *fail, bool &ok)
{
    const DevProj &w = a.dn;
    const int nc = a.I >> 2;
    const int g = rd / nd, i = rd - g * nd;
    ok = s1_wait(const_cast<uint64_t *>(bars) + kS1BarDown + g, a.err, fail);
    const float4 *hs4 = reinterpret_cast<const float4 *>(smem + L.h);
    const float *hsum = reinterpret_cast<const float *>(smem + L.hsum);
    const uint8_t *b = smem + L.dn + (size_t)g * L.dr * L.dn_row;
    const uint8_t *q = b + (size_t)i * w.qs_row, *sc = b + (size_t)nd * w.qs_row + (size_t)i * w.sr_row,
                  *qh = b + (size_t)nd * (w.qs_row + w.sr_row) + (size_t)i * w.qh_row;
    const float half_ts = FMT == MOE_FMT_NVFP4 ? half_ts_base * __ldg(w.ts + grp_e[g]) : 0.5f;
    float v = 0.f;
    if (!ok) return v;
    if (NU <= LPR) {  // one unit per lane
        float4 hr[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) hr[j] = hs4[g * nc + sl * 8 + (j ^ (sl & 7))];
        const float hsr = FMT == MOE_FMT_Q5_1 ? hsum[g * NU + sl] : 0.f;
        v = unit_dot_reg<FMT>(lds_unit<FMT>(q, sc, qh, sl), hr, hsr, a.tab_dn, half_ts, 0.f);
    } else {
        const int xoff[1] = {g * nc}, xsoff[1] = {g * NU};
        float acc[1] = {0.f};
        for (int u = sl; u < NU; u += LPR)
            unit_dot<FMT, 1>(lds_unit<FMT>(q, sc, qh, u), u, hs4, hsum, xoff, xsoff, 1, a.tab_dn, half_ts, acc);
        v = acc[0];
    }
    return v;
}

template <int FMT>
__device__ __forceinline__ void s1_down(const FusedArgs &a, const S1Layout &L, uint8_t *smem, int r0, int nd, const int *grp_e,
                        const float *grp_gate, int *fail)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NU = a.I >> 5;
    const int ng = L.ng;
    float *part = reinterpret_cast<float *>(smem + L.part);
    const uint64_t *bars = reinterpret_cast<const uint64_t *>(smem + L.bars);
    const int LPR = lanes_per_row(NU), RPW = 32 / LPR;
    const int sub = lane / LPR, sl = lane - sub * LPR;
    const int nrd = ng * nd, nsteps = (nrd + RPW - 1) / RPW;
#pragma unroll 1
    for (int s0 = warp; s0 < nsteps; s0 += 2 * kS1Warps) {
        const int s1 = s0 + kS1Warps;
        const int rd0 = s0 * RPW + sub, rd1 = s1 * RPW + sub;
        const bool v0ok = rd0 < nrd, v1ok = s1 < nsteps && rd1 < nrd;
        bool ok0 = false, ok1 = false;
        float v0 = s1_row_dot<FMT>(a, L, smem, nd, v0ok ? rd0 : nrd - 1, sl, LPR, NU, 0.5f, grp_e, bars, fail, ok0);
        float v1 = 0.f;
        if (s1 < nsteps)  // warp-uniform
            v1 = s1_row_dot<FMT>(a, L, smem, nd, v1ok ? rd1 : nrd - 1, sl, LPR, NU, 0.5f, grp_e, bars, fail, ok1);
        for (int o = LPR >> 1; o >= 1; o >>= 1) {
            v0 += __shfl_xor_sync(0xffffffffu, v0, o);
            v1 += __shfl_xor_sync(0xffffffffu, v1, o);
        }
        if (sl == 0) {
            if (v0ok) {
                const int g = rd0 / nd;
                part[g * L.dr + rd0 - g * nd] = grp_gate[g] * v0;
            }
            if (v1ok) {
                const int g = rd1 / nd;
                part[g * L.dr + rd1 - g * nd] = grp_gate[g] * v1;
            }
        }
    }
    if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[30] = clock64();
    __syncthreads();
    for (int i = threadIdx.x; i < nd; i += kS1Threads) {
        float o = 0.f;
        for (int g = 0; g < ng; ++g) o += part[g * L.dr + i];
        a.out[r0 + i] = o;
    }
}

template <int FG, int FD>
__global__ void __launch_bounds__(kS1Threads, 1) stream1_kernel(const FusedArgs a)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int G = gridDim.x, c = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const S1Layout L = s1_layout(a, G);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
    int *grp_e = reinterpret_cast<int *>(smem + L.meta);
    float *grp_gate = reinterpret_cast<float *>(grp_e + kS1MaxGroups);
    int *flags = reinterpret_cast<int *>(grp_gate + kS1MaxGroups);  // [0] a wait failed, [1] armed barriers
    float4 *xs4 = reinterpret_cast<float4 *>(smem + L.x);
    float *xsum = reinterpret_cast<float *>(smem + L.xsum);
    const bool stamp = a.stamps && c == 0 && threadIdx.x == 0;
    if (stamp) a.stamps[0] = clock64();

    const int k = a.k, hs = a.has_shared ? 1 : 0;
    // 32-bit products: E, ng * I and H times the grid stay far below 2^31 for the shapes taken
    const int e0 = a.E * c / G, e1 = a.E * (c + 1) / G;
    const int P = L.ng * a.I;
    const int p0 = P * c / G, p1 = P * (c + 1) / G;
    const int r0 = a.H * c / G, r1 = a.H * (c + 1) / G;
    const int nd = r1 - r0;
    Seg *seg = reinterpret_cast<Seg *>(flags + 8 + 128);  // this CTA's gate/up chunks
    // copy sources and the layout, for the issuing code (256-byte slots after the chunks)
    S1Src *src = reinterpret_cast<S1Src *>(smem + L.meta + ((4 * (2 * kS1MaxGroups + 8 + 2 * 32 + 2 * 32) +
                                                             sizeof(int) * 5 * kS1MaxSeg + 15) & ~(size_t)15));
    S1Layout *Ls = reinterpret_cast<S1Layout *>(reinterpret_cast<uint8_t *>(src) + 256);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kS1NumBars; ++i) mbar_init(bars + i, 1);
        tc::fence_mbar_init();
        flags[0] = 0;
        flags[1] = 0;
        flags[2] = s1_segments(p0, p1, a.I, L.gu_pair, s1_chunk_pairs(L.gp), seg);
        const DevProj *pr[2] = {&a.gu, &a.dn};
        for (int j = 0; j < 2; ++j) {
            src->q[j] = pr[j]->qs;
            src->s[j] = pr[j]->sr;
            src->h[j] = pr[j]->qh;
            src->qstr[j] = pr[j]->qs_stride;
            src->sstr[j] = pr[j]->sr_stride;
            src->hstr[j] = pr[j]->qh_stride;
            src->qrow[j] = pr[j]->qs_row;
            src->srow[j] = pr[j]->sr_row;
            src->hrow[j] = pr[j]->qh_row;
        }
        src->I = a.I;
        *Ls = L;
        if (hs) {
            grp_e[k] = a.E;  // the shared expert is stored after the routed ones
            grp_gate[k] = 1.f;
        }
    }
    __syncthreads();
    const int nseg = flags[2];
    grid_event(a.stamps, 0);
    if (stamp) a.stamps[24] = clock64();
    // ---- prologue: bytes that do not depend on the routing, one warp per item -------
    if (lane == 0) {
        if (warp == 0 && e1 > e0) {
            mbar_arrive_expect_tx(bars + kS1BarRouter, (uint32_t)((e1 - e0) * a.H * 2));
            bulk_g2s(smem + L.h, a.wr + (size_t)e0 * a.H, (uint32_t)((e1 - e0) * a.H * 2), bars + kS1BarRouter);
            atomicOr(flags + 1, 1 << kS1BarRouter);
        }
        if (hs)
            for (int it = (warp + 1) % kS1Warps; it < nseg + L.ng; it += kS1Warps)
                issue_item(src, Ls, smem, seg, nseg, it, false, k, grp_e, r0, nd, flags + 1);
        if (stamp) a.stamps[25] = clock64();
    }
    pdl_wait();  // x, the workspace and out may belong to the previous kernel until here

    // ---- x as fp32 in shared memory (16-byte chunks swizzled per 32-weight unit) -----
    {
        const int H = a.H, nc = H >> 2;
        for (int i = threadIdx.x; i < nc; i += kS1Threads) {
            float4 v;
            if (a.x_dtype == MOE_DT_BF16) {
                const uint2 b = __ldg(reinterpret_cast<const uint2 *>(reinterpret_cast<const uint16_t *>(a.x) + i * 4));
                v = make_float4(bf16lo(b.x), bf16hi(b.x), bf16lo(b.y), bf16hi(b.y));
            } else {
                v = __ldg(reinterpret_cast<const float4 *>(a.x) + i);
            }
            const int u = i >> 3, j = i & 7;
            xs4[u * 8 + (j ^ (u & 7))] = v;
        }
        if (stamp) a.stamps[27] = clock64();
        if (c == 0)  // routing readback: counts are zero except for the selected experts
            for (int e = threadIdx.x; e <= a.E; e += kS1Threads) a.cnt_out[e] = e < a.E ? 0 : hs;
        if (FG == MOE_FMT_Q5_1) {
            __syncthreads();
            for (int u = threadIdx.x; u < (H >> 5); u += kS1Threads) {
                const float4 *p = xs4 + u * 8;
                float s = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 q = p[j];
                    s += q.x;
                    s += q.y;
                    s += q.z;
                    s += q.w;
                }
                xsum[u] = s;
            }
        }
        __syncthreads();
    }
    if (stamp) a.stamps[1] = clock64();

    // ---- router logits of rows [e0, e1) -----------------------------------------------
    if (warp < e1 - e0) {
        const int H = a.H, nch = H >> 3;
        const uint16_t *wr = reinterpret_cast<const uint16_t *>(smem + L.h);
        const bool ok = s1_wait(bars + kS1BarRouter, a.err, flags);
        for (int e = warp; ok && e < e1 - e0; e += kS1Warps) {
            const uint16_t *row = wr + (size_t)e * H;
            float acc = 0.f;
            for (int ch = lane; ch < nch; ch += 32) {
                const uint4 v = *reinterpret_cast<const uint4 *>(row + ch * 8);
                const int u = ch >> 2, j0 = (2 * ch) & 7;
                const float4 x0 = xs4[u * 8 + (j0 ^ (u & 7))];
                const float4 x1 = xs4[u * 8 + ((j0 + 1) ^ (u & 7))];
                acc = fmaf(bf16lo(v.x), x0.x, acc);
                acc = fmaf(bf16hi(v.x), x0.y, acc);
                acc = fmaf(bf16lo(v.y), x0.z, acc);
                acc = fmaf(bf16hi(v.y), x0.w, acc);
                acc = fmaf(bf16lo(v.z), x1.x, acc);
                acc = fmaf(bf16hi(v.z), x1.y, acc);
                acc = fmaf(bf16lo(v.w), x1.z, acc);
                acc = fmaf(bf16hi(v.w), x1.w, acc);
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) a.logits[e0 + e] = acc;
        }
    }
    if (stamp) a.stamps[2] = clock64();
    grid_event(a.stamps, 1);

    // ---- every logit here, top-k, then the routed experts' copies ----------------------
    const float *lg = reinterpret_cast<const float *>(smem + L.h);
    const bool have_logits = s1_exchange(a.xcnt + 1, a.logits, smem + L.h, (uint32_t)s1_al16((size_t)a.E * 4),
                                         bars + kS1BarLogits, a.err, flags, kS1BarLogits);
    if (stamp) a.stamps[26] = clock64();
    if (warp == 0 && have_logits) {
        int my_e;
        float my_g;
        unsigned *cand = reinterpret_cast<unsigned *>(flags + 8);
        if (a.E <= 512) topk_threshold<16>(lg, a.E, k, my_e, my_g, cand);
        else topk_threshold<32>(lg, a.E, k, my_e, my_g, cand);
        if (stamp) a.stamps[3] = clock64();
        if (lane < k) {
            grp_e[lane] = my_e;
            grp_gate[lane] = my_g;
            if (c == 0) {
                a.idx_out[lane] = my_e;
                a.gate_out[lane] = my_g;
                a.cnt_out[my_e] = 1;
            }
        }
    }
    __syncthreads();
    const bool routed = flags[0] == 0;
    // the gate/up chunks first: their bytes are needed first, and the SM's copy
    // engine and the memory system serve requests roughly in issue order; the
    // down rows (not read before the h hand-over) are issued after a barrier
    if (routed && lane == 0)
        for (int it = warp; it < nseg; it += kS1Warps)
            issue_item(src, Ls, smem, seg, nseg, it, true, k, grp_e, r0, nd, flags + 1);
    __syncthreads();
    if (routed && lane == 0)
        for (int it = nseg + warp; it < nseg + L.ng; it += kS1Warps)
            issue_item(src, Ls, smem, seg, nseg, it, true, k, grp_e, r0, nd, flags + 1);
    if (stamp) a.stamps[28] = clock64();
    if (stamp) a.stamps[4] = clock64();
    grid_event(a.stamps, 2);

    // ---- gate/up + SwiGLU -----------------------------------------------------------
    if (routed) s1_gateup<FG>(a, L, smem, seg, nseg, p1 - p0, xs4, xsum, grp_e, flags);
    if (a.stamps) __syncthreads();  // profiling: the whole CTA's gate/up
    if (stamp) a.stamps[5] = clock64();
    grid_event(a.stamps, 3);
    pdl_trigger();

    // ---- every group's h here, then down + combine ------------------------------------
    const bool have_h = s1_exchange(a.xcnt + 2, a.h, smem + L.h, (uint32_t)((size_t)L.ng * a.I * 4), bars + kS1BarH,
                                    a.err, flags, kS1BarH);
    if (FD == MOE_FMT_Q5_1 && have_h) s1_h_sums(L, smem, a.I);
    if (stamp) a.stamps[6] = clock64();
    if (routed && have_h && nd > 0) s1_down<FD>(a, L, smem, r0, nd, grp_e, grp_gate, flags);
    if (stamp) {
        a.stamps[7] = clock64();
        a.stamps[9] = clock64();
    }
    // every issued copy must have landed before the CTA's shared memory is
    // released; the last CTA to get here resets the hand-over counters
    __syncthreads();
    grid_event(a.stamps, 4);
    if (threadIdx.x == 0) {
        if (flags[0]) {
            const unsigned armed = (unsigned)flags[1];
            for (int i = 0; i < kS1NumBars; ++i)
                if ((armed >> i) & 1u) mbar_wait(bars + i, 0);
        }
        __threadfence();
        if (atomicAdd(a.xcnt, 1u) == (unsigned)G - 1u) {
            a.xcnt[1] = 0u;
            a.xcnt[2] = 0u;
            __threadfence();
            a.xcnt[0] = 0u;
        }
        if (stamp) a.stamps[31] = clock64();
    }
}

using S1Kernel = void (*)(const FusedArgs);

template <int FG>
S1Kernel s1_pick_down(int fd)
{
    switch (fd) {
    case MOE_FMT_Q8_0: return stream1_kernel<FG, MOE_FMT_Q8_0>;
    case MOE_FMT_Q5_1: return stream1_kernel<FG, MOE_FMT_Q5_1>;
    case MOE_FMT_IQ4_NL: return stream1_kernel<FG, MOE_FMT_IQ4_NL>;
    default: return stream1_kernel<FG, MOE_FMT_NVFP4>;
    }
}

S1Kernel s1_pick(int fg, int fd)
{
    switch (fg) {
    case MOE_FMT_Q8_0: return s1_pick_down<MOE_FMT_Q8_0>(fd);
    case MOE_FMT_Q5_1: return s1_pick_down<MOE_FMT_Q5_1>(fd);
    case MOE_FMT_IQ4_NL: return s1_pick_down<MOE_FMT_IQ4_NL>(fd);
    default: return s1_pick_down<MOE_FMT_NVFP4>(fd);
    }
}

}  // namespace

size_t stream1_smem_bytes(const FusedArgs &a, int grid) { return s1_layout(a, grid).total; }

bool stream1_supported(const FusedArgs &a, int grid, size_t smem_limit)
{
    if (a.T != 1 || grid < 1 || a.k > kFusedMaxK || a.E > 1024) return false;
    // 32-bit work splits in the kernel: every product (size x grid) must fit
    if ((long long)(kFusedMaxK + 1) * a.I * grid >= (1ll << 31) || (long long)a.H * grid >= (1ll << 31)) return false;
    if (!a.xcnt || !a.logits || !a.h) return false;
    // bulk copies move whole rows: every plane's row must be a multiple of 16 bytes
    const DevProj *ps[2] = {&a.gu, &a.dn};
    for (const DevProj *p : ps) {
        if (p->qs_row % 16 || p->sr_row % 16 || p->qh_row % 16 || !p->sr) return false;
        if (p->qs_stride % 16 || p->sr_stride % 16 || p->qh_stride % 16) return false;
    }
    if (a.H % 8 || a.I % 256) return false;  // I % 256: see s1_stage_h
    const S1Layout L = s1_layout(a, grid);
    // chunks: at most 8 by size, plus one per group boundary in the range
    if (L.gp > 2 * a.I || L.gp / s1_chunk_pairs(L.gp) + 4 > kS1MaxSeg) return false;
    return L.total <= smem_limit && L.total <= (size_t)kS1SmemLimit;
}

// CTAs of this kernel that fit on one SM at once with `smem` bytes of dynamic
// shared memory (0 when the query fails).  Its CTAs hand data to one another,
// so the forward uses it only when one CTA per SM fits: grid = SMs.
int stream1_blocks_per_sm(const FusedArgs &a, size_t smem)
{
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, s1_pick(a.gu.fmt, a.dn.fmt), kS1Threads, smem) !=
        cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

cudaError_t stream1_set_attributes()
{
    const int fmts[4] = {MOE_FMT_Q8_0, MOE_FMT_Q5_1, MOE_FMT_IQ4_NL, MOE_FMT_NVFP4};
    for (int fg : fmts)
        for (int fd : fmts) {
            const cudaError_t e =
                cudaFuncSetAttribute(s1_pick(fg, fd), cudaFuncAttributeMaxDynamicSharedMemorySize, kS1SmemLimit);
            if (e != cudaSuccess) return e;
        }
    return cudaSuccess;
}

cudaError_t launch_stream1(const FusedArgs &a, int grid, size_t smem, int pdl, cudaStream_t s)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kS1Threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (pdl) {
        // CTAs hand data to one another, so all must be resident: one CTA per
        // SM (the shared-memory footprint allows no second), grid = SMs
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
    } else {
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, s1_pick(a.gu.fmt, a.dn.fmt), a);
}

}  // namespace moe
