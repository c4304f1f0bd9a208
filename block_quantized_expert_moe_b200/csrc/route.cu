// Router GEMV + softmax/top-k + device-side plan, fused in one launch.
//
// The "Qwen3.8-Flash-Next UD-IQ2_XS (L4 fix) for Basalt" model card, section
// "What was changed", calls its fast decode path a device-planned MoE tail:
// the per-expert token lists are built on the GPU, with no host round trip.
// Here the plan is built at the end of the router launch:
//
//   phase 1 (all CTAs)   logits[t][e] = sum_h Wr[e][h] x[t][h], fp32 accumulate;
//                        CTA b takes token block b % NB (<= 8 tokens) and a
//                        slice of the expert rows; one thread bulk-copies the
//                        slice's router rows and the tokens' x rows into shared
//                        memory, four rows per warp (gemv_staged; rows read
//                        from global memory, one per warp, when the slice does
//                        not fit)
//   phase 2 (last CTA of each token block)  one warp per token: the threshold
//                        top-k (candidates at or above the k-th largest lane
//                        maximum, ranked in one pass; ties to the lower expert
//                        index), gates exp(l - lmax) / sum over the selected
//   phase 3 (last block) plan: per-expert counts by shared-memory atomics, an
//                        exclusive scan to slot offsets, and a stable slot
//                        order (tokens ascending inside an expert) from 64-bit
//                        token masks and popcounts, so the plan is identical
//                        from run to run; then the list of work groups
//                        {expert, first slot, tokens <= tt} for the grouped
//                        kernels, the shared expert's groups last (plan_small
//                        for <= 64 tokens: four barriers; plan_phase above).
//
// "Last" is decided by global tickets (atomicAdd after a fence: one per token
// block, one over blocks); no CTA ever waits on another.
#include <climits>

#include "decode_common.cuh"
#include "moe_internal.cuh"
#include "quant_dot.cuh"
#include "tc_common.cuh"

namespace moe {

namespace {

constexpr int kRouteMaxBlockGroups = 14;  // per-group tickets at words 2..15 of the ticket area
constexpr int kPlanIdxCache = 4096;       // selections the plan keeps in shared memory
constexpr size_t kRouteWrSmem = 128 * 1024;  // router rows a CTA may stage in shared memory
constexpr int kSmallPlanT = 64;           // token masks of one 64-bit word: the short plan

__host__ __device__ inline size_t route_al16(size_t v) { return (v + 15) & ~(size_t)15; }

// Shared-memory regions of the kernel, from (H, rt, E, rows per CTA); host and
// device compute them alike.
struct RouteSmem {
    bool staged;     // the CTA's router rows are bulk-copied into shared memory
    size_t wr, red;  // x rows as given (bf16 or fp32) at 0, then the router rows, partials
    size_t gemv;     // bytes of the logit phase
    size_t idx;      // the selections (short plan), after the top-k rows and the plan
    size_t total;
};

__host__ __device__ inline RouteSmem route_smem(int H, int rt, int E, int rmax)
{
    RouteSmem m;
    const size_t xb = (size_t)rt * H * 4;  // room for rt fp32 rows
    m.staged = (size_t)rmax * H * 2 <= kRouteWrSmem;
    m.wr = xb;
    m.red = m.wr + route_al16((size_t)rmax * H * 2);
    m.gemv = m.staged ? m.red + (size_t)(kThreads / 32) * 32 * 4 : xb;
    const size_t topk = (size_t)(kThreads / 32) * (E + 128) * 4;
    const size_t plan = (size_t)E * 8 + (size_t)4 * (E + 1) * 4 + 64 * 4;
    m.idx = route_al16(topk > plan ? topk : plan);
    size_t t = m.idx + (size_t)kPlanIdxCache * 4;
    // the general top-k fallback (k > 32 or E > 1024): two rows per warp and flags
    const size_t fb = (size_t)2 * (kThreads / 32) * E * 4 + (kThreads / 32) * 32 * 4;
    if (fb > t) t = fb;
    m.total = m.gemv > t ? m.gemv : t;
    return m;
}

// 8 consecutive x values of token t starting at element 8c, from the raw rows
// in shared memory, as four (even, odd) pairs.
template <bool XBF16>
__device__ __forceinline__ void x_chunk(const unsigned char *xs, int H, int t, int c, float2 (&x)[4])
{
    if constexpr (XBF16) {
        const uint4 v = *reinterpret_cast<const uint4 *>(xs + ((size_t)t * H + c * 8) * 2);
        x[0] = make_float2(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u));
        x[1] = make_float2(__uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
        x[2] = make_float2(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xFFFF0000u));
        x[3] = make_float2(__uint_as_float(v.w << 16), __uint_as_float(v.w & 0xFFFF0000u));
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(xs + ((size_t)t * H + c * 8) * 4);
        const float4 lo = p[0], hi = p[1];
        x[0] = make_float2(lo.x, lo.y);
        x[1] = make_float2(lo.z, lo.w);
        x[2] = make_float2(hi.x, hi.y);
        x[3] = make_float2(hi.z, hi.w);
    }
}

// Profiling only: thread 0 folds the global timer into event ev's first/last pair.
__device__ __forceinline__ void route_event(long long *st, int ev)
{
    if (!st || threadIdx.x != 0) return;
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    atomicMax(st + 10 + 2 * ev, (1ll << 62) - (long long)t);
    atomicMax(st + 11 + 2 * ev, (long long)t);
}

// Profiling only: thread 0 records its SM clock in word i of the stamps.
__device__ __forceinline__ void route_clock(long long *st, int i, bool on)
{
    if (st && on && threadIdx.x == 0) st[i] = clock64();
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint4 ldg_nc16(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// In-place exclusive scan of n <= 4*kThreads ints in shared memory; returns
// the total to every thread.  Uses `tmp` (>= 32 ints) for warp totals.
__device__ __forceinline__ int block_exclusive_scan(int *v, int n, int *tmp)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int loc[4], s = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int j = tid * 4 + i;
        loc[i] = j < n ? v[j] : 0;
        s += loc[i];
    }
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kThreads / 32 ? tmp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int u = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += u;
        }
        if (lane < kThreads / 32) tmp[lane] = wi - w;  // exclusive warp offsets
        if (lane == kThreads / 32 - 1) tmp[kThreads / 32] = wi;
    }
    __syncthreads();
    int run = tmp[warp] + incl - s;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int j = tid * 4 + i;
        if (j < n) v[j] = run;
        run += loc[i];
    }
    int total = tmp[kThreads / 32];
    __syncthreads();
    return total;
}

__device__ __forceinline__ void topk_phase(const RouteArgs &a, unsigned char *smem, int t_begin, int t_end, int *idx_s)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = kThreads / 32;
    const int E = a.E, k = a.k;
    if (k <= 32 && E <= 1024) {
        // one warp per token: the row into shared memory, then the threshold
        // selection (candidates at or above the k-th largest lane maximum)
        float *row = reinterpret_cast<float *>(smem) + (size_t)warp * (E + 128);
        for (int t = t_begin + warp; t < t_end; t += nw) {
            if (E <= 512) stage_logits<16>(a.logits + (size_t)t * E, row, E, lane);
            else stage_logits<32>(a.logits + (size_t)t * E, row, E, lane);
            __syncwarp();
            route_clock(a.stamps, 1, t == 0);
            int me;
            float mg;
            unsigned *cand = reinterpret_cast<unsigned *>(row + E);
            if (E <= 512) topk_threshold<16>(row, E, k, me, mg, cand);
            else topk_threshold<32>(row, E, k, me, mg, cand);
            route_clock(a.stamps, 2, t == 0);
            if (lane < k) {
                a.idx[(size_t)t * k + lane] = me;
                a.gate[(size_t)t * k + lane] = mg;
                if (idx_s) idx_s[t * k + lane] = me;
            }
            __syncwarp();
        }
        return;
    }
    float *row = reinterpret_cast<float *>(smem) + warp * E;
    float *selv = reinterpret_cast<float *>(smem) + nw * E + warp * E;
    uint32_t *taken = reinterpret_cast<uint32_t *>(smem + (size_t)2 * nw * E * sizeof(float)) + warp * 32;
    for (int t = t_begin + warp; t < t_end; t += nw) {
        for (int e = lane; e < E; e += 32) row[e] = __ldcg(a.logits + (size_t)t * E + e);
        taken[lane] = 0u;
        __syncwarp();
        float den = 0.f, vmax = 0.f;
        for (int j = 0; j < k; ++j) {
            float bv = -INFINITY;
            int bi = INT_MAX;
            for (int e = lane; e < E; e += 32) {
                if ((taken[e >> 5] >> (e & 31)) & 1u) continue;
                float v = row[e];
                if (bi == INT_MAX || v > bv) { bv = v; bi = e; }
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (oi != INT_MAX && (bi == INT_MAX || ov > bv || (ov == bv && oi < bi))) {
                    bv = ov;
                    bi = oi;
                }
            }
            if (j == 0) vmax = bv;
            den += expf(bv - vmax);
            if (lane == 0) {
                taken[bi >> 5] |= 1u << (bi & 31);
                selv[j] = bv;
                a.idx[(size_t)t * k + j] = bi;
                if (idx_s) idx_s[t * k + j] = bi;
            }
            __syncwarp();
        }
        for (int j = lane; j < k; j += 32) a.gate[(size_t)t * k + j] = expf(selv[j] - vmax) / den;
        __syncwarp();
    }
}

// Dense-batched plan: active expert a (ascending id, the shared expert last)
// owns slots a*T .. a*T+T-1, one per token of the batch; its gate for token t is
// the routing gate if t selected it, else 0.
__device__ __forceinline__ void plan_dense(const RouteArgs &a, unsigned char *smem)
{
    const int tid = threadIdx.x;
    const int E = a.E, k = a.k, T = a.T, tt = a.tt;
    int *cnt = reinterpret_cast<int *>(smem);
    int *act = cnt + (E + 1);
    int *tmp = act + (E + 1);
    for (int e = tid; e < E; e += kThreads) cnt[e] = 0;
    __syncthreads();
    for (int i = tid; i < T * k; i += kThreads) atomicAdd(&cnt[__ldcg(a.idx + i)], 1);
    __syncthreads();
    for (int e = tid; e < E; e += kThreads) act[e] = cnt[e] > 0 ? 1 : 0;
    __syncthreads();
    const int n_routed = block_exclusive_scan(act, E, tmp);
    const int n_act = n_routed + (a.has_shared ? 1 : 0);
    const int chunks = (T + tt - 1) / tt;
    if (n_act * chunks > a.max_groups) {
        if (tid == 0) {
            atomicExch(a.err, (int)MOE_ERR_DEVICE);
            *a.n_groups = 0;
        }
        return;
    }
    for (int i = tid; i < n_act * T; i += kThreads) {
        a.perm_tok[i] = i % T;
        a.dgate[i] = (a.has_shared && i >= n_routed * T) ? 1.f : 0.f;
    }
    for (int e = tid; e < E; e += kThreads) {
        a.cnt[e] = cnt[e];
        if (cnt[e] > 0)
            for (int c = 0; c < chunks; ++c)
                a.groups[act[e] * chunks + c] = make_int4(e, act[e] * T + c * tt, min(tt, T - c * tt), 0);
    }
    if (a.has_shared)
        for (int c = tid; c < chunks; c += kThreads)
            a.groups[n_routed * chunks + c] = make_int4(E, n_routed * T + c * tt, min(tt, T - c * tt), 0);
    __syncthreads();  // dgate zeroed before the routed gates land
    for (int i = tid; i < T * k; i += kThreads) {
        const int e = __ldcg(a.idx + i);
        a.dgate[act[e] * T + i / k] = __ldcg(a.gate + i);
    }
    if (tid == 0) {
        a.cnt[E] = a.has_shared ? T : 0;
        *a.n_groups = n_act * chunks;
        *a.n_dense_rows = n_act * T;
    }
}

// Plan for at most 64 tokens with four barriers: per-expert counts and 64-bit
// token masks (shared-memory atomics); a block-wide scan of the counts and of
// the group counts (thread i owns experts EPT i .. EPT i + EPT - 1, EPT = E / 256
// rounded up; warp totals through shared memory, read back by every thread)
// that also writes the groups; then
// every selection's slot is its expert's offset plus the number of earlier
// tokens in the expert's mask, so slots follow token order inside an expert.
// `local`: the selections are already in idx_s (this CTA selected every token).
__device__ __forceinline__ void plan_small(const RouteArgs &a, unsigned char *smem, int *idx_s, bool local)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = kThreads / 32;
    const int E = a.E, k = a.k, T = a.T, tt = a.tt, n = T * k;
    unsigned long long *mask = reinterpret_cast<unsigned long long *>(smem);
    int *cnt = reinterpret_cast<int *>(mask + E);
    int *off = cnt + (E + 1);
    int *wsum = off + (E + 1);  // [2][nw] warp totals of counts and groups
    if (!local)
        for (int i0 = tid; i0 < n; i0 += 4 * kThreads) {
            int v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] = i0 + q * kThreads < n ? __ldcg(a.idx + i0 + q * kThreads) : 0;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (i0 + q * kThreads < n) idx_s[i0 + q * kThreads] = v[q];
        }
    for (int e = tid; e < E; e += kThreads) {
        cnt[e] = 0;
        mask[e] = 0ull;
    }
    __syncthreads();
    for (int i = tid; i < n; i += kThreads) {
        const int e = idx_s[i];
        atomicAdd(&cnt[e], 1);
        atomicOr(&mask[e], 1ull << (i / k));
    }
    __syncthreads();
    route_clock(a.stamps, 5, true);
    // experts EPT tid .. EPT tid + EPT - 1 (E <= 1024 = 4 x 256: up to four each)
    const int EPT = (E + kThreads - 1) / kThreads, eb = tid * EPT;
    int c[4], cs = 0, gs = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        c[q] = q < EPT && eb + q < E ? cnt[eb + q] : 0;
        cs += c[q];
        gs += (c[q] + tt - 1) / tt;
    }
    int ci = cs, gi = gs;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, ci, o), w = __shfl_up_sync(0xffffffffu, gi, o);
        if (lane >= o) {
            ci += u;
            gi += w;
        }
    }
    if (lane == 31) {
        wsum[warp] = ci;
        wsum[nw + warp] = gi;
    }
    __syncthreads();
    int co = ci - cs, go = gi - gs, slots = 0, routed_groups = 0;
#pragma unroll
    for (int w = 0; w < nw; ++w) {
        const int a0 = wsum[w], a1 = wsum[nw + w];
        if (w < warp) {
            co += a0;
            go += a1;
        }
        slots += a0;
        routed_groups += a1;
    }
    const int shared_groups = a.has_shared ? (T + tt - 1) / tt : 0;
    const bool bad = routed_groups + shared_groups > a.max_groups || slots != n;
    if (bad) {
        if (tid == 0) {
            atomicExch(a.err, (int)MOE_ERR_DEVICE);
            *a.n_groups = 0;
        }
        return;  // uniform: every thread computed the same totals
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = eb + q;
        if (q < EPT && e < E) {
            off[e] = co;
            a.cnt[e] = c[q];
            a.off[e] = co;
            for (int j = 0; j * tt < c[q]; ++j) a.groups[go + j] = make_int4(e, co + j * tt, min(tt, c[q] - j * tt), 0);
            co += c[q];
            go += (c[q] + tt - 1) / tt;
        }
    }
    for (int j = tid; j < shared_groups; j += kThreads)
        a.groups[routed_groups + j] = make_int4(E, n + j * tt, min(tt, T - j * tt), 0);
    if (tid == 0) {
        a.cnt[E] = a.has_shared ? T : 0;
        a.off[E] = n;
        *a.n_groups = routed_groups + shared_groups;
    }
    __syncthreads();
    route_clock(a.stamps, 6, true);
    route_clock(a.stamps, 7, true);
    for (int i = tid; i < n; i += kThreads) {
        const int t = i / k, e = idx_s[i];
        const int pos = off[e] + __popcll(mask[e] & ((1ull << t) - 1ull));
        a.perm_tok[pos] = t;
        a.slot_pos[i] = pos;
    }
    for (int t = tid; t < (a.has_shared ? T : 0); t += kThreads) a.perm_tok[n + t] = t;
    route_clock(a.stamps, 8, true);
}

__device__ __forceinline__ void plan_phase(const RouteArgs &a, unsigned char *smem)
{
    const int tid = threadIdx.x;
    const int E = a.E, k = a.k, T = a.T, tt = a.tt;
    unsigned long long *mask = reinterpret_cast<unsigned long long *>(smem);
    int *cnt = reinterpret_cast<int *>(mask + E);
    int *off = cnt + (E + 1);
    int *run = off + (E + 1);
    int *gbase = run + (E + 1);
    int *tmp = gbase + (E + 1);
    // the selections, read three times below, into shared memory once when they
    // fit (four loads in flight per thread), else read from L2 each time
    int *idx_s = tmp + 64;
    const bool cached = T * k <= kPlanIdxCache;
    if (cached)
        for (int i0 = tid; i0 < T * k; i0 += 4 * kThreads) {
            int v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] = i0 + q * kThreads < T * k ? __ldcg(a.idx + i0 + q * kThreads) : 0;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (i0 + q * kThreads < T * k) idx_s[i0 + q * kThreads] = v[q];
        }
    const int *sel = cached ? idx_s : a.idx;
    for (int e = tid; e < E; e += kThreads) { cnt[e] = 0; run[e] = 0; }
    __syncthreads();
    for (int i = tid; i < T * k; i += kThreads) atomicAdd(&cnt[cached ? sel[i] : __ldcg(sel + i)], 1);
    __syncthreads();
    route_clock(a.stamps, 5, true);
    for (int e = tid; e < E; e += kThreads) {
        off[e] = cnt[e];
        gbase[e] = (cnt[e] + tt - 1) / tt;
    }
    __syncthreads();
    const int slots = block_exclusive_scan(off, E, tmp);
    const int routed_groups = block_exclusive_scan(gbase, E, tmp);
    route_clock(a.stamps, 6, true);
    const int shared_groups = a.has_shared ? (T + tt - 1) / tt : 0;
    const int total_groups = routed_groups + shared_groups;
    if (total_groups > a.max_groups || slots != T * k) {
        if (tid == 0) {
            atomicExch(a.err, (int)MOE_ERR_DEVICE);
            *a.n_groups = 0;
        }
        return;
    }
    for (int e = tid; e < E; e += kThreads) {
        a.cnt[e] = cnt[e];
        a.off[e] = off[e];
        for (int c = 0; c * tt < cnt[e]; ++c)
            a.groups[gbase[e] + c] = make_int4(e, off[e] + c * tt, min(tt, cnt[e] - c * tt), 0);
    }
    for (int c = tid; c < shared_groups; c += kThreads)
        a.groups[routed_groups + c] = make_int4(E, T * k + c * tt, min(tt, T - c * tt), 0);
    if (tid == 0) {
        a.cnt[E] = a.has_shared ? T : 0;
        a.off[E] = T * k;
        *a.n_groups = total_groups;
    }
    for (int t = tid; t < (a.has_shared ? T : 0); t += kThreads) a.perm_tok[T * k + t] = t;
    route_clock(a.stamps, 7, true);
    // stable slot order: within expert e, slots follow token order
    for (int c0 = 0; c0 < T; c0 += 64) {
        const int nt = min(64, T - c0);
        for (int e = tid; e < E; e += kThreads) mask[e] = 0ull;
        __syncthreads();
        for (int i = tid; i < nt * k; i += kThreads) {
            int t = c0 + i / k;
            const size_t at = (size_t)t * k + i % k;
            int e = cached ? sel[at] : __ldcg(sel + at);
            atomicOr(&mask[e], 1ull << (t - c0));
        }
        __syncthreads();
        for (int i = tid; i < nt * k; i += kThreads) {
            int t = c0 + i / k, j = i % k;
            const size_t at = (size_t)t * k + j;
            int e = cached ? sel[at] : __ldcg(sel + at);
            unsigned long long below = (t - c0) ? (mask[e] & ((1ull << (t - c0)) - 1ull)) : 0ull;
            int pos = off[e] + run[e] + __popcll(below);
            a.perm_tok[pos] = t;
            a.slot_pos[(size_t)t * k + j] = pos;
        }
        __syncthreads();
        for (int e = tid; e < E; e += kThreads) run[e] += __popcll(mask[e]);
        __syncthreads();
    }
    route_clock(a.stamps, 8, true);
}

// Sum over the warp's lanes of each of v[0..31], transposed: lane l ends with
// the total of v[l] in v[0] (31 shuffles in five halving steps).
__device__ __forceinline__ float warp_transpose_sum(float (&v)[32])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int j = 0; j < o; ++j) {
            const float send = up ? v[j] : v[j + o];
            const float keep = up ? v[j + o] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0];
}

// Logits of the CTA's staged router rows for the nt tokens of this pass.
// Rows go four to a warp (each x chunk read from shared memory feeds four
// rows); lane l takes 16-byte weight chunks l, l + 32, ... of the rows, so a
// warp's 32 chunk loads cover consecutive bytes; when the CTA has fewer row
// quads than warps, the chunks of a quad are split over several warps and
// their partial sums added in warp order.
template <bool XBF16>
__device__ __forceinline__ void gemv_staged(const RouteArgs &a, const unsigned char *smem, const RouteSmem &m, int e0,
                                            int nrow, int t0, int nt)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = kThreads / 32;
    const int H = a.H, E = a.E, nch = H >> 3, NI = (nch + 31) / 32;
    const uint16_t *wrs = reinterpret_cast<const uint16_t *>(smem + m.wr);
    float *red = reinterpret_cast<float *>(const_cast<unsigned char *>(smem) + m.red);
    const int nq = (nrow + 3) / 4;
    const int wpq = nq >= nw ? 1 : nw / nq, qpp = nw / wpq;  // warps per quad, quads per pass
    const int part = warp % wpq;
    for (int q = warp / wpq; q < nq; q += qpp) {
        float2 acc[4][8];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int t = 0; t < 8; ++t) acc[r][t] = make_float2(0.f, 0.f);
        for (int i = part; i < NI; i += wpq) {
            const int c = lane + 32 * i;
            if (c >= nch) break;
            float2 w[4][4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const uint4 v = 4 * q + r < nrow
                                    ? *reinterpret_cast<const uint4 *>(wrs + (size_t)(4 * q + r) * H + c * 8)
                                    : make_uint4(0, 0, 0, 0);
                w[r][0] = make_float2(bf16lo(v.x), bf16hi(v.x));
                w[r][1] = make_float2(bf16lo(v.y), bf16hi(v.y));
                w[r][2] = make_float2(bf16lo(v.z), bf16hi(v.z));
                w[r][3] = make_float2(bf16lo(v.w), bf16hi(v.w));
            }
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                if (t < nt) {
                    float2 x[4];
                    x_chunk<XBF16>(smem, H, t, c, x);
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        float2 s2 = acc[r][t];
#pragma unroll
                        for (int h = 0; h < 4; ++h) s2 = qd::fma2(w[r][h], x[h], s2);
                        acc[r][t] = s2;
                    }
                }
            }
        }
        float v[32];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int t = 0; t < 8; ++t) v[r * 8 + t] = acc[r][t].x + acc[r][t].y;
        const float sum = warp_transpose_sum(v);  // lane = 8 r + t
        const int r = lane >> 3, t = lane & 7;
        if (wpq == 1) {
            if (t < nt && 4 * q + r < nrow) a.logits[(size_t)(t0 + t) * E + e0 + 4 * q + r] = sum;
        } else {
            red[(q * wpq + part) * 32 + lane] = sum;
        }
    }
    if (wpq > 1) {
        __syncthreads();
        for (int i = threadIdx.x; i < nq * 32; i += kThreads) {
            const int q = i >> 5, l = i & 31, r = l >> 3, t = l & 7;
            float sum = 0.f;
            for (int p = 0; p < wpq; ++p) sum += red[(q * wpq + p) * 32 + l];
            if (t < nt && 4 * q + r < nrow) a.logits[(size_t)(t0 + t) * E + e0 + 4 * q + r] = sum;
        }
    }
}

// Logits of rows [e0, e1) for the nt tokens of this pass, router rows read from
// global memory (CTAs whose rows do not fit the staging area), one row per warp.
template <bool XBF16>
__device__ __forceinline__ void gemv_global(const RouteArgs &a, const unsigned char *xs, int e0, int e1, int t0, int nt)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = kThreads / 32;
    const int H = a.H, E = a.E, nch = H >> 3;
    for (int e = e0 + warp; e < e1; e += nw) {
        const uint16_t *wrow = a.wr + (size_t)e * H;
        float2 acc[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) acc[t] = make_float2(0.f, 0.f);
        for (int cb = 0; cb < nch; cb += 32 * 8) {
            uint4 wv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                int c = cb + lane + 32 * i;
                wv[i] = c < nch ? ldg_nc16(wrow + c * 8) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                int c = cb + lane + 32 * i;
                if (c >= nch) break;
                const float2 w[4] = {make_float2(bf16lo(wv[i].x), bf16hi(wv[i].x)),
                                     make_float2(bf16lo(wv[i].y), bf16hi(wv[i].y)),
                                     make_float2(bf16lo(wv[i].z), bf16hi(wv[i].z)),
                                     make_float2(bf16lo(wv[i].w), bf16hi(wv[i].w))};
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    if (t < nt) {
                        float2 x[4];
                        x_chunk<XBF16>(xs, H, t, c, x);
#pragma unroll
                        for (int h = 0; h < 4; ++h) acc[t] = qd::fma2(w[h], x[h], acc[t]);
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            float v = acc[t].x + acc[t].y;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && t < nt) a.logits[(size_t)(t0 + t) * E + e] = v;
        }
    }
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     tc::smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
                 : "memory");
}

__global__ void __launch_bounds__(kThreads) route_kernel(const RouteArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_last;
    __shared__ __align__(8) uint64_t wr_bar, x_bar;
    route_event(a.stamps, 0);
    const int H = a.H, E = a.E;
    // CTA b takes token block b % NB and a slice of the expert rows (token
    // blocks of rt tokens dealt to NB block groups: with more blocks than
    // groups a CTA takes blocks j, j + NB, ...), so every CTA stages its tokens
    // once and the grid covers the SMs
    const int ntb = (a.T + a.rt - 1) / a.rt, NB = min(ntb, kRouteMaxBlockGroups), per = gridDim.x / NB;
    const int tb = blockIdx.x % NB, slice = blockIdx.x / NB;
    const int e0 = slice < per ? (int)((long long)E * slice / per) : E;
    const int e1 = slice < per ? (int)((long long)E * (slice + 1) / per) : E;
    const RouteSmem m = route_smem(H, a.rt, E, (E + per - 1) / per);
    const bool xbf16 = a.x_dtype == MOE_DT_BF16;
    const uint32_t xrow = (uint32_t)H * (xbf16 ? 2u : 4u);
    // bulk copies: the CTA's router rows (contiguous, once) and each pass's x
    // rows as given, all issued by one thread and landing together
    const bool staged = m.staged && e1 > e0;
    if (threadIdx.x == 0) {
        tc::mbar_init(&wr_bar, 1);
        tc::mbar_init(&x_bar, 1);
        tc::fence_mbar_init();
        if (staged) {
            const uint32_t bytes = (uint32_t)((e1 - e0) * H * 2);
            tc::mbar_arrive_expect_tx(&wr_bar, bytes);
            bulk_g2s(smem + m.wr, a.wr + (size_t)e0 * H, bytes, &wr_bar);
        }
    }
    for (int t0 = tb * a.rt, pass = 0; t0 < a.T && e1 > e0; t0 += NB * a.rt, ++pass) {
        const int nt = min(a.rt, a.T - t0);
        __syncthreads();  // the previous pass's x is consumed (and the barriers initialised)
        if (threadIdx.x == 0) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc::mbar_arrive_expect_tx(&x_bar, (uint32_t)nt * xrow);
            for (int t = 0; t < nt; ++t)
                bulk_g2s(smem + (size_t)t * xrow, static_cast<const unsigned char *>(a.x) + (size_t)(t0 + t) * xrow,
                         xrow, &x_bar);
        }
        // bounded waits; the CTA agrees on the outcome so its barriers stay uniform
        bool ok = tc::mbar_wait(&x_bar, pass & 1);
        if (staged && pass == 0) ok = tc::mbar_wait(&wr_bar, 0) && ok;
        if (__syncthreads_or(!ok)) {
            // record the error, give the copies in flight a second bounded wait
            // before shared memory is reused, and skip the logits
            if (threadIdx.x == 0) {
                if (a.err) atomicExch(a.err, (int)MOE_ERR_TIMEOUT);
                tc::mbar_wait(&x_bar, pass & 1);
                if (staged) tc::mbar_wait(&wr_bar, 0);
            }
            __syncthreads();
            break;
        }
        if (pass == 0) route_event(a.stamps, 1);
        if (staged) {
            if (xbf16) gemv_staged<true>(a, smem, m, e0, e1 - e0, t0, nt);
            else gemv_staged<false>(a, smem, m, e0, e1 - e0, t0, nt);
        } else {
            if (xbf16) gemv_global<true>(a, smem, e0, e1, t0, nt);
            else gemv_global<false>(a, smem, e0, e1, t0, nt);
        }
    }
    // the last CTA of this token block selects its tokens' experts; the last
    // token block to finish builds the plan (tickets: [0] blocks, [2 + tb] CTAs)
    __syncthreads();
    route_event(a.stamps, 2);
    if (threadIdx.x == 0) {
        __threadfence();
        const int ticket = atomicAdd(a.ticket + 2 + tb, 1);
        s_last = ticket == per - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    route_clock(a.stamps, 0, tb == 0);
    // the short plan (<= 64 tokens) reads the selections from shared memory;
    // with one block group this CTA selects every token and writes them there
    const bool small = a.do_plan && !a.dense && a.T <= kSmallPlanT && a.T * a.k <= kPlanIdxCache && a.k <= 32 &&
                       E <= 1024;
    int *idx_s = reinterpret_cast<int *>(smem + m.idx);
    for (int t0 = tb * a.rt; t0 < a.T; t0 += NB * a.rt)
        topk_phase(a, smem, t0, min(a.T, t0 + a.rt), small && NB == 1 ? idx_s : nullptr);
    __syncthreads();
    route_event(a.stamps, 3);
    // SM clocks are per SM: with several token blocks the plan may run on another
    // CTA's SM, so the selection's end is recorded only when one CTA does both
    route_clock(a.stamps, 3, tb == 0 && NB == 1);
    if (threadIdx.x == 0) {
        a.ticket[2 + tb] = 0;
        if (NB > 1) {  // one block group: this CTA is already the last
            __threadfence();
            const int ticket = atomicAdd(a.ticket, 1);
            s_last = ticket == NB - 1;
        }
    }
    __syncthreads();
    if (!s_last) return;
    if (NB > 1) __threadfence();
    route_clock(a.stamps, 4, true);
    if (a.do_plan) {
        __syncthreads();
        if (a.dense) plan_dense(a, smem);
        else if (small) plan_small(a, smem, idx_s, NB == 1);
        else plan_phase(a, smem);
    }
    __syncthreads();
    route_event(a.stamps, 4);
    route_clock(a.stamps, 9, true);
    if (threadIdx.x == 0) *a.ticket = 0;
}

}  // namespace

int route_tokens_per_pass(int H)
{
    int rt = 65536 / (4 * H);
    return rt < 1 ? 1 : (rt > 8 ? 8 : rt);
}

size_t route_smem_bytes(int H, int rt, int E, int grid, int T)
{
    const int NB = min((T + rt - 1) / rt, kRouteMaxBlockGroups), per = grid / NB;
    return route_smem(H, rt, E, (E + per - 1) / per).total;
}

int route_grid(int E, int T, int rt, int num_sms)
{
    const int ntb = min((T + rt - 1) / rt, kRouteMaxBlockGroups);  // block groups
    int per = (E + 3) / 4;  // row slices: at least one quad of rows each
    if (per * ntb > num_sms) per = num_sms / ntb > 0 ? num_sms / ntb : 1;
    return per * ntb;
}

cudaError_t route_set_attributes()
{
    return cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
}

cudaError_t launch_route(const RouteArgs &a, int grid, cudaStream_t s)
{
    size_t smem = route_smem_bytes(a.H, a.rt, a.E, grid, a.T);
    route_kernel<<<grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
