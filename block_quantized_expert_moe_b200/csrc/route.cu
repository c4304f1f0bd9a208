// Router GEMV + softmax/top-k + device-side plan, fused in one launch.
//
// The "Qwen3.8-Flash-Next UD-IQ2_XS (L4 fix) for Basalt" model card, section
// "What was changed", calls its fast decode path a device-planned MoE tail:
// the per-expert token lists are built on the GPU, with no host round trip.
// Here the plan is built at the end of the router launch:
//
//   phase 1 (all CTAs)   logits[t][e] = sum_h Wr[e][h] x[t][h], fp32 accumulate;
//                        CTA b takes token block b % ntb (8 tokens, staged in
//                        shared memory as fp32 once) and a slice of the expert
//                        rows, one warp per row
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
//                        matvecs, the shared expert's groups last.
//
// "Last" is decided by global tickets (atomicAdd after a fence: one per token
// block, one over blocks); no CTA ever waits on another.
#include <climits>

#include "decode_common.cuh"
#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kRouteMaxBlockGroups = 14;  // per-group tickets at words 2..15 of the ticket area

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
__device__ int block_exclusive_scan(int *v, int n, int *tmp)
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

__device__ void topk_phase(const RouteArgs &a, unsigned char *smem, int t_begin, int t_end)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = kThreads / 32;
    const int E = a.E, k = a.k;
    if (k <= 32 && E <= 1024) {
        // one warp per token: the row into shared memory, then the threshold
        // selection (candidates at or above the k-th largest lane maximum)
        float *row = reinterpret_cast<float *>(smem) + (size_t)warp * (E + 128);
        unsigned *cand = reinterpret_cast<unsigned *>(row + E);
        for (int t = t_begin + warp; t < t_end; t += nw) {
            for (int e = lane; e < E; e += 32) row[e] = __ldcg(a.logits + (size_t)t * E + e);
            __syncwarp();
            int me;
            float mg;
            if (E <= 512) topk_threshold<16>(row, E, k, me, mg, cand);
            else topk_threshold<32>(row, E, k, me, mg, cand);
            if (lane < k) {
                a.idx[(size_t)t * k + lane] = me;
                a.gate[(size_t)t * k + lane] = mg;
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
__device__ void plan_dense(const RouteArgs &a, unsigned char *smem)
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

__device__ void plan_phase(const RouteArgs &a, unsigned char *smem)
{
    const int tid = threadIdx.x;
    const int E = a.E, k = a.k, T = a.T, tt = a.tt;
    unsigned long long *mask = reinterpret_cast<unsigned long long *>(smem);
    int *cnt = reinterpret_cast<int *>(mask + E);
    int *off = cnt + (E + 1);
    int *run = off + (E + 1);
    int *gbase = run + (E + 1);
    int *tmp = gbase + (E + 1);
    for (int e = tid; e < E; e += kThreads) { cnt[e] = 0; run[e] = 0; }
    __syncthreads();
    for (int i = tid; i < T * k; i += kThreads) atomicAdd(&cnt[__ldcg(a.idx + i)], 1);
    __syncthreads();
    for (int e = tid; e < E; e += kThreads) {
        off[e] = cnt[e];
        gbase[e] = (cnt[e] + tt - 1) / tt;
    }
    __syncthreads();
    const int slots = block_exclusive_scan(off, E, tmp);
    const int routed_groups = block_exclusive_scan(gbase, E, tmp);
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
    // stable slot order: within expert e, slots follow token order
    for (int c0 = 0; c0 < T; c0 += 64) {
        const int nt = min(64, T - c0);
        for (int e = tid; e < E; e += kThreads) mask[e] = 0ull;
        __syncthreads();
        for (int i = tid; i < nt * k; i += kThreads) {
            int t = c0 + i / k;
            int e = __ldcg(a.idx + (size_t)t * k + i % k);
            atomicOr(&mask[e], 1ull << (t - c0));
        }
        __syncthreads();
        for (int i = tid; i < nt * k; i += kThreads) {
            int t = c0 + i / k, j = i % k;
            int e = __ldcg(a.idx + (size_t)t * k + j);
            unsigned long long below = (t - c0) ? (mask[e] & ((1ull << (t - c0)) - 1ull)) : 0ull;
            int pos = off[e] + run[e] + __popcll(below);
            a.perm_tok[pos] = t;
            a.slot_pos[(size_t)t * k + j] = pos;
        }
        __syncthreads();
        for (int e = tid; e < E; e += kThreads) run[e] += __popcll(mask[e]);
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kThreads) route_kernel(const RouteArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_last;
    float *xs = reinterpret_cast<float *>(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = kThreads / 32;
    const int H = a.H, E = a.E;
    // CTA b takes token block b % ntb (rt tokens) and a slice of the expert rows,
    // so every CTA stages its tokens once and the grid covers all SMs
    // token blocks of rt tokens, dealt to NB block groups (more blocks than
    // groups: a CTA handles blocks j, j + NB, ...)
    const int ntb = (a.T + a.rt - 1) / a.rt, NB = min(ntb, kRouteMaxBlockGroups), per = gridDim.x / NB;
    const int tb = blockIdx.x % NB, slice = blockIdx.x / NB;
    const int e0 = slice < per ? (int)((long long)E * slice / per) : E;
    const int e1 = slice < per ? (int)((long long)E * (slice + 1) / per) : E;
    const int nch = H >> 3;  // 16-byte chunks of 8 bf16 in a router row
    for (int t0 = tb * a.rt; t0 < a.T && e1 > e0; t0 += NB * a.rt) {
        const int nt = min(a.rt, a.T - t0);
        __syncthreads();
        for (int i0 = threadIdx.x; i0 < nt * nch; i0 += 4 * kThreads) {
            float4 lo[4], hi[4];  // four chunks' loads in flight before any store
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = i0 + q * kThreads;
                if (i >= nt * nch) break;
                const int t = i / nch, c = i - t * nch;
                if (a.x_dtype == MOE_DT_BF16) {
                    uint4 v = ldg_nc16(reinterpret_cast<const uint16_t *>(a.x) + (size_t)(t0 + t) * H + c * 8);
                    lo[q] = make_float4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y));
                    hi[q] = make_float4(bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w));
                } else {
                    const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.x) +
                                                                       (size_t)(t0 + t) * H + c * 8);
                    lo[q] = __ldg(p);
                    hi[q] = __ldg(p + 1);
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = i0 + q * kThreads;
                if (i >= nt * nch) break;
                const int t = i / nch, c = i - t * nch;
                float4 *d = reinterpret_cast<float4 *>(xs + (size_t)t * H + c * 8);
                d[0] = lo[q];
                d[1] = hi[q];
            }
        }
        __syncthreads();
        for (int e = e0 + warp; e < e1; e += nw) {
            const uint16_t *wrow = a.wr + (size_t)e * H;
            float acc[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) acc[t] = 0.f;
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
                    float w0 = bf16lo(wv[i].x), w1 = bf16hi(wv[i].x), w2 = bf16lo(wv[i].y), w3 = bf16hi(wv[i].y);
                    float w4 = bf16lo(wv[i].z), w5 = bf16hi(wv[i].z), w6 = bf16lo(wv[i].w), w7 = bf16hi(wv[i].w);
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        if (t < nt) {
                            const float4 *xp = reinterpret_cast<const float4 *>(xs + (size_t)t * H + c * 8);
                            float4 x0 = xp[0], x1 = xp[1];
                            float s = acc[t];
                            s = fmaf(w0, x0.x, s); s = fmaf(w1, x0.y, s);
                            s = fmaf(w2, x0.z, s); s = fmaf(w3, x0.w, s);
                            s = fmaf(w4, x1.x, s); s = fmaf(w5, x1.y, s);
                            s = fmaf(w6, x1.z, s); s = fmaf(w7, x1.w, s);
                            acc[t] = s;
                        }
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                float v = acc[t];
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0 && t < nt) a.logits[(size_t)(t0 + t) * E + e] = v;
            }
        }
    }
    // the last CTA of this token block selects its tokens' experts; the last
    // token block to finish builds the plan (tickets: [0] blocks, [2 + tb] CTAs)
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int ticket = atomicAdd(a.ticket + 2 + tb, 1);
        s_last = ticket == per - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int t0 = tb * a.rt; t0 < a.T; t0 += NB * a.rt) topk_phase(a, smem, t0, min(a.T, t0 + a.rt));
    __syncthreads();
    if (threadIdx.x == 0) {
        a.ticket[2 + tb] = 0;
        __threadfence();
        const int ticket = atomicAdd(a.ticket, 1);
        s_last = ticket == NB - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (a.do_plan) {
        __syncthreads();
        if (a.dense) plan_dense(a, smem);
        else plan_phase(a, smem);
    }
    __syncthreads();
    if (threadIdx.x == 0) *a.ticket = 0;
}

}  // namespace

int route_tokens_per_pass(int H)
{
    int rt = 65536 / (4 * H);
    return rt < 1 ? 1 : (rt > 8 ? 8 : rt);
}

size_t route_smem_bytes(int H, int rt, int E)
{
    size_t stage = (size_t)rt * H * sizeof(float);
    size_t topk = (size_t)2 * (kThreads / 32) * E * sizeof(float) + (kThreads / 32) * 32 * sizeof(uint32_t);
    const size_t topk_thr = (size_t)(kThreads / 32) * (E + 128) * sizeof(float);  // row + candidates per warp
    if (topk_thr > topk) topk = topk_thr;
    size_t plan = (size_t)E * 8 + (size_t)4 * (E + 1) * sizeof(int) + 64 * sizeof(int);
    size_t m = stage > topk ? stage : topk;
    return m > plan ? m : plan;
}

int route_grid(int E, int T, int rt, int num_sms)
{
    const int ntb = min((T + rt - 1) / rt, kRouteMaxBlockGroups);  // block groups
    int per = (E + (kThreads / 32) - 1) / (kThreads / 32);  // row slices: >= one warp's row each
    if (per * ntb > num_sms) per = num_sms / ntb > 0 ? num_sms / ntb : 1;
    return per * ntb;
}

cudaError_t route_set_attributes()
{
    return cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
}

cudaError_t launch_route(const RouteArgs &a, int grid, cudaStream_t s)
{
    size_t smem = route_smem_bytes(a.H, a.rt, a.E);
    route_kernel<<<grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
