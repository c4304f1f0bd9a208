// Pieces shared by the one-launch decode kernels: the bounded grid-wide
// barrier, the warp top-k of one token's router logits and the lane split of a
// row's 32-weight units.
#pragma once

#include <climits>
#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(unsigned *p, unsigned v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid-wide barrier; false (and *err = MOE_ERR_TIMEOUT) if the wait ran out.
__device__ bool grid_sync(unsigned *bar, int32_t *err)
{
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned gen = ld_acquire(bar + 1);
        __threadfence();
        const unsigned arrived = atomicAdd(bar, 1u) + 1u;
        int ok = 1;
        if (arrived == gridDim.x) {
            bar[0] = 0u;
            st_release(bar + 1, gen + 1u);
        } else {
            const long long t0 = clock64();
            while (ld_acquire(bar + 1) == gen) {
                if (clock64() - t0 > (1ll << 32)) {
                    atomicExch(err, (int)MOE_ERR_TIMEOUT);
                    ok = 0;
                    break;
                }
                __nanosleep(64);
            }
        }
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

// Order-preserving key of a float (larger float -> larger unsigned key).
__device__ __forceinline__ unsigned fkey(float f)
{
    const unsigned u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k of one token's logits by warp `warp`: k rounds of (lane-local best,
// warp max of the order-preserving key with redux, lowest index among the
// lanes holding it).  Writes the selected experts (descending logit) and gates.
__device__ void warp_topk(const FusedArgs &a, int t, int *sel_e, float *sel_g)
{
    const int lane = threadIdx.x & 31;
    const int E = a.E, k = a.k;
    float v[32];
    uint32_t taken = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int e = lane + 32 * i;
        if (e < E) v[i] = __ldcg(a.logits + (size_t)t * E + e);
        else { v[i] = -INFINITY; taken |= 1u << i; }
    }
    float vmax = 0.f, den = 0.f;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 32;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (!((taken >> i) & 1u) && (bi == 32 || v[i] > bv)) {
                bv = v[i];
                bi = i;
            }
        const unsigned key = bi < 32 ? fkey(bv) : 0u;
        const unsigned kmax = __reduce_max_sync(0xffffffffu, key);
        const unsigned cand = (key == kmax && bi < 32) ? (unsigned)(lane + 32 * bi) : 0xffffffffu;
        const unsigned win = __reduce_min_sync(0xffffffffu, cand);
        if ((int)(win & 31) == lane) taken |= 1u << (win >> 5);
        const float wv = __shfl_sync(0xffffffffu, bv, win & 31);
        if (j == 0) vmax = wv;
        den += expf(wv - vmax);
        if (lane == 0) {
            sel_e[t * k + j] = (int)win;
            sel_g[t * k + j] = wv;  // logit for now, gate below
        }
    }
    __syncwarp();
    if (lane < k) sel_g[t * k + lane] = expf(sel_g[t * k + lane] - vmax) / den;
    __syncwarp();
}

__device__ __forceinline__ int lanes_per_row(int NU)
{
    return NU >= 32 ? 32 : NU >= 16 ? 16 : NU >= 8 ? 8 : NU >= 4 ? 4 : NU >= 2 ? 2 : 1;
}

__device__ __forceinline__ float key_to_float(unsigned key)
{
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Row t of the logits into shared memory with all of a lane's loads in flight
// (a loop of dependent load/store pairs would pay one L2 round trip per
// element of the lane).
template <int NPL>
__device__ __forceinline__ void stage_logits(const float *src, float *row, int E, int lane)
{
    float v[NPL];
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
        const int e = lane + 32 * j;
        v[j] = e < E ? __ldcg(src + e) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
        const int e = lane + 32 * j;
        if (e < E) row[e] = v[j];
    }
}

// Best (largest key, lowest position on ties) of a lane's NPL keys, as a tree.
template <int NPL>
__device__ __forceinline__ void lane_best(const unsigned (&key)[NPL], unsigned &bk, int &bi)
{
    unsigned k[NPL];
    int ix[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        k[i] = key[i];
        ix[i] = i;
    }
#pragma unroll
    for (int w = 1; w < NPL; w <<= 1) {
#pragma unroll
        for (int i = 0; i < NPL; i += 2 * w) {
            const bool p = k[i + w] > k[i];  // right side wins only if strictly larger
            k[i] = p ? k[i + w] : k[i];
            ix[i] = p ? ix[i + w] : ix[i];
        }
    }
    bk = k[0];
    bi = ix[0];
}

// Warp-wide top-k over one token's logits (k <= 32), held in shared memory:
// lane l takes logits e = l + 32 i as order-preserving keys.  The candidates
// are the keys at or above the k-th largest lane maximum (at least k keys
// reach it, so every selected key is among them); when at most 32, each is
// ranked against all of them (larger key first, then lower expert id) in one
// pass; otherwise k rounds of warp maxima.  `cand` is 128 words of shared
// scratch.  Lane j < k ends with the j-th selected expert and its gate.
template <int NPL>
__device__ void topk_threshold(const float *lg, int E, int k, int &my_e, float &my_g, unsigned *cand)
{
    const int lane = threadIdx.x & 31;
    unsigned key[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) key[i] = lane + 32 * i < E ? fkey(lg[lane + 32 * i]) : 0u;
    float my_l = 0.f;
    my_e = 0;
    // threshold: the k-th largest of the 32 lane maxima; at least k keys reach
    // it, so it bounds the k-th largest key from below and every selected key
    // is among the keys >= theta
    unsigned lm = 0u;
#pragma unroll
    for (int i = 0; i < NPL; ++i) lm = max(lm, key[i]);
    int lrank = 0;
#pragma unroll
    for (int l = 0; l < 32; ++l) {  // independent shuffles: fully unrolled
        const unsigned o = __shfl_sync(0xffffffffu, lm, l);
        lrank += (o > lm || (o == lm && l < lane)) ? 1 : 0;
    }
    const unsigned tb = __ballot_sync(0xffffffffu, lrank == k - 1);
    const unsigned theta = __shfl_sync(0xffffffffu, lm, __ffs(tb) - 1);
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) cnt += key[i] >= theta ? 1 : 0;
    const int total = (int)__reduce_add_sync(0xffffffffu, (unsigned)cnt);
    if (total <= 32) {
        // gather the candidates, then rank each against all of them
        int pos = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, pos, o);
            if (lane >= o) pos += v;
        }
        pos -= cnt;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (key[i] >= theta) {
                cand[pos] = key[i];
                cand[32 + pos] = (unsigned)(lane + 32 * i);
                ++pos;
            }
        __syncwarp();
        const unsigned ck = lane < total ? cand[lane] : 0u, ce = lane < total ? cand[32 + lane] : 0xffffffffu;
        // lanes >= total hold key 0 / id ~0, which never outrank a candidate:
        // a fixed 32-step, fully unrolled loop needs no bound
        int r = 0;
#pragma unroll
        for (int q = 0; q < 32; ++q) {
            const unsigned qk = __shfl_sync(0xffffffffu, ck, q), qe = __shfl_sync(0xffffffffu, ce, q);
            r += (qk > ck || (qk == ck && qe < ce)) ? 1 : 0;
        }
        __syncwarp();
        if (lane < total && r < k) {
            cand[64 + r] = ck;
            cand[96 + r] = ce;
        }
        __syncwarp();
        if (lane < k) {
            my_e = (int)cand[96 + lane];
            my_l = key_to_float(cand[64 + lane]);
        }
    } else {
        // many keys tie at the top: k rounds of warp maximum
        unsigned bk;
        int bi;
        lane_best<NPL>(key, bk, bi);
        for (int j = 0; j < k; ++j) {
            const unsigned kmax = __reduce_max_sync(0xffffffffu, bk);
            const unsigned cnd = (bk == kmax) ? (unsigned)(lane + 32 * bi) : 0xffffffffu;
            const unsigned win = __reduce_min_sync(0xffffffffu, cnd);
            if (lane == j) {
                my_e = (int)win;
                my_l = key_to_float(kmax);
            }
            if ((int)(win & 31) == lane) {
                const int taken = (int)(win >> 5);
#pragma unroll
                for (int i = 0; i < NPL; ++i)
                    if (i == taken) key[i] = 0u;
                lane_best<NPL>(key, bk, bi);
            }
        }
    }
    // renormalised softmax over the selected logits: exp(l_j - l_max) / sum
    const float lmax = __shfl_sync(0xffffffffu, my_l, 0);
    const float ex = lane < k ? expf(my_l - lmax) : 0.f;
    float den = ex;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    my_g = ex / den;
}

}  // namespace
}  // namespace moe
