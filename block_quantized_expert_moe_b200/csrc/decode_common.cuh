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

}  // namespace
}  // namespace moe
