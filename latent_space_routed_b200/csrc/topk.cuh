// Biased top-k of one token held by a warp ("Stable LatentMoE", equation for
// T_k(x): TopK(r + b, k); equal scores go to the lower expert index, as the
// cooking-agi LatentMoE page's routed_example picks index 0 when v0 >= v1).
// Shared by the routing kernels and the tensor-core router's fused epilogue.
#pragma once

#include <float.h>

#include "lmoe_internal.cuh"

namespace lmoe {

// "a before b": larger biased score first, equal scores to the lower index.
__device__ __forceinline__ bool ahead(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

// Bitonic sort of a lane's N (score, expert) pairs into "ahead" order, in registers.
template <int N>
__device__ __forceinline__ void sort_lane(float (&v)[N], int (&ix)[N])
{
#pragma unroll
    for (int kk = 2; kk <= N; kk <<= 1)
#pragma unroll
        for (int j = kk >> 1; j > 0; j >>= 1)
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int m = i ^ j;
                if (m > i) {
                    const bool first_ahead = ahead(v[i], ix[i], v[m], ix[m]);
                    if (((i & kk) == 0) != first_ahead) {
                        const float tv = v[i]; v[i] = v[m]; v[m] = tv;
                        const int ti = ix[i]; ix[i] = ix[m]; ix[m] = ti;
                    }
                }
            }
}

// Order-preserving 32-bit key of a score: a > b as floats exactly when
// key(a) > key(b) as unsigned integers (for -0 and +0 alike only if the caller
// made -0 into +0, which it does).
__device__ __forceinline__ uint32_t score_key(float v)
{
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k of one token held by a warp.  Lane L holds experts L, L + 32, ...
// (EPL of them, padded with -inf) as (biased score, expert) pairs, sorts them,
// and the k rounds are a tournament over the 32 lane heads: the largest head
// score (one warp max-reduction over the score keys), then the lowest expert
// index among the heads with that score (one min-reduction), so equal scores
// go to the lower index; the winning lane pops its head.  Selection j is kept
// by lane j % 32 (in *mine0 for j < 32, *mine1 above).  One more round gives
// the (k+1)-th biased score, the Quantile-Balancing cutoff (-inf when k = E).
template <int EPL>
__device__ __forceinline__ void warp_topk(float (&v)[EPL], int (&ix)[EPL], int k, int E, int lane, int *mine0,
                                          int *mine1, float *cut)
{
    sort_lane<EPL>(v, ix);
    int m0 = 0, m1 = 0;
    for (int j = 0; j < k; ++j) {
        const uint32_t key = score_key(v[0]);
        const uint32_t best = __reduce_max_sync(0xffffffffu, key);
        const int bi = (int)__reduce_min_sync(0xffffffffu, key == best ? (uint32_t)ix[0] : 0xffffffffu);
        if (lane == (bi & 31)) {            // the winner pops its head
#pragma unroll
            for (int i = 0; i + 1 < EPL; ++i) { v[i] = v[i + 1]; ix[i] = ix[i + 1]; }
            v[EPL - 1] = -INFINITY;
            ix[EPL - 1] = 0x7fffffff;
        }
        if (lane == (j & 31)) {
            if (j < 32) m0 = bi; else m1 = bi;
        }
    }
    const uint32_t key = score_key(v[0]);
    const uint32_t best = __reduce_max_sync(0xffffffffu, key);
    const int bi = (int)__reduce_min_sync(0xffffffffu, key == best ? (uint32_t)ix[0] : 0xffffffffu);
    const float cv = __shfl_sync(0xffffffffu, v[0], bi & 31);
    *cut = k < E ? cv : -INFINITY;
    *mine0 = m0;
    *mine1 = m1;
}

// Biased key of expert e for the tournament: NaN / -inf map to -FLT_MAX so
// that a real candidate always beats the padding; adding +0 turns -0 into +0,
// so equal scores get equal keys.
__device__ __forceinline__ float biased_key(float r, float b) { return fmaxf(r + b, -FLT_MAX) + 0.0f; }

}  // namespace lmoe
