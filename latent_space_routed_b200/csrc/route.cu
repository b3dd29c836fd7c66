// Selection and dispatch: biased top-k with raw-score renormalisation, and a
// stable counting sort of the T*k (token, slot) pairs by expert.
//
// Selection ("Stable LatentMoE", equations for T_k(x) and p_i): s = r + b,
// T_k = TopK(s, k) with equal scores going to the lower expert index (the
// cooking-agi LatentMoE page's routed_example picks index 0 when v0 >= v1),
// p_i = r_i / sum_{j in T_k} r_j over the raw scores r.
//
// Dispatch: slot rows are ordered by (expert, token); a token selects an
// expert at most once, so the position of (t, j) with e = sel[t, j] is
//   offsets[e] + #{t' < t : t' selected e}.
// The top-k kernel (one warp per token) counts each expert's selections per
// block of ROUTE_TPB tokens, one block scans the counts over blocks and
// experts (scan kernel), and each block of ROUTE_TPB tokens ranks its tokens
// within an expert with a bit mask and popcounts (dispatch kernel).
// Integer-only, hence bit-exact and deterministic.
#include <float.h>

#include "lmoe_internal.cuh"

namespace lmoe {
namespace {

constexpr int TOPK_WARPS = 8;   // one token per warp, 8 tokens per block
constexpr int KMAX = 64;

template <typename TO>
__global__ void __launch_bounds__(TOPK_WARPS * 32)
topk_kernel(const float *__restrict__ r, const float *__restrict__ bias, int64_t T, int E, int k,
            int32_t *__restrict__ sel, float *__restrict__ p32, TO *__restrict__ p_out,
            int32_t *__restrict__ blockhist)
{
    extern __shared__ float smem[];
    __shared__ int chosen[TOPK_WARPS][KMAX];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float *sw = smem + warp * 2 * E;   // biased scores of this warp's token (taken -> -inf)
    float *rw = sw + E;                // raw scores
    const int64_t t = (int64_t)blockIdx.x * TOPK_WARPS + warp;
    if (t >= T) return;
    for (int e = lane; e < E; e += 32) {
        const float rv = r[t * E + e];
        rw[e] = rv;
        // NaN / -inf map to -FLT_MAX so that a candidate always exists and
        // the chosen index stays in range whatever the input holds
        sw[e] = fmaxf(rv + bias[e], -FLT_MAX);
    }
    __syncwarp();
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            const float v = sw[e];
            if (v > bv) { bv = v; bi = e; }   // ascending e: strict > keeps the lower index
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if (lane == 0) {
            chosen[warp][j] = bi;
            sw[bi] = -INFINITY;
        }
        __syncwarp();
    }
    float sum = 0.f;   // every lane sums in selection order: identical result
    for (int j = 0; j < k; ++j) sum += rw[chosen[warp][j]];
    int32_t *hist = blockhist + (t / ROUTE_TPB) * E;
    for (int j = lane; j < k; j += 32) {
        const int e = chosen[warp][j];
        const float p = rw[e] / sum;
        sel[t * k + j] = e;
        p32[t * k + j] = p;
        p_out[t * k + j] = from_f32<TO>(p);
        atomicAdd(&hist[e], 1);
    }
}

// One block: per-expert totals and per-(block, expert) starting positions.
__global__ void __launch_bounds__(1024)
scan_kernel(const int32_t *__restrict__ blockhist, int nb, int E, int bm, int32_t *__restrict__ counts,
            int32_t *__restrict__ offsets, int32_t *__restrict__ base, int32_t *__restrict__ tile_off)
{
    __shared__ int s_cnt[1024];
    __shared__ int s_tiles[1024];
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += blockDim.x) {
        int run = 0;
        for (int b = 0; b < nb; ++b) {
            const int64_t i = (int64_t)b * E + e;
            const int h = blockhist[i];
            base[i] = run;
            run += h;
        }
        counts[e] = run;
        s_cnt[e] = run;
        s_tiles[e] = (run + bm - 1) / bm;
    }
    __syncthreads();
    if (tid == 0) {   // E <= 1024: a serial exclusive scan is a few microseconds at most
        int acc = 0, tacc = 0;
        for (int e = 0; e < E; ++e) {
            offsets[e] = acc;
            tile_off[e] = tacc;
            const int c = s_cnt[e], tt = s_tiles[e];
            s_cnt[e] = acc;
            acc += c;
            tacc += tt;
        }
        offsets[E] = acc;
        tile_off[E] = tacc;
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        const int off = s_cnt[e];
        for (int b = 0; b < nb; ++b) base[(int64_t)b * E + e] += off;
    }
}

constexpr int WORDS = ROUTE_TPB / 32;

__global__ void __launch_bounds__(256)
dispatch_kernel(const int32_t *__restrict__ sel, const float *__restrict__ p32, const int32_t *__restrict__ base,
                int64_t T, int E, int k, int32_t *__restrict__ slot_of, int32_t *__restrict__ perm_tok,
                float *__restrict__ perm_w)
{
    extern __shared__ uint32_t bits[];   // [E][WORDS]: bit i of expert e = token t_begin+i chose e
    const int64_t t_begin = (int64_t)blockIdx.x * ROUTE_TPB;
    const int ntok = (int)min((int64_t)ROUTE_TPB, T - t_begin);
    for (int i = threadIdx.x; i < E * WORDS; i += blockDim.x) bits[i] = 0u;
    __syncthreads();
    const int n = ntok * k;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int tl = i / k;
        const int e = sel[t_begin * k + i];
        atomicOr(&bits[e * WORDS + (tl >> 5)], 1u << (tl & 31));
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int tl = i / k;
        const int e = sel[t_begin * k + i];
        const uint32_t *w = bits + e * WORDS;
        int rank = __popc(w[tl >> 5] & ((1u << (tl & 31)) - 1u));
        for (int q = 0; q < (tl >> 5); ++q) rank += __popc(w[q]);
        const int pos = base[(int64_t)blockIdx.x * E + e] + rank;
        slot_of[t_begin * k + i] = pos;
        perm_tok[pos] = (int32_t)(t_begin + tl);
        perm_w[pos] = p32[t_begin * k + i];
    }
}

// Router for a few tokens: one block per (expert row e, ROUTER_TB tokens).
// The block's 8 warps stream W[e] (fp32, 16-byte loads) in interleaved
// 512-byte pieces against the same columns of each token; each warp adds its
// lanes in a fixed butterfly order and the warps' partial sums are added in
// warp order, so the result does not depend on timing.
constexpr int ROUTER_TB = 8;
constexpr int ROUTER_WARPS = 8;

__global__ void __launch_bounds__(ROUTER_WARPS * 32)
router_small_kernel(const bf16 *__restrict__ x, const float *__restrict__ W, int64_t T, int E, int d,
                    float *__restrict__ r)
{
    __shared__ float part[ROUTER_WARPS][ROUTER_TB];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.x;
    const int64_t t0 = (int64_t)blockIdx.y * ROUTER_TB;
    float acc[ROUTER_TB];
#pragma unroll
    for (int j = 0; j < ROUTER_TB; ++j) acc[j] = 0.f;
    const float4 *w = reinterpret_cast<const float4 *>(W + (int64_t)e * d);
    for (int c = warp * 32 + lane; c < d / 4; c += ROUTER_WARPS * 32) {
        const float4 wv = __ldg(w + c);
#pragma unroll
        for (int j = 0; j < ROUTER_TB; ++j) {
            if (t0 + j < T) {
                const uint2 xv = __ldg(reinterpret_cast<const uint2 *>(x + (t0 + j) * d) + c);
                const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xv.x));
                const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xv.y));
                acc[j] = fmaf(wv.x, a.x, acc[j]);
                acc[j] = fmaf(wv.y, a.y, acc[j]);
                acc[j] = fmaf(wv.z, b.x, acc[j]);
                acc[j] = fmaf(wv.w, b.y, acc[j]);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < ROUTER_TB; ++j) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
    }
    if (lane == 0) {
#pragma unroll
        for (int j = 0; j < ROUTER_TB; ++j) part[warp][j] = acc[j];
    }
    __syncthreads();
    if (threadIdx.x < ROUTER_TB && t0 + threadIdx.x < T) {
        float a = 0.f;
#pragma unroll
        for (int q = 0; q < ROUTER_WARPS; ++q) a += part[q][threadIdx.x];
        r[(t0 + threadIdx.x) * E + e] = sigmoidf_(a);
    }
}

// Zp[m, :] = z[perm_tok[m], :]: one warp per slot row, 16-byte vectors.
__global__ void __launch_bounds__(256)
permute_rows_kernel(const uint4 *__restrict__ z, const int32_t *__restrict__ perm_tok, uint4 *__restrict__ Zp,
                    int64_t S, int vec_per_row)
{
    const int64_t m = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (m >= S) return;
    const int lane = threadIdx.x & 31;
    const uint4 *src = z + (int64_t)perm_tok[m] * vec_per_row;
    uint4 *dst = Zp + m * vec_per_row;
    for (int i = lane; i < vec_per_row; i += 32) dst[i] = src[i];
}

}  // namespace

cudaError_t launch_router_small(const bf16 *x, const float *W, int64_t T, int E, int d, float *r, cudaStream_t s)
{
    if (T == 0) return cudaSuccess;
    if (d % 4) return cudaErrorInvalidValue;
    dim3 grid((unsigned)E, (unsigned)((T + ROUTER_TB - 1) / ROUTER_TB));
    router_small_kernel<<<grid, ROUTER_WARPS * 32, 0, s>>>(x, W, T, E, d, r);
    return cudaGetLastError();
}

cudaError_t launch_permute_rows(const void *z, const int32_t *perm_tok, void *Zp, int64_t S, int l, int elem_bytes,
                                cudaStream_t s)
{
    if (S == 0) return cudaSuccess;
    if (((int64_t)l * elem_bytes) % 16) return cudaErrorInvalidValue;
    const int vpr = (int)((int64_t)l * elem_bytes / 16);
    permute_rows_kernel<<<(unsigned)((S + 7) / 8), 256, 0, s>>>((const uint4 *)z, perm_tok, (uint4 *)Zp, S, vpr);
    return cudaGetLastError();
}

cudaError_t launch_topk(const float *r, const float *bias, int64_t T, int E, int k, int32_t *sel, float *p32,
                        void *p_out, int out_bf16, int32_t *blockhist, cudaStream_t s)
{
    if (k > KMAX) return cudaErrorInvalidValue;
    const int64_t nhb = (T + ROUTE_TPB - 1) / ROUTE_TPB;
    cudaError_t e = cudaMemsetAsync(blockhist, 0, sizeof(int32_t) * nhb * E, s);
    if (e != cudaSuccess) return e;
    const unsigned nb = (unsigned)((T + TOPK_WARPS - 1) / TOPK_WARPS);
    const size_t smem = sizeof(float) * 2 * TOPK_WARPS * E;
    if (out_bf16) {
        cudaFuncSetAttribute(topk_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        topk_kernel<bf16><<<nb, TOPK_WARPS * 32, smem, s>>>(r, bias, T, E, k, sel, p32, (bf16 *)p_out, blockhist);
    } else {
        cudaFuncSetAttribute(topk_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        topk_kernel<float><<<nb, TOPK_WARPS * 32, smem, s>>>(r, bias, T, E, k, sel, p32, (float *)p_out,
                                                               blockhist);
    }
    return cudaGetLastError();
}

cudaError_t launch_scan(const int32_t *blockhist, int nb, int E, int bm, int32_t *counts, int32_t *offsets,
                        int32_t *base, int32_t *tile_off, cudaStream_t s)
{
    if (E > 1024) return cudaErrorInvalidValue;
    scan_kernel<<<1, 1024, 0, s>>>(blockhist, nb, E, bm, counts, offsets, base, tile_off);
    return cudaGetLastError();
}

cudaError_t launch_dispatch(const int32_t *sel, const float *p32, const int32_t *base, int64_t T, int E, int k,
                            int32_t *slot_of, int32_t *perm_tok, float *perm_w, cudaStream_t s)
{
    const int nb = (int)((T + ROUTE_TPB - 1) / ROUTE_TPB);
    const size_t smem = sizeof(uint32_t) * E * WORDS;
    dispatch_kernel<<<nb, 256, smem, s>>>(sel, p32, base, T, E, k, slot_of, perm_tok, perm_w);
    return cudaGetLastError();
}

}  // namespace lmoe
