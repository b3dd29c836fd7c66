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
// block of ROUTE_TPB tokens (expert-major), one block per expert scans its
// counts over the token blocks (scan kernel), and each block of ROUTE_TPB
// tokens scans the expert totals into offsets and ranks its tokens within an
// expert with one bit word per expert and popcounts (dispatch kernel).
// Integer-only, hence bit-exact and deterministic.
#include <float.h>

#include "lmoe_internal.cuh"

namespace lmoe {
namespace {

constexpr int TOPK_WARPS = 8;   // one token per warp, 8 tokens per block
constexpr int KMAX = 64;

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

// Top-k for one token per warp.  Lane L holds experts L, L + 32, ... (EPL of
// them, padded with -inf), sorts them, and the k rounds are a tournament over
// the 32 lane heads: the largest head score (one warp max-reduction over the
// score keys), then the lowest expert index among the heads with that score
// (one min-reduction), so equal scores go to the lower index; the winning lane
// pops its head.  The raw scores of the chosen experts are normalised by their
// sum (a fixed butterfly order, so the result does not depend on timing).
//
// nsplit = 0: r_in holds the router scores r [T, E].  nsplit > 0: r_in holds
// nsplit fp32 partial slabs [nsplit, T, E] of the router logits (split-K
// GEMM); the kernel sums them in slab order, applies the sigmoid and writes r
// to r_out.
template <typename TO, int EPL>
__global__ void __launch_bounds__(TOPK_WARPS * 32)
topk_kernel(const float *__restrict__ r_in, int nsplit, float *r_out, const float *__restrict__ bias, int64_t T,
            int E, int k, int32_t *__restrict__ sel, float *__restrict__ p32, TO *__restrict__ p_out,
            int32_t *__restrict__ blockhist, int nb, float *__restrict__ cutoff)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t = (int64_t)blockIdx.x * TOPK_WARPS + warp;
    if (t >= T) return;
    float v[EPL];
    int ix[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        ix[i] = e;
        float r = 0.f;
        if (e < E) {
            if (nsplit == 0) {
                r = r_in[t * E + e];
            } else {
                float a = 0.f;
                for (int q = 0; q < nsplit; ++q) a += r_in[((int64_t)q * T + t) * E + e];
                r = sigmoidf_(a);
                r_out[t * E + e] = r;
            }
        }
        // NaN / -inf map to -FLT_MAX so that a real candidate always beats the
        // padding; adding +0 turns -0 into +0, so equal scores get equal keys
        v[i] = e < E ? fmaxf(r + bias[e], -FLT_MAX) + 0.0f : -INFINITY;
    }
    sort_lane<EPL>(v, ix);
    int mine0 = 0, mine1 = 0;    // selection j kept by lane j % 32 (slot j / 32)
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
            if (j < 32) mine0 = bi; else mine1 = bi;
        }
    }
    // Quantile-Balancing cutoff: the (k+1)-th biased score, one more round
    // (-inf when k = E leaves nothing unselected)
    {
        const uint32_t key = score_key(v[0]);
        const uint32_t best = __reduce_max_sync(0xffffffffu, key);
        const int bi = (int)__reduce_min_sync(0xffffffffu, key == best ? (uint32_t)ix[0] : 0xffffffffu);
        const float cv = __shfl_sync(0xffffffffu, v[0], bi & 31);
        if (lane == 0) cutoff[t] = k < E ? cv : -INFINITY;
    }
    const float *rr = nsplit ? r_out : r_in;
    if (nsplit) __syncwarp();               // r_out of this token, written by every lane, is visible
    const float r0 = lane < k ? rr[t * E + mine0] : 0.f;
    const float r1 = lane + 32 < k ? rr[t * E + mine1] : 0.f;
    float sum = r0 + r1;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const int64_t tb = t / ROUTE_TPB;   // counts are expert-major: blockhist[e][token block]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int j = lane + 32 * h;
        if (j < k) {
            const int e = h ? mine1 : mine0;
            const float p = (h ? r1 : r0) / sum;
            sel[t * k + j] = e;
            p32[t * k + j] = p;
            p_out[t * k + j] = from_f32<TO>(p);
            atomicAdd(&blockhist[(int64_t)e * nb + tb], 1);
        }
    }
}

// Exclusive scan of one int per thread over an NT-thread block; returns this
// thread's exclusive prefix and the block total in *total.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int *s_warp, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < NT / 32 ? s_warp[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += o;
        }
        if (lane < NT / 32) s_warp[lane] = w;   // inclusive over warps
    }
    __syncthreads();
    const int before = warp ? s_warp[warp - 1] : 0;
    *total = s_warp[NT / 32 - 1];
    __syncthreads();
    return before + incl - v;
}

// One block per expert: the expert's per-token-block counts (contiguous,
// expert-major) are scanned into per-block starting ranks within the expert,
// and their total is the expert's count.  Chunks of SCAN_NT * 4 token blocks
// are scanned in order with a running carry.
constexpr int SCAN_NT = 256;

__global__ void __launch_bounds__(SCAN_NT)
scan_cols_kernel(const int32_t *__restrict__ blockhist, int nb, int32_t *__restrict__ base,
                 int32_t *__restrict__ counts)
{
    __shared__ int s_warp[SCAN_NT / 32];
    const int e = blockIdx.x;
    const int32_t *h = blockhist + (int64_t)e * nb;
    int32_t *o = base + (int64_t)e * nb;
    int carry = 0;
    for (int c0 = 0; c0 < nb; c0 += SCAN_NT * 4) {
        const int i0 = c0 + threadIdx.x * 4;
        int v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = (i0 + q < nb) ? h[i0 + q] : 0;
        int total = 0;
        int run = carry + block_exclusive_scan<SCAN_NT>(v[0] + v[1] + v[2] + v[3], s_warp, &total);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (i0 + q < nb) o[i0 + q] = run;
            run += v[q];
        }
        carry += total;
    }
    if (threadIdx.x == 0) counts[e] = carry;
}

// Dispatch for one block of ROUTE_TPB = 32 tokens.  Every block first scans
// the expert counts into expert offsets (block 0 also publishes the offsets
// and the m-tile prefix of the grouped GEMMs), marks which of its tokens chose
// each expert in one bit word per expert, and places slot (t, j) with
// e = sel[t, j] at offsets[e] + base[e][block] + #{earlier tokens of this
// block that chose e}.
constexpr int DISP_NT = 256;

__global__ void __launch_bounds__(DISP_NT)
dispatch_kernel(const int32_t *__restrict__ sel, const float *__restrict__ p32, const int32_t *__restrict__ base,
                const int32_t *__restrict__ counts, int64_t T, int E, int k, int nb, int bm,
                int32_t *__restrict__ offsets, int32_t *__restrict__ tile_off, int32_t *__restrict__ slot_of,
                int32_t *__restrict__ perm_tok, float *__restrict__ perm_w)
{
    extern __shared__ int s_dyn[];
    int *s_off = s_dyn;                             // [E + 1]
    uint32_t *bits = (uint32_t *)(s_dyn + E + 1);   // [E]
    __shared__ int s_warp[DISP_NT / 32];
    {   // expert offsets: E <= 1024 counts, four per thread
        const int e0 = threadIdx.x * 4;
        int v[4], tv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            v[q] = (e0 + q < E) ? counts[e0 + q] : 0;
            tv[q] = (v[q] + bm - 1) / bm;
        }
        int total = 0;
        int run = block_exclusive_scan<DISP_NT>(v[0] + v[1] + v[2] + v[3], s_warp, &total);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (e0 + q < E) s_off[e0 + q] = run;
            run += v[q];
        }
        if (threadIdx.x == 0) s_off[E] = total;
        if (blockIdx.x == 0) {   // uniform across the block
            int ttot = 0;
            int trun = block_exclusive_scan<DISP_NT>(tv[0] + tv[1] + tv[2] + tv[3], s_warp, &ttot);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (e0 + q < E) tile_off[e0 + q] = trun;
                trun += tv[q];
            }
            if (threadIdx.x == 0) tile_off[E] = ttot;
        }
    }
    for (int i = threadIdx.x; i < E; i += DISP_NT) bits[i] = 0u;
    __syncthreads();
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i <= E; i += DISP_NT) offsets[i] = s_off[i];
    const int64_t t_begin = (int64_t)blockIdx.x * ROUTE_TPB;
    const int ntok = (int)min((int64_t)ROUTE_TPB, T - t_begin);
    const int n = ntok * k;
    for (int i = threadIdx.x; i < n; i += DISP_NT) {
        const int tl = i / k;
        atomicOr(&bits[sel[t_begin * k + i]], 1u << tl);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += DISP_NT) {
        const int tl = i / k;
        const int e = sel[t_begin * k + i];
        const int rank = __popc(bits[e] & ((1u << tl) - 1u));
        const int pos = s_off[e] + base[(int64_t)e * nb + blockIdx.x] + rank;
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

namespace {

template <typename TO, int EPL>
cudaError_t run_topk(const float *r_in, int nsplit, float *r_out, const float *bias, int64_t T, int E, int k,
                     int32_t *sel, float *p32, void *p_out, int32_t *blockhist, int nb, float *cutoff, cudaStream_t s)
{
    const unsigned nblk = (unsigned)((T + TOPK_WARPS - 1) / TOPK_WARPS);
    topk_kernel<TO, EPL><<<nblk, TOPK_WARPS * 32, 0, s>>>(r_in, nsplit, r_out, bias, T, E, k, sel, p32, (TO *)p_out,
                                                         blockhist, nb, cutoff);
    return cudaGetLastError();
}

template <typename TO>
cudaError_t run_topk_epl(const float *r_in, int nsplit, float *r_out, const float *bias, int64_t T, int E, int k,
                         int32_t *sel, float *p32, void *p_out, int32_t *blockhist, int nb, float *cutoff,
                         cudaStream_t s)
{
    const int epl = (E + 31) / 32;
#define LMOE_TOPK(N) run_topk<TO, N>(r_in, nsplit, r_out, bias, T, E, k, sel, p32, p_out, blockhist, nb, cutoff, s)
    if (epl <= 1) return LMOE_TOPK(1);
    if (epl <= 2) return LMOE_TOPK(2);
    if (epl <= 4) return LMOE_TOPK(4);
    if (epl <= 8) return LMOE_TOPK(8);
    if (epl <= 16) return LMOE_TOPK(16);
    return LMOE_TOPK(32);
#undef LMOE_TOPK
}

}  // namespace

cudaError_t launch_topk(const float *r_in, int nsplit, float *r_out, const float *bias, int64_t T, int E, int k,
                        int32_t *sel, float *p32, void *p_out, int out_bf16, int32_t *blockhist, float *cutoff,
                        cudaStream_t s)
{
    if (k > KMAX || E > 1024 || nsplit < 0) return cudaErrorInvalidValue;
    const int64_t nb = (T + ROUTE_TPB - 1) / ROUTE_TPB;
    cudaError_t e = cudaMemsetAsync(blockhist, 0, sizeof(int32_t) * nb * E, s);
    if (e != cudaSuccess) return e;
    if (out_bf16)
        return run_topk_epl<bf16>(r_in, nsplit, r_out, bias, T, E, k, sel, p32, p_out, blockhist, (int)nb, cutoff, s);
    return run_topk_epl<float>(r_in, nsplit, r_out, bias, T, E, k, sel, p32, p_out, blockhist, (int)nb, cutoff, s);
}

cudaError_t launch_scan(const int32_t *blockhist, int nb, int E, int32_t *counts, int32_t *base, cudaStream_t s)
{
    scan_cols_kernel<<<E, SCAN_NT, 0, s>>>(blockhist, nb, base, counts);
    return cudaGetLastError();
}

cudaError_t launch_dispatch(const int32_t *sel, const float *p32, const int32_t *base, const int32_t *counts,
                            int64_t T, int E, int k, int bm, int32_t *offsets, int32_t *tile_off, int32_t *slot_of,
                            int32_t *perm_tok, float *perm_w, cudaStream_t s)
{
    if (E > 1024) return cudaErrorInvalidValue;
    const int nb = (int)((T + ROUTE_TPB - 1) / ROUTE_TPB);
    const size_t smem = sizeof(int) * (2 * (size_t)E + 1);
    dispatch_kernel<<<nb, DISP_NT, smem, s>>>(sel, p32, base, counts, T, E, k, nb, bm, offsets, tile_off, slot_of,
                                               perm_tok, perm_w);
    return cudaGetLastError();
}

}  // namespace lmoe
