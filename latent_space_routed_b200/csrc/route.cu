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

#include <algorithm>

#include "lmoe_internal.cuh"
#include "topk.cuh"

namespace lmoe {
namespace {

constexpr int TOPK_WARPS = 8;   // one token per warp, 8 tokens per block
constexpr int KMAX = 64;

// Top-k for one token per warp (warp_topk_radix for 9 <= k <= 32, else
// warp_topk), then the raw scores of the chosen experts normalised by their
// sum (a fixed butterfly order, so the result does not depend on timing), and
// each block's per-expert selection counts.
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
    extern __shared__ __align__(16) uint8_t topk_scratch[];   // TOPK_SCRATCH_BYTES per warp when radix
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t = (int64_t)blockIdx.x * TOPK_WARPS + warp;
    griddep_wait();
    griddep_launch_dependents();
    if (t >= T) return;
    const bool radix = topk_radix(k);
    uint32_t *hist = reinterpret_cast<uint32_t *>(topk_scratch + warp * TOPK_SCRATCH_BYTES);
    if (radix) {
        reinterpret_cast<uint4 *>(hist)[lane] = make_uint4(0u, 0u, 0u, 0u);
        reinterpret_cast<uint4 *>(hist)[lane + 32] = make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();
    }
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
        v[i] = e < E ? biased_key(r, bias[e]) : -INFINITY;
    }
    int mine0, mine1 = 0;
    float cv;
    if (radix)
        warp_topk_radix<EPL>(v, k, E, lane, hist, &mine0, &cv);
    else
        warp_topk<EPL>(v, ix, k, E, lane, &mine0, &mine1, &cv);
    if (lane == 0) cutoff[t] = cv;
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
    griddep_wait();
    griddep_launch_dependents();
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
    griddep_wait();
    griddep_launch_dependents();
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

// The whole routing of a few tokens (T <= ROUTE_SMALL_MAX_T) in one launch.
//
// Every block first computes the router scores of one expert row e for all T
// tokens: its 8 warps split W_r[e] (fp32) into interleaved 4 KB pieces, each
// lane keeping four 16-byte loads in flight, against the same columns of every
// token; lanes are added in a fixed butterfly order and warps in warp order
// (deterministic), and r[t, e] = sigmoid of the sum.  The block then counts
// itself done on a ticket; the last block to finish (all scores are written
// and, by the writers' fences, visible) does the rest:
//   top-k of each token (one warp per token, as in topk_kernel), the
//   Quantile-Balancing cutoff, p from the raw scores;
//   the stable counting sort of the T k slots by expert in shared memory: one
//   bit word per expert marks the tokens that chose it, counts are popcounts,
//   offsets and the m-tile prefix (tiles of bm rows) are block scans, and slot
//   (t, j) with e = sel[t, j] goes to offsets[e] + #{t' < t that chose e};
//   the touched experts (count > 0) in ascending order, for the grouped GEMVs;
// and puts the ticket back to zero for the next call.
constexpr int RS_WARPS = 8;

template <typename TO, int EPL>
__global__ void __launch_bounds__(RS_WARPS * 32)
route_small_kernel(const bf16 *__restrict__ x, const float *__restrict__ Wr, const float *__restrict__ bias, int T,
                   int E, int d, int k, int bm, float *__restrict__ r, int32_t *__restrict__ sel,
                   float *__restrict__ p32, TO *__restrict__ p_out, float *__restrict__ cutoff,
                   int32_t *__restrict__ counts, int32_t *__restrict__ offsets, int32_t *__restrict__ tile_off,
                   int32_t *__restrict__ slot_of, int32_t *__restrict__ perm_tok, float *__restrict__ perm_w,
                   int32_t *__restrict__ touched, int32_t *__restrict__ n_touched, int32_t *ticket)
{
    __shared__ float part[RS_WARPS][ROUTE_SMALL_MAX_T];
    __shared__ int s_last;
    __shared__ uint32_t s_bits[1024];
    __shared__ int s_off[1024 + 1];
    __shared__ int s_sel[ROUTE_SMALL_MAX_T * KMAX];
    __shared__ float s_p[ROUTE_SMALL_MAX_T * KMAX];
    __shared__ int s_warp[RS_WARPS];
    __shared__ __align__(16) uint8_t scratch[RS_WARPS][TOPK_SCRATCH_BYTES];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.x;
    griddep_wait();
    griddep_launch_dependents();

    // ---- router scores of expert e
    float acc[ROUTE_SMALL_MAX_T];
#pragma unroll
    for (int t = 0; t < ROUTE_SMALL_MAX_T; ++t) acc[t] = 0.f;
    const float4 *w = reinterpret_cast<const float4 *>(Wr + (int64_t)e * d);
    const int nv = d / 4;
    constexpr int STEP = RS_WARPS * 32;
    for (int c0 = warp * 32 + lane; c0 < nv; c0 += 4 * STEP) {
        float4 wv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) wv[u] = c0 + u * STEP < nv ? __ldg(w + c0 + u * STEP) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int t = 0; t < ROUTE_SMALL_MAX_T; ++t) {
            if (t < T) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (c0 + u * STEP < nv) {
                        const uint2 xv = __ldg(reinterpret_cast<const uint2 *>(x + (int64_t)t * d) + c0 + u * STEP);
                        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xv.x));
                        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xv.y));
                        acc[t] = fmaf(wv[u].x, a.x, acc[t]);
                        acc[t] = fmaf(wv[u].y, a.y, acc[t]);
                        acc[t] = fmaf(wv[u].z, b.x, acc[t]);
                        acc[t] = fmaf(wv[u].w, b.y, acc[t]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < ROUTE_SMALL_MAX_T; ++t)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
    if (lane == 0) {
#pragma unroll
        for (int t = 0; t < ROUTE_SMALL_MAX_T; ++t) part[warp][t] = acc[t];
    }
    __syncthreads();
    if (threadIdx.x < T) {
        float a = 0.f;
#pragma unroll
        for (int q = 0; q < RS_WARPS; ++q) a += part[q][threadIdx.x];
        r[(int64_t)threadIdx.x * E + e] = sigmoidf_(a);
        __threadfence();                       // the score is visible before the ticket counts this block
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = atomicAdd(ticket, 1) == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---- the last block: top-k, p, cutoff (one warp per token)
    for (int i = threadIdx.x; i < E; i += blockDim.x) s_bits[i] = 0u;
    const bool radix = topk_radix(k);
    uint32_t *hist = reinterpret_cast<uint32_t *>(scratch[warp]);
    reinterpret_cast<uint4 *>(hist)[lane] = make_uint4(0u, 0u, 0u, 0u);
    reinterpret_cast<uint4 *>(hist)[lane + 32] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    for (int t = warp; t < T; t += RS_WARPS) {
        float v[EPL];
        int ix[EPL];
        float rv[EPL];
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int ee = lane + 32 * i;
            ix[i] = ee;
            rv[i] = ee < E ? __ldcg(r + (int64_t)t * E + ee) : 0.f;
            v[i] = ee < E ? biased_key(rv[i], bias[ee]) : -INFINITY;
        }
        int mine0, mine1 = 0;
        float cv;
        if (radix)
            warp_topk_radix<EPL>(v, k, E, lane, hist, &mine0, &cv);
        else
            warp_topk<EPL>(v, ix, k, E, lane, &mine0, &mine1, &cv);
        if (lane == 0) cutoff[t] = cv;
        const float r0 = lane < k ? __ldcg(r + (int64_t)t * E + mine0) : 0.f;
        const float r1 = lane + 32 < k ? __ldcg(r + (int64_t)t * E + mine1) : 0.f;
        float sum = r0 + r1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = lane + 32 * h;
            if (j < k) {
                const int ee = h ? mine1 : mine0;
                const float p = (h ? r1 : r0) / sum;
                sel[(int64_t)t * k + j] = ee;
                p32[(int64_t)t * k + j] = p;
                p_out[(int64_t)t * k + j] = from_f32<TO>(p);
                s_sel[t * k + j] = ee;
                s_p[t * k + j] = p;
                atomicOr(&s_bits[ee], 1u << t);
            }
        }
    }
    __syncthreads();

    // ---- counting sort of the T k slots by expert
    {
        const int e0 = threadIdx.x * 4;
        int c[4], tl[4], used[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            c[q] = e0 + q < E ? __popc(s_bits[e0 + q]) : 0;
            tl[q] = (c[q] + bm - 1) / bm;
            used[q] = c[q] > 0 ? 1 : 0;
        }
        int total = 0;
        int run = block_exclusive_scan<RS_WARPS * 32>(c[0] + c[1] + c[2] + c[3], s_warp, &total);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (e0 + q < E) {
                s_off[e0 + q] = run;
                offsets[e0 + q] = run;
                counts[e0 + q] = c[q];
            }
            run += c[q];
        }
        if (threadIdx.x == 0) {
            s_off[E] = total;
            offsets[E] = total;
        }
        int ttot = 0;
        int trun = block_exclusive_scan<RS_WARPS * 32>(tl[0] + tl[1] + tl[2] + tl[3], s_warp, &ttot);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (e0 + q < E) tile_off[e0 + q] = trun;
            trun += tl[q];
        }
        if (threadIdx.x == 0) tile_off[E] = ttot;
        int ntot = 0;
        int nrun = block_exclusive_scan<RS_WARPS * 32>(used[0] + used[1] + used[2] + used[3], s_warp, &ntot);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (used[q]) touched[nrun] = e0 + q;
            nrun += used[q];
        }
        if (threadIdx.x == 0) *n_touched = ntot;
    }
    __syncthreads();
    const int S = T * k;
    for (int i = threadIdx.x; i < S; i += blockDim.x) {
        const int t = i / k;
        const int ee = s_sel[i];
        const int pos = s_off[ee] + __popc(s_bits[ee] & ((1u << t) - 1u));
        slot_of[i] = pos;
        perm_tok[pos] = t;
        perm_w[pos] = s_p[i];
    }
    if (threadIdx.x == 0) *ticket = 0;
}

// Zp[slot_of[t, j], :] = z[t, :] for j < k: G warps per token, warp g holding
// the token's z row in registers (V 16-byte vectors per lane, longer rows in
// pieces of 32 V vectors) and storing it to the slot rows j = g, g + G, ...
// With many tokens G = 1: z is read once and few, long-lived warps stream the
// slot rows' writes (the HBM traffic); with few tokens G grows up to k so that
// enough warps share the writes.
template <int V>
__global__ void __launch_bounds__(256)
permute_tokens_kernel(const uint4 *__restrict__ z, const int32_t *__restrict__ slot_of, uint4 *__restrict__ Zp,
                      int64_t T, int k, int G, int vec_per_row)
{
    const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    griddep_wait();
    griddep_launch_dependents();
    const int64_t t = w / G;
    const int g = (int)(w - t * G);
    if (t >= T) return;
    const int lane = threadIdx.x & 31;
    const int s0 = lane < k ? slot_of[t * k + lane] : 0;
    const int s1 = lane + 32 < k ? slot_of[t * k + lane + 32] : 0;
    for (int base = 0; base < vec_per_row; base += 32 * V) {   // one pass for rows up to 512 V bytes
        uint4 v[V];
#pragma unroll
        for (int u = 0; u < V; ++u)
            if (base + lane + 32 * u < vec_per_row) v[u] = z[t * vec_per_row + base + lane + 32 * u];
        for (int j = g; j < k; j += G) {
            const int slot = __shfl_sync(0xffffffffu, j < 32 ? s0 : s1, j & 31);
            uint4 *dst = Zp + (int64_t)slot * vec_per_row + base;
#pragma unroll
            for (int u = 0; u < V; ++u)
                if (base + lane + 32 * u < vec_per_row) dst[lane + 32 * u] = v[u];
        }
    }
}

}  // namespace

cudaError_t launch_permute_tokens(const void *z, const int32_t *slot_of, void *Zp, int64_t T, int k, int l,
                                  int elem_bytes, cudaStream_t s)
{
    if (T == 0) return cudaSuccess;
    if (((int64_t)l * elem_bytes) % 16 || k > KMAX) return cudaErrorInvalidValue;
    const int vpr = (int)((int64_t)l * elem_bytes / 16);
    // warps per token: about 4096 warps in all, at most one per slot row
    int G = (int)std::min<int64_t>((int64_t)k, std::max<int64_t>(1, 4096 / T));
    const dim3 grid((unsigned)((T * G + 7) / 8));
#define LMOE_PERMUTE(V) launch_pdl(permute_tokens_kernel<V>, grid, dim3(256), 0, s, (const uint4 *)z, slot_of, \
                                   (uint4 *)Zp, T, k, G, vpr)
    if (vpr <= 32) return LMOE_PERMUTE(1);
    if (vpr <= 64) return LMOE_PERMUTE(2);
    if (vpr <= 128) return LMOE_PERMUTE(4);
    if (vpr <= 256) return LMOE_PERMUTE(8);
    return LMOE_PERMUTE(16);   // rows above 8 KB in pieces of 8 KB
#undef LMOE_PERMUTE
}

namespace {

template <typename TO, int EPL>
cudaError_t run_topk(const float *r_in, int nsplit, float *r_out, const float *bias, int64_t T, int E, int k,
                     int32_t *sel, float *p32, void *p_out, int32_t *blockhist, int nb, float *cutoff, cudaStream_t s)
{
    const unsigned nblk = (unsigned)((T + TOPK_WARPS - 1) / TOPK_WARPS);
    const size_t smem = topk_radix(k) ? (size_t)TOPK_WARPS * TOPK_SCRATCH_BYTES : 0;
    return launch_pdl(topk_kernel<TO, EPL>, dim3(nblk), dim3(TOPK_WARPS * 32), smem, s, r_in, nsplit, r_out, bias, T,
                      E, k, sel, p32, (TO *)p_out, blockhist, nb, cutoff);
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
    if (out_bf16)
        return run_topk_epl<bf16>(r_in, nsplit, r_out, bias, T, E, k, sel, p32, p_out, blockhist, (int)nb, cutoff, s);
    return run_topk_epl<float>(r_in, nsplit, r_out, bias, T, E, k, sel, p32, p_out, blockhist, (int)nb, cutoff, s);
}

namespace {

template <typename TO, int EPL>
cudaError_t run_route_small(const SmallRouteArgs &a, cudaStream_t s)
{
    return launch_pdl(route_small_kernel<TO, EPL>, dim3((unsigned)a.E), dim3(RS_WARPS * 32), 0, s, a.x, a.Wr, a.bias,
                      a.T, a.E, a.d, a.k, a.bm, a.r, a.sel, a.p32, (TO *)a.p_out, a.cutoff, a.counts, a.offsets,
                      a.tile_off, a.slot_of, a.perm_tok, a.perm_w, a.touched, a.n_touched, a.ticket);
}

template <typename TO>
cudaError_t run_route_small_epl(const SmallRouteArgs &a, cudaStream_t s)
{
    const int epl = (a.E + 31) / 32;
    if (epl <= 1) return run_route_small<TO, 1>(a, s);
    if (epl <= 2) return run_route_small<TO, 2>(a, s);
    if (epl <= 4) return run_route_small<TO, 4>(a, s);
    if (epl <= 8) return run_route_small<TO, 8>(a, s);
    if (epl <= 16) return run_route_small<TO, 16>(a, s);
    return run_route_small<TO, 32>(a, s);
}

}  // namespace

cudaError_t launch_route_small(const SmallRouteArgs &a, int out_bf16, cudaStream_t s)
{
    if (a.T < 1 || a.T > ROUTE_SMALL_MAX_T || a.k > KMAX || a.E > 1024 || a.d % 4 || a.bm < 1)
        return cudaErrorInvalidValue;
    if (out_bf16) return run_route_small_epl<bf16>(a, s);
    return run_route_small_epl<float>(a, s);
}

cudaError_t launch_scan(const int32_t *blockhist, int nb, int E, int32_t *counts, int32_t *base, cudaStream_t s)
{
    return launch_pdl(scan_cols_kernel, dim3(E), dim3(SCAN_NT), 0, s, blockhist, nb, base, counts);
}

cudaError_t launch_dispatch(const int32_t *sel, const float *p32, const int32_t *base, const int32_t *counts,
                            int64_t T, int E, int k, int bm, int32_t *offsets, int32_t *tile_off, int32_t *slot_of,
                            int32_t *perm_tok, float *perm_w, cudaStream_t s)
{
    if (E > 1024) return cudaErrorInvalidValue;
    const int nb = (int)((T + ROUTE_TPB - 1) / ROUTE_TPB);
    const size_t smem = sizeof(int) * (2 * (size_t)E + 1);
    return launch_pdl(dispatch_kernel, dim3(nb), dim3(DISP_NT), smem, s, sel, p32, base, counts, T, E, k, nb, bm,
                      offsets, tile_off, slot_of, perm_tok, perm_w);
}

}  // namespace lmoe
