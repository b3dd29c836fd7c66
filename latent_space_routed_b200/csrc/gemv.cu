// Weight-streaming GEMMs of a few rows on CUDA cores:
// out[t, n] = epilogue(sum_k x[t, k] W[n, k]) with x [rows, K] and W [N, K] bf16.
//
// At a handful of tokens the GEMMs of a decode step only stream their weights
// (the down-projection, the shared experts' gate/up and the final GEMM: 25 to
// 117 MB each at d = 7168; the touched routed experts: 22 MB each), so what
// matters is keeping enough bytes in flight on every SM, not tensor cores
// ("at low latency and small batch size, MoE is bound by the memory bandwidth
// of loading weights").
//
// One warp owns a block of RB = 8 weight rows at a time (for the gate: 4 gate
// rows and the matching 4 up rows of the interleaved layout) and runs over
// the whole of K: each lane issues 16-byte non-allocating loads of its 8 rows
// two steps ahead (256 bytes in flight per lane) and multiplies them with the
// same columns of each input row (x is small and stays in L1).  Lane partial
// sums are added with a fixed butterfly, so the result does not depend on
// timing.  A persistent grid of 4-warp blocks hands row blocks out warp by
// warp, so every SM streams until the work runs out.
//
// Dense mode: one matrix, input rows 0..T-1, output row t.
// Grouped mode (the routed experts): work items are (touched expert, row
// block); the expert's slot rows [offsets[e], offsets[e+1]) are its input rows
// (through the slot -> token map amap when given, e.g. z rows of the tokens)
// and its output rows; W is the expert's slice.
#include "lmoe_internal.cuh"

namespace lmoe {
namespace {

constexpr int RB = 8;            // weight rows per warp item
constexpr int GV_WARPS = 4;      // warps per block

__device__ __forceinline__ uint4 ld_stream(const bf16 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float dot8(const uint4 &w, const uint4 &x, float acc)
{
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w}, xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ws[i]));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xs[i]));
        acc = fmaf(a.x, b.x, acc);
        acc = fmaf(a.y, b.y, acc);
    }
    return acc;
}

struct GemvParams {
    const bf16 *x;            // input rows [*, K]
    int64_t ldx;
    const bf16 *W;            // [N, K] (dense) or [E, N, K] (grouped)
    int64_t w_group_stride;   // elements between experts' slices
    int K, N;                 // N: weight rows per matrix (GLU: 2 F interleaved)
    int T;                    // dense: input rows
    // grouped
    const int32_t *offsets;   // [E + 1] slot offsets, or NULL (dense)
    const int32_t *touched;   // [n] experts with at least one slot, ascending
    const int32_t *n_touched; // device count
    const int32_t *amap;      // input row of each slot (NULL: the slot itself)
    EpiArgs epi;              // out / ldo / act / caps / ib / row_w (COMBINE) / residual
};

// Rows of the item and, for GLU, the first output column.
template <int MODE>
__device__ __forceinline__ void item_rows(const GemvParams &p, int rb, int64_t *rows, int *col0)
{
    if (MODE == EPI_GLU) {
        const int j0 = rb * (RB / 2);                         // 4 outputs: gate rows then up rows
        const int g = (j0 / p.epi.ib) * 2 * p.epi.ib + (j0 % p.epi.ib);
#pragma unroll
        for (int r = 0; r < RB / 2; ++r) {
            rows[r] = g + r;
            rows[r + RB / 2] = g + p.epi.ib + r;
        }
        *col0 = j0;
    } else {
        const int n0 = rb * RB;
#pragma unroll
        for (int r = 0; r < RB; ++r) rows[r] = n0 + r < p.N ? n0 + r : p.N - 1;   // clamped rows are dropped
        *col0 = n0;
    }
}

template <int TT, int MODE>
__global__ void __launch_bounds__(GV_WARPS * 32)
stream_gemv_kernel(const GemvParams p)
{
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * GV_WARPS + (threadIdx.x >> 5);
    const int total_warps = gridDim.x * GV_WARPS;
    const int nrb = MODE == EPI_GLU ? p.N / RB : (p.N + RB - 1) / RB;
    griddep_wait();
    griddep_launch_dependents();
    const int groups = p.offsets ? *p.n_touched : 1;
    const int items = groups * nrb;
    const int nv = p.K / 8;   // 16-byte vectors per row
    for (int item = gw; item < items; item += total_warps) {
        const int grp = item / nrb, rb = item % nrb;
        int64_t rows[RB];
        int col0;
        item_rows<MODE>(p, rb, rows, &col0);
        const bf16 *W = p.W;
        int s0 = 0, cnt = p.T;
        if (p.offsets) {
            const int e = p.touched[grp];
            W += (int64_t)e * p.w_group_stride;
            s0 = p.offsets[e];
            cnt = p.offsets[e + 1] - s0;
        }
        const bf16 *xr[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            const int s = s0 + (t < cnt ? t : 0);
            const int64_t src = p.amap ? (int64_t)p.amap[s] : (int64_t)s;
            xr[t] = p.x + src * p.ldx;
        }
        float acc[TT][RB];
#pragma unroll
        for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int r = 0; r < RB; ++r) acc[t][r] = 0.f;
#pragma unroll 2
        for (int c = lane; c < nv; c += 32) {
            uint4 wv[RB];
#pragma unroll
            for (int r = 0; r < RB; ++r) wv[r] = ld_stream(W + rows[r] * p.K + (int64_t)c * 8);
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                if (t < cnt) {
                    const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(xr[t]) + c);
#pragma unroll
                    for (int r = 0; r < RB; ++r) acc[t][r] = dot8(wv[r], xv, acc[t][r]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int r = 0; r < RB; ++r)
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) acc[t][r] += __shfl_xor_sync(0xffffffffu, acc[t][r], off);
        // every lane holds every sum; lane (t, q) writes one output
        bf16 *out = (bf16 *)p.epi.out;
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            if (t >= cnt) break;
            const int64_t orow = p.offsets ? (int64_t)(s0 + t) : (int64_t)t;
            if (MODE == EPI_GLU) {
#pragma unroll
                for (int q = 0; q < RB / 2; ++q)
                    if (lane == t * RB + q)
                        out[orow * p.epi.ldo + col0 + q] = __float2bfloat16_rn(
                            glu_act(p.epi.act, acc[t][q], acc[t][q + RB / 2], p.epi.gate_cap, p.epi.up_cap));
            } else {
#pragma unroll
                for (int q = 0; q < RB; ++q) {
                    if (lane == t * RB + q && col0 + q < p.N) {
                        float v = acc[t][q];
                        if (MODE == EPI_COMBINE) v *= p.epi.row_w[orow];
                        if (p.epi.residual) v += __bfloat162float(((const bf16 *)p.epi.residual)[orow * p.epi.ldr + col0 + q]);
                        out[orow * p.epi.ldo + col0 + q] = __float2bfloat16_rn(v);
                    }
                }
            }
        }
    }
}

int g_sms = 0;

template <int TT>
cudaError_t run(int mode, const GemvParams &p, int max_items, cudaStream_t s)
{
    if (g_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
        if (g_sms <= 0) g_sms = 148;
    }
    // persistent grid: at most 4 blocks per SM (register-bound), no more warps than items
    int blocks = (max_items + GV_WARPS - 1) / GV_WARPS;
    if (blocks > 4 * g_sms) blocks = 4 * g_sms;
    if (blocks < 1) blocks = 1;
    const dim3 grid(blocks), block(GV_WARPS * 32);
    if (mode == EPI_GLU) return launch_pdl(stream_gemv_kernel<TT, EPI_GLU>, grid, block, 0, s, p);
    if (mode == EPI_COMBINE) return launch_pdl(stream_gemv_kernel<TT, EPI_COMBINE>, grid, block, 0, s, p);
    return launch_pdl(stream_gemv_kernel<TT, EPI_STORE>, grid, block, 0, s, p);
}

cudaError_t dispatch_tt(int tt, int mode, const GemvParams &p, int max_items, cudaStream_t s)
{
    if (tt <= 1) return run<1>(mode, p, max_items, s);
    if (tt <= 2) return run<2>(mode, p, max_items, s);
    return run<4>(mode, p, max_items, s);
}

}  // namespace

cudaError_t launch_gemv(int mode, const GemmArgs &g, cudaStream_t s)
{
    if (g.M < 1 || g.M > GEMV_MAX_T) return cudaErrorInvalidValue;
    if (mode != EPI_STORE && mode != EPI_GLU) return cudaErrorInvalidValue;
    if (g.K % 8 || g.lda % 8 || g.ldb != g.K) return cudaErrorInvalidValue;
    if (mode == EPI_GLU && (g.N % RB || g.epi.ib % (RB / 2))) return cudaErrorInvalidValue;
    if (((uintptr_t)g.A | (uintptr_t)g.B) & 15u) return cudaErrorMisalignedAddress;
    GemvParams p = {};
    p.x = (const bf16 *)g.A;
    p.ldx = g.lda;
    p.W = (const bf16 *)g.B;
    p.K = g.K;
    p.N = g.N;
    p.T = g.M;
    p.epi = g.epi;
    const int nrb = mode == EPI_GLU ? g.N / RB : (g.N + RB - 1) / RB;
    return dispatch_tt(g.M, mode, p, nrb, s);
}

cudaError_t launch_gemv_grouped(int mode, const GemmArgs &g, const int32_t *touched, const int32_t *n_touched,
                                int max_touched, const int32_t *amap, int max_rows_per_group, cudaStream_t s)
{
    if (max_rows_per_group < 1 || max_rows_per_group > GEMV_MAX_T) return cudaErrorInvalidValue;
    if (mode != EPI_GLU && mode != EPI_COMBINE) return cudaErrorInvalidValue;
    if (!g.offsets || !touched || !n_touched) return cudaErrorInvalidValue;
    if (g.K % 8 || g.lda % 8 || g.ldb != g.K) return cudaErrorInvalidValue;
    if (mode == EPI_GLU && (g.N % RB || g.epi.ib % (RB / 2))) return cudaErrorInvalidValue;
    if (((uintptr_t)g.A | (uintptr_t)g.B) & 15u) return cudaErrorMisalignedAddress;
    GemvParams p = {};
    p.x = (const bf16 *)g.A;
    p.ldx = g.lda;
    p.W = (const bf16 *)g.B;
    p.w_group_stride = g.b_group_stride;
    p.K = g.K;
    p.N = g.N;
    p.offsets = g.offsets;
    p.touched = touched;
    p.n_touched = n_touched;
    p.amap = amap;
    p.epi = g.epi;
    const int nrb = mode == EPI_GLU ? g.N / RB : (g.N + RB - 1) / RB;
    return dispatch_tt(max_rows_per_group, mode, p, max_touched * nrb, s);
}

}  // namespace lmoe
