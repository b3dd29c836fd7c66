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
// Dense (one matrix, input rows 0..T-1): a block of 8 warps owns 4 weight rows
// (for the gate: 2 gate rows and the matching 2 up rows of the interleaved
// layout); its warps split K into interleaved 512-byte pieces, each lane
// keeping 16 loads of 16 bytes in flight, and the warps' sums are added in
// warp order.  Many small blocks keep every SM streaming even for the 26 MB
// down-projection (N = 1792 rows).
//
// Grouped (the routed experts): one warp owns a block of RB = 8 weight rows
// at a time (4 gate + 4 up rows for the gate) of one touched expert and runs
// over the whole of K, 16 loads of 16 bytes in flight per lane; a persistent
// grid of 4-warp blocks gives each warp a contiguous run of (touched expert,
// row block) items.  The expert's slot rows [offsets[e], offsets[e+1]) are its input rows
// (through the slot -> token map amap when given: the z rows of the tokens)
// and its output rows; W is the expert's slice.
//
// Either way each weight vector meets the same columns of every input row (x
// is small and stays in L1), lane sums are added with a fixed butterfly and
// nothing depends on timing.
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

constexpr int DV_ROWS = 4;       // dense: weight rows per block
constexpr int DV_WARPS = 8;      // dense: warps per block (split K)

template <int TT, int MODE>
__global__ void __launch_bounds__(DV_WARPS * 32)
dense_gemv_kernel(const bf16 *__restrict__ x, int64_t ldx, int T, int K, const bf16 *__restrict__ W, int64_t ldw, int N,
                  EpiArgs e)
{
    __shared__ float part[DV_WARPS][TT][DV_ROWS];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    griddep_wait();
    griddep_launch_dependents();
    int64_t rows[DV_ROWS];
    int64_t out0;
    if (MODE == EPI_GLU) {
        // outputs j0, j0 + 1: gate rows (j / ib) 2 ib + j % ib, up rows ib after them
        const int64_t j0 = (int64_t)blockIdx.x * 2;
        const int64_t g = (j0 / e.ib) * 2 * e.ib + (j0 % e.ib);
        rows[0] = g;
        rows[1] = g + 1;
        rows[2] = g + e.ib;
        rows[3] = g + e.ib + 1;
        out0 = j0;
    } else {
        out0 = (int64_t)blockIdx.x * DV_ROWS;
#pragma unroll
        for (int r = 0; r < DV_ROWS; ++r) rows[r] = out0 + r < N ? out0 + r : N - 1;   // clamped rows are dropped
    }
    float acc[TT][DV_ROWS];
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
        for (int r = 0; r < DV_ROWS; ++r) acc[t][r] = 0.f;
    const int nv = K / 8;   // 16-byte vectors per row
#pragma unroll 4
    for (int c = warp * 32 + lane; c < nv; c += DV_WARPS * 32) {
        uint4 wv[DV_ROWS];
#pragma unroll
        for (int r = 0; r < DV_ROWS; ++r) wv[r] = ld_stream(W + rows[r] * ldw + (int64_t)c * 8);
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            if (t < T) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(x + (int64_t)t * ldx) + c);
#pragma unroll
                for (int r = 0; r < DV_ROWS; ++r) acc[t][r] = dot8(wv[r], xv, acc[t][r]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
        for (int r = 0; r < DV_ROWS; ++r)
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc[t][r] += __shfl_xor_sync(0xffffffffu, acc[t][r], off);
    if (lane == 0) {
#pragma unroll
        for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int r = 0; r < DV_ROWS; ++r) part[warp][t][r] = acc[t][r];
    }
    __syncthreads();
    // thread (t, r) adds the warps' sums in warp order and writes its output
    const int t = threadIdx.x / DV_ROWS, r = threadIdx.x % DV_ROWS;
    if (t >= TT || t >= T) return;
    bf16 *out = (bf16 *)e.out;
    if (MODE == EPI_GLU) {
        if (r >= 2) return;
        float gsum = 0.f, usum = 0.f;
#pragma unroll
        for (int w = 0; w < DV_WARPS; ++w) {
            gsum += part[w][t][r];
            usum += part[w][t][r + 2];
        }
        out[(int64_t)t * e.ldo + out0 + r] = __float2bfloat16_rn(glu_act(e.act, gsum, usum, e.gate_cap, e.up_cap));
    } else {
        const int64_t n = out0 + r;
        if (n >= N) return;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < DV_WARPS; ++w) v += part[w][t][r];
        if (MODE == EPI_STORE_F32) {   // fp32 partial of a GEMV split along K
            ((float *)e.out)[(int64_t)t * e.ldo + n] = v;
            return;
        }
        if (e.residual32) v += e.residual32[(int64_t)t * e.ldo + n];
        if (e.residual) v += __bfloat162float(((const bf16 *)e.residual)[(int64_t)t * e.ldr + n]);
        out[(int64_t)t * e.ldo + n] = __float2bfloat16_rn(v);
    }
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
    // each warp takes a contiguous run of items: consecutive row blocks of the
    // same expert, whose rows are contiguous in memory and whose expert, slot
    // rows and input rows are looked up once per expert, not per item
    const int per = (items + total_warps - 1) / total_warps;
    const int i_end = min(items, (gw + 1) * per);
    int cur = -1, s0 = 0, cnt = p.T;
    const bf16 *W = p.W;
    const bf16 *xr[TT];
    for (int item = gw * per; item < i_end; ++item) {
        const int grp = item / nrb, rb = item % nrb;
        int64_t rows[RB];
        int col0;
        item_rows<MODE>(p, rb, rows, &col0);
        if (grp != cur) {
            cur = grp;
            if (p.offsets) {
                const int e = p.touched[grp];
                W = p.W + (int64_t)e * p.w_group_stride;
                s0 = p.offsets[e];
                cnt = p.offsets[e + 1] - s0;
            }
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const int s = s0 + (t < cnt ? t : 0);
                const int64_t src = p.amap ? (int64_t)p.amap[s] : (int64_t)s;
                xr[t] = p.x + src * p.ldx;
            }
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

namespace {

template <int TT>
cudaError_t run_dense(int mode, const GemmArgs &g, cudaStream_t s)
{
    const bf16 *x = (const bf16 *)g.A, *W = (const bf16 *)g.B;
    if (mode == EPI_GLU)
        return launch_pdl(dense_gemv_kernel<TT, EPI_GLU>, dim3((unsigned)(g.N / 4)), dim3(DV_WARPS * 32), 0, s, x,
                          g.lda, g.M, g.K, W, g.ldb, g.N, g.epi);
    if (mode == EPI_STORE_F32)
        return launch_pdl(dense_gemv_kernel<TT, EPI_STORE_F32>, dim3((unsigned)((g.N + DV_ROWS - 1) / DV_ROWS)),
                          dim3(DV_WARPS * 32), 0, s, x, g.lda, g.M, g.K, W, g.ldb, g.N, g.epi);
    return launch_pdl(dense_gemv_kernel<TT, EPI_STORE>, dim3((unsigned)((g.N + DV_ROWS - 1) / DV_ROWS)),
                      dim3(DV_WARPS * 32), 0, s, x, g.lda, g.M, g.K, W, g.ldb, g.N, g.epi);
}

}  // namespace

cudaError_t launch_gemv(int mode, const GemmArgs &g, cudaStream_t s)
{
    if (g.M < 1 || g.M > GEMV_MAX_T) return cudaErrorInvalidValue;
    if (mode != EPI_STORE && mode != EPI_GLU && mode != EPI_STORE_F32) return cudaErrorInvalidValue;
    if (g.K % 8 || g.lda % 8 || g.ldb % 8 || g.ldb < g.K) return cudaErrorInvalidValue;
    if (mode == EPI_GLU && (g.N % 4 || g.epi.ib % 2)) return cudaErrorInvalidValue;
    if (((uintptr_t)g.A | (uintptr_t)g.B) & 15u) return cudaErrorMisalignedAddress;
    if (g.M <= 1) return run_dense<1>(mode, g, s);
    if (g.M <= 2) return run_dense<2>(mode, g, s);
    return run_dense<4>(mode, g, s);
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
