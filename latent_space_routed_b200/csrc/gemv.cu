// Dense GEMMs of one or two tokens (T <= GEMV_MAX_T) on CUDA cores:
// out[t, n] = epilogue(sum_k x[t, k] W[n, k]) with x [T, K] and W [N, K] bf16.
//
// At a handful of tokens these GEMMs only stream their weights (the
// down-projection, the shared experts' gate/up and the final GEMM of a decode
// step: 25 to 117 MB each at d = 7168), so what matters is bytes in flight, not
// tensor cores.  A block owns 4 weight rows (for the gate: 2 gate rows and the
// matching 2 up rows of the interleaved layout), its 8 warps split K and
// stream those rows with 16-byte non-allocating loads, each against the same
// columns of every token (x is tiny and stays in L1); the warps' partial sums
// are added in warp order, so the result does not depend on timing.  (At 8
// tokens the L1 reads of x outweigh the weight stream and split-K tensor-core
// tiles do better, measured.)
#include "lmoe_internal.cuh"

namespace lmoe {
namespace {

constexpr int GV_ROWS = 4;
constexpr int GV_WARPS = 8;

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

template <int TT, int MODE>
__global__ void __launch_bounds__(GV_WARPS * 32)
gemv_kernel(const bf16 *__restrict__ x, int T, int K, const bf16 *__restrict__ W, int N, EpiArgs e)
{
    __shared__ float part[GV_WARPS][TT][GV_ROWS];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t rows[GV_ROWS];
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
        out0 = (int64_t)blockIdx.x * GV_ROWS;
#pragma unroll
        for (int r = 0; r < GV_ROWS; ++r) rows[r] = out0 + r < N ? out0 + r : N - 1;   // clamped rows are dropped
    }
    float acc[TT][GV_ROWS];
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
        for (int r = 0; r < GV_ROWS; ++r) acc[t][r] = 0.f;
    const int nv = K / 8;   // 16-byte vectors per row
#pragma unroll 2
    for (int c = warp * 32 + lane; c < nv; c += GV_WARPS * 32) {
        uint4 wv[GV_ROWS];
#pragma unroll
        for (int r = 0; r < GV_ROWS; ++r) wv[r] = ld_stream(W + rows[r] * K + (int64_t)c * 8);
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            if (t < T) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(x + (int64_t)t * K) + c);
#pragma unroll
                for (int r = 0; r < GV_ROWS; ++r) acc[t][r] = dot8(wv[r], xv, acc[t][r]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
        for (int r = 0; r < GV_ROWS; ++r) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc[t][r] += __shfl_xor_sync(0xffffffffu, acc[t][r], off);
        }
    if (lane == 0) {
#pragma unroll
        for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int r = 0; r < GV_ROWS; ++r) part[warp][t][r] = acc[t][r];
    }
    __syncthreads();
    // thread (t, r) adds the warps' sums in warp order and writes its output
    const int t = threadIdx.x / GV_ROWS, r = threadIdx.x % GV_ROWS;
    if (t >= TT || t >= T) return;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < GV_WARPS; ++w) v += part[w][t][r];
    bf16 *out = (bf16 *)e.out;
    if (MODE == EPI_GLU) {
        if (r >= 2) return;
        float gsum = 0.f, usum = 0.f;
#pragma unroll
        for (int w = 0; w < GV_WARPS; ++w) {
            gsum += part[w][t][r];
            usum += part[w][t][r + 2];
        }
        out[(int64_t)t * e.ldo + out0 + r] = __float2bfloat16_rn(glu_act(e.act, gsum, usum, e.gate_cap, e.up_cap));
    } else {
        const int64_t n = out0 + r;
        if (n >= N) return;
        if (e.residual) v += __bfloat162float(((const bf16 *)e.residual)[(int64_t)t * e.ldr + n]);
        out[(int64_t)t * e.ldo + n] = __float2bfloat16_rn(v);
    }
}

template <int TT>
cudaError_t run_gemv(int mode, const GemmArgs &g, cudaStream_t s)
{
    const int T = g.M;
    if (mode == EPI_GLU) {
        const int blocks = g.N / 2 / 2;
        gemv_kernel<TT, EPI_GLU><<<blocks, GV_WARPS * 32, 0, s>>>((const bf16 *)g.A, T, g.K, (const bf16 *)g.B, g.N,
                                                                   g.epi);
    } else {
        const int blocks = (g.N + GV_ROWS - 1) / GV_ROWS;
        gemv_kernel<TT, EPI_STORE><<<blocks, GV_WARPS * 32, 0, s>>>((const bf16 *)g.A, T, g.K, (const bf16 *)g.B,
                                                                     g.N, g.epi);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemv(int mode, const GemmArgs &g, cudaStream_t s)
{
    if (g.M < 1 || g.M > GEMV_MAX_T) return cudaErrorInvalidValue;
    if (mode != EPI_STORE && mode != EPI_GLU) return cudaErrorInvalidValue;
    if (g.K % 8 || g.lda != g.K || g.ldb != g.K) return cudaErrorInvalidValue;
    if (mode == EPI_GLU && (g.N % 4 || g.epi.ib % 2)) return cudaErrorInvalidValue;
    if (((uintptr_t)g.A | (uintptr_t)g.B) & 15u) return cudaErrorMisalignedAddress;
    if (g.M <= 1) return run_gemv<1>(mode, g, s);
    return run_gemv<2>(mode, g, s);
}

}  // namespace lmoe
