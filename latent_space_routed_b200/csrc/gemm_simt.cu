// CUDA-core GEMM with the layer's fused epilogues.
//
// C[m, n] = sum_k A[m, k] B[n, k] in fp32 FFMA, A and B K-major (row-major
// "out x in" weights, as in W @ x).  This is the fp32 path (tensor-core TF32
// would not hold the fp32 workload's 1e-4 tolerance) and a cross-check path
// for bf16.  Tile 64 x 128 x 16, 256 threads, 4 x 8 outputs per thread; the
// accumulator tile is staged through shared memory so every epilogue sees
// whole row chunks.
//
// Grouped mode (offsets != nullptr): the rows of A are the expert-sorted slot
// rows; m-tile i belongs to the expert e with tile_off[e] <= i < tile_off[e+1]
// and covers rows offsets[e] + 64 (i - tile_off[e]) .. min(+64, offsets[e+1]);
// B for that expert starts at B + e * b_group_stride.
#include "lmoe_internal.cuh"

namespace lmoe {
namespace {

constexpr int BM = SIMT_BM, BN = SIMT_BN, BK = 16, NT = 256;

template <typename T> __device__ __forceinline__ float ldg_f32(const T *p) { return to_f32(*p); }

template <typename TA, typename TB, typename TO, int MODE>
__global__ void __launch_bounds__(NT) simt_gemm_kernel(GemmArgs g)
{
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[BK][BN + 4];
    __shared__ float Cs[BM][BN + 4];

    const int tid = threadIdx.x;
    int64_t row0, row_end;
    const TB *B = (const TB *)g.B;
    if (g.offsets) {
        const int mt = blockIdx.x;
        if (mt >= g.tile_off[g.E]) return;
        int lo = 0, hi = g.E - 1;  // last e with tile_off[e] <= mt
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (g.tile_off[mid] <= mt) lo = mid; else hi = mid - 1;
        }
        const int e = lo;
        row0 = (int64_t)g.offsets[e] + (int64_t)(mt - g.tile_off[e]) * BM;
        row_end = g.offsets[e + 1];
        B += (int64_t)e * g.b_group_stride;
    } else {
        row0 = (int64_t)blockIdx.x * BM;
        row_end = g.M;
    }
    const int n0 = blockIdx.y * BN;
    const TA *A = (const TA *)g.A;

    const int ty = tid / 16, tx = tid % 16;
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    // load assignment: A 64 rows x 16 k (4 per thread), B 128 rows x 16 k (8 per thread)
    const int a_r = tid / 4, a_k = (tid % 4) * 4;
    const int b_r = tid / 2, b_k = (tid % 2) * 8;
    const int64_t a_row = row0 + a_r;
    const bool a_ok = a_row < row_end;
    const int b_row = n0 + b_r;
    const bool b_ok = b_row < g.N;

    for (int k0 = 0; k0 < g.K; k0 += BK) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int kk = k0 + a_k + i;
            As[a_k + i][a_r] = (a_ok && kk < g.K) ? ldg_f32(A + a_row * g.lda + kk) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int kk = k0 + b_k + i;
            Bs[b_k + i][b_r] = (b_ok && kk < g.K) ? ldg_f32(B + (int64_t)b_row * g.ldb + kk) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[4], b[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 8; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }

#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) Cs[ty * 4 + i][tx + 16 * j] = acc[i][j];
    __syncthreads();

    // epilogue: 4 threads per row
    const int r = tid / 4, q = tid % 4;
    const int64_t row = row0 + r;
    if (row >= row_end) return;
    if (MODE == EPI_GLU) {
        // columns [0, BN/2) of the tile are gate rows, [BN/2, BN) the matching up rows
        const int half = BN / 2;
        if (n0 + half > g.N) return;
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int c = q * 16 + i;
            v[i] = glu_act(g.epi.act, Cs[r][c], Cs[r][c + half], g.epi.gate_cap, g.epi.up_cap);
        }
        epi_store_chunk<MODE, TO>(g.epi, row, (int64_t)(n0 / 2) + q * 16, v, 16);
    } else {
        float v[32];
        const int c0 = q * 32;
        int n = g.N - (n0 + c0);
        if (n <= 0) return;
        if (n > 32) n = 32;
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = Cs[r][c0 + i];
        epi_store_chunk<MODE, TO>(g.epi, row, (int64_t)n0 + c0, v, n);
    }
}

template <typename TA, typename TB, typename TO, int MODE>
cudaError_t run(const GemmArgs &g, int max_mtiles, cudaStream_t s)
{
    dim3 grid(g.offsets ? max_mtiles : (g.M + BM - 1) / BM, (g.N + BN - 1) / BN);
    if (grid.x == 0 || grid.y == 0) return cudaSuccess;
    simt_gemm_kernel<TA, TB, TO, MODE><<<grid, NT, 0, s>>>(g);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_simt_gemm(int mode, int ta, int tb, int to, const GemmArgs &g, int max_mtiles, cudaStream_t s)
{
    // instantiated combinations: token dtype for A; B is the token dtype or fp32 (router)
#define LMOE_SIMT_CASE(TA_, TB_, TO_, M_)                                                        \
    if (ta == (sizeof(TA_) == 4 ? 0 : 1) && tb == (sizeof(TB_) == 4 ? 0 : 1) &&                \
        to == (sizeof(TO_) == 4 ? 0 : 1) && mode == M_)                                          \
        return run<TA_, TB_, TO_, M_>(g, max_mtiles, s);
    LMOE_SIMT_CASE(float, float, float, EPI_STORE)
    LMOE_SIMT_CASE(float, float, float, EPI_SIGMOID)
    LMOE_SIMT_CASE(float, float, float, EPI_GLU)
    LMOE_SIMT_CASE(float, float, float, EPI_COMBINE)
    LMOE_SIMT_CASE(bf16, bf16, bf16, EPI_STORE)
    LMOE_SIMT_CASE(bf16, float, float, EPI_SIGMOID)
    LMOE_SIMT_CASE(bf16, bf16, bf16, EPI_GLU)
    LMOE_SIMT_CASE(bf16, bf16, bf16, EPI_COMBINE)
#undef LMOE_SIMT_CASE
    return cudaErrorInvalidValue;
}

}  // namespace lmoe
