// Internal declarations shared by the kernel files of liblmoe (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lmoe.h"

namespace lmoe {

typedef __nv_bfloat16 bf16;

// Record `msg` as the calling thread's lmoe_last_error() and return `s`.
lmoe_status report_error(lmoe_status s, const char *msg);

// Device the handle was created on (its weights live there).
int handle_device(const lmoe_handle *h);

// Device address of the library's built-in scratch area (lmoe_forward_noalloc)
// on the handle's device, which must be current: LMOE_ERR_INVALID_ARG when it
// is not, LMOE_ERR_CUDA when the address lookup fails.  *bytes gets its size.
lmoe_status noalloc_area_for(const lmoe_handle *h, void **area, size_t *bytes);

// ---------------------------------------------------------------- conversions
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ float sigmoidf_(float a) { return 1.0f / (1.0f + expf(-a)); }

// Programmatic dependent launch.  Kernels of the forward are launched with
// programmatic stream serialization (launch_pdl), so a kernel may start while
// its predecessor on the stream is still finishing; griddep_wait() blocks
// until that predecessor has completed and its writes are visible, and every
// kernel calls it before it reads a predecessor's output or writes anything a
// predecessor may still read.  Without a predecessor it returns at once.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the next kernel on the stream start launching (it still waits for this
// one's completion in its own griddep_wait).
__device__ __forceinline__ void griddep_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, kern, args...);
}

// Gate of every expert: SwiGLU silu(g) * v, or the capped SiTU-GLU
// cg tanh(g/cg) sigmoid(g) * cu tanh(v/cu) ("Stable LatentMoE" names SiTU-GLU;
// this capped form reproduces its worked example).
__device__ __forceinline__ float glu_act(int act, float g, float v, float cg, float cu)
{
    const float sg = sigmoidf_(g);
    if (act == LMOE_ACT_SITU) return cg * tanhf(g / cg) * sg * (cu * tanhf(v / cu));
    return g * sg * v;
}

// ---------------------------------------------------------------- epilogues
// Every GEMM here computes C[m, n] = sum_k A[m, k] B[n, k] (both K-major) and
// hands each row chunk of fp32 accumulators to one of these epilogues.
enum EpiMode {
    EPI_STORE = 0,    // out[m, n] = C                      (final GEMM -> y)
    EPI_SIGMOID = 1,  // out32[m, n] = sigmoid(C)           (router -> r)
    EPI_GLU = 3,      // out[m, n'] = act(C[gate], C[up])   (gate/up GEMMs -> h)
    EPI_COMBINE = 4,  // out[m, n] = w[m] * C               (routed down -> p-weighted rows)
    EPI_GLU_SITU = 5, // EPI_GLU with the SiTU gate, as its own instantiation
    EPI_STORE_F32 = 6, // out32[m, n] = C                   (split-K partial tiles)
    EPI_SIGMOID_PARTIAL = 7  // router split-K: EPI_STORE_F32 partials, sigmoid in the reduction
};

struct EpiArgs {
    void *out;
    int64_t ldo;             // row stride of out, elements
    const float *row_w;      // EPI_COMBINE: weight of each row
    int act;                 // EPI_GLU
    float gate_cap, up_cap;
    int ib;                  // EPI_GLU: gate/up interleave block (columns)
    const void *residual;    // EPI_STORE: out = C + residual[m, n] (token dtype) when not NULL
    int64_t ldr;             // row stride of residual, elements
    const float *residual32; // dense GEMV, EPI_STORE: out = C + residual32[m, n] (fp32, row stride ldo) when not NULL
};

// Write n <= 32 consecutive values v[0..n) of row `row` starting at output column `col`.
template <int MODE, typename TO>
__device__ __forceinline__ void epi_store_chunk(const EpiArgs &e, int64_t row, int64_t col, const float *v, int n)
{
    if (MODE == EPI_SIGMOID) {
        float *o = (float *)e.out + row * e.ldo + col;
        #pragma unroll
        for (int i = 0; i < 32; ++i) if (i < n) o[i] = sigmoidf_(v[i]);
    } else if (MODE == EPI_COMBINE) {
        TO *o = (TO *)e.out + row * e.ldo + col;
        const float w = e.row_w[row];
        #pragma unroll
        for (int i = 0; i < 32; ++i) if (i < n) o[i] = from_f32<TO>(w * v[i]);
    } else {
        TO *o = (TO *)e.out + row * e.ldo + col;
        const TO *res = e.residual ? (const TO *)e.residual + row * e.ldr + col : nullptr;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (i < n) o[i] = from_f32<TO>(res ? v[i] + to_f32(res[i]) : v[i]);
    }
}

// ---------------------------------------------------------------- GEMM description
struct GemmArgs {
    const void *A;
    int64_t lda;        // elements
    const void *B;
    int64_t ldb;        // elements
    int64_t b_group_stride;  // elements between consecutive experts' B
    int M, N, K;        // dense: M rows; grouped: M = total rows (upper bound)
    const int32_t *offsets;   // grouped: [E+1] row offsets, else nullptr
    const int32_t *tile_off;  // grouped: [E+1] m-tile prefix for this kernel's BM
    int E;
    EpiArgs epi;
    // 1: launch without programmatic dependent launch, so that the kernel's
    // CTAs take SMs only once its stream predecessor has finished (instead of
    // waiting on them early, where another stream's kernel would run)
    int no_early_launch;
};

// ---------------------------------------------------------------- launchers
// CUDA-core GEMM (fp32 FFMA): the fp32 path, and a cross-check path for bf16.
// ta/tb/to: 0 = fp32, 1 = bf16.  Returns the launch error.
cudaError_t launch_simt_gemm(int mode, int ta, int tb, int to, const GemmArgs &g, int max_mtiles, cudaStream_t s);
constexpr int SIMT_BM = 64;
constexpr int SIMT_BN = 128;

// Router top-k + renormalisation + per-block expert histogram.
constexpr int ROUTE_TPB = 32;   // tokens per counting block (also the dispatch block)
// nsplit = 0: r_in is r [T, E]; nsplit > 0: r_in holds nsplit fp32 partial
// slabs [nsplit, T, E] of the router logits, summed in order, put through the
// sigmoid and written to r_out [T, E].  cutoff [T] gets each token's (k+1)-th
// biased score (-inf when k = E).
cudaError_t launch_topk(const float *r_in, int nsplit, float *r_out, const float *bias, int64_t T, int E, int k,
                        int32_t *sel, float *p32, void *p_out, int out_bf16, int32_t *blockhist, float *cutoff,
                        cudaStream_t s);
// Quantile-Balancing statistics: add the margin histogram of T tokens to hist
// [E, bins]; and the next bias b - q from an accumulated histogram.
cudaError_t launch_qb_histogram(const float *r, const float *bias, const float *cutoff, int64_t T, int E, int bins,
                                float lo, float hi, int32_t *hist, cudaStream_t s);
cudaError_t launch_qb_bias_update(const int32_t *hist, const float *bias, int E, int bins, float lo, float hi,
                                  int64_t target, float *bias_out, cudaStream_t s);
// blockhist is expert-major [E][nb]; base (same layout) gets each block's
// starting rank within its expert, counts[e] the expert totals.
cudaError_t launch_scan(const int32_t *blockhist, int nb, int E, int32_t *counts, int32_t *base, cudaStream_t s);
// Also writes offsets[E+1] and the m-tile prefix tile_off[E+1] for tiles of bm rows.
cudaError_t launch_dispatch(const int32_t *sel, const float *p32, const int32_t *base, const int32_t *counts,
                            int64_t T, int E, int k, int bm, int32_t *offsets, int32_t *tile_off, int32_t *slot_of,
                            int32_t *perm_tok, float *perm_w, cudaStream_t s);
// Zp[slot_of[t, j]] = z[t] for every token t and j < k (rows of l elements of
// elem_bytes; l elem_bytes a multiple of 16).
cudaError_t launch_permute_tokens(const void *z, const int32_t *slot_of, void *Zp, int64_t T, int k, int l,
                                  int elem_bytes, cudaStream_t s);
// Yp in the token dtype.
// hs = NULL: u only (no RMSNorm; the standard-MoE form).
cudaError_t launch_combine_norm(const void *Yp, const int32_t *slot_of, int64_t T, int l, int k, float eps,
                                void *u_out, void *hs, int64_t ld_hs, int64_t col0, int tok_bf16, cudaStream_t s);

// Sum ksplit fp32 partial tiles [ksplit][M][N] in split order and apply the
// epilogue: EPI_STORE (bf16 out[m, n]), EPI_GLU (gate/up column pairs
// interleaved in blocks of ib, bf16 out[m, n'] for n' < N / 2) or EPI_SIGMOID
// (fp32 out[m, n] = sigmoid(sum)).
cudaError_t launch_splitk_reduce(const float *partial, int ksplit, int64_t M, int N, int mode, int act, float gate_cap,
                                 float up_cap, int ib, void *out, int64_t ldo, cudaStream_t s,
                                 const void *residual = nullptr, int64_t ldr = 0);
// Dense bf16 GEMM of a few tokens (g.M = T <= GEMV_MAX_T, B rows g.ldb >= K
// elements apart, K a multiple of 8) on CUDA cores, streaming B: EPI_STORE
// (with the optional residual and fp32 residual32), EPI_STORE_F32 (fp32
// output) or EPI_GLU (gate/up rows interleaved in blocks of ib).
// (measured on B200, decode_d7168: at T = 3 and 4 the GEMVs, whose loads serve
// only the one or two slot rows most touched experts have, took 0.60 and 0.73
// ms against 0.42 and 0.50 ms for the tensor-core tiles; equal at T = 1, 2)
constexpr int GEMV_MAX_T = 2;
cudaError_t launch_gemv(int mode, const GemmArgs &g, cudaStream_t s);
// The routed experts' GEMMs of a few slot rows per expert, streaming only the
// touched experts' weights: g.offsets [E+1] gives each expert's slot rows
// (at most max_rows_per_group <= GEMV_MAX_T of them), touched[0 .. *n_touched)
// the experts with at least one (max_touched bounds the count); input row of
// slot s is amap[s] (or s when amap is NULL), output row s.  EPI_GLU
// (g.epi.ib-interleaved gate/up rows) or EPI_COMBINE (g.epi.row_w[s] * sum).
cudaError_t launch_gemv_grouped(int mode, const GemmArgs &g, const int32_t *touched, const int32_t *n_touched,
                                int max_touched, const int32_t *amap, int max_rows_per_group, cudaStream_t s);
// The whole routing of T <= ROUTE_SMALL_MAX_T tokens in one launch: router
// scores r [T, E] (fp32, CUDA cores), top-k, p (fp32 and token dtype), the
// Quantile-Balancing cutoff, expert counts, offsets [E+1], the m-tile prefix
// for tiles of bm rows, slot_of, the slot -> token map and slot weights, and
// the touched experts in ascending order with their count.  *ticket must be
// zero at launch; the kernel leaves it zero.
constexpr int ROUTE_SMALL_MAX_T = 8;
struct SmallRouteArgs {
    const bf16 *x;
    const float *Wr, *bias;
    int T, E, d, k, bm;
    float *r;
    int32_t *sel;
    float *p32;
    void *p_out;
    float *cutoff;
    int32_t *counts, *offsets, *tile_off, *slot_of, *perm_tok;
    float *perm_w;
    int32_t *touched, *n_touched, *ticket;
};
cudaError_t launch_route_small(const SmallRouteArgs &a, int out_bf16, cudaStream_t s);

// Weight repacking (create time).
cudaError_t launch_pack_glu(const void *G, const void *U, void *P, int nE, int F, int K, int ib, int elem_bytes,
                            cudaStream_t s);
cudaError_t launch_pack_cat(const void *Ds, const void *Wup, void *P, int d, int fs, int l, int elem_bytes,
                            cudaStream_t s);
cudaError_t launch_split_router(const float *Wr, bf16 *split, int64_t n, cudaStream_t s);

// ---------------------------------------------------------------- tensor-core GEMM (sm_100a)
struct TcGemm;  // defined in gemm_tc.cu
constexpr int TC_BM = 128;
constexpr int TC_BN = 256;
constexpr int TC_BK = 64;

}  // namespace lmoe
