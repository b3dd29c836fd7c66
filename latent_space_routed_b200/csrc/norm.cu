// Weighted combine + RMSNorm, and create-time weight repacking.
//
// combine_norm ("Stable LatentMoE", equations for u and y): for token t,
//   u = sum_j Y[slot_of[t, j]]        (rows already scaled by p_j, stored in the
//                                      token dtype, summed in fp32 in slot
//                                      order j = 0..k-1: deterministic)
//   n = u / sqrt(mean(u^2) + eps)     (RMSNorm, unit gain, eps inside the root)
// u is written out as latent_routed_aggregate (token dtype); n goes to the
// columns [col0, col0 + l) of the final GEMM's A operand, right after the
// shared experts' hidden columns, so that W_up n and both shared down
// projections are one K-concatenated GEMM.
#include "gemm_tc.cuh"
#include "lmoe_internal.cuh"

namespace lmoe {
namespace {

// Eight consecutive values as fp32 (16-byte loads) and back.
__device__ __forceinline__ void load8(const bf16 *p, float *v)
{
    const uint4 q = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float *p, float *v)
{
    const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void store8(bf16 *p, const float *v)
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ void store8(float *p, const float *v)
{
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// One block per token, one thread per 8 consecutive latent columns: the
// thread loads its columns from the token's k slot rows (eight rows in flight
// at a time), adds them in fp32 in slot order, and keeps u in registers for
// the norm.  DEEP (few tokens, blocks on a fraction of the SMs): a register
// budget that keeps all eight bf16 rows in flight; otherwise the compiler's
// smaller budget, which keeps more blocks resident.
template <typename TT, bool DEEP>
__global__ void __launch_bounds__(1024, DEEP ? 1 : 0)
combine_norm_kernel(const TT *__restrict__ Yp, const int32_t *__restrict__ slot_of, int l, int k, float eps,
                    TT *__restrict__ u_out, TT *__restrict__ hs, int64_t ld_hs, int64_t col0)
{
    __shared__ int slots[64];
    __shared__ float red[32];
    const int64_t t = blockIdx.x;
    griddep_wait();
    griddep_launch_dependents();
    for (int j = threadIdx.x; j < k; j += blockDim.x) slots[j] = slot_of[t * k + j];
    __syncthreads();
    const int c0 = threadIdx.x * 8;
    const bool active = c0 < l;
    float u[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (active) {
        int j = 0;
        if (DEEP && sizeof(TT) == 2) {
            for (; j + 8 <= k; j += 8) {  // eight rows in flight as raw 16-byte vectors, added in slot order
                uint4 raw[8];
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    raw[q] = *reinterpret_cast<const uint4 *>(Yp + (int64_t)slots[j + q] * l + c0);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float v[8];
                    load8(reinterpret_cast<const bf16 *>(&raw[q]), v);
#pragma unroll
                    for (int i = 0; i < 8; ++i) u[i] += v[i];
                }
            }
        }
        for (; j + 8 <= k; j += 8) {      // eight rows in flight, added in slot order
            float v[8][8];
#pragma unroll
            for (int q = 0; q < 8; ++q) load8(Yp + (int64_t)slots[j + q] * l + c0, v[q]);
#pragma unroll
            for (int q = 0; q < 8; ++q)
#pragma unroll
                for (int i = 0; i < 8; ++i) u[i] += v[q][i];
        }
        for (; j + 4 <= k; j += 4) {
            float v[4][8];
#pragma unroll
            for (int q = 0; q < 4; ++q) load8(Yp + (int64_t)slots[j + q] * l + c0, v[q]);
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int i = 0; i < 8; ++i) u[i] += v[q][i];
        }
        for (; j < k; ++j) {
            float v[8];
            load8(Yp + (int64_t)slots[j] * l + c0, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) u[i] += v[i];
        }
    }
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) ss += u[i] * u[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    const int nw = blockDim.x >> 5;
    for (int w = 0; w < nw; ++w) tot += red[w];
    const float inv = 1.0f / sqrtf(tot / (float)l + eps);
    if (active) {
        store8(u_out + t * l + c0, u);
        if (hs) {
            float n[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) n[i] = u[i] * inv;
            store8(hs + t * ld_hs + col0 + c0, n);
        }
    }
}

// P[e, 2F, K]: for every block q of ib rows, ib gate rows then the matching ib up rows.
template <typename T>
__global__ void pack_glu_kernel(const T *__restrict__ G, const T *__restrict__ U, T *__restrict__ P, int nE, int F,
                                int K, int ib)
{
    const int64_t total = (int64_t)nE * 2 * F * K;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t kk = i % K;
        const int64_t row = (i / K) % (2 * F);
        const int64_t e = i / ((int64_t)K * 2 * F);
        const int64_t q = row / (2 * ib), w = row % (2 * ib);
        const int64_t src_row = q * ib + (w % ib);
        const T *src = (w < ib) ? G : U;
        P[i] = src[(e * F + src_row) * K + kk];
    }
}

// P[d, 2 fs + l] = [Ds[0] | Ds[1] | W_up] row by row.
template <typename T>
__global__ void pack_cat_kernel(const T *__restrict__ Ds, const T *__restrict__ Wup, T *__restrict__ P, int d, int fs,
                                int l)
{
    const int64_t W = 2 * (int64_t)fs + l;
    const int64_t total = (int64_t)d * W;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = i / W, c = i % W;
        T v;
        if (c < fs) v = Ds[row * fs + c];
        else if (c < 2 * fs) v = Ds[((int64_t)d + row) * fs + (c - fs)];
        else v = Wup[row * l + (c - 2 * fs)];
        P[i] = v;
    }
}

// fp32 W -> three bf16 terms hi + mid + lo (each the rounding of what is left),
// stored as [3][n]; with bf16 activations every product is exact in fp32, so the
// three tensor-core passes reproduce an fp32 router to ~2^-24 relative.
__global__ void split_router_kernel(const float *__restrict__ W, bf16 *__restrict__ out, int64_t n)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float w = W[i];
        const bf16 hi = __float2bfloat16_rn(w);
        const float r1 = w - __bfloat162float(hi);
        const bf16 mid = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(mid);
        out[i] = hi;
        out[n + i] = mid;
        out[2 * n + i] = __float2bfloat16_rn(r2);
    }
}

// Split-K reduction: out[m, :] from the sum over splits of partial[s, m, :],
// four output columns per thread, splits summed in order (deterministic).
template <int MODE>
__global__ void __launch_bounds__(256)
splitk_reduce_kernel(const float *__restrict__ partial, int ksplit, int64_t M, int N, int act, float gate_cap,
                     float up_cap, int ib, void *__restrict__ out_, int64_t ldo,
                     const bf16 *__restrict__ residual, int64_t ldr)
{
    const int64_t m = blockIdx.y;
    const int nout = (MODE == EPI_GLU) ? N / 2 : N;
    const int j0 = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    griddep_wait();
    griddep_launch_dependents();
    if (j0 >= nout) return;
    const int64_t slab = M * (int64_t)N;
    float r[4];
    if (MODE == EPI_SIGMOID) {
        r[0] = r[1] = r[2] = r[3] = 0.f;
        const int n = N - j0 < 4 ? N - j0 : 4;
        float *o = reinterpret_cast<float *>(out_) + m * ldo + j0;
        if (n == 4 && (N & 3) == 0 && (ldo & 3) == 0) {
            for (int sp = 0; sp < ksplit; ++sp) {
                const float4 a = *reinterpret_cast<const float4 *>(partial + sp * slab + m * N + j0);
                r[0] += a.x; r[1] += a.y; r[2] += a.z; r[3] += a.w;
            }
            *reinterpret_cast<float4 *>(o) = make_float4(sigmoidf_(r[0]), sigmoidf_(r[1]), sigmoidf_(r[2]),
                                                         sigmoidf_(r[3]));
        } else {
            for (int sp = 0; sp < ksplit; ++sp)
                for (int i = 0; i < n; ++i) r[i] += partial[sp * slab + m * N + j0 + i];
            for (int i = 0; i < n; ++i) o[i] = sigmoidf_(r[i]);
        }
        return;
    }
    if (MODE == EPI_GLU) {
        // output column j: gate column (j / ib) 2 ib + j % ib, up column ib after it
        const int g0 = (j0 / ib) * 2 * ib + (j0 % ib);
        float gv[4] = {0.f, 0.f, 0.f, 0.f}, uv[4] = {0.f, 0.f, 0.f, 0.f};
        for (int sp = 0; sp < ksplit; ++sp) {
            const float4 a = *reinterpret_cast<const float4 *>(partial + sp * slab + m * N + g0);
            const float4 b = *reinterpret_cast<const float4 *>(partial + sp * slab + m * N + g0 + ib);
            gv[0] += a.x; gv[1] += a.y; gv[2] += a.z; gv[3] += a.w;
            uv[0] += b.x; uv[1] += b.y; uv[2] += b.z; uv[3] += b.w;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) r[i] = glu_act(act, gv[i], uv[i], gate_cap, up_cap);
    } else {
        r[0] = r[1] = r[2] = r[3] = 0.f;
        for (int sp = 0; sp < ksplit; ++sp) {
            const float4 a = *reinterpret_cast<const float4 *>(partial + sp * slab + m * N + j0);
            r[0] += a.x; r[1] += a.y; r[2] += a.z; r[3] += a.w;
        }
        if (residual) {   // standard MoE: y = shared + u
#pragma unroll
            for (int i = 0; i < 4; ++i) r[i] += __bfloat162float(residual[m * ldr + j0 + i]);
        }
    }
    bf16 *out = reinterpret_cast<bf16 *>(out_);
    const __nv_bfloat162 p0 = __floats2bfloat162_rn(r[0], r[1]);
    const __nv_bfloat162 p1 = __floats2bfloat162_rn(r[2], r[3]);
    uint2 w;
    w.x = *reinterpret_cast<const uint32_t *>(&p0);
    w.y = *reinterpret_cast<const uint32_t *>(&p1);
    *reinterpret_cast<uint2 *>(out + m * ldo + j0) = w;
}

}  // namespace

cudaError_t launch_splitk_reduce(const float *partial, int ksplit, int64_t M, int N, int mode, int act, float gate_cap,
                                 float up_cap, int ib, void *out, int64_t ldo, cudaStream_t s, const void *residual,
                                 int64_t ldr)
{
    if (M == 0) return cudaSuccess;
    if (mode != EPI_SIGMOID && (N % 8 || ldo % 4 || (mode == EPI_GLU && ib % 4))) return cudaErrorInvalidValue;
    const int nout = mode == EPI_GLU ? N / 2 : N;
    const int nvec = (nout + 3) / 4;
    const int threads = nvec < 256 ? ((nvec + 31) / 32) * 32 : 256;
    dim3 grid((unsigned)((nvec + threads - 1) / threads), (unsigned)M);
    if (mode == EPI_GLU)
        return launch_pdl(splitk_reduce_kernel<EPI_GLU>, grid, dim3(threads), 0, s, partial, ksplit, M, N, act,
                          gate_cap, up_cap, ib, out, ldo, (const bf16 *)nullptr, (int64_t)0);
    if (mode == EPI_SIGMOID)
        return launch_pdl(splitk_reduce_kernel<EPI_SIGMOID>, grid, dim3(threads), 0, s, partial, ksplit, M, N, act,
                          gate_cap, up_cap, ib, out, ldo, (const bf16 *)nullptr, (int64_t)0);
    return launch_pdl(splitk_reduce_kernel<EPI_STORE>, grid, dim3(threads), 0, s, partial, ksplit, M, N, act, gate_cap,
                      up_cap, ib, out, ldo, (const bf16 *)residual, ldr);
}

cudaError_t launch_combine_norm(const void *Yp, const int32_t *slot_of, int64_t T, int l, int k, float eps,
                                void *u_out, void *hs, int64_t ld_hs, int64_t col0, int tok_bf16, cudaStream_t s)
{
    if (T == 0) return cudaSuccess;
    if (k > 64 || l % 8 || l > 8192 || ld_hs % 8 || col0 % 8) return cudaErrorInvalidValue;
    const int threads = ((l / 8 + 31) / 32) * 32;
    const int sms = tc_num_sms() > 0 ? tc_num_sms() : 148;
#define LMOE_COMBINE(TT, DEEP)                                                                                   \
    launch_pdl(combine_norm_kernel<TT, DEEP>, dim3((unsigned)T), dim3(threads), 0, s, (const TT *)Yp, slot_of, l, k, \
               eps, (TT *)u_out, (TT *)hs, ld_hs, col0)
    if (tok_bf16) return T < 2 * sms ? LMOE_COMBINE(bf16, true) : LMOE_COMBINE(bf16, false);
    return T < 2 * sms ? LMOE_COMBINE(float, true) : LMOE_COMBINE(float, false);
#undef LMOE_COMBINE
}

cudaError_t launch_pack_glu(const void *G, const void *U, void *P, int nE, int F, int K, int ib, int elem_bytes,
                            cudaStream_t s)
{
    if (elem_bytes == 2)
        pack_glu_kernel<bf16><<<2048, 256, 0, s>>>((const bf16 *)G, (const bf16 *)U, (bf16 *)P, nE, F, K, ib);
    else
        pack_glu_kernel<float><<<2048, 256, 0, s>>>((const float *)G, (const float *)U, (float *)P, nE, F, K, ib);
    return cudaGetLastError();
}

cudaError_t launch_pack_cat(const void *Ds, const void *Wup, void *P, int d, int fs, int l, int elem_bytes,
                            cudaStream_t s)
{
    if (elem_bytes == 2)
        pack_cat_kernel<bf16><<<1024, 256, 0, s>>>((const bf16 *)Ds, (const bf16 *)Wup, (bf16 *)P, d, fs, l);
    else
        pack_cat_kernel<float><<<1024, 256, 0, s>>>((const float *)Ds, (const float *)Wup, (float *)P, d, fs, l);
    return cudaGetLastError();
}

cudaError_t launch_split_router(const float *Wr, bf16 *split, int64_t n, cudaStream_t s)
{
    split_router_kernel<<<256, 256, 0, s>>>(Wr, split, n);
    return cudaGetLastError();
}

}  // namespace lmoe
