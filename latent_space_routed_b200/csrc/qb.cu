// Quantile-Balancing statistics of the router (cooking-agi LatentMoE page,
// section "Quantile Balancing: measure now, use next step"): the (k+1)-th
// biased score of each token is the cutoff (the top-k kernel writes it), the
// margins m[t, e] = s[t, e] - cutoff[t] of every expert go into per-expert
// histograms ("global quantiles are approximated with histograms"), and the
// next step's bias moves each expert by the histogram estimate of the margin
// that leaves `target` tokens above it (the page's fixed-cutoff rule).
//
// Bin of a margin (every operation in fp32, round to nearest):
//   x = (m - lo) * (bins / (hi - lo)),  bin = 0 if x < 0, bins - 1 if x >= bins,
//   floor(x) otherwise.
#include "lmoe_internal.cuh"

namespace lmoe {
namespace {

constexpr int QB_TOKENS = 64;   // tokens per block of the histogram kernel

// Thread e of a block takes expert e (and e + blockDim, ...) over QB_TOKENS
// tokens: reads of r are coalesced across the experts, and the threads of a
// block never add to the same counter.
__global__ void qb_hist_kernel(const float *__restrict__ r, const float *__restrict__ bias,
                               const float *__restrict__ cutoff, int64_t T, int E, int bins, float lo, float inv_w,
                               int32_t *__restrict__ hist)
{
    const int64_t t0 = (int64_t)blockIdx.x * QB_TOKENS;
    const int64_t t1 = t0 + QB_TOKENS < T ? t0 + QB_TOKENS : T;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const float be = bias[e];
        for (int64_t t = t0; t < t1; ++t) {
            const float s = __fadd_rn(r[t * E + e], be);
            const float m = __fsub_rn(s, cutoff[t]);
            const float x = __fmul_rn(__fsub_rn(m, lo), inv_w);
            const int j = x < 0.f ? 0 : (x >= (float)bins ? bins - 1 : (int)x);
            atomicAdd(&hist[(int64_t)e * bins + j], 1);
        }
    }
}

// One thread per expert: scan its bins from the top; the target-th largest
// margin (0-based) lies in the bin j with C <= target < C + h_j (C = count in
// the bins above j) and is placed at the centre of its rank inside that bin.
__global__ void qb_bias_kernel(const int32_t *__restrict__ hist, const float *__restrict__ bias, int E, int bins,
                               double lo, double w, int64_t target, float *__restrict__ bias_out)
{
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    double q = lo;
    int64_t above = 0;
    for (int j = bins - 1; j >= 0; --j) {
        const int64_t h = hist[(int64_t)e * bins + j];
        if (above <= target && target < above + h) {
            q = lo + (j + 1) * w - w * ((double)(target - above) + 0.5) / (double)h;
            break;
        }
        above += h;
    }
    bias_out[e] = (float)((double)bias[e] - q);
}

}  // namespace

cudaError_t launch_qb_histogram(const float *r, const float *bias, const float *cutoff, int64_t T, int E, int bins,
                                float lo, float hi, int32_t *hist, cudaStream_t s)
{
    if (T <= 0) return cudaSuccess;
    const float inv_w = (float)bins / (hi - lo);   // fp32, as the histogram definition states
    const int threads = E < 256 ? ((E + 31) / 32) * 32 : 256;
    const unsigned blocks = (unsigned)((T + QB_TOKENS - 1) / QB_TOKENS);
    qb_hist_kernel<<<blocks, threads, 0, s>>>(r, bias, cutoff, T, E, bins, lo, inv_w, hist);
    return cudaGetLastError();
}

cudaError_t launch_qb_bias_update(const int32_t *hist, const float *bias, int E, int bins, float lo, float hi,
                                  int64_t target, float *bias_out, cudaStream_t s)
{
    const double w = ((double)hi - (double)lo) / bins;
    qb_bias_kernel<<<(E + 127) / 128, 128, 0, s>>>(hist, bias, E, bins, (double)lo, w, target, bias_out);
    return cudaGetLastError();
}

}  // namespace lmoe
