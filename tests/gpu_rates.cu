// Two rate measurements behind the tile shapes of the library's tensor-core
// GEMM (a standalone program, built and run by tests/test_gpu_rates.py):
//
//   mma   cycles per tcgen05.mma (kind::f16, bf16 operands, fp32 accumulator,
//         K = 16) for a given cta_group, M and N, with `nacc` independent
//         accumulators in flight: operands sit in shared memory, one thread
//         issues `iters` rounds of 4 k-steps x nacc MMAs (interleaved: each
//         k-step to every accumulator in turn; blocked: all 4 k-steps to one
//         accumulator, then the next), then one commit; the issuing thread
//         times issue + completion with its cycle counter.
//   bulk  bytes per second moved from global memory into shared memory by the
//         bulk-copy engine (cp.async.bulk ... complete_tx), one CTA per SM,
//         each keeping `stages` copies of `chunk` bytes in flight over a buffer
//         of `span` bytes (L2-resident when small, HBM-bound when large).
//
// Every wait is bounded (about 2 s of SM cycles); a wait that gives up sets
// *status, the CTA drains what it still has in flight (again bounded) and
// returns.  Output: one JSON object per line on stdout.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#define CK(x)                                                                                   \
    do {                                                                                        \
        cudaError_t e_ = (x);                                                                   \
        if (e_ != cudaSuccess) {                                                                \
            fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));                            \
            exit(2);                                                                            \
        }                                                                                       \
    } while (0)

static constexpr long long LIMIT = 4000000000ll;

__device__ __forceinline__ uint32_t su32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ bool try_wait(uint32_t bar, uint32_t par)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(par) : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t par)
{
    const long long t0 = clock64();
    while (!try_wait(bar, par))
        if (clock64() - t0 > LIMIT) return false;
    return true;
}

__device__ __forceinline__ uint64_t desc_sw128(uint32_t a)
{
    return (uint64_t)((a & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// ------------------------------------------------------------------ mma
template <int CG>
__global__ void __launch_bounds__(128, 1)
mma_kernel(int M, int N, int nacc, int blocked, int iters, unsigned long long *cycles, int *status)
{
    extern __shared__ uint8_t dyn[];                  // A 128 rows, B up to 256 rows (K = 64), 1024-aligned
    constexpr int OPS = 128 * 128 + 256 * 128;
    uint8_t *ops = dyn + ((1024 - (su32(dyn) & 1023)) & 1023);
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tmem_holder;
    uint32_t rank = 0;
    if (CG == 2) asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    for (int i = threadIdx.x; i < OPS / 2; i += blockDim.x)
        reinterpret_cast<__nv_bfloat16 *>(ops)[i] = __float2bfloat16((float)((i * 7) % 13 - 6) * 0.125f);
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&bar)) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (threadIdx.x < 32) {
        if (CG == 2) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(su32(&tmem_holder)) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(su32(&tmem_holder)) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (CG == 2) asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_holder;
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
    const uint32_t sa = su32(ops), sb = sa + 128 * 128;
    if (threadIdx.x == 0 && rank == 0) {
        const long long t0 = clock64();
        for (int it = 0; it < iters; ++it) {
            // interleaved: k-step outer, accumulator inner; blocked: accumulator
            // outer, so one accumulator takes all 4 k-steps of a 64-wide slice
            for (int q = 0; q < 4 * nacc; ++q) {
                const int k = blocked ? q % 4 : q / nacc, a = blocked ? q / 4 : q % nacc;
                const uint64_t ad = desc_sw128(sa + 32u * k), bd = desc_sw128(sb + 32u * k);
                {
                    const uint32_t d = tmem + (uint32_t)(a * N);
                    const uint32_t acc = (it > 0 || k > 0) ? 1u : 0u;
                    if (CG == 2)
                        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                     "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                                     ::"r"(d), "l"(ad), "l"(bd), "r"(idesc), "r"(acc));
                    else
                        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                     "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                                     ::"r"(d), "l"(ad), "l"(bd), "r"(idesc), "r"(acc));
                }
            }
        }
        if (CG == 2)
            asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                         ::"r"(su32(&bar)), "h"((uint16_t)0x3) : "memory");
        else
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(&bar)) : "memory");
        const bool ok = wait_bounded(su32(&bar), 0);
        const long long t1 = clock64();
        if (!ok) atomicOr(status, 1);
        cycles[blockIdx.x / CG] = (unsigned long long)(t1 - t0);
    } else if (threadIdx.x == 0) {
        if (!wait_bounded(su32(&bar), 0)) atomicOr(status, 2);    // the peer's commit arrives here too
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (CG == 2) asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (threadIdx.x < 32) {
        if (CG == 2) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
        else asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

static constexpr int MMA_SMEM = 128 * 128 + 256 * 128 + 1024;

// ------------------------------------------------------------------ bulk copies
constexpr int MAX_STAGES = 12;

__global__ void __launch_bounds__(32, 1)
bulk_kernel(const uint8_t *src, size_t span, int chunk, int stages, int iters, int *status)
{
    extern __shared__ __align__(1024) uint8_t buf[];
    __shared__ __align__(8) uint64_t bars[MAX_STAGES];
    if (threadIdx.x != 0) return;
    for (int s = 0; s < stages; ++s) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&bars[s])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    const size_t nchunks = span / (size_t)chunk;
    size_t pos = ((size_t)blockIdx.x * 977) % nchunks;
    int issued = 0, done = 0;
    bool ok = true;
    for (int it = 0; it < iters && ok; ++it) {
        const int s = it % stages;
        if (it >= stages) {   // the copy that used this stage last has landed
            ok = wait_bounded(su32(&bars[s]), (uint32_t)((it / stages - 1) & 1));
            if (!ok) break;
            ++done;
        }
        const uint32_t bar = su32(&bars[s]);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(chunk) : "memory");
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                     ::"r"(su32(buf + (size_t)s * chunk)), "l"(src + pos * chunk), "r"(chunk), "r"(bar) : "memory");
        ++issued;
        pos += 148 * 3 + 1;
        if (pos >= nchunks) pos %= nchunks;
    }
    // drain every copy still in flight (bounded)
    for (int i = done; i < issued; ++i)
        if (!wait_bounded(su32(&bars[i % stages]), (uint32_t)((i / stages) & 1))) { ok = false; break; }
    if (!ok) atomicOr(status, 4);
}

int main(int argc, char **argv)
{
    int dev = 0, sms = 0;
    CK(cudaGetDevice(&dev));
    CK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    int clk_khz = 0;
    cudaDeviceGetAttribute(&clk_khz, cudaDevAttrClockRate, dev);
    int *status;
    unsigned long long *cycles;
    CK(cudaMalloc(&status, sizeof(int)));
    CK(cudaMalloc(&cycles, sizeof(unsigned long long) * sms));
    CK(cudaMemset(status, 0, sizeof(int)));

    CK(cudaFuncSetAttribute(mma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, MMA_SMEM));
    CK(cudaFuncSetAttribute(mma_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, MMA_SMEM));
    // (cta_group, M, N): the kind::f16 shapes of both groups
    const int shapes[][3] = {{1, 128, 256}, {1, 128, 192}, {1, 128, 128}, {1, 128, 64}, {1, 64, 256}, {1, 64, 128},
                             {2, 256, 256}, {2, 256, 192}, {2, 256, 128}, {2, 256, 64}, {2, 128, 256}};
    const int iters = 2000;
    for (const auto &sh : shapes) {
        const int cg = sh[0], M = sh[1], N = sh[2];
        for (int mode = 0; mode < 5; ++mode) {
            const int nacc = mode < 3 ? (1 << mode) : (mode == 3 ? 2 : 4), blocked = mode >= 3;
            if (nacc * N > 512) continue;
            const int groups = sms / cg;
            cudaLaunchConfig_t lc = {};
            lc.gridDim = dim3(groups * cg);
            lc.blockDim = dim3(128);
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = cg;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            lc.attrs = at;
            lc.numAttrs = 1;
            lc.dynamicSmemBytes = MMA_SMEM;
            for (int rep = 0; rep < 2; ++rep) {   // the first launch warms up
                if (cg == 2) CK(cudaLaunchKernelEx(&lc, mma_kernel<2>, M, N, nacc, blocked, iters, cycles, status));
                else CK(cudaLaunchKernelEx(&lc, mma_kernel<1>, M, N, nacc, blocked, iters, cycles, status));
                CK(cudaDeviceSynchronize());
            }
            unsigned long long h[256];
            CK(cudaMemcpy(h, cycles, sizeof(unsigned long long) * groups, cudaMemcpyDeviceToHost));
            double mean = 0;
            for (int g = 0; g < groups; ++g) mean += (double)h[g];
            mean /= groups;
            const double n_mma = (double)iters * 4 * nacc;
            const double cyc = mean / n_mma;                         // cycles per instruction
            const double flop = 2.0 * M * N * 16;                    // per instruction (whole cta group)
            printf("{\"probe\": \"mma\", \"cta_group\": %d, \"M\": %d, \"N\": %d, \"nacc\": %d, "
                   "\"order\": \"%s\", \"cycles_per_mma\": %.2f, \"flop_per_clk_per_sm\": %.1f}\n",
                   cg, M, N, nacc, blocked ? "blocked" : "interleaved", cyc, flop / cyc / cg);
        }
    }

    // bulk copies: an L2-resident span and an HBM-sized one
    const size_t spans[] = {(size_t)16 << 20, (size_t)48 << 20, (size_t)4 << 30};
    // (chunk bytes, stages): 128 KB and 192 KB in flight per SM in 16 KB copies, 192 KB in 32 KB copies
    const int cases[][2] = {{16384, 8}, {16384, 12}, {32768, 6}};
    uint8_t *src;
    CK(cudaMalloc(&src, spans[2]));
    CK(cudaMemset(src, 1, spans[2]));
    for (size_t span : spans) {
        for (const auto &cs : cases) {
            const int chunk = cs[0], stages = cs[1];
            const size_t smem = (size_t)chunk * stages;
            CK(cudaFuncSetAttribute(bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
            const int iters = (int)(((size_t)8 << 30) / ((size_t)sms * chunk));   // 8 GiB in all
            cudaEvent_t a, b;
            CK(cudaEventCreate(&a));
            CK(cudaEventCreate(&b));
            float best = 1e30f;
            for (int rep = 0; rep < 3; ++rep) {
                CK(cudaEventRecord(a));
                bulk_kernel<<<sms, 32, smem>>>(src, span, chunk, stages, iters, status);
                CK(cudaEventRecord(b));
                CK(cudaEventSynchronize(b));
                float ms = 0;
                CK(cudaEventElapsedTime(&ms, a, b));
                if (ms < best) best = ms;
            }
            const double bytes = (double)sms * iters * chunk;
            printf("{\"probe\": \"bulk\", \"span_bytes\": %zu, \"chunk\": %d, \"stages\": %d, \"ctas\": %d, "
                   "\"GBps\": %.1f}\n", span, chunk, stages, sms, bytes / (best * 1e-3) / 1e9);
            cudaEventDestroy(a);
            cudaEventDestroy(b);
        }
    }
    int st = 0;
    CK(cudaMemcpy(&st, status, sizeof st, cudaMemcpyDeviceToHost));
    printf("{\"probe\": \"done\", \"status\": %d, \"sms\": %d, \"clock_khz\": %d}\n", st, sms, clk_khz);
    return st != 0 ? 3 : 0;
}
