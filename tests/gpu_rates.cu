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
//         of `span` bytes (L2-resident when small, HBM-bound when large), issued
//         by one thread or split over two;
//   tile  the same with tiled tensor copies (cp.async.bulk.tensor.2d, 128-byte
//         swizzle, boxes of 64 bf16 x R rows: the GEMM's operand loads).
//
// Every wait is bounded (about 2 s of SM cycles); a wait that gives up sets
// *status, the CTA drains what it still has in flight (again bounded) and
// returns.  Output: one JSON object per line on stdout.
#include <cuda.h>
#include <cudaTypedefs.h>
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

// CLUSTER: wait with cluster-scope acquire semantics; otherwise the default
// (acquire, CTA scope).
template <bool CLUSTER = false>
__device__ __forceinline__ bool try_wait(uint32_t bar, uint32_t par)
{
    uint32_t ok;
    if (CLUSTER)
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(ok) : "r"(bar), "r"(par) : "memory");
    else
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(ok) : "r"(bar), "r"(par) : "memory");
    return ok != 0;
}

template <bool CLUSTER = false>
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t par)
{
    const long long t0 = clock64();
    while (!try_wait<CLUSTER>(bar, par))
        if (clock64() - t0 > LIMIT) return false;
    return true;
}

__device__ __forceinline__ uint64_t desc_sw128(uint32_t a)
{
    return (uint64_t)((a & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// ------------------------------------------------------------------ mma
template <int CG, int NACC, bool BLOCKED>
__global__ void __launch_bounds__(128, 1)
mma_kernel(int M, int N, int commit_every, int iters, unsigned long long *cycles, int *status)
{
    extern __shared__ uint8_t dyn[];                  // A 128 rows, B up to 256 rows (K = 64), 1024-aligned
    constexpr int OPS = 128 * 128 + 256 * 128;
    uint8_t *ops = dyn + ((1024 - (su32(dyn) & 1023)) & 1023);
    __shared__ __align__(8) uint64_t bar;
    __shared__ __align__(8) uint64_t step_bar;      // commit_every > 0: a commit per that many k-step rounds
    __shared__ uint32_t tmem_holder;
    uint32_t rank = 0;
    if (CG == 2) asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    for (int i = threadIdx.x; i < OPS / 2; i += blockDim.x)
        reinterpret_cast<__nv_bfloat16 *>(ops)[i] = __float2bfloat16((float)((i * 7) % 13 - 6) * 0.125f);
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&bar)) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&step_bar)) : "memory");
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
        uint64_t ad[4], bd[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            ad[k] = desc_sw128(sa + 32u * k);
            bd[k] = desc_sw128(sb + 32u * k);
        }
        auto mma = [&](uint32_t d, int k, uint32_t acc) {
            if (CG == 2)
                asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                             "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                             ::"r"(d), "l"(ad[k]), "l"(bd[k]), "r"(idesc), "r"(acc));
            else
                asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                             "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                             ::"r"(d), "l"(ad[k]), "l"(bd[k]), "r"(idesc), "r"(acc));
        };
        // the issuing loop is kept to a few instructions per MMA (precomputed
        // descriptors, compile-time accumulator count and order, no division):
        // a heavier loop throttles the issue itself
        const int group_len = commit_every > 0 ? commit_every : iters;
        for (int it0 = 0; it0 < iters; it0 += group_len) {
            for (int it = it0; it < it0 + group_len && it < iters; ++it) {
                if (BLOCKED) {      // accumulator outer: one accumulator takes all 4 k-steps of a 64-wide slice
#pragma unroll
                    for (int a = 0; a < NACC; ++a)
#pragma unroll
                        for (int k = 0; k < 4; ++k) mma(tmem + (uint32_t)(a * N), k, (it > 0 || k > 0) ? 1u : 0u);
                } else {            // k-step outer, accumulator inner
#pragma unroll
                    for (int k = 0; k < 4; ++k)
#pragma unroll
                        for (int a = 0; a < NACC; ++a) mma(tmem + (uint32_t)(a * N), k, (it > 0 || k > 0) ? 1u : 0u);
                }
            }
            if (commit_every > 0) {
                // the GEMM's per-stage pattern: a commit to a barrier (here never
                // waited for) after a stage's MMAs, then the next stage's wait on
                // an already complete barrier
                if (CG == 2)
                    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                                 ::"r"(su32(&step_bar)), "h"((uint16_t)0x3) : "memory");
                else
                    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                                 ::"r"(su32(&step_bar)) : "memory");
                (void)try_wait(su32(&bar), 1);
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

// ------------------------------------------------------------------ bulk and tile copies
constexpr int MAX_STAGES = 24;

// One ring of `stages` copies per issuing thread (threads 0 and 32 when
// issuers = 2, each with its own half of the buffer and barriers).
template <bool TILED, bool CLUSTER>
__global__ void __launch_bounds__(64, 1)
copy_kernel(const uint8_t *src, size_t span, const __grid_constant__ CUtensorMap tm, int tile_rows, int rows_total,
            int kblocks, int chunk, int stages, int issuers, int iters, int *status)
{
    extern __shared__ uint8_t dynbuf[];
    __shared__ __align__(8) uint64_t bars[MAX_STAGES];
    uint8_t *buf = dynbuf + ((1024 - (su32(dynbuf) & 1023)) & 1023);   // 1024-aligned (128-byte swizzle)
    const int who = threadIdx.x == 0 ? 0 : (threadIdx.x == 32 && issuers == 2 ? 1 : -1);
    if (who < 0) return;
    const int st = stages / issuers, s_base = who * st;
    for (int s = 0; s < st; ++s) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&bars[s_base + s])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    const size_t nchunks = TILED ? (size_t)(rows_total / tile_rows) * kblocks : span / (size_t)chunk;
    size_t pos = ((size_t)blockIdx.x * 977 + who * 131) % nchunks;
    const int my_iters = iters / issuers;
    int issued = 0, done = 0;
    bool ok = true;
    for (int it = 0; it < my_iters && ok; ++it) {
        const int s = it % st;
        if (it >= st) {   // the copy that used this stage last has landed
            ok = wait_bounded<CLUSTER>(su32(&bars[s_base + s]), (uint32_t)((it / st - 1) & 1));
            if (!ok) break;
            ++done;
        }
        const uint32_t bar = su32(&bars[s_base + s]);
        const uint32_t dst = su32(buf + (size_t)(s_base + s) * chunk);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(chunk) : "memory");
        if (TILED) {
            const int c0 = (int)(pos % kblocks) * 64, c1 = (int)(pos / kblocks) * tile_rows;
            asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                         " [%0], [%1, {%3, %4}], [%2];"
                         ::"r"(dst), "l"((uint64_t)&tm), "r"(bar), "r"(c0), "r"(c1) : "memory");
        } else {
            asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                         ::"r"(dst), "l"(src + pos * chunk), "r"(chunk), "r"(bar) : "memory");
        }
        ++issued;
        pos += 148 * 3 + 1;
        if (pos >= nchunks) pos %= nchunks;
    }
    // drain every copy still in flight (bounded)
    for (int i = done; i < issued; ++i)
        if (!wait_bounded<CLUSTER>(su32(&bars[s_base + i % st]), (uint32_t)((i / st) & 1))) { ok = false; break; }
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

#define LMOE_SMEM(CGV)                                                                                          \
    CK(cudaFuncSetAttribute(mma_kernel<CGV, 1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, MMA_SMEM)); \
    CK(cudaFuncSetAttribute(mma_kernel<CGV, 2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, MMA_SMEM)); \
    CK(cudaFuncSetAttribute(mma_kernel<CGV, 2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, MMA_SMEM));  \
    CK(cudaFuncSetAttribute(mma_kernel<CGV, 4, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, MMA_SMEM)); \
    CK(cudaFuncSetAttribute(mma_kernel<CGV, 4, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, MMA_SMEM));
    LMOE_SMEM(1)
    LMOE_SMEM(2)
#undef LMOE_SMEM
    // (cta_group, M, N): the kind::f16 shapes of both groups
    const int shapes[][3] = {{1, 128, 256}, {1, 128, 192}, {1, 128, 128}, {1, 128, 64}, {1, 64, 256}, {1, 64, 128},
                             {2, 256, 256}, {2, 256, 192}, {2, 256, 128}, {2, 256, 64}, {2, 128, 256}};
    const int iters = 2000;
    for (const auto &sh : shapes) {
        const int cg = sh[0], M = sh[1], N = sh[2];
        for (int mode = 0; mode < 8; ++mode) {
            // modes 0-4: accumulator counts and orders; 5-7: one accumulator with a
            // commit + wait after every 1, 2 or 4 rounds of 4 k-steps
            const int nacc = mode < 3 ? (1 << mode) : (mode == 3 ? 2 : (mode == 4 ? 4 : 1));
            const int blocked = mode == 3 || mode == 4;
            const int commit_every = mode == 5 ? 1 : (mode == 6 ? 2 : (mode == 7 ? 4 : 0));
            if (nacc * N > 512) continue;
            if (commit_every && !((cg == 2 && M == 256 && N == 256) || (cg == 1 && M == 128 && N == 256))) continue;
            void (*kern)(int, int, int, int, unsigned long long *, int *) = nullptr;
#define LMOE_PICK(CGV)                                                                                   \
            kern = nacc == 1 ? mma_kernel<CGV, 1, false>                                                 \
                 : nacc == 2 ? (blocked ? mma_kernel<CGV, 2, true> : mma_kernel<CGV, 2, false>)         \
                             : (blocked ? mma_kernel<CGV, 4, true> : mma_kernel<CGV, 4, false>);
            if (cg == 2) { LMOE_PICK(2) } else { LMOE_PICK(1) }
#undef LMOE_PICK
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
                CK(cudaLaunchKernelEx(&lc, kern, M, N, commit_every, iters, cycles, status));
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
                   "\"order\": \"%s\", \"commit_every\": %d, \"cycles_per_mma\": %.2f, "
                   "\"flop_per_clk_per_sm\": %.1f}\n",
                   cg, M, N, nacc, blocked ? "blocked" : "interleaved", commit_every, cyc, flop / cyc / cg);
        }
    }

    // copies: L2-resident and HBM-sized spans; bulk (1D) and tiled (2D, the GEMM's form)
    uint8_t *src;
    const size_t big = (size_t)4 << 30;
    CK(cudaMalloc(&src, big));
    CK(cudaMemset(src, 1, big));
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        CK(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
        encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
    }
    CK(cudaFuncSetAttribute(copy_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, 196608 + 1024));
    CK(cudaFuncSetAttribute(copy_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, 196608 + 1024));
    CK(cudaFuncSetAttribute(copy_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, 196608 + 1024));
    CK(cudaFuncSetAttribute(copy_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, 196608 + 1024));
    // (tiled, span bytes, chunk bytes, stages, issuers); every case runs with
    // CTA-scope and with cluster-scope waits
    struct Case { int tiled; size_t span; int chunk, stages, issuers; };
    const Case cases[] = {
        {0, (size_t)48 << 20, 8192, 8, 1},  {0, (size_t)48 << 20, 8192, 24, 1}, {0, (size_t)48 << 20, 16384, 4, 1},
        {0, (size_t)48 << 20, 16384, 8, 1}, {0, (size_t)48 << 20, 16384, 12, 1}, {0, (size_t)48 << 20, 16384, 12, 2},
        {0, (size_t)48 << 20, 32768, 2, 1}, {0, (size_t)48 << 20, 32768, 4, 1}, {0, (size_t)48 << 20, 32768, 6, 1},
        {0, (size_t)48 << 20, 32768, 6, 2}, {0, (size_t)48 << 20, 65536, 3, 1}, {0, (size_t)16 << 20, 32768, 6, 1},
        {0, big, 16384, 8, 1},               {0, big, 32768, 6, 1},               {0, big, 65536, 3, 1},
        {1, (size_t)48 << 20, 16384, 4, 1}, {1, (size_t)48 << 20, 16384, 8, 1}, {1, (size_t)48 << 20, 16384, 12, 1},
        {1, (size_t)48 << 20, 16384, 12, 2}, {1, (size_t)48 << 20, 32768, 3, 1}, {1, (size_t)48 << 20, 32768, 6, 1},
        {1, (size_t)48 << 20, 32768, 6, 2}, {1, big, 16384, 12, 1},              {1, big, 32768, 6, 1}};
    for (int scope = 0; scope < 2; ++scope)
    for (const Case &cs : cases) {
        const size_t smem = (size_t)cs.chunk * cs.stages + 1024;
        CUtensorMap tm;
        memset(&tm, 0, sizeof tm);
        const int K = 1024, rows = cs.chunk / 128;            // tiles: 64 bf16 (128 bytes) x rows
        const int rows_total = (int)(cs.span / (K * 2));
        if (cs.tiled) {
            cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows_total};
            cuuint64_t strides[1] = {(cuuint64_t)K * 2};
            cuuint32_t box[2] = {64, (cuuint32_t)rows};
            cuuint32_t estr[2] = {1, 1};
            if (encode(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, src, dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
                fprintf(stderr, "tensor map encode failed\n");
                return 2;
            }
        }
        const int iters = (int)(((size_t)8 << 30) / ((size_t)sms * cs.chunk));   // 8 GiB in all
        cudaEvent_t a, b;
        CK(cudaEventCreate(&a));
        CK(cudaEventCreate(&b));
        float best = 1e30f;
        for (int rep = 0; rep < 3; ++rep) {
            CK(cudaEventRecord(a));
            auto kern = cs.tiled ? (scope ? copy_kernel<true, true> : copy_kernel<true, false>)
                                 : (scope ? copy_kernel<false, true> : copy_kernel<false, false>);
            kern<<<sms, 64, smem>>>(src, cs.span, tm, rows, rows_total, K / 64, cs.chunk, cs.stages, cs.issuers, iters,
                                    status);
            CK(cudaGetLastError());
            CK(cudaEventRecord(b));
            CK(cudaEventSynchronize(b));
            float ms = 0;
            CK(cudaEventElapsedTime(&ms, a, b));
            if (ms < best) best = ms;
        }
        const double bytes = (double)sms * (iters / cs.issuers * cs.issuers) * cs.chunk;
        printf("{\"probe\": \"%s\", \"wait_scope\": \"%s\", \"span_bytes\": %zu, \"chunk\": %d, "
               "\"stages\": %d, \"issuers\": %d, \"ctas\": %d, \"GBps\": %.1f}\n", cs.tiled ? "tile" : "bulk",
               scope ? "cluster" : "cta", cs.span, cs.chunk, cs.stages, cs.issuers, sms, bytes / (best * 1e-3) / 1e9);
        cudaEventDestroy(a);
        cudaEventDestroy(b);
    }
    int st = 0;
    CK(cudaMemcpy(&st, status, sizeof st, cudaMemcpyDeviceToHost));
    printf("{\"probe\": \"done\", \"status\": %d, \"sms\": %d, \"clock_khz\": %d}\n", st, sms, clk_khz);
    return st != 0 ? 3 : 0;
}
