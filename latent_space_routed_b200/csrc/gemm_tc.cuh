// Host interface of the sm_100a tensor-core GEMM (tcgen05 + TMEM + TMA).
#pragma once

#include "lmoe_internal.cuh"

namespace lmoe {

// LMOE_OK if the current device is sm_100 and the driver exposes the
// tensor-map encoder; LMOE_ERR_UNSUPPORTED otherwise.
lmoe_status tc_check_device();

// C = A B^T with the epilogue `mode` (EPI_GLU, EPI_COMBINE, EPI_STORE), A and
// B bf16 K-major, K a multiple of 64, rows 16-byte aligned.  cg = 1: 128 x 256
// tiles on one CTA; cg = 2: 256 x 256 tiles on a two-CTA cluster.  Grouped when
// g.offsets != nullptr (tile_off built for 128 cg rows per m-tile; max_mtiles
// bounds the m-tiles of all experts).  Bounded waits that give up OR a code
// into *status.
// ksplit > 1 (dense, mode EPI_STORE_F32 only): the K range is split into
// ksplit parts whose fp32 partial tiles go to rows [split M, split M + M) of
// g.epi.out; launch_splitk_reduce sums them and applies the real epilogue.
cudaError_t tc_gemm(int mode, const GemmArgs &g, int max_mtiles, int cg, int32_t *status, cudaStream_t s,
                    int ksplit = 1);

// Number of SMs of the current device (after tc_check_device).
int tc_num_sms();

// Failure-detection test hook: the next tensor-core GEMM launch makes its MMA
// warp wait on a barrier that nothing signals; the bounded wait runs out, the
// status word records it and the kernel returns.
void tc_debug_stall_next();

// Router r = sigmoid(x W_r^T) from the three-term bf16 split of fp32 W_r
// (Wr3 = [3, E, d]): the three products accumulate into one fp32 TMEM tile,
// on (128 cg)-row tiles.  ksplit > 1: the 3 d/64 k-blocks are split into
// ksplit ranges whose raw fp32 partial tiles go to g.epi.out slabs (the top-k
// kernel sums them and applies the sigmoid).
cudaError_t tc_gemm_router(const bf16 *Wr3, const GemmArgs &g, int cg, int32_t *status, cudaStream_t s,
                           int ksplit = 1);

// Router scores, biased top-k and renormalisation in one launch (tensor
// cores, fp32 router through its three-term bf16 split Wr3 = [3, E, d]) for
// T tokens of x [T, d]: r [T, E] fp32, sel / p32 / p_out (token dtype) [T, k],
// the Quantile-Balancing cutoff [T] and the per-32-token expert counts added
// into blockhist [E][ceil(T / 32)] (zeroed by the caller).  The split
// logits are summed through the cluster's shared memory: no workspace.
// tc_router_topk_splits: CTAs per 128-token tile (a cluster), or 0 when this
// path does not apply (E > 256 or E not a multiple of 32) or does not pay
// (tiles enough to give every CTA a whole 128-token tile of its own).
int tc_router_topk_splits(int64_t T, int E, int d);
cudaError_t tc_router_topk(const bf16 *x, const bf16 *Wr3, const float *bias, int64_t T, int E, int d, int k,
                           float *r, int32_t *sel, float *p32, void *p_out, int out_bf16,
                           float *cutoff, int32_t *blockhist, int32_t *status, cudaStream_t s);

}  // namespace lmoe
