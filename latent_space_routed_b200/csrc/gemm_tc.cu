// Persistent tensor-core GEMM for sm_100a: TMA -> shared memory -> tcgen05.mma
// -> TMEM -> fused epilogue.
//
// C[m, n] = sum_k A[m, k] B[n, k], A and B bf16 and K-major (the "out x in"
// weights of the layer), fp32 accumulation in tensor memory.
//
// CTA = 6 warps, one CTA per SM, tiles of 128 x 256 x 64:
//   warp 0      TMA producer: one thread streams A (128 x 64) and B (256 x 64)
//               tiles into a 4-stage ring (SWIZZLE_128B), completing the
//               stage's "full" mbarrier by transaction bytes;
//   warp 1      TMEM owner and MMA issuer: one thread issues four
//               tcgen05.mma (M=128, N=256, K=16) per stage into one of two
//               256-column fp32 accumulators and commits the stage's "empty"
//               barrier, then the accumulator's "full" barrier per tile;
//   warps 2-5   epilogue: each warp owns one 32-lane quarter of TMEM (= 32
//               rows), reads 32-column chunks with tcgen05.ld and applies the
//               fused epilogue, then frees the accumulator, so the epilogue of
//               tile i overlaps the main loop of tile i+1.
// Tiles are handed out round-robin over a grid of min(SMs, tiles) CTAs, with
// the n-tile index fastest so that CTAs running together share the A tile.
//
// Grouped mode: m-tile i of the expert-sorted slot rows belongs to the expert
// e with tile_off[e] <= i < tile_off[e+1]; rows past offsets[e+1] are computed
// on whatever the TMA brought in (the next expert's rows, or zero fill past the
// end) and discarded by the epilogue.
//
// Every mbarrier wait is bounded by a cycle-count limit (about 2 s); a wait that gives up
// ORs a code into the status word, stops its role's loop, and the CTA drains
// the copies and MMAs it still has in flight (again bounded) before it frees
// its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "gemm_tc.cuh"

namespace lmoe {
namespace {

constexpr int BM = TC_BM, BN = TC_BN, BK = TC_BK, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 320;   // 2 role warps + 8 epilogue warps
constexpr int TMEM_COLS = 2 * BN;
constexpr long long WAIT_LIMIT_CYCLES = 4000000000ll;   // about 2 s at 2 GHz
constexpr int MAX_E = 1024;
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256 + 2 * sizeof(int) * (MAX_E + 1);

// status codes (OR-ed together)
constexpr int ST_PRODUCER = 0x1, ST_MMA = 0x2, ST_EPILOGUE = 0x4, ST_DRAIN = 0x8;

struct TcParams {
    int M;                      // dense rows
    int N;                      // valid output columns
    int nkb;                    // k-blocks per B term
    int nterms;                 // B terms summed into one accumulator (router: 3)
    int64_t term_rows;          // rows of B between terms
    int ntn;                    // n tiles
    int64_t group_rows;         // rows of B per expert (grouped)
    const int32_t *offsets;
    const int32_t *tile_off;
    int E;
    int max_tiles;              // dense: exact tile count
    EpiArgs epi;
    int32_t *status;
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete; false after the limit.
// The limit is counted on the SM's own cycle counter (cheap to read, unlike
// the global nanosecond timer, which is a long-latency read).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > WAIT_LIMIT_CYCLES) return false;
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"((uint64_t)map), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map) : "memory");
}

// UMMA shared-memory descriptor, K-major, 128-byte swizzle: rows of 128 bytes,
// 8-row atoms 1024 bytes apart (stride byte offset), leading byte offset 16.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major, M x N.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// bf16 outputs only: the gate with the hardware exp2 and reciprocal
// approximations (a few ulp of fp32, far below the bf16 rounding that follows).
__device__ __forceinline__ float rcp_approx(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <bool SITU>
__device__ __forceinline__ float glu_fast(float g, float v, float cg, float cu)
{
    const float sg = rcp_approx(1.0f + __expf(-g));
    if (SITU) return cg * tanhf(g * rcp_approx(cg)) * sg * (cu * tanhf(v * rcp_approx(cu)));
    return g * sg * v;
}

// Two 32x32b.x32 loads in flight, then one wait.
__device__ __forceinline__ void tmem_ld32_pair(uint32_t ta, uint32_t tb, float *va, float *vb)
{
    uint32_t r[32], s[32];
#define LMOE_TMEM_LD(dst, addr)                                                                                  \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "                                                      \
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "                       \
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"       \
                 : "=r"(dst[0]), "=r"(dst[1]), "=r"(dst[2]), "=r"(dst[3]), "=r"(dst[4]), "=r"(dst[5]),            \
                   "=r"(dst[6]), "=r"(dst[7]), "=r"(dst[8]), "=r"(dst[9]), "=r"(dst[10]), "=r"(dst[11]),          \
                   "=r"(dst[12]), "=r"(dst[13]), "=r"(dst[14]), "=r"(dst[15]), "=r"(dst[16]), "=r"(dst[17]),      \
                   "=r"(dst[18]), "=r"(dst[19]), "=r"(dst[20]), "=r"(dst[21]), "=r"(dst[22]), "=r"(dst[23]),      \
                   "=r"(dst[24]), "=r"(dst[25]), "=r"(dst[26]), "=r"(dst[27]), "=r"(dst[28]), "=r"(dst[29]),      \
                   "=r"(dst[30]), "=r"(dst[31])                                                                   \
                 : "r"(addr))
    LMOE_TMEM_LD(r, ta);
    LMOE_TMEM_LD(s, tb);
#undef LMOE_TMEM_LD
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        va[i] = __uint_as_float(r[i]);
        vb[i] = __uint_as_float(s[i]);
    }
}

// ------------------------------------------------------------------ epilogue stores
__device__ __forceinline__ void store32(bf16 *dst, const float *v)
{
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 p = __floats2bfloat162_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t *>(&p);
        }
        d[q] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__device__ __forceinline__ void store32(float *dst, const float *v)
{
    float4 *d = reinterpret_cast<float4 *>(dst);
#pragma unroll
    for (int q = 0; q < 8; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

template <typename TO>
__device__ __forceinline__ void store_n(TO *dst, const float *v, int n)
{
    if (n == 32 && ((uintptr_t)dst & 15u) == 0) {
        store32(dst, v);
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (i < n) dst[i] = from_f32<TO>(v[i]);
    }
}

// ------------------------------------------------------------------ tile decode
struct Tile {
    int64_t row0, row_end;  // A rows [row0, row_end) are real for this tile
    int64_t brow;           // first B row of this tile (term 0)
    int n0;                 // first output column (GEMM n)
};

// Grouped mode reads the expert row offsets and m-tile prefix from shared
// memory (staged once per CTA), so decoding a tile costs no global round trip.
__device__ __forceinline__ Tile decode(const TcParams &p, const int *s_tile_off, const int *s_offsets, int tile)
{
    Tile t;
    const int mt = tile / p.ntn, nt = tile % p.ntn;
    t.n0 = nt * BN;
    if (p.offsets) {
        int lo = 0, hi = p.E - 1;  // last e with tile_off[e] <= mt
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_tile_off[mid] <= mt) lo = mid; else hi = mid - 1;
        }
        t.row0 = (int64_t)s_offsets[lo] + (int64_t)(mt - s_tile_off[lo]) * BM;
        t.row_end = s_offsets[lo + 1];
        t.brow = (int64_t)lo * p.group_rows + t.n0;
    } else {
        t.row0 = (int64_t)mt * BM;
        t.row_end = p.M;
        t.brow = t.n0;
    }
    return t;
}

template <int MODE, typename TO>
__global__ void __launch_bounds__(THREADS, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;           // 1024-aligned stage ring
    uint8_t *gbase = smem_raw + (sbase - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(gbase + (size_t)STAGES * STAGE_BYTES);
    // bars[0..S) full, [S..2S) empty, [2S..2S+2) acc full, [2S+2..2S+4) acc empty
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 4);
    int *abort_flag = reinterpret_cast<int *>(tmem_holder + 1);
    int *drain_counts = abort_flag + 1;                      // [0] loads issued, [1] stages consumed
    int *s_tile_off = reinterpret_cast<int *>(gbase + (size_t)STAGES * STAGE_BYTES + 256);   // [E+1]
    int *s_offsets = s_tile_off + (MAX_E + 1);                                              // [E+1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto accf_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
    auto acce_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(accf_bar(a), 1);
            mbar_init(acce_bar(a), 8);   // one arrival per epilogue warp
        }
        *abort_flag = 0;
        drain_counts[0] = drain_counts[1] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (p.offsets) {
        for (int i = threadIdx.x; i <= p.E; i += THREADS) {
            s_tile_off[i] = p.tile_off[i];
            s_offsets[i] = p.offsets[i];
        }
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int total = p.offsets ? s_tile_off[p.E] * p.ntn : p.max_tiles;
    const int nkb_total = p.nkb * p.nterms;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------- TMA producer
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const Tile t = decode(p, s_tile_off, s_offsets, tile);
                for (int kb = 0; kb < nkb_total; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (!mbar_wait(empty_bar(s), ph ^ 1u) || *(volatile int *)abort_flag) {
                        atomicOr(p.status, ST_PRODUCER);
                        *(volatile int *)abort_flag = 1;
                        ok = false;
                        break;
                    }
                    const int term = kb / p.nkb, kk = (kb % p.nkb) * BK;
                    const uint32_t sa = sbase + (uint32_t)s * STAGE_BYTES;
                    mbar_expect_tx(full_bar(s), STAGE_BYTES);
                    tma_load_2d(sa, &tmA, full_bar(s), kk, (int)t.row0);
                    tma_load_2d(sa + A_BYTES, &tmB, full_bar(s), kk, (int)(t.brow + term * p.term_rows));
                    drain_counts[0] = it + 1;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------- MMA issuer
            int it = 0, local = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++local) {
                const int acc = local & 1;
                const uint32_t aph = (uint32_t)(local >> 1) & 1u;
                if (!mbar_wait(acce_bar(acc), aph ^ 1u)) {
                    atomicOr(p.status, ST_MMA);
                    *(volatile int *)abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t dt = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < nkb_total; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (!mbar_wait(full_bar(s), ph) || *(volatile int *)abort_flag) {
                        atomicOr(p.status, ST_MMA);
                        *(volatile int *)abort_flag = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = sbase + (uint32_t)s * STAGE_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        const uint64_t ad = sdesc_sw128(sa + 32u * k);
                        const uint64_t bd = sdesc_sw128(sa + A_BYTES + 32u * k);
                        umma_bf16(dt, ad, bd, (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit(empty_bar(s));
                    drain_counts[1] = it + 1;
                }
                if (ok) umma_commit(accf_bar(acc));
            }
        }
    } else {
        // -------------------------------------------------------- epilogue warps 2..9
        // Two warps per TMEM lane quarter; warp set h = 0/1 takes the 32-column
        // chunks c = 32 h + 64 i, so each warp drains half of its 32 rows' tile.
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int hset = (warp - 2) >> 2;       // 0 for warps 2..5, 1 for warps 6..9
        int local = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
            const int acc = local & 1;
            const uint32_t aph = (uint32_t)(local >> 1) & 1u;
            const bool got = mbar_wait(accf_bar(acc), aph);
            if (!got || *(volatile int *)abort_flag) {
                if (lane == 0) {
                    atomicOr(p.status, ST_EPILOGUE);
                    *(volatile int *)abort_flag = 1;
                }
                break;
            }
            tc_fence_after();
            const Tile t = decode(p, s_tile_off, s_offsets, tile);
            const int64_t row = t.row0 + 32 * q + lane;
            const bool valid = row < t.row_end;
            const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * BN);
            float v[32], u[32];
            if (MODE == EPI_GLU || MODE == EPI_GLU_SITU) {
                const int half = BN / 2;
#pragma unroll 1
                for (int c = 32 * hset; c < half; c += 64) {
                    __syncwarp();
                    tmem_ld32_pair(tq + c, tq + half + c, v, u);   // gate and up columns, one wait
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = glu_fast<MODE == EPI_GLU_SITU>(v[i], u[i], p.epi.gate_cap,
                                                                                       p.epi.up_cap);
                    if (valid) store_n((TO *)p.epi.out + row * p.epi.ldo + t.n0 / 2 + c, v, 32);
                }
            } else {
#pragma unroll 1
                for (int c = 32 * hset; c < BN; c += 128) {
                    __syncwarp();
                    tmem_ld32_pair(tq + c, tq + c + 64, v, u);     // warp-collective: every lane
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
                        float *x = part ? u : v;
                        const int col = t.n0 + c + 64 * part;
                        int n = p.N - col;
                        if (n > 32) n = 32;
                        if (!valid || n <= 0) {
                            // nothing to store for this lane
                        } else if (MODE == EPI_SIGMOID) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) x[i] = sigmoidf_(x[i]);
                            store_n((float *)p.epi.out + row * p.epi.ldo + col, x, n);
                        } else if (MODE == EPI_COMBINE) {
                            const float w = p.epi.row_w[row];
#pragma unroll
                            for (int i = 0; i < 32; ++i) x[i] *= w;
                            store_n((float *)p.epi.out + row * p.epi.ldo + col, x, n);
                        } else {
                            store_n((TO *)p.epi.out + row * p.epi.ldo + col, x, n);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce_bar(acc));
        }
    }

    __syncthreads();
    if (*(volatile int *)abort_flag && threadIdx.x == 0) {
        // Drain: loads issued but never consumed, then the MMAs behind the last commit.
        const int issued = drain_counts[0], consumed = drain_counts[1];
        bool ok = true;
        for (int i = consumed; i < issued; ++i)
            ok &= mbar_wait(full_bar(i % STAGES), (uint32_t)(i / STAGES) & 1u);
        if (consumed > 0) {
            const int i = consumed - 1;
            ok &= mbar_wait(empty_bar(i % STAGES), (uint32_t)(i / STAGES) & 1u);
        }
        if (!ok) atomicOr(p.status, ST_DRAIN);
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
int g_num_sms = 0;

bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_outer)
{
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_outer};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int MODE, typename TO>
cudaError_t launch(const CUtensorMap &a, const CUtensorMap &b, const TcParams &p, int grid, cudaStream_t s)
{
    const cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<MODE, TO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    tc_gemm_kernel<MODE, TO><<<grid, THREADS, SMEM_BYTES, s>>>(a, b, p);
    return cudaGetLastError();
}

cudaError_t run(int mode, const GemmArgs &g, int max_mtiles, int nterms, int64_t term_rows, int64_t b_rows_total,
                int32_t *status, cudaStream_t s)
{
    if (!g_encode) return cudaErrorInitializationError;
    if (g.K % BK) return cudaErrorInvalidValue;
    if (((uintptr_t)g.A | (uintptr_t)g.B) & 15u) return cudaErrorMisalignedAddress;
    if ((g.lda * 2) % 16 || (g.ldb * 2) % 16) return cudaErrorMisalignedAddress;
    TcParams p = {};
    p.M = g.M;
    p.N = g.N;
    p.nkb = g.K / BK;
    p.nterms = nterms;
    p.term_rows = term_rows;
    p.ntn = mode == EPI_GLU ? g.N / BN : (g.N + BN - 1) / BN;   // GLU: N = 2F, F % (BN/2) == 0
    p.group_rows = g.offsets ? g.b_group_stride / g.ldb : 0;
    p.offsets = g.offsets;
    p.tile_off = g.tile_off;
    p.E = g.E;
    const int mtiles = g.offsets ? max_mtiles : (g.M + BM - 1) / BM;
    p.max_tiles = mtiles * p.ntn;
    p.epi = g.epi;
    p.status = status;
    if (p.max_tiles == 0) return cudaSuccess;
    const int64_t a_rows = g.M;   // grouped: M = total slot rows
    CUtensorMap ta, tb;
    if (!make_map(&ta, g.A, (uint64_t)g.K, (uint64_t)a_rows, (uint64_t)g.lda * 2, BM)) return cudaErrorInvalidValue;
    if (!make_map(&tb, g.B, (uint64_t)g.K, (uint64_t)b_rows_total, (uint64_t)g.ldb * 2, BN))
        return cudaErrorInvalidValue;
    const int grid = p.max_tiles < g_num_sms ? p.max_tiles : g_num_sms;
    switch (mode) {
    case EPI_SIGMOID: return launch<EPI_SIGMOID, float>(ta, tb, p, grid, s);
    case EPI_GLU:
        if (g.epi.act == LMOE_ACT_SITU) return launch<EPI_GLU_SITU, bf16>(ta, tb, p, grid, s);
        return launch<EPI_GLU, bf16>(ta, tb, p, grid, s);
    case EPI_COMBINE: return launch<EPI_COMBINE, float>(ta, tb, p, grid, s);
    case EPI_STORE: return launch<EPI_STORE, bf16>(ta, tb, p, grid, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

lmoe_status tc_check_device()
{
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LMOE_ERR_CUDA;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return LMOE_ERR_UNSUPPORTED;
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (!g_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return LMOE_ERR_UNSUPPORTED;
        g_encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
    }
    return LMOE_OK;
}

cudaError_t tc_gemm(int mode, const GemmArgs &g, int max_mtiles, int32_t *status, cudaStream_t s)
{
    // B rows: dense N; grouped E * (rows per expert)
    const int64_t b_rows = g.offsets ? (int64_t)g.E * (g.b_group_stride / g.ldb) : g.N;
    return run(mode, g, max_mtiles, 1, 0, b_rows, status, s);
}

cudaError_t tc_gemm_router(const bf16 *Wr3, const GemmArgs &g, int32_t *status, cudaStream_t s)
{
    GemmArgs r = g;
    r.B = Wr3;
    r.ldb = g.K;
    return run(EPI_SIGMOID, r, 0, 3, g.N, 3 * (int64_t)g.N, status, s);
}

}  // namespace lmoe
