// Persistent tensor-core GEMM for sm_100a: TMA -> shared memory -> tcgen05.mma
// -> TMEM -> fused epilogue.
//
// C[m, n] = sum_k A[m, k] B[n, k], A and B bf16 and K-major (the "out x in"
// weights of the layer), fp32 accumulation in tensor memory.  Output tiles are
// (128 CG) x 256 with K steps of 64:
//
//   CG = 1  one CTA per tile, tcgen05.mma.cta_group::1 with M = 128, N = 256;
//   CG = 2  a cluster of two CTAs per tile, tcgen05.mma.cta_group::2 with
//           M = 256, N = 256: CTA r holds A rows 128 r .. 128 r + 127 and B rows
//           (output columns) 128 r .. 128 r + 127 of every k-step, the even
//           ("leader") CTA issues the MMAs for both, and each CTA's tensor memory
//           receives its own 128 accumulator rows.  Each SM then moves and reads
//           32 KB of operands per k-step instead of 48 KB for the same work per
//           SM; with 48 KB the shared-memory traffic of TMA writes plus MMA reads
//           holds the MMA at about half its rate.
//
// Warp roles in each CTA (10 warps):
//   warp 0      TMA producer (one thread): streams its A and B shares into a
//               STAGES-deep ring (SWIZZLE_128B) and signals the leader CTA's
//               "full" barrier of the stage (transaction bytes);
//   warp 1      TMEM owner; in the leader CTA one thread issues the MMAs into one
//               of two 256-column fp32 accumulators, commits each stage's "empty"
//               barrier (in both CTAs) once its MMAs have read it, then the
//               accumulator's "full" barrier (in both CTAs) per tile;
//   warps 2-9   epilogue: two warps per 32-lane TMEM quarter read 32-column
//               chunks with tcgen05.ld, apply the fused epilogue, and arrive on
//               the leader's accumulator "empty" barrier, so the epilogue of
//               tile i overlaps the main loop of tile i+1.
// Tiles are handed out round-robin over min(SMs / CG, tiles) CTA groups, with
// the n-tile index fastest so that groups running together share the A tile.
//
// Grouped mode: m-tile i of the expert-sorted slot rows belongs to the expert
// e with tile_off[e] <= i < tile_off[e+1] (tile_off built for 128 CG rows);
// rows past offsets[e+1] are computed on whatever the TMA brought in (the next
// expert's rows, or zero fill past the end) and discarded by the epilogue.
//
// Every mbarrier wait is bounded by a cycle-count limit (about 2 s); a wait
// that gives up ORs a code into the status word, stops its role's loop, and the
// CTA drains what it still has in flight (again bounded) before it frees its
// TMEM and returns.
#include <atomic>
#include <cstring>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "gemm_tc.cuh"
#include "topk.cuh"

namespace lmoe {
namespace {

constexpr int BN = TC_BN, BK = TC_BK;
// Warps: 0, 10 and 11 TMA producers, 1 MMA issuer / TMEM owner, 2..9 epilogue.
// Each thread's tensor copies go out one after another (measured on B200: one
// issuing thread moves 16 KB tiles at about 6.4 TB/s across the chip, two
// threads at twice that), so up to three producers share the k-steps (with
// two k-blocks per copy that keeps the CTA-pair GEMMs fed: a fourth producer
// warp measured no faster).  Twelve warps of 128 registers leave room on each
// of the SM's four schedulers for a small kernel's warps beside a GEMM CTA
// (with thirteen, one scheduler's register file is full), so the latency-bound
// routing kernels can run beside the shared-expert GEMM.
//
// Producer q of P takes k-steps it = q (mod P) into ring slot it % S and first
// waits for that slot's previous use to be consumed, by the parity of the
// slot's "empty" barrier.  A parity wait is only sound while the barrier is at
// most one phase behind, i.e. while the use before the previous one has been
// consumed: the producer's own previous wait (k-step it - P) guaranteed the
// consumption of it - P - S, which covers it - 2 S exactly when P <= S.  So a
// ring of S stages runs min(NPROD, S) producers.
constexpr int NPROD = 3;
constexpr int THREADS = 32 * (2 + 8 + NPROD - 1);
__device__ __forceinline__ int producer_index(int warp) { return warp == 0 ? 0 : (warp >= 10 ? warp - 9 : -1); }
constexpr int TMEM_COLS = 2 * BN;
constexpr long long WAIT_LIMIT_CYCLES = 4000000000ll;   // about 2 s at 2 GHz
constexpr int MAX_E = 1024;
// KPS: 64-wide k-blocks per ring stage.  The MMA issuer commits each stage's
// "empty" barrier once, and a commit costs tensor-pipe time: measured on B200,
// a commit after every 4 MMAs holds them at 75 % of the pipe's rate, after
// every 8 (CTA pairs) at 93 %, after every 16 at 100 %.  So the CTA-pair
// GEMMs with bf16 outputs (the large ones) take two k-blocks per stage, laid
// out as [A kb0][A kb1][B kb0][B kb1], each a standard 128-byte-swizzled tile.
template <int CG, int KPS = 1> struct Tiles {
    static constexpr int A_SUB = 128 * BK * 2;                  // this CTA's 128 A rows, one k-block
    static constexpr int B_SUB = (BN / CG) * BK * 2;            // this CTA's share of B rows, one k-block
    static constexpr int A_BYTES = KPS * A_SUB;
    static constexpr int B_BYTES = KPS * B_SUB;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TILE_M = 128 * CG;
    // kind::f16, D fp32, A and B bf16, both K-major, M = 128 CG, N = BN
    static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                      ((uint32_t)(TILE_M >> 4) << 24);
};

// Shared memory of one CTA for output elements of OB bytes: the expert tables,
// one 32 x 32 output chunk of staging per epilogue warp (written swizzled and
// stored by TMA), and as many operand stages as fit (at most 6): the weight
// tiles of a grouped GEMM mostly come from HBM, and the ring is what keeps
// their loads in flight.
template <int CG, int OB, int KPS_ = (CG == 2 && OB == 2) ? 2 : 1> struct Cfg : Tiles<CG, KPS_> {
    static constexpr int KPS = KPS_;
    static constexpr int EPI_CHUNK = 32 * 32 * OB;
    static constexpr int EPI_STAGING = 8 * EPI_CHUNK;
    static constexpr int TABLES = 2 * (int)sizeof(int) * (MAX_E + 1);
    static constexpr int FIXED = 1024 + EPI_STAGING + 256 + TABLES;
    static constexpr int STAGES_FIT = (232448 - FIXED) / Tiles<CG, KPS_>::STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
    static constexpr size_t SMEM = (size_t)FIXED + (size_t)STAGES * Tiles<CG, KPS_>::STAGE_BYTES;
    static_assert(STAGES >= 3, "operand ring too shallow");
};

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
    int ksplit;                 // >1: K split into ksplit ranges, partial tiles to row slab `split`
    int64_t split_rows;         // rows of one partial slab (= M)
    EpiArgs epi;
    int out_cols;               // columns of the output tensor map
    int stall_test;             // failure-detection test: the MMA warp waits on a barrier nobody signals
    int tma_store;              // 1: full chunks leave through TMA stores
    int load3d;                 // 1: the tensor maps are 3D (KPS k-blocks per copy)
    int half_tiles;             // 1: an expert's last m-tile of at most 64 CG rows runs as an M = 64 CG MMA
    int no_early_launch;        // 1: launched without programmatic dependent launch
    int32_t *status;
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Arrive on a barrier given by its shared::cluster address (own CTA or peer).
// Default semantics (release, CTA scope): what the arrive orders is this
// warp's TMEM reads, already fenced by tcgen05.fence::before_thread_sync.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Default semantics (acquire, CTA scope).  A phase completes only when its
// transaction bytes (TMA, including a peer CTA's copies into this pair) and
// its arrivals are in, which is what orders the consumers' reads; measured, a
// cluster-scope acquire on every wait of the MMA issuer costs tensor-pipe time.
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
// The limit is counted on the SM's own cycle counter (cheap to read).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > WAIT_LIMIT_CYCLES) return false;
    }
}

// 2D tile load into this CTA's shared memory; completion bytes go to `bar`,
// a shared::cluster address that is the leader CTA's barrier when CG = 2.
template <int CG>
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1)
{
    if (CG == 2)
        asm volatile(
            "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%3, %4}], [%2];"
            ::"r"(dst), "l"((uint64_t)map), "r"(bar), "r"(c0), "r"(c1)
            : "memory");
    else
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%3, %4}], [%2];"
            ::"r"(dst), "l"((uint64_t)map), "r"(bar), "r"(c0), "r"(c1)
            : "memory");
}

// 3D tile load: coordinates {k inside the k-block, row, k-block}; with a box
// of {64, rows, KPS} it brings KPS consecutive k-blocks of the same rows as KPS
// standard 128-byte-swizzled tiles, one after another, in one copy.
template <int CG>
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c1, int c2)
{
    if (CG == 2)
        asm volatile(
            "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%3, %4, %5}], [%2];"
            ::"r"(dst), "l"((uint64_t)map), "r"(bar), "r"(0), "r"(c1), "r"(c2)
            : "memory");
    else
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%3, %4, %5}], [%2];"
            ::"r"(dst), "l"((uint64_t)map), "r"(bar), "r"(0), "r"(c1), "r"(c2)
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

template <int CG>
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    if (CG == 2)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Arrive on `bar` (the same offset in every CTA of the group) once all MMAs
// issued so far by this thread have completed.
template <int CG>
__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    if (CG == 2)
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
            ::"r"(bar), "h"((uint16_t)0x3)
            : "memory");
    else
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                     : "memory");
}

// 2D tile store from this CTA's shared memory (bulk group of the calling thread).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int c0, int c1)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"((uint64_t)map), "r"(src), "r"(c0), "r"(c1)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Write this lane's 32 outputs as row `lane` of the warp's 32 x 32 staging
// chunk, in the layout a SWIZZLE_64B (bf16: 64-byte rows) or SWIZZLE_128B
// (fp32: 128-byte rows) tensor map expects: 16-byte piece c of row r sits at
// piece c ^ ((r >> 1) & 3), resp. c ^ (r & 7); the pieces of one instruction
// then fall in distinct banks.
__device__ __forceinline__ void stage_row(uint32_t buf, int lane, const float *v, bf16 *)
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 pr = __floats2bfloat162_rn(v[c * 8 + 2 * i], v[c * 8 + 2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t *>(&pr);
        }
        st_shared_v4(buf + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4), w[0], w[1], w[2], w[3]);
    }
}

__device__ __forceinline__ void stage_row(uint32_t buf, int lane, const float *v, float *)
{
#pragma unroll
    for (int c = 0; c < 8; ++c)
        st_shared_v4(buf + lane * 128 + ((c ^ (lane & 7)) << 4), __float_as_uint(v[4 * c]),
                     __float_as_uint(v[4 * c + 1]), __float_as_uint(v[4 * c + 2]), __float_as_uint(v[4 * c + 3]));
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

// sigmoid(x) = (1 + tanh(x / 2)) / 2: one tanh.approx (a single MUFU
// operation) instead of an exponential and a reciprocal; its error, a few
// units in 2^-11, is below the bf16 rounding that follows.
__device__ __forceinline__ float tanh_approx(float x)
{
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <bool SITU>
__device__ __forceinline__ float glu_fast(float g, float v, float cg, float cu)
{
    const float sg = fmaf(0.5f, tanh_approx(0.5f * g), 0.5f);
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
    int64_t row0, row_end;  // A rows [row0, row_end) of the whole (128 CG)-row tile are real
    int64_t brow;           // first B row of this tile (term 0)
    int n0;                 // first output column (GEMM n)
    bool half;              // half tile: 64 rows per CTA, M = 64 CG
};

// Grouped mode reads the expert row offsets and m-tile prefix from shared
// memory (staged once per CTA), so decoding a tile costs no global round trip.
template <int CG>
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
        t.row0 = (int64_t)s_offsets[lo] + (int64_t)(mt - s_tile_off[lo]) * Tiles<CG>::TILE_M;
        t.row_end = s_offsets[lo + 1];
        t.brow = (int64_t)lo * p.group_rows + t.n0;
        t.half = CG == 2 && p.half_tiles && t.row_end - t.row0 <= 64 * CG;
    } else {
        t.row0 = (int64_t)mt * Tiles<CG>::TILE_M;
        t.row_end = p.M;
        t.brow = t.n0;
        t.half = false;
    }
    return t;
}

template <int MODE, typename TO, int CG>
__global__ void __launch_bounds__(THREADS, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAh,
               const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC, const TcParams p)
{
    using C = Cfg<CG, (int)sizeof(TO)>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;           // 1024-aligned stage ring
    uint8_t *gbase = smem_raw + (sbase - raw);
    const uint32_t epi_base = sbase + (uint32_t)(STAGES * C::STAGE_BYTES);   // 1024-aligned staging
    uint64_t *bars = reinterpret_cast<uint64_t *>(gbase + (size_t)STAGES * C::STAGE_BYTES + C::EPI_STAGING);
    // bars[0..S) full, [S..2S) empty, [2S..2S+2) acc full, [2S+2..2S+4) acc empty
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 4);
    int *abort_flag = reinterpret_cast<int *>(tmem_holder + 1);
    int *drain_counts = abort_flag + 1;   // [0, NPROD) k-steps issued by each producer, [NPROD] consumed
    int *s_half = drain_counts + NPROD + 1;   // [STAGES] half-tile flag of the k-step in ring slot s
    int *s_tile_off = reinterpret_cast<int *>(gbase + (size_t)STAGES * C::STAGE_BYTES + C::EPI_STAGING + 256);
    int *s_offsets = s_tile_off + (MAX_E + 1);                                                 // [E+1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = CG == 2 ? cluster_rank() : 0u;
    const bool leader = rank == 0;
    const int group = blockIdx.x / CG, ngroups = gridDim.x / CG;
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto accf_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
    auto acce_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);      // the leader's producer arms it for the whole group
            mbar_init(empty_bar(s), 1);     // one MMA commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(accf_bar(a), 1);
            mbar_init(acce_bar(a), 8 * CG);  // every epilogue warp of the group
        }
        *abort_flag = 0;
        for (int i = 0; i <= NPROD; ++i) drain_counts[i] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (p.half_tiles) tma_prefetch_desc(&tmAh);
    }
    if (warp == 1) {
        if (CG == 2) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                         ::"r"(smem_u32(tmem_holder)), "r"(TMEM_COLS) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                         ::"r"(smem_u32(tmem_holder)), "r"(TMEM_COLS) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    // the prologue above overlaps the previous kernel's tail; from here on this
    // kernel reads its inputs (A rows, expert tables) and writes its outputs
    griddep_wait();
    griddep_launch_dependents();
    if (p.offsets) {
        for (int i = threadIdx.x; i <= p.E; i += THREADS) {
            s_tile_off[i] = p.tile_off[i];
            s_offsets[i] = p.offsets[i];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (CG == 2) cluster_sync();     // peer barriers initialised before any remote signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int total = (p.offsets ? s_tile_off[p.E] * p.ntn : p.max_tiles) * p.ksplit;   // work items
    const int nkb_total = p.nkb * p.nterms;
    const int pw = producer_index(warp);
    constexpr int NP = NPROD < STAGES ? NPROD : STAGES;   // producers in use (see NPROD)

    if (pw >= 0) {
        if (lane == 0 && pw < NP) {
            // ---------------------------------------------------- TMA producers
            // Producer pw issues the loads of k-steps it with it % NP == pw:
            // a thread's tensor copies go out one after another, so several
            // issuing threads are what keeps the operand ring full.
            int it = 0;
            bool ok = true;
            for (int item = group; item < total && ok; item += ngroups) {
                const Tile t = decode<CG>(p, s_tile_off, s_offsets, item / p.ksplit);
                const int split = item % p.ksplit;
                const int kb_end = (split + 1) * nkb_total / p.ksplit;
                for (int kb = split * nkb_total / p.ksplit; kb < kb_end; kb += C::KPS, ++it) {
                    if (it % NP != pw) continue;
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (!mbar_wait(empty_bar(s), ph ^ 1u) || *(volatile int *)abort_flag) {
                        atomicOr(p.status, ST_PRODUCER);
                        *(volatile int *)abort_flag = 1;
                        ok = false;
                        break;
                    }
                    const int nk = kb_end - kb < C::KPS ? kb_end - kb : C::KPS;   // k-blocks in this stage
                    const uint32_t sa = sbase + (uint32_t)s * C::STAGE_BYTES;
                    if (leader) s_half[s] = t.half;   // published to the MMA thread by the arrive below
                    const uint32_t fb = CG == 2 ? map_to_rank(full_bar(s), 0) : full_bar(s);
                    if (C::KPS > 1 && p.load3d) {
                        // one copy per operand; a k-block past the end reads as zeros
                        // (and its MMAs are skipped) but still counts its bytes
                        if (t.half) {   // 64 A rows per CTA: [kb0 64 rows][kb1 64 rows]
                            if (leader) mbar_expect_tx(full_bar(s), CG * (C::A_BYTES / 2 + C::B_BYTES));
                            tma_load_3d<CG>(sa, &tmAh, fb, (int)(t.row0 + 64 * rank), kb);
                        } else {
                            if (leader) mbar_expect_tx(full_bar(s), CG * C::STAGE_BYTES);
                            tma_load_3d<CG>(sa, &tmA, fb, (int)(t.row0 + 128 * rank), kb);
                        }
                        tma_load_3d<CG>(sa + C::A_BYTES, &tmB, fb, (int)(t.brow + (BN / CG) * rank), kb);
                    } else {
                        if (leader) mbar_expect_tx(full_bar(s), CG * nk * (C::A_SUB + C::B_SUB));
                        for (int j = 0; j < nk; ++j) {
                            const int term = (kb + j) / p.nkb, kk = ((kb + j) % p.nkb) * BK;
                            tma_load_2d<CG>(sa + j * C::A_SUB, &tmA, fb, kk, (int)(t.row0 + 128 * rank));
                            tma_load_2d<CG>(sa + C::A_BYTES + j * C::B_SUB, &tmB, fb, kk,
                                            (int)(t.brow + (BN / CG) * rank + term * p.term_rows));
                        }
                    }
                    drain_counts[pw] = it + 1;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------------------------------------------- MMA issuer (leader CTA)
            // Between MMAs this thread does as little as it can (measured: a few
            // extra instructions per MMA cost tensor-pipe time): the ring slot
            // and phase advance incrementally, the shared-memory descriptors
            // are a base plus constants, and the abort flag and the TMEM fence
            // are looked at once per tile, not per k-step.
            const uint64_t desc_base = sdesc_sw128(sbase);
            constexpr uint32_t STAGE16 = C::STAGE_BYTES >> 4, A16 = C::A_BYTES >> 4;
            constexpr uint32_t ASUB16 = C::A_SUB >> 4, BSUB16 = C::B_SUB >> 4;
            constexpr uint32_t IDESC_HALF = (C::IDESC & ~(0x1fu << 24)) | ((uint32_t)((64 * CG) >> 4) << 24);
            int it = 0, local = 0;
            int s = 0;
            uint32_t ph = 0u;
            bool ok = true;
            for (int item = group; item < total && ok; item += ngroups, ++local) {
                const int acc = local & 1;
                const uint32_t aph = (uint32_t)(local >> 1) & 1u;
                const int split = item % p.ksplit;
                const int kb_begin = split * nkb_total / p.ksplit, kb_end = (split + 1) * nkb_total / p.ksplit;
                // half tile: M = 64 CG, this CTA's k-blocks of A 64 rows (8 KB) apart; the
                // flag comes with the tile's first stage (no table search in this thread)
                uint32_t idesc = C::IDESC, astep = ASUB16;
                if (!mbar_wait(acce_bar(acc), aph ^ 1u) || *(volatile int *)abort_flag) {
                    atomicOr(p.status, ST_MMA);
                    *(volatile int *)abort_flag = 1;
                    break;
                }
                tc_fence_after();
                if (p.stall_test && local == 0 && !mbar_wait(accf_bar(acc), 0u)) {
                    // only this thread commits that barrier: the wait runs out by design
                    atomicOr(p.status, ST_MMA);
                    *(volatile int *)abort_flag = 1;
                    break;
                }
                const uint32_t dt = tmem_base + (uint32_t)(acc * BN);
                uint32_t accumulate = 0u;      // the tile's first MMA overwrites the accumulator
                for (int kb = kb_begin; kb < kb_end; kb += C::KPS, ++it) {
                    if (!mbar_wait(full_bar(s), ph)) {
                        atomicOr(p.status, ST_MMA);
                        *(volatile int *)abort_flag = 1;
                        ok = false;
                        break;
                    }
                    if (kb == kb_begin && p.half_tiles && s_half[s]) {
                        idesc = IDESC_HALF;
                        astep = ASUB16 / 2;
                    }
                    const uint64_t da = desc_base + (uint64_t)(s * STAGE16);
#pragma unroll
                    for (int j = 0; j < C::KPS; ++j) {
                        if (j > 0 && kb + j >= kb_end) break;      // a tile's odd last k-block
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k) {
                            umma_bf16<CG>(dt, da + (uint64_t)(j * astep + 2 * k),
                                          da + (uint64_t)(A16 + j * BSUB16 + 2 * k), idesc, accumulate);
                            accumulate = 1u;
                        }
                    }
                    umma_commit<CG>(empty_bar(s));
                    drain_counts[NPROD] = it + 1;
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (ok) umma_commit<CG>(accf_bar(acc));
            }
        }
    } else {
        // -------------------------------------------------------- epilogue warps 2..9
        // Two warps per TMEM lane quarter; warp set h = 0/1 takes the 32-column
        // chunk pairs (c, c + 64) with c = 32 h + 128 i, so each warp drains half
        // of its 32 rows' tile.  A half tile (M = 64 CG) holds this CTA's 64 rows
        // with GEMM columns [0, 128) in lanes 0-63 and [128, 256) in lanes 64-127,
        // both at TMEM columns [0, 128): quarter q has rows 32 (q & 1) + lane and
        // GEMM columns 128 (q >> 1) + [0, 128), one chunk pair per warp.
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int hset = (warp - 2) >> 2;       // 0 for warps 2..5, 1 for warps 6..9
        const uint32_t ebuf = epi_base + (uint32_t)(warp - 2) * C::EPI_CHUNK;
        int local = 0;
        for (int item = group; item < total; item += ngroups, ++local) {
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
            const Tile t = decode<CG>(p, s_tile_off, s_offsets, item / p.ksplit);
            const int64_t slab = (int64_t)(item % p.ksplit) * p.split_rows;   // 0 unless split K
            const int64_t chunk_row = t.half ? t.row0 + 64 * rank + 32 * (q & 1) : t.row0 + 128 * rank + 32 * q;
            const int cbase = t.half ? 128 * (q >> 1) : 0;   // GEMM column of this quarter's TMEM column 0
            const int npair = t.half ? 1 : 2;                // chunk pairs per warp
            const int64_t row = chunk_row + lane;
            const bool valid = row < t.row_end;
            const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * BN);
            float v[32], u[32];
            // Emit 32 output columns [col, col + n) of this warp's 32 rows: whole
            // chunks go through the staging buffer and one TMA store; chunks that
            // straddle an expert's last row (or a ragged column edge) store per lane.
            const bool rows_ok = (p.offsets || p.ksplit > 1) ? (chunk_row + 32 <= t.row_end) : true;
            auto emit = [&](const float *x, int col, int n) {
                if (p.tma_store && rows_ok && n == 32) {
                    // the warp's previous store must have finished reading its chunk
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
                    const uint32_t buf = ebuf;
                    stage_row(buf, lane, x, (TO *)nullptr);
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) tma_store_2d(&tmC, buf, col, (int)(slab + chunk_row));
                } else if (valid) {
                    store_n((TO *)p.epi.out + (slab + row) * p.epi.ldo + col, x, n);
                }
            };
            if (MODE == EPI_GLU || MODE == EPI_GLU_SITU) {
                // gate/up rows interleaved in blocks of 64: GEMM columns [128 i, 128 i + 64)
                // are gates of outputs 64 i + [0, 64), the next 64 their ups
#pragma unroll 1
                for (int i = 0; i < npair; ++i) {
                    const int c = 32 * hset + 128 * i;
                    __syncwarp();
                    tmem_ld32_pair(tq + c, tq + c + 64, v, u);     // gate and up columns, one wait
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = glu_fast<MODE == EPI_GLU_SITU>(v[e], u[e], p.epi.gate_cap,
                                                                                       p.epi.up_cap);
                    emit(v, (t.n0 + cbase) / 2 + 32 * hset + 64 * i, 32);
                }
            } else {
#pragma unroll 1
                for (int i = 0; i < npair; ++i) {
                    const int c = 32 * hset + 128 * i;
                    __syncwarp();
                    tmem_ld32_pair(tq + c, tq + c + 64, v, u);     // warp-collective: every lane
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
                        float *x = part ? u : v;
                        const int col = t.n0 + cbase + c + 64 * part;
                        int n = p.N - col;
                        if (n > 32) n = 32;
                        if (n <= 0) continue;             // uniform across the warp
                        if (MODE == EPI_SIGMOID) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) x[i] = sigmoidf_(x[i]);
                        } else if (MODE == EPI_STORE && sizeof(TO) == 2) {
                            if (p.epi.residual && valid) {   // standard MoE: y = shared + u
                                const bf16 *res = (const bf16 *)p.epi.residual + (slab + row) * p.epi.ldr + col;
                                if (n == 32 && ((uintptr_t)res & 15u) == 0) {
#pragma unroll
                                    for (int q8 = 0; q8 < 4; ++q8) {   // four 16-byte loads
                                        const uint4 w = *reinterpret_cast<const uint4 *>(res + 8 * q8);
                                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                                        for (int i = 0; i < 4; ++i) {
                                            const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162 *>(&ws[i]);
                                            x[8 * q8 + 2 * i] += __low2float(h2);
                                            x[8 * q8 + 2 * i + 1] += __high2float(h2);
                                        }
                                    }
                                } else {
#pragma unroll
                                    for (int i = 0; i < 32; ++i)
                                        if (i < n) x[i] += __bfloat162float(res[i]);
                                }
                            }
                        } else if (MODE == EPI_COMBINE) {
                            const float w = valid ? p.epi.row_w[row] : 0.f;   // bf16 rows: p-weighted here
#pragma unroll
                            for (int i = 0; i < 32; ++i) x[i] *= w;
                        }
                        emit(x, col, n);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(CG == 2 ? map_to_rank(acce_bar(acc), 0) : acce_bar(acc));
        }
        if (lane == 0) bulk_wait_all();             // this warp's TMA stores are complete
    }

    __syncthreads();
    if (*(volatile int *)abort_flag && threadIdx.x == 0 && leader) {
        // Drain: loads issued but never consumed (each producer's own k-steps),
        // then the MMAs behind the last commit.
        const int consumed = drain_counts[NPROD];
        bool ok = true;
        for (int q = 0; q < NP; ++q)
            for (int i = consumed; i < drain_counts[q]; ++i)
                if (i % NP == q) ok &= mbar_wait(full_bar(i % STAGES), (uint32_t)(i / STAGES) & 1u);
        if (consumed > 0) {
            const int i = consumed - 1;
            ok &= mbar_wait(empty_bar(i % STAGES), (uint32_t)(i / STAGES) & 1u);
        }
        if (!ok) atomicOr(p.status, ST_DRAIN);
    }
    tc_fence_before();
    __syncthreads();
    if (CG == 2) cluster_sync();     // no CTA leaves while its peer may still touch its memory
    tc_fence_after();
    if (warp == 1) {
        if (CG == 2)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                         : "memory");
    }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::atomic<int> g_stall_next{0};
int g_num_sms = 0;

// Output map: 32 x 32 boxes, swizzled to match stage_row.
bool make_out_map(CUtensorMap *m, void *base, bool f32, uint64_t cols, uint64_t rows, uint64_t row_bytes)
{
    if (((uintptr_t)base & 15u) || (row_bytes & 15u)) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base,
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3D view {64 k (contiguous), rows (row_bytes apart), k-blocks (128 bytes
// apart)} of a K-major bf16 matrix, box {64, box_rows, kps}: one copy lands
// kps k-blocks of box_rows rows as kps 128-byte-swizzled tiles back to back.
bool make_map3(CUtensorMap *m, const void *base, uint64_t K, uint64_t rows, uint64_t row_bytes, uint32_t box_rows,
               uint32_t kps)
{
    cuuint64_t dims[3] = {(cuuint64_t)BK, rows, K / BK};
    cuuint64_t strides[2] = {row_bytes, (cuuint64_t)BK * 2};
    cuuint32_t box[3] = {(cuuint32_t)BK, box_rows, kps};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

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

// Per-device, per-instantiation launch setup (shared-memory opt-in and, for
// CTA pairs, how many pairs fit at once), done on first use and cached.
constexpr int MAX_DEVICES = 64;

template <int MODE, typename TO, int CG>
cudaError_t group_capacity(int *max_groups)
{
    static std::atomic<int> cached[MAX_DEVICES];   // 0 = not yet known
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < MAX_DEVICES && cached[dev] > 0) {
        *max_groups = cached[dev];
        return cudaSuccess;
    }
    auto kern = tc_gemm_kernel<MODE, TO, CG>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg<CG, (int)sizeof(TO)>::SMEM);
    if (e != cudaSuccess) return e;
    int groups = g_num_sms / CG;
    if (CG > 1) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(g_num_sms / CG * CG);
        q.blockDim = dim3(THREADS);
        q.dynamicSmemBytes = Cfg<CG, (int)sizeof(TO)>::SMEM;
        cudaLaunchAttribute qa[1];
        qa[0].id = cudaLaunchAttributeClusterDimension;
        qa[0].val.clusterDim.x = CG;
        qa[0].val.clusterDim.y = 1;
        qa[0].val.clusterDim.z = 1;
        q.attrs = qa;
        q.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &q) == cudaSuccess && n > 0 && n < groups) groups = n;
        cudaGetLastError();
    }
    if (dev >= 0 && dev < MAX_DEVICES) cached[dev] = groups;
    *max_groups = groups;
    return cudaSuccess;
}

// Persistent grid: min(work items, CTA groups that can be resident at once).
template <int MODE, typename TO, int CG>
cudaError_t launch(const CUtensorMap &a, const CUtensorMap &ah, const CUtensorMap &b, const CUtensorMap &c,
                   const TcParams &p, cudaStream_t s)
{
    auto kern = tc_gemm_kernel<MODE, TO, CG>;
    int max_groups = 0;
    const cudaError_t e = group_capacity<MODE, TO, CG>(&max_groups);
    if (e != cudaSuccess) return e;
    const int items = p.max_tiles * p.ksplit;
    const int groups = items < max_groups ? items : max_groups;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(groups * CG);
    lc.blockDim = dim3(THREADS);
    lc.dynamicSmemBytes = Cfg<CG, (int)sizeof(TO)>::SMEM;
    lc.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CG;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see griddep_wait
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = p.no_early_launch ? 1 : 2;
    return cudaLaunchKernelEx(&lc, kern, a, ah, b, c, p);
}

template <int CG>
cudaError_t run(int mode, const GemmArgs &g, int max_mtiles, int nterms, int64_t term_rows, int64_t b_rows_total,
                int ksplit, int32_t *status, cudaStream_t s)
{
    if (!g_encode) return cudaErrorInitializationError;
    if (g.K % BK) return cudaErrorInvalidValue;
    if (((uintptr_t)g.A | (uintptr_t)g.B) & 15u) return cudaErrorMisalignedAddress;
    if ((g.lda * 2) % 16 || (g.ldb * 2) % 16) return cudaErrorMisalignedAddress;
    if (g.offsets && g.E > MAX_E) return cudaErrorInvalidValue;
    TcParams p = {};
    p.M = g.M;
    p.N = g.N;
    p.nkb = g.K / BK;
    p.nterms = nterms;
    p.term_rows = term_rows;
    p.ntn = (mode == EPI_GLU) ? g.N / BN : (g.N + BN - 1) / BN;   // GLU: N = 2F, F % (BN/2) == 0
    p.group_rows = g.offsets ? g.b_group_stride / g.ldb : 0;
    p.offsets = g.offsets;
    p.tile_off = g.tile_off;
    p.E = g.E;
    const int mtiles = g.offsets ? max_mtiles : (g.M + Tiles<CG>::TILE_M - 1) / Tiles<CG>::TILE_M;
    p.max_tiles = mtiles * p.ntn;
    p.ksplit = ksplit < 1 ? 1 : ksplit;
    p.split_rows = g.M;
    if (p.ksplit > 1 && (g.offsets || (mode != EPI_STORE_F32 && mode != EPI_SIGMOID_PARTIAL) ||
                         p.ksplit > p.nkb * nterms))
        return cudaErrorInvalidValue;

    p.epi = g.epi;
    p.status = status;
    p.no_early_launch = g.no_early_launch;
    p.stall_test = g_stall_next.exchange(0);
    if (p.max_tiles == 0) return cudaSuccess;
    CUtensorMap ta, tah, tb;
    memset(&tah, 0, sizeof tah);
    if (mode == EPI_SIGMOID_PARTIAL) mode = EPI_STORE_F32;   // raw fp32 partial tiles; sigmoid after the sum
    const bool out_f32 = (mode == EPI_SIGMOID || mode == EPI_STORE_F32);
    const int kps = Cfg<CG, 2>::KPS;
    p.load3d = 0;
    if (!out_f32 && kps > 1 && nterms == 1 && p.ksplit == 1 &&
        make_map3(&ta, g.A, (uint64_t)g.K, (uint64_t)g.M, (uint64_t)g.lda * 2, 128, kps) &&
        make_map3(&tb, g.B, (uint64_t)g.K, (uint64_t)b_rows_total, (uint64_t)g.ldb * 2, BN / CG, kps)) {
        p.load3d = 1;
        // grouped: an expert's last m-tile of at most 128 rows loads 64 rows per CTA
        p.half_tiles = (CG == 2 && g.offsets &&
                        make_map3(&tah, g.A, (uint64_t)g.K, (uint64_t)g.M, (uint64_t)g.lda * 2, 64, kps)) ? 1 : 0;
    } else {
        if (!make_map(&ta, g.A, (uint64_t)g.K, (uint64_t)g.M, (uint64_t)g.lda * 2, 128)) return cudaErrorInvalidValue;
        if (!make_map(&tb, g.B, (uint64_t)g.K, (uint64_t)b_rows_total, (uint64_t)g.ldb * 2, BN / CG))
            return cudaErrorInvalidValue;
    }
    p.out_cols = (mode == EPI_GLU) ? g.N / 2 : g.N;
    CUtensorMap tc;
    memset(&tc, 0, sizeof tc);
    p.tma_store = make_out_map(&tc, g.epi.out, out_f32, (uint64_t)p.out_cols, (uint64_t)g.M * p.ksplit,
                               (uint64_t)g.epi.ldo * (out_f32 ? 4 : 2)) ? 1 : 0;
    switch (mode) {
    case EPI_SIGMOID: return launch<EPI_SIGMOID, float, CG>(ta, tah, tb, tc, p, s);
    case EPI_GLU:
        if (g.epi.act == LMOE_ACT_SITU) return launch<EPI_GLU_SITU, bf16, CG>(ta, tah, tb, tc, p, s);
        return launch<EPI_GLU, bf16, CG>(ta, tah, tb, tc, p, s);
    case EPI_COMBINE: return launch<EPI_COMBINE, bf16, CG>(ta, tah, tb, tc, p, s);
    case EPI_STORE: return launch<EPI_STORE, bf16, CG>(ta, tah, tb, tc, p, s);
    case EPI_STORE_F32: return launch<EPI_STORE, float, CG>(ta, tah, tb, tc, p, s);
    default: return cudaErrorInvalidValue;
    }
}


// ------------------------------------------------------------------ router + top-k
// Router scores, biased top-k and renormalisation in one launch ("Stable
// LatentMoE", equations for r, T_k(x) and p_i), for E <= 256 experts.
//
// A cluster of KS >= 2 CTAs takes one 128-token tile: CTA `rank` runs the
// k-blocks [rank, rank + 1) * NKB / KS of x against the same k-blocks of the
// three bf16 terms of the fp32 router weight (hi + mid + lo; with bf16 tokens
// every product is exact in fp32): each ring stage holds one k-block of x and
// of all three terms, so x is loaded once for the three, and tcgen05.mma adds
// them into one fp32 TMEM accumulator of E columns.  Its eight epilogue warps
// move the partial logits into its own shared memory (the drained operand
// ring: 128 rows of E floats, each row's 16-byte chunks swizzled by the row's
// low three bits so that the warps' row-per-lane stores and the
// column-per-lane reads below hit distinct banks).  After a cluster
// barrier each CTA owns 128 / KS tokens of the tile.  All its threads read the
// KS partials of those rows, chunk by chunk, from the cluster's shared memory,
// sum them in rank order (fixed order, deterministic), apply the sigmoid and
// write r to global memory and over their own partial.  Then one warp per
// token runs the top-k on r + b (warp_topk_radix for 9 <= k <= 32, else the
// tournament warp_topk; equal scores to the lower index) and writes the
// selection, p from the raw scores, the Quantile-Balancing cutoff and the
// per-32-token expert counts that the counting sort scans.  A last cluster
// barrier keeps every CTA's shared memory alive until its peers have read it.
constexpr int RT_SMEM_FIXED = 1024 + 256;   // alignment slack, barriers and flags
constexpr int RT_MAX_KS = 8;                 // CTAs per cluster (portable cluster size)
// The GEMM's warp roles plus four warps that wait out the MMA phase and join
// the r and top-k phases, which are latency bound.
constexpr int RT_THREADS = THREADS + 4 * 32;

__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

struct RtParams {
    int T, E, k;
    int nkb;                 // k-blocks of 64 per term (d / 64)
    int ks;                  // CTAs per cluster (split of the 3 nkb k-blocks)
    int halves, n_half;      // MMA column halves (1 or 2) and columns per half
    uint32_t idesc;          // kind::f16, M = 128, N = n_half
    int stages, stage_bytes, tmem_cols;
    const float *bias;
    float *r;                // [T][E]
    int32_t *sel;
    float *p32;
    void *p_out;
    float *cutoff;
    int32_t *blockhist;
    int nb;
    int stall_test;
    int32_t *status;
};

template <typename TO, int EPL>
__global__ void __launch_bounds__(RT_THREADS, 1)
router_topk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const RtParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (sbase - raw);
    const int STAGES = p.stages;
    uint64_t *bars = reinterpret_cast<uint64_t *>(gbase + (size_t)STAGES * p.stage_bytes);
    // bars[0..S) full, [S..2S) empty, [2S] accumulator full
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_holder + 1);
    int *drain_counts = abort_flag + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)(blockIdx.x % p.ks);
    const int64_t row0 = (int64_t)(blockIdx.x / p.ks) * 128;
    const int kb_begin = rank * p.nkb / p.ks, kb_end = (rank + 1) * p.nkb / p.ks;   // k-blocks of x
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    const uint32_t accf = bar0 + 8u * (2 * STAGES);
    const int a_bytes = 128 * BK * 2, bh_bytes = p.n_half * BK * 2;
    float *tile = reinterpret_cast<float *>(gbase);   // logit tile over the drained ring: [128][E], chunk-swizzled

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(accf, 1);
        *abort_flag = 0;
        for (int i = 0; i <= NPROD; ++i) drain_counts[i] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_holder)), "r"(p.tmem_cols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    griddep_wait();
    griddep_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int pw = producer_index(warp);
    const int NP = NPROD < STAGES ? NPROD : STAGES;   // producers in use (see NPROD)
    if (pw >= 0) {
        if (lane == 0 && pw < NP) {   // ------------------------------------ TMA producers (k-step it % NP)
            // k-steps it = pw, pw + NP, ...; slot and phase advance incrementally (NP <= STAGES)
            int s = pw;
            uint32_t ph = 0u;
            for (int it = pw; kb_begin + it < kb_end; it += NP) {
                if (!mbar_wait(empty_bar(s), ph ^ 1u)) {
                    atomicOr(p.status, ST_PRODUCER);
                    *(volatile int *)abort_flag = 1;
                    break;
                }
                // one stage: a k-block of x and the same k-block of all three W_r terms
                const int kk = (kb_begin + it) * BK;
                const uint32_t sa = sbase + (uint32_t)s * p.stage_bytes;
                mbar_expect_tx(full_bar(s), a_bytes + 3 * p.halves * bh_bytes);
                tma_load_2d<1>(sa, &tmA, full_bar(s), kk, (int)row0);
                for (int th = 0; th < 3 * p.halves; ++th)   // term th / halves, column half th % halves
                    tma_load_2d<1>(sa + a_bytes + th * bh_bytes, &tmB, full_bar(s), kk,
                                   (th / p.halves) * p.E + (th % p.halves) * p.n_half);
                drain_counts[pw] = it + 1;
                s += NP;
                if (s >= STAGES) {
                    s -= STAGES;
                    ph ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {   // ------------------------------------------------ MMA issuer
            // as in the GEMM: incremental slot and phase, descriptors as a base plus
            // constants, and nothing else between the MMAs of a stage
            bool ok = true;
            if (p.stall_test && !mbar_wait(accf, 0u)) {
                // only this thread commits that barrier: the wait runs out by design
                atomicOr(p.status, ST_MMA);
                *(volatile int *)abort_flag = 1;
                ok = false;
            }
            const uint64_t desc0 = sdesc_sw128(sbase);
            const uint32_t st16 = (uint32_t)p.stage_bytes >> 4, a16 = (uint32_t)a_bytes >> 4,
                           bh16 = (uint32_t)bh_bytes >> 4;
            int s = 0, it = 0;
            uint32_t ph = 0u;
            for (int kb = kb_begin; kb < kb_end && ok; ++kb, ++it) {
                if (!mbar_wait(full_bar(s), ph)) {
                    atomicOr(p.status, ST_MMA);
                    *(volatile int *)abort_flag = 1;
                    ok = false;
                    break;
                }
                const uint64_t da = desc0 + (uint64_t)(s * st16);
                // the three terms of this k-block, term by term, into the same accumulator;
                // each half's first MMA of the CTA's range overwrites
                for (int th = 0; th < 3 * p.halves; ++th) {
                    const int h = th % p.halves;
                    const uint32_t acc0 = (kb > kb_begin || th >= p.halves) ? 1u : 0u;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        const uint64_t ad = da + (uint64_t)(2 * k);
                        const uint64_t bd = da + (uint64_t)(a16 + th * bh16 + 2 * k);
                        asm volatile(
                            "{\n\t.reg .pred q;\n\t"
                            "setp.ne.b32 q, %4, 0;\n\t"
                            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, q;\n\t}"
                            ::"r"(tmem_base + (uint32_t)(h * 256)), "l"(ad), "l"(bd), "r"(p.idesc),
                              "r"(k > 0 ? 1u : acc0));
                    }
                }
                umma_commit<1>(empty_bar(s));
                drain_counts[NPROD] = it + 1;
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (ok) umma_commit<1>(accf);
        }
    } else if (warp <= 9) {
        // ---------------------------------------------------------------- epilogue warps 2..9
        const int q = warp & 3, hset = (warp - 2) >> 2;
        const bool got = mbar_wait(accf, 0u);
        if (!got || *(volatile int *)abort_flag) {
            if (lane == 0) {
                atomicOr(p.status, ST_EPILOGUE);
                *(volatile int *)abort_flag = 1;
            }
        } else {
            // every MMA has completed, so the operand ring is free for the logit tile
            tc_fence_after();
            const int lrow = 32 * q + lane;
            const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16);
            float *srow = tile + lrow * p.E;
            const int sw = lrow & 7;
            for (int c = 32 * hset; c < p.E; c += 64) {
                uint32_t v[32];
                asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                             "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                             "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                             : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                               "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
                               "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
                               "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
                               "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
                               "=r"(v[31])
                             : "r"(tq + (uint32_t)c));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                // 16-byte chunk i of these 32 columns goes to chunk position i ^ (row & 7):
                // the 32 rows of a warp store spread over all banks
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<float4 *>(srow + c + 4 * (i ^ sw)) =
                        make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                    __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            }
        }
    }
    // every CTA of the cluster passes exactly these barriers, whatever happened above
    __syncwarp();
    __threadfence();
    tc_fence_before();
    __syncthreads();
    cluster_sync();                   // every rank's partial logit tile is written and visible

    const int own = 128 / p.ks;       // this CTA's tokens: tile rows [rank * own, (rank + 1) * own)
    const int nch = p.E / 4;          // 16-byte chunks per row
    if (!*(volatile int *)abort_flag) {
        // ------------------------------------------------ r = sigmoid(sum of the KS partial logits)
        // Every thread takes chunks of this CTA's rows: the KS partials of the chunk
        // from the cluster's shared memory, summed in rank order (fixed order,
        // deterministic), the sigmoid, r to global memory and back over this CTA's
        // own partial (no peer reads this CTA's rows).
        uint32_t peer[RT_MAX_KS];
#pragma unroll
        for (int qq = 0; qq < RT_MAX_KS; ++qq) peer[qq] = qq < p.ks ? map_to_rank(sbase, (uint32_t)qq) : 0u;
        for (int u0 = threadIdx.x; u0 < own * nch; u0 += 2 * RT_THREADS) {
            // two chunks per thread at a time: all their loads are issued before any sum
            float4 part[2][RT_MAX_KS];
            uint32_t off[2];
            int64_t tok[2];
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const int u = u0 + b * RT_THREADS;
                const int lrow = rank * own + u / nch, c4 = u % nch;
                tok[b] = u < own * nch ? row0 + lrow : (int64_t)p.T;
                off[b] = 4u * (uint32_t)(lrow * p.E + 4 * (c4 ^ (lrow & 7)));
                if (tok[b] < p.T) {
#pragma unroll
                    for (int qq = 0; qq < RT_MAX_KS; ++qq)
                        if (qq < p.ks) part[b][qq] = ld_cluster_f32x4(peer[qq] + off[b]);
                }
            }
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                if (tok[b] >= p.T) continue;
                const int c4 = (u0 + b * RT_THREADS) % nch;
                float4 a = part[b][0];
#pragma unroll
                for (int qq = 1; qq < RT_MAX_KS; ++qq)
                    if (qq < p.ks) {
                        a.x += part[b][qq].x;
                        a.y += part[b][qq].y;
                        a.z += part[b][qq].z;
                        a.w += part[b][qq].w;
                    }
                a = make_float4(sigmoidf_(a.x), sigmoidf_(a.y), sigmoidf_(a.z), sigmoidf_(a.w));
                *reinterpret_cast<float4 *>(p.r + tok[b] * p.E + 4 * c4) = a;
                *reinterpret_cast<float4 *>(reinterpret_cast<uint8_t *>(tile) + off[b]) = a;
            }
        }
    }
    __syncthreads();                  // this CTA's rows of r are in its shared memory

    if (!*(volatile int *)abort_flag) {
        // ---------------------------------------------------------------- top-k, one warp per token
        float bias[EPL];              // this lane's experts' selection biases, for every token
#pragma unroll
        for (int j = 0; j < EPL; ++j) bias[j] = lane + 32 * j < p.E ? p.bias[lane + 32 * j] : 0.f;
        const bool radix = topk_radix(p.k);
        // per-warp scratch of the radix selection, past the tile in the drained ring
        uint32_t *hist = reinterpret_cast<uint32_t *>(gbase + (size_t)128 * p.E * 4 + (size_t)warp * TOPK_SCRATCH_BYTES);
        if (radix) {
            reinterpret_cast<uint4 *>(hist)[lane] = make_uint4(0u, 0u, 0u, 0u);
            reinterpret_cast<uint4 *>(hist)[lane + 32] = make_uint4(0u, 0u, 0u, 0u);
            __syncwarp();
        }
        for (int i = warp; i < own; i += RT_THREADS / 32) {
            const int lrow = rank * own + i;
            const int64_t t = row0 + lrow;
            if (t >= p.T) break;
            const float *srow = tile + lrow * p.E;
            const int sw = lrow & 7;
            auto r_of = [&](int e) { return srow[4 * ((e >> 2) ^ sw) + (e & 3)]; };
            float v[EPL];
            int ix[EPL];
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                const int e = lane + 32 * j;
                ix[j] = e;
                v[j] = e < p.E ? biased_key(r_of(e), bias[j]) : -INFINITY;
            }
            int mine0, mine1 = 0;
            float cv;
            if (radix)
                warp_topk_radix<EPL>(v, p.k, p.E, lane, hist, &mine0, &cv);
            else
                warp_topk<EPL>(v, ix, p.k, p.E, lane, &mine0, &mine1, &cv);
            if (lane == 0) p.cutoff[t] = cv;
            const float r0 = lane < p.k ? r_of(mine0) : 0.f;
            const float r1 = lane + 32 < p.k ? r_of(mine1) : 0.f;
            float sum = r0 + r1;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            const int64_t tb = t / ROUTE_TPB;   // per-block counts, expert-major
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = lane + 32 * h;
                if (j < p.k) {
                    const int e = h ? mine1 : mine0;
                    const float pv = (h ? r1 : r0) / sum;
                    p.sel[t * p.k + j] = e;
                    p.p32[t * p.k + j] = pv;
                    ((TO *)p.p_out)[t * p.k + j] = from_f32<TO>(pv);
                    atomicAdd(&p.blockhist[(int64_t)e * p.nb + tb], 1);
                }
            }
        }
    }
    cluster_sync();                   // no CTA leaves while a peer may still read its logit tile

    __syncthreads();
    if (*(volatile int *)abort_flag && threadIdx.x == 0) {
        // Drain: loads issued but never consumed (each producer's own k-steps),
        // then the MMAs behind the last commit.
        const int consumed = drain_counts[NPROD];
        bool ok = true;
        for (int q = 0; q < NP; ++q)
            for (int i = consumed; i < drain_counts[q]; ++i)
                if (i % NP == q) ok &= mbar_wait(full_bar(i % STAGES), (uint32_t)(i / STAGES) & 1u);
        if (consumed > 0) {
            const int i = consumed - 1;
            ok &= mbar_wait(empty_bar(i % STAGES), (uint32_t)(i / STAGES) & 1u);
        }
        if (!ok) atomicOr(p.status, ST_DRAIN);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(p.tmem_cols)
                     : "memory");
}


// Stages and bytes of the router + top-k kernel for E experts.
void rt_shape(int E, int *halves, int *n_half, int *stages, int *stage_bytes, int *tmem_cols)
{
    *halves = E > 256 ? 2 : 1;
    *n_half = E > 256 ? 256 : E;
    *stage_bytes = 128 * BK * 2 + 3 * *halves * *n_half * BK * 2;   // x and the three W_r terms
    int st = (232448 - RT_SMEM_FIXED) / *stage_bytes;
    *stages = st > 6 ? 6 : st;
    int cols = 32;
    while (cols < E) cols *= 2;
    *tmem_cols = cols;
}

template <typename TO, int EPL>
cudaError_t launch_rt(const CUtensorMap &a, const CUtensorMap &b, const RtParams &p, int tiles, cudaStream_t s)
{
    auto kern = router_topk_kernel<TO, EPL>;
    const size_t smem = RT_SMEM_FIXED + (size_t)p.stages * p.stage_bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3((unsigned)(tiles * p.ks));
    lc.blockDim = dim3(RT_THREADS);
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see griddep_wait
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 2;
    return cudaLaunchKernelEx(&lc, kern, a, b, p);
}

template <typename TO>
cudaError_t launch_rt_epl(const CUtensorMap &a, const CUtensorMap &b, const RtParams &p, int tiles, cudaStream_t s)
{
    const int epl = (p.E + 31) / 32;
    if (epl <= 1) return launch_rt<TO, 1>(a, b, p, tiles, s);
    if (epl <= 2) return launch_rt<TO, 2>(a, b, p, tiles, s);
    if (epl <= 4) return launch_rt<TO, 4>(a, b, p, tiles, s);
    if (epl <= 8) return launch_rt<TO, 8>(a, b, p, tiles, s);
    return launch_rt<TO, 16>(a, b, p, tiles, s);
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

cudaError_t tc_gemm(int mode, const GemmArgs &g, int max_mtiles, int cg, int32_t *status, cudaStream_t s,
                    int ksplit)
{
    // B rows: dense N; grouped E * (rows per expert)
    const int64_t b_rows = g.offsets ? (int64_t)g.E * (g.b_group_stride / g.ldb) : g.N;
    if (cg == 2) return run<2>(mode, g, max_mtiles, 1, 0, b_rows, ksplit, status, s);
    return run<1>(mode, g, max_mtiles, 1, 0, b_rows, ksplit, status, s);
}

int tc_num_sms() { return g_num_sms; }

void tc_debug_stall_next() { g_stall_next.store(1); }

cudaError_t tc_gemm_router(const bf16 *Wr3, const GemmArgs &g, int cg, int32_t *status, cudaStream_t s, int ksplit)
{
    GemmArgs r = g;
    r.B = Wr3;
    r.ldb = g.K;
    const int mode = ksplit > 1 ? EPI_SIGMOID_PARTIAL : EPI_SIGMOID;
    if (cg == 2) return run<2>(mode, r, 0, 3, g.N, 3 * (int64_t)g.N, ksplit, status, s);
    return run<1>(mode, r, 0, 3, g.N, 3 * (int64_t)g.N, ksplit, status, s);
}

}  // namespace lmoe

namespace lmoe {

int tc_router_topk_splits(int64_t T, int E, int d)
{
    // the logit tile (128 rows of E floats) and the top-k scratch must fit in the drained operand ring
    if (T <= 0 || E > 256 || E % 32 || d % BK) return 0;
    int halves, n_half, stages, stage_bytes, tmem_cols;
    rt_shape(E, &halves, &n_half, &stages, &stage_bytes, &tmem_cols);
    if ((size_t)128 * E * sizeof(float) + (size_t)(RT_THREADS / 32) * TOPK_SCRATCH_BYTES > (size_t)stages * stage_bytes)
        return 0;
    const int sms = g_num_sms > 0 ? g_num_sms : 148;
    const int64_t tiles = (T + 127) / 128;
    const int nkb = d / BK;
    int ks = 1;
    while (ks < RT_MAX_KS && tiles * ks * 2 <= sms && 2 * ks <= nkb) ks *= 2;   // >= 1 k-block of x per CTA
    // One CTA per tile leaves 128 tokens' top-k to its warps, one token after
    // another; measured on B200 (T = 16384, E = 256, k = 6) that phase is latency
    // bound (about 1100 instructions per token at 13 cycles each) and the router
    // GEMM plus the one-warp-per-token top-k kernel is faster.  From two CTAs per
    // tile on, the fused launch is as fast or faster (T = 4096, E = 256).
    return ks >= 2 ? ks : 0;
}

cudaError_t tc_router_topk(const bf16 *x, const bf16 *Wr3, const float *bias, int64_t T, int E, int d, int k,
                           float *r, int32_t *sel, float *p32, void *p_out, int out_bf16,
                           float *cutoff, int32_t *blockhist, int32_t *status, cudaStream_t s)
{
    const int ks = tc_router_topk_splits(T, E, d);
    if (!ks || k < 1 || k > 64 || k > E) return cudaErrorInvalidValue;
    if (!g_encode) return cudaErrorInitializationError;
    if (((uintptr_t)x | (uintptr_t)Wr3) & 15u) return cudaErrorMisalignedAddress;
    RtParams p = {};
    p.T = (int)T;
    p.E = E;
    p.k = k;
    p.nkb = d / BK;
    p.ks = ks;
    rt_shape(E, &p.halves, &p.n_half, &p.stages, &p.stage_bytes, &p.tmem_cols);
    p.idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(p.n_half >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    p.bias = bias;
    p.r = r;
    p.sel = sel;
    p.p32 = p32;
    p.p_out = p_out;
    p.cutoff = cutoff;
    p.blockhist = blockhist;
    p.nb = (int)((T + ROUTE_TPB - 1) / ROUTE_TPB);
    p.stall_test = g_stall_next.exchange(0);
    p.status = status;
    CUtensorMap ta, tb;
    if (!make_map(&ta, x, (uint64_t)d, (uint64_t)T, (uint64_t)d * 2, 128)) return cudaErrorInvalidValue;
    if (!make_map(&tb, Wr3, (uint64_t)d, (uint64_t)3 * E, (uint64_t)d * 2, (uint32_t)p.n_half))
        return cudaErrorInvalidValue;
    const int tiles = (int)((T + 127) / 128);
    if (out_bf16) return launch_rt_epl<bf16>(ta, tb, p, tiles, s);
    return launch_rt_epl<float>(ta, tb, p, tiles, s);
}

}  // namespace lmoe
