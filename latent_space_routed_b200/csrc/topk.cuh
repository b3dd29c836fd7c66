// Biased top-k of one token held by a warp ("Stable LatentMoE", equation for
// T_k(x): TopK(r + b, k); equal scores go to the lower expert index, as the
// cooking-agi LatentMoE page's routed_example picks index 0 when v0 >= v1).
// Shared by the routing kernels and the tensor-core router's fused epilogue.
#pragma once

#include <float.h>

#include "lmoe_internal.cuh"

namespace lmoe {

// "a before b": larger biased score first, equal scores to the lower index.
__device__ __forceinline__ bool ahead(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

// Bitonic sort of a lane's N (score, expert) pairs into "ahead" order, in registers.
template <int N>
__device__ __forceinline__ void sort_lane(float (&v)[N], int (&ix)[N])
{
#pragma unroll
    for (int kk = 2; kk <= N; kk <<= 1)
#pragma unroll
        for (int j = kk >> 1; j > 0; j >>= 1)
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int m = i ^ j;
                if (m > i) {
                    const bool first_ahead = ahead(v[i], ix[i], v[m], ix[m]);
                    if (((i & kk) == 0) != first_ahead) {
                        const float tv = v[i]; v[i] = v[m]; v[m] = tv;
                        const int ti = ix[i]; ix[i] = ix[m]; ix[m] = ti;
                    }
                }
            }
}

// Order-preserving 32-bit key of a score: a > b as floats exactly when
// key(a) > key(b) as unsigned integers (for -0 and +0 alike only if the caller
// made -0 into +0, which it does).
__device__ __forceinline__ uint32_t score_key(float v)
{
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k of one token held by a warp.  Lane L holds experts L, L + 32, ...
// (EPL of them, padded with -inf) as (biased score, expert) pairs, sorts them,
// and the k rounds are a tournament over the 32 lane heads: the largest head
// score (one warp max-reduction over the score keys), then the lowest expert
// index among the heads with that score (one min-reduction), so equal scores
// go to the lower index; the winning lane pops its head.  Selection j is kept
// by lane j % 32 (in *mine0 for j < 32, *mine1 above).  One more round gives
// the (k+1)-th biased score, the Quantile-Balancing cutoff (-inf when k = E).
template <int EPL>
__device__ __forceinline__ void warp_topk(float (&v)[EPL], int (&ix)[EPL], int k, int E, int lane, int *mine0,
                                          int *mine1, float *cut)
{
    sort_lane<EPL>(v, ix);
    int m0 = 0, m1 = 0;
    for (int j = 0; j < k; ++j) {
        const uint32_t key = score_key(v[0]);
        const uint32_t best = __reduce_max_sync(0xffffffffu, key);
        const int bi = (int)__reduce_min_sync(0xffffffffu, key == best ? (uint32_t)ix[0] : 0xffffffffu);
        if (lane == (bi & 31)) {            // the winner pops its head
#pragma unroll
            for (int i = 0; i + 1 < EPL; ++i) { v[i] = v[i + 1]; ix[i] = ix[i + 1]; }
            v[EPL - 1] = -INFINITY;
            ix[EPL - 1] = 0x7fffffff;
        }
        if (lane == (j & 31)) {
            if (j < 32) m0 = bi; else m1 = bi;
        }
    }
    const uint32_t key = score_key(v[0]);
    const uint32_t best = __reduce_max_sync(0xffffffffu, key);
    const int bi = (int)__reduce_min_sync(0xffffffffu, key == best ? (uint32_t)ix[0] : 0xffffffffu);
    const float cv = __shfl_sync(0xffffffffu, v[0], bi & 31);
    *cut = k < E ? cv : -INFINITY;
    *mine0 = m0;
    *mine1 = m1;
}

// Biased key of expert e for the tournament: NaN / -inf map to -FLT_MAX so
// that a real candidate always beats the padding; adding +0 turns -0 into +0,
// so equal scores get equal keys.
__device__ __forceinline__ float biased_key(float r, float b) { return fmaxf(r + b, -FLT_MAX) + 0.0f; }

// The float whose score_key is `key`.
__device__ __forceinline__ float key_score(uint32_t key)
{
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Shared-memory scratch of warp_topk_radix, per warp: a 256-bin histogram,
// zero on entry and left zero on return (its first 384 bytes also hold the
// chosen candidates and their order for a moment).
constexpr int TOPK_SCRATCH_BYTES = 256 * 4;

// warp_topk_radix serves 9 <= k <= 32: below, the tournament's k + 1 rounds
// cost fewer instructions than the radix passes; above, a selection no longer
// fits one lane each.
__host__ __device__ __forceinline__ bool topk_radix(int k) { return k >= 9 && k <= 32; }

// The same selection and cutoff as warp_topk, by radix selection on the 32-bit
// score keys (k <= 32).  Lane L holds experts L, L + 32, ... (v: biased scores,
// padding past E ignored).  The bits above the highest bit on which the keys
// differ are common to all of them (a warp AND and OR); from that bit down,
// 8-bit digits, each pass a shared-memory histogram of the keys that still
// match the digits chosen so far (lane L reads bins 255 - 8L down to 248 - 8L
// and a warp scan finds the bin holding the k-th largest key); a pass whose bin
// holds exactly the keys still wanted ends the search.  Then every key above
// the chosen digits is selected, and of the keys equal to them as many as are
// still wanted, lowest expert index first (ties remain only when all bits are
// equal).  The k chosen (score, index) pairs are compacted, and each one's
// place in the selection is the number of chosen pairs ahead of it on the
// packed key (score key, then inverted index), so that lane j holds selection
// j: the order warp_topk gives, because both order by score and then by lower
// index.  The cutoff is the largest key below the selection, or the chosen key
// itself when ties were left unselected.
template <int EPL>
__device__ __forceinline__ void warp_topk_radix(const float (&v)[EPL], int k, int E, int lane, uint32_t *hist,
                                                int *mine0, float *cut)
{
    constexpr unsigned FULL = 0xffffffffu;
    uint32_t key[EPL];
    uint32_t kand = FULL, kor = 0u;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
        key[j] = lane + 32 * j < E ? score_key(v[j]) : 0u;   // real keys > 0
        if (lane + 32 * j < E) {
            kand &= key[j];
            kor |= key[j];
        }
    }
    kand = __reduce_and_sync(FULL, kand);
    kor = __reduce_or_sync(FULL, kor);
    const uint32_t diff = kand ^ kor;
    const int top = diff ? 31 - __clz(diff) : -1;     // highest bit on which the keys differ
    uint32_t pmask = top >= 31 ? 0u : FULL << (top + 1);
    uint32_t prefix = kand & pmask;
    int want = k, cnt = E;                            // every real key matches the common bits
    uint4 *mine = reinterpret_cast<uint4 *>(hist + 248 - 8 * lane);
#pragma unroll 1
    for (int hi = top; hi >= 0 && cnt != want; hi -= 8) {
        const int lo = hi >= 7 ? hi - 7 : 0;
        const uint32_t dmask = (2u << (hi - lo)) - 1u;
#pragma unroll
        for (int j = 0; j < EPL; ++j)
            if (key[j] != 0u && (key[j] & pmask) == prefix) atomicAdd(&hist[(key[j] >> lo) & dmask], 1u);
        __syncwarp();
        const uint4 h0 = mine[0], h1 = mine[1];
        mine[0] = make_uint4(0u, 0u, 0u, 0u);   // each lane reads and clears only its own bins
        mine[1] = make_uint4(0u, 0u, 0u, 0u);
        const int c[8] = {(int)h1.w, (int)h1.z, (int)h1.y, (int)h1.x, (int)h0.w, (int)h0.z, (int)h0.y, (int)h0.x};
        int sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) sum += c[i];
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int t = __shfl_up_sync(FULL, incl, off);
            if (lane >= off) incl += t;
        }
        const int excl = incl - sum;
        const int owner = __ffs(__ballot_sync(FULL, excl < want && want <= incl)) - 1;
        int a = excl, dsel = 0, asel = 0, csel = 0;
        bool found = false;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const bool hit = !found && a + c[i] >= want;
            if (hit) {
                dsel = 255 - 8 * lane - i;
                asel = a;
                csel = c[i];
            }
            found = found || hit;
            a += c[i];
        }
        prefix |= (uint32_t)__shfl_sync(FULL, dsel, owner) << lo;
        pmask |= dmask << lo;
        want -= __shfl_sync(FULL, asel, owner);
        cnt = __shfl_sync(FULL, csel, owner);
        __syncwarp();                          // the bins are clear before the next pass adds to them
    }
    // selection: above the chosen bits, or equal to them and among the first `want` by index
    unsigned long long *cand = reinterpret_cast<unsigned long long *>(hist);
    const unsigned lt = (1u << lane) - 1u;
    int eq_before = 0, pos = 0;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
        const uint32_t m = key[j] & pmask;
        const bool eq = key[j] != 0u && m == prefix;
        const unsigned be = __ballot_sync(FULL, eq);
        const bool s = m > prefix || (eq && eq_before + __popc(be & lt) < want);
        eq_before += __popc(be);
        const unsigned bs = __ballot_sync(FULL, s);
        const int slot = pos + __popc(bs & lt);
        if (s && slot < 32)                    // exactly k <= 32 are selected; the test only bounds the store
            cand[slot] =
                ((unsigned long long)key[j] << 32) | (unsigned long long)(0xffffffffu - (uint32_t)(lane + 32 * j));
        pos += __popc(bs);
    }
    __syncwarp();
    // order: candidate i's place is the number of candidates ahead of it (the
    // packed keys are distinct), and the expert index goes to that place
    uint32_t *ranked = hist + 64;
    if (lane < k) {
        const unsigned long long x = cand[lane];
        int place = 0;
        for (int i = 0; i < k; ++i) place += cand[i] > x;
        ranked[place] = 0xffffffffu - (uint32_t)x;
    }
    __syncwarp();
    *mine0 = (int)ranked[lane];
    __syncwarp();
    cand[lane] = 0ull;                         // the histogram is zero again
    ranked[lane] = 0u;
    uint32_t ck = prefix;
    if (cnt == want) {                         // every key equal to the chosen bits was selected
        uint32_t m = 0u;
#pragma unroll
        for (int j = 0; j < EPL; ++j)
            if ((key[j] & pmask) < prefix && key[j] > m) m = key[j];
        ck = __reduce_max_sync(FULL, m);
    }
    *cut = k < E && ck != 0u ? key_score(ck) : -INFINITY;
    __syncwarp();                              // the scratch is clear before the next token uses it
}

}  // namespace lmoe
