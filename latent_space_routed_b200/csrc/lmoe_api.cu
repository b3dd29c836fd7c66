// Host runtime behind the C ABI of include/lmoe.h: configuration checks,
// handle-owned repacked weights, the workspace plan, and the launch sequence
// of one layer forward on one stream.
//
// Forward sequence for T tokens (S = T k slot rows):
//   1 router GEMM      r = sigmoid(x W_r^T)                     [T, E] fp32
//   2 top-k            sel, p (fp32 and token dtype), per-block expert counts
//   3 scan             counts, offsets, per-block bases, m-tile prefix
//   4 dispatch         slot_of[t, j], token and weight of every slot row
//   5 down GEMM        z = x W_down^T                           [T, l]
//   6 permute          Zp[m] = z[token of slot m]               [S, l]
//   7 gate/up GEMM     per expert: h = act(G z, U z)            [S, f]
//   8 down GEMM        per expert: Y = p * (h D^T)              [S, l] token dtype
//   9 combine+norm     u = sum_j Y[slot_of[t, j]], n = RMSNorm(u)
//  10 shared gate/up   h_s = act([G_1; G_2] x, [U_1; U_2] x)    [T, 2 f_s]
//  11 final GEMM       y = [h_s | n] [D_s1 | D_s2 | W_up]^T     [T, d]
// The standard-MoE form (config.standard) skips 5, permutes x, skips the norm
// in 9 and computes y = h_s [D_s1 | D_s2]^T + u in 11.
//
// Tensor-core path: for E <= 256 (a multiple of 32) and tiles split over a
// cluster, stages 1 and 2 are one launch (tc_router_topk: router GEMM,
// sigmoid, top-k, p, cutoff, per-block counts).  Few tokens: up to ROUTE_SMALL_MAX_T tokens,
// stages 1-4 are one launch (route_small_kernel); up to GEMV_MAX_T tokens the
// dense GEMMs and the routed experts' GEMMs are weight-streaming GEMVs, the
// routed ones over the touched experts only, reading z through the slot ->
// token map (no permute).
#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "lmoe_internal.cuh"
#include "gemm_tc.cuh"

using namespace lmoe;

namespace {

thread_local std::string g_err;
std::atomic<int> g_fail_alloc_at{0};   // test hook: this allocation of the next lmoe_create fails

lmoe_status fail(lmoe_status s, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

#define LMOE_CUDA(call)                                                                         \
    do {                                                                                        \
        cudaError_t e_ = (call);                                                                \
        if (e_ != cudaSuccess)                                                                  \
            return fail(LMOE_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_),  \
                        __FILE__, __LINE__);                                                    \
    } while (0)

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Columns of [h_s | RMSNorm(u)], the final GEMM's A (no norm columns in the
// standard-MoE form, which adds u in the final GEMM's epilogue instead).
int64_t hs_cols(const lmoe_config &c) { return 2 * (int64_t)c.f_shared + (c.standard ? 0 : c.l); }

struct Layout {
    size_t r32, p32, blockhist, base, counts, offsets, tile_off, slot_of, perm_tok, perm_w, z, Zp, H, Yp, HS, partial,
        partial_side, cutoff, status, touched, final32;
    size_t total;
};

// Words of the 256-byte control slot at the start of every workspace.
constexpr int CTL_STATUS = 0;      // device status word (bounded waits that gave up)
constexpr int CTL_TICKET = 1;      // route_small_kernel's block ticket (zero at launch)
constexpr int CTL_NTOUCHED = 2;    // number of touched experts (few-token plan)

}  // namespace

lmoe_status lmoe::report_error(lmoe_status s, const char *msg)
{
    g_err = msg;
    return s;
}

namespace {
constexpr int HOST_MAX_CHUNKS = 8;   // chunks of one lmoe_forward_host call
}  // namespace

struct lmoe_handle {
    lmoe_config cfg;
    int device;
    bool tc;          // tensor-core GEMMs
    int ib;           // gate/up interleave block
    size_t tb;        // token dtype bytes
    float *Wr;        // [E, d] fp32 (CUDA-core router)
    bf16 *Wr3;        // [3, E, d] bf16 split (tensor-core router)
    float *b;         // [E]
    void *Wdown;      // [l, d]
    void *Wgu;        // [E, 2f, l] interleaved
    void *D;          // [E, l, f]
    void *Wgu_s;      // [4 f_s, d] interleaved (both shared experts as one of width 2 f_s)
    void *Wcat;       // [d, 2 f_s + l]
    void *const *stage_events;  // caller's cudaEvent_t[LMOE_NUM_STAGES + 1] or NULL
    cudaStream_t side = nullptr;  // tensor-core path: the shared experts' gate/up runs here, overlapped
    cudaEvent_t ev_fork = nullptr, ev_z = nullptr, ev_join = nullptr;
    std::mutex fork_mutex;
    // lmoe_forward_host: copy streams and events of its chunk pipeline
    cudaStream_t copy_in = nullptr, copy_out = nullptr;
    cudaEvent_t ev_host[2 + 2 * HOST_MAX_CHUNKS] = {};
    std::mutex host_mutex;
};

int lmoe::handle_device(const lmoe_handle *h) { return h->device; }

namespace {

// Few-token plans.  The router runs on CUDA cores for a handful of tokens;
// a dense tensor-core GEMM (the router included) whose tiles cover fewer than
// half the SMs is split along K into as many parts as keep all parts in one
// wave (fp32 partial tiles, then an ordered reduction that applies the
// epilogue).
constexpr int SPLIT_MAX = 16;

// Few-token plans of the tensor-core path.
bool small_route(const lmoe_handle *h, int64_t T) { return h->tc && T <= ROUTE_SMALL_MAX_T; }
bool gemv_experts(const lmoe_handle *h, int64_t T) { return h->tc && T <= GEMV_MAX_T; }
// Few tokens, latent form: the final GEMV's shared-expert columns (K = 2 f_s of
// 2 f_s + l) run as their own GEMV into an fp32 partial on the side stream,
// beside the routed GEMVs; the final GEMV after the combine + RMSNorm then
// streams only W_up and adds the partial.
bool split_final(const lmoe_handle *h, int64_t T) { return gemv_experts(h, T) && !h->cfg.standard; }

// K splits for a dense GEMM of M rows, N columns on (128 cg) x 256 tiles, nkb
// k-blocks of 64.
int plan_ksplit(const lmoe_handle *h, int64_t M, int64_t N, int64_t nkb, bool any_m = false, int cg = 1)
{
    if (!h->tc) return 1;
    if (!any_m && M >= 256) return 1;   // 256-row pair tiles without a split do better there
    const int sms = tc_num_sms() > 0 ? tc_num_sms() : 148;
    const int groups = sms / cg;
    const int64_t tiles = ((M + TC_BM * cg - 1) / (TC_BM * cg)) * ((N + TC_BN - 1) / TC_BN);
    if (tiles * 2 >= groups) return 1;
    int64_t ks = groups / tiles;
    if (ks > nkb / 4) ks = nkb / 4;
    if (ks > SPLIT_MAX) ks = SPLIT_MAX;
    return ks >= 2 ? (int)ks : 1;
}

// Tile rows of the tensor-core router: CTA pairs from 256 tokens on.
int router_cg(int64_t T) { return T >= 256 ? 2 : 1; }

struct SplitPlan {
    int router, down, shared, final_;
    bool fused_router;            // router + top-k in one launch (tc_router_topk)
    size_t partial_floats;        // router and final GEMMs: largest ks * T * N
    size_t partial_side_floats;   // down and shared gate/up GEMMs (the side stream's)
};

SplitPlan plan_splits(const lmoe_handle *h, int64_t T)
{
    const lmoe_config &c = h->cfg;
    const int64_t ld_hs = hs_cols(c);
    SplitPlan sp;
    const int fused_ks = (h->tc && T > ROUTE_SMALL_MAX_T) ? tc_router_topk_splits(T, c.E, c.d) : 0;
    sp.fused_router = fused_ks > 0;
    sp.router = sp.fused_router ? fused_ks
                : (h->tc && T > ROUTE_SMALL_MAX_T) ? plan_ksplit(h, T, c.E, 3 * (int64_t)c.d / TC_BK, true, router_cg(T))
                                                   : 1;
    const bool gemv = h->tc && T <= GEMV_MAX_T;   // few tokens: dense GEMMs as weight-streaming GEMVs
    sp.down = (c.standard || gemv) ? 1 : plan_ksplit(h, T, c.l, c.d / TC_BK);
    sp.shared = gemv ? 1 : plan_ksplit(h, T, 4 * (int64_t)c.f_shared, c.d / TC_BK);
    sp.final_ = gemv ? 1 : plan_ksplit(h, T, c.d, ld_hs / TC_BK);
    auto need = [&](int ks, int64_t n) -> size_t { return ks > 1 ? (size_t)ks * (size_t)n * (size_t)T : 0; };
    sp.partial_floats = std::max(need(sp.fused_router ? 1 : sp.router, c.E), need(sp.final_, c.d));
    sp.partial_side_floats = std::max(need(sp.down, c.l), need(sp.shared, 4 * (int64_t)c.f_shared));
    return sp;
}

// The two-stream order: tensor-core path and no stage events (those time the
// stages one after another on one stream).
bool use_side_stream(const lmoe_handle *h) { return h->tc && h->side && !h->stage_events; }

// Chunks of a host-buffer forward (lmoe_forward_host): the copies of chunk
// j + 1 in and chunk j - 1 out overlap the compute of chunk j.  Rows are
// independent, so chunking changes no row's arithmetic (only how a batch is
// cut into launches); each chunk keeps at least 2048 tokens and enough slot
// rows per expert (192 E / k tokens) for CTA-pair tiles.
int host_chunks(const lmoe_config &c, int64_t T, int64_t *Tc)
{
    int64_t minc = (192LL * c.E + c.k - 1) / c.k;
    if (minc < 2048) minc = 2048;
    int64_t nc = T / minc;
    if (nc > HOST_MAX_CHUNKS) nc = HOST_MAX_CHUNKS;
    if (nc < 2) {
        *Tc = T;
        return 1;
    }
    *Tc = (T + nc - 1) / nc;
    return (int)nc;
}

Layout plan(const lmoe_handle *h, int64_t T)
{
    const lmoe_config &c = h->cfg;
    const int64_t S = T * c.k;
    const int64_t nb = (T + ROUTE_TPB - 1) / ROUTE_TPB;
    Layout L;
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
    L.status = take(256);   // control slot first: the same offset for every T (chunked host forwards share it)
    L.r32 = take(sizeof(float) * T * c.E);
    L.p32 = take(sizeof(float) * S);
    L.blockhist = take(sizeof(int32_t) * nb * c.E);
    L.base = take(sizeof(int32_t) * nb * c.E);
    L.counts = take(sizeof(int32_t) * c.E);
    L.offsets = take(sizeof(int32_t) * (c.E + 1));
    L.tile_off = take(sizeof(int32_t) * (c.E + 1));
    L.slot_of = take(sizeof(int32_t) * S);
    L.perm_tok = take(sizeof(int32_t) * S);
    L.perm_w = take(sizeof(float) * S);
    L.z = take(c.standard ? 0 : h->tb * T * c.l);   // the standard form permutes x itself
    L.Zp = take(h->tb * S * c.l);
    L.H = take(h->tb * S * c.f);
    L.Yp = take(h->tb * S * c.l);
    L.HS = take(h->tb * T * (2 * (int64_t)c.f_shared + c.l));
    const SplitPlan sp = plan_splits(h, T);
    L.partial = take(sizeof(float) * sp.partial_floats);
    L.partial_side = take(sizeof(float) * sp.partial_side_floats);
    L.cutoff = take(sizeof(float) * T);
    L.touched = take(sizeof(int32_t) * c.E);
    L.final32 = take(split_final(h, T) ? sizeof(float) * T * c.d : 0);
    L.total = o;
    return L;
}

lmoe_status check_config(const lmoe_config *c, bool *tc)
{
    if (!c) return fail(LMOE_ERR_INVALID_ARG, "config is NULL");
    if (c->d < 1 || c->l < 1 || c->f < 1 || c->E < 1 || c->f_shared < 1)
        return fail(LMOE_ERR_INVALID_ARG, "dimensions must be positive");
    if (c->l > c->d) return fail(LMOE_ERR_INVALID_ARG, "latent width l=%d exceeds d=%d", c->l, c->d);
    if (c->k < 1 || c->k > c->E) return fail(LMOE_ERR_INVALID_ARG, "k=%d must satisfy 1 <= k <= E=%d", c->k, c->E);
    if (c->n_shared != 2) return fail(LMOE_ERR_INVALID_ARG, "exactly two shared experts are required");
    if (!(c->eps >= 0.f)) return fail(LMOE_ERR_INVALID_ARG, "eps must be >= 0");
    if (c->dtype != LMOE_F32 && c->dtype != LMOE_BF16) return fail(LMOE_ERR_INVALID_ARG, "unknown dtype");
    if (c->act != LMOE_ACT_SWIGLU && c->act != LMOE_ACT_SITU) return fail(LMOE_ERR_INVALID_ARG, "unknown act");
    if (c->act == LMOE_ACT_SITU && !(c->gate_cap > 0.f && c->up_cap > 0.f))
        return fail(LMOE_ERR_INVALID_ARG, "SiTU caps must be positive");
    if (c->gemm != 0 && c->gemm != 1) return fail(LMOE_ERR_INVALID_ARG, "gemm must be 0 or 1");
    if (c->standard != 0 && c->standard != 1) return fail(LMOE_ERR_INVALID_ARG, "standard must be 0 or 1");
    if (c->standard && c->l != c->d)
        return fail(LMOE_ERR_INVALID_ARG, "the standard-MoE form needs l = d (got l=%d, d=%d)", c->l, c->d);
    if (c->E > 1024) return fail(LMOE_ERR_UNSUPPORTED, "E=%d > 1024", c->E);
    if (c->l > 8192) return fail(LMOE_ERR_UNSUPPORTED, "l=%d > 8192", c->l);
    if (c->k > 64) return fail(LMOE_ERR_UNSUPPORTED, "k=%d > 64", c->k);
    if (c->d % 64 || c->l % 64 || c->f % 64 || c->f_shared % 64)
        return fail(LMOE_ERR_UNSUPPORTED, "d, l, f and f_shared must be multiples of 64");
    *tc = (c->dtype == LMOE_BF16 && c->gemm == 0);
    if (*tc && (c->f % (TC_BN / 2) || c->f_shared % (TC_BN / 2)))
        return fail(LMOE_ERR_UNSUPPORTED, "tensor-core path needs f and f_shared multiples of %d", TC_BN / 2);
    return LMOE_OK;
}

void free_handle(lmoe_handle *h)
{
    if (!h) return;
    void *ptrs[] = {h->Wr, h->Wr3, h->b, h->Wdown, h->Wgu, h->D, h->Wgu_s, h->Wcat};
    for (void *p : ptrs)
        if (p) cudaFree(p);
    if (h->side) cudaStreamDestroy(h->side);
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    if (h->ev_z) cudaEventDestroy(h->ev_z);
    if (h->copy_in) cudaStreamDestroy(h->copy_in);
    if (h->copy_out) cudaStreamDestroy(h->copy_out);
    for (cudaEvent_t e : h->ev_host)
        if (e) cudaEventDestroy(e);
    if (h->ev_join) cudaEventDestroy(h->ev_join);
    delete h;
}

}  // namespace

extern "C" {

const char *lmoe_last_error(void) { return g_err.c_str(); }

lmoe_status lmoe_config_from_base(int32_t d, int32_t m, int32_t N, int32_t K, int32_t alpha, int32_t n_shared,
                                  const char *variant, lmoe_config *out)
{
    g_err.clear();
    if (!out || !variant) return fail(LMOE_ERR_INVALID_ARG, "NULL argument");
    if (d < 1 || m < 1 || N < 1 || K < 1 || alpha < 1 || n_shared < 1)
        return fail(LMOE_ERR_INVALID_ARG, "all base values must be positive");
    if (d % alpha) return fail(LMOE_ERR_INVALID_ARG, "alpha=%d does not divide d=%d", alpha, d);
    int k;
    const bool standard = !strcmp(variant, "std");
    if (!strcmp(variant, "eff") || standard) k = K;
    else if (!strcmp(variant, "acc")) k = alpha * K;
    else return fail(LMOE_ERR_INVALID_ARG, "variant must be \"acc\", \"eff\" or \"std\"");
    const int E = standard ? N : alpha * N;
    if (k > E) return fail(LMOE_ERR_INVALID_ARG, "top-k %d exceeds %d experts", k, E);
    lmoe_config c;
    memset(&c, 0, sizeof c);
    c.d = d; c.l = standard ? d : d / alpha; c.f = m; c.E = E; c.k = k; c.f_shared = m; c.n_shared = n_shared;
    c.eps = 1e-6f; c.dtype = LMOE_BF16; c.act = LMOE_ACT_SWIGLU; c.gate_cap = 4.f; c.up_cap = 25.f; c.gemm = 0;
    c.standard = standard ? 1 : 0;
    *out = c;
    return LMOE_OK;
}

lmoe_status lmoe_create(const lmoe_config *cfg, const lmoe_weights *w, void *stream, lmoe_handle **out)
{
    g_err.clear();
    if (!out) return fail(LMOE_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    bool tc = false;
    lmoe_status st = check_config(cfg, &tc);
    if (st != LMOE_OK) return st;
    if (!w || !w->W_r || !w->b || !w->G || !w->U || !w->D || !w->Gs || !w->Us || !w->Ds ||
        (!cfg->standard && (!w->W_down || !w->W_up)))
        return fail(LMOE_ERR_INVALID_ARG, "a weight pointer is NULL");
    if (tc) {
        st = tc_check_device();
        if (st != LMOE_OK) return st;
    }
    cudaStream_t s = (cudaStream_t)stream;
    lmoe_handle *h = new lmoe_handle();
    h->cfg = *cfg;
    cudaGetDevice(&h->device);
    h->tc = tc;
    h->ib = tc ? TC_BN / 4 : SIMT_BN / 2;   // tensor cores: 64-row blocks (see the GLU epilogue)
    h->tb = cfg->dtype == LMOE_BF16 ? 2 : 4;
    const lmoe_config &c = *cfg;
    const size_t tb = h->tb;
    const int64_t fs = c.f_shared;

    int alloc_index = 0;
    const int fail_at = g_fail_alloc_at.exchange(0);
#define ALLOC(ptr, bytes)                                                                        \
    do {                                                                                         \
        ++alloc_index;                                                                           \
        if (alloc_index == fail_at || cudaMalloc((void **)&(ptr), (bytes)) != cudaSuccess) {   \
            cudaGetLastError();                                                                  \
            free_handle(h);                                                                      \
            return fail(LMOE_ERR_OOM, "cudaMalloc of %zu bytes failed", (size_t)(bytes));        \
        }                                                                                        \
    } while (0)
#define STEP(call)                                                                               \
    do {                                                                                         \
        cudaError_t e_ = (call);                                                                 \
        if (e_ != cudaSuccess) {                                                                 \
            free_handle(h);                                                                      \
            return fail(LMOE_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_));                 \
        }                                                                                        \
    } while (0)

    ALLOC(h->Wr, sizeof(float) * c.E * c.d);
    ALLOC(h->b, sizeof(float) * c.E);
    if (!c.standard) ALLOC(h->Wdown, tb * c.l * c.d);
    ALLOC(h->Wgu, tb * (size_t)c.E * 2 * c.f * c.l);
    ALLOC(h->D, tb * (size_t)c.E * c.l * c.f);
    ALLOC(h->Wgu_s, tb * 4 * fs * c.d);
    ALLOC(h->Wcat, tb * c.d * hs_cols(c));
    STEP(cudaMemcpyAsync(h->Wr, w->W_r, sizeof(float) * c.E * c.d, cudaMemcpyDeviceToDevice, s));
    STEP(cudaMemcpyAsync(h->b, w->b, sizeof(float) * c.E, cudaMemcpyDeviceToDevice, s));
    if (!c.standard) STEP(cudaMemcpyAsync(h->Wdown, w->W_down, tb * c.l * c.d, cudaMemcpyDeviceToDevice, s));
    STEP(cudaMemcpyAsync(h->D, w->D, tb * (size_t)c.E * c.l * c.f, cudaMemcpyDeviceToDevice, s));
    STEP(launch_pack_glu(w->G, w->U, h->Wgu, c.E, c.f, c.l, h->ib, (int)tb, s));
    // [2, f_s, d] stacks are the rows of one expert of width 2 f_s
    STEP(launch_pack_glu(w->Gs, w->Us, h->Wgu_s, 1, 2 * c.f_shared, c.d, h->ib, (int)tb, s));
    // standard: [D_s1 | D_s2] only (u is added in the final GEMM's epilogue)
    STEP(launch_pack_cat(w->Ds, w->W_up, h->Wcat, c.d, c.f_shared, c.standard ? 0 : c.l, (int)tb, s));
    if (tc) {
        ALLOC(h->Wr3, sizeof(bf16) * 3 * c.E * c.d);
        STEP(launch_split_router(h->Wr, h->Wr3, (int64_t)c.E * c.d, s));
        STEP(cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking));
        STEP(cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming));
        STEP(cudaEventCreateWithFlags(&h->ev_z, cudaEventDisableTiming));
        STEP(cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming));
    }
    STEP(cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking));
    STEP(cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking));
    for (cudaEvent_t &e : h->ev_host) STEP(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    STEP(cudaStreamSynchronize(s));
#undef ALLOC
#undef STEP
    *out = h;
    return LMOE_OK;
}

void lmoe_destroy(lmoe_handle *h) { free_handle(h); }

lmoe_status lmoe_workspace_size(const lmoe_handle *h, int64_t T, size_t *bytes)
{
    g_err.clear();
    if (!h || !bytes) return fail(LMOE_ERR_INVALID_ARG, "NULL argument");
    if (T < 0) return fail(LMOE_ERR_INVALID_ARG, "T < 0");
    *bytes = T == 0 ? 0 : plan(h, T).total;
    return LMOE_OK;
}

lmoe_status lmoe_workspace_region(const lmoe_handle *h, int64_t T, int32_t region, size_t *offset, size_t *bytes)
{
    g_err.clear();
    if (!h || !offset || !bytes) return fail(LMOE_ERR_INVALID_ARG, "NULL argument");
    if (T < 1) return fail(LMOE_ERR_INVALID_ARG, "T < 1");
    const Layout L = plan(h, T);
    const lmoe_config &c = h->cfg;
    const int64_t S = T * c.k;
    switch (region) {
    case 0: *offset = L.r32; *bytes = sizeof(float) * T * c.E; break;
    case 1: *offset = L.p32; *bytes = sizeof(float) * S; break;
    case 2: *offset = L.counts; *bytes = sizeof(int32_t) * c.E; break;
    case 3: *offset = L.offsets; *bytes = sizeof(int32_t) * (c.E + 1); break;
    case 4: *offset = L.slot_of; *bytes = sizeof(int32_t) * S; break;
    case 5: *offset = L.perm_tok; *bytes = sizeof(int32_t) * S; break;
    case 6: *offset = L.z; *bytes = c.standard ? 0 : h->tb * T * c.l; break;
    case 7: *offset = L.H; *bytes = h->tb * S * c.f; break;
    case 8: *offset = L.Yp; *bytes = h->tb * S * c.l; break;
    case 9: *offset = L.HS; *bytes = h->tb * T * (2 * (int64_t)c.f_shared + c.l); break;
    case 10: *offset = L.status; *bytes = sizeof(int32_t); break;
    case 11: *offset = L.cutoff; *bytes = sizeof(float) * T; break;
    case 12: *offset = L.Zp; *bytes = gemv_experts(h, T) ? 0 : h->tb * S * c.l; break;
    default: return fail(LMOE_ERR_INVALID_ARG, "unknown region %d", region);
    }
    return LMOE_OK;
}

lmoe_status lmoe_debug_inject(int32_t what, int32_t arg)
{
    g_err.clear();
    if (what == LMOE_INJECT_STALL_NEXT_GEMM) {
        tc_debug_stall_next();
        return LMOE_OK;
    }
    if (what == LMOE_INJECT_FAIL_ALLOC) {
        if (arg < 1) return fail(LMOE_ERR_INVALID_ARG, "allocation index must be >= 1");
        g_fail_alloc_at.store(arg);
        return LMOE_OK;
    }
    return fail(LMOE_ERR_INVALID_ARG, "unknown injection %d", what);
}

lmoe_status lmoe_set_stage_events(lmoe_handle *h, void *const *events, int32_t n)
{
    g_err.clear();
    if (!h) return fail(LMOE_ERR_INVALID_ARG, "handle is NULL");
    if (n == 0 && !events) { h->stage_events = nullptr; return LMOE_OK; }
    if (n != LMOE_NUM_STAGES + 1 || !events)
        return fail(LMOE_ERR_INVALID_ARG, "need %d events", LMOE_NUM_STAGES + 1);
    h->stage_events = events;
    return LMOE_OK;
}

lmoe_status lmoe_launch_count(const lmoe_handle *h, int64_t T, int32_t *launches)
{
    g_err.clear();
    if (!h || !launches) return fail(LMOE_ERR_INVALID_ARG, "NULL argument");
    // kernels: router, top-k, scan, dispatch (one kernel for few tokens), down
    // (none in the standard form), permute (none when the routed GEMVs read z
    // through the slot map), gate/up, down+combine, norm, shared, final; plus one
    // reduction per split-K GEMM other than the router's (which the top-k kernel
    // reduces).  Memsets (control words, per-block expert counts) are not kernels
    // and are not counted.
    if (T == 0) { *launches = 0; return LMOE_OK; }
    const lmoe_config &c = h->cfg;
    const SplitPlan sp = plan_splits(h, T);
    *launches = 11 - (c.standard ? 1 : 0) + (sp.down > 1) + (sp.shared > 1) + (sp.final_ > 1) -
                (small_route(h, T) ? 3 : 0) - (gemv_experts(h, T) ? 1 : 0) - (sp.fused_router ? 1 : 0) +
                (split_final(h, T) ? 1 : 0);
    return LMOE_OK;
}

lmoe_status lmoe_set_bias(lmoe_handle *h, const float *b, void *stream)
{
    g_err.clear();
    if (!h || !b) return fail(LMOE_ERR_INVALID_ARG, "NULL argument");
    LMOE_CUDA(cudaMemcpyAsync(h->b, b, sizeof(float) * h->cfg.E, cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
    return LMOE_OK;
}

lmoe_status lmoe_qb_histogram(const lmoe_handle *h, const void *workspace, int64_t T, int32_t bins, float lo, float hi,
                              int32_t *hist, void *stream)
{
    g_err.clear();
    if (!h || !hist) return fail(LMOE_ERR_INVALID_ARG, "NULL argument");
    if (!workspace && T > 0) {   // the built-in area of lmoe_forward_noalloc
        void *area = nullptr;
        size_t area_bytes = 0;
        const lmoe_status st = noalloc_area_for(h, &area, &area_bytes);
        if (st != LMOE_OK) return st;
        if (plan(h, T).total > area_bytes) return fail(LMOE_ERR_WORKSPACE, "T exceeds the built-in area");
        workspace = area;
    }
    if (T < 0) return fail(LMOE_ERR_INVALID_ARG, "T < 0");
    if (bins < 1 || bins > (1 << 20)) return fail(LMOE_ERR_INVALID_ARG, "bins=%d outside [1, 2^20]", bins);
    if (!std::isfinite(lo) || !std::isfinite(hi) || !(hi > lo)) return fail(LMOE_ERR_INVALID_ARG, "need finite lo < hi");
    if (T == 0) return LMOE_OK;
    const Layout L = plan(h, T);
    const char *ws = (const char *)workspace;
    LMOE_CUDA(launch_qb_histogram((const float *)(ws + L.r32), h->b, (const float *)(ws + L.cutoff), T, h->cfg.E,
                                  bins, lo, hi, hist, (cudaStream_t)stream));
    return LMOE_OK;
}

lmoe_status lmoe_qb_bias_update(const lmoe_handle *h, const int32_t *hist, int32_t bins, float lo, float hi,
                                int64_t target, float *bias_out, void *stream)
{
    g_err.clear();
    if (!h || !hist || !bias_out) return fail(LMOE_ERR_INVALID_ARG, "NULL argument");
    if (bins < 1 || bins > (1 << 20)) return fail(LMOE_ERR_INVALID_ARG, "bins=%d outside [1, 2^20]", bins);
    if (!std::isfinite(lo) || !std::isfinite(hi) || !(hi > lo)) return fail(LMOE_ERR_INVALID_ARG, "need finite lo < hi");
    if (target < 0) return fail(LMOE_ERR_INVALID_ARG, "target < 0");
    LMOE_CUDA(launch_qb_bias_update(hist, h->b, h->cfg.E, bins, lo, hi, target, bias_out, (cudaStream_t)stream));
    return LMOE_OK;
}

// The forward of lmoe_forward; reset_status = false keeps the device status
// word as it is (the chunks of one lmoe_forward_host call after the first).
static lmoe_status forward_body(lmoe_handle *h, const void *x, int64_t T, void *output, int32_t *selected_experts,
                                void *mixture_weights, void *latent_routed_aggregate, void *workspace,
                                size_t ws_bytes, void *stream, bool reset_status)
{
    if (!h) return fail(LMOE_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0) return fail(LMOE_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return LMOE_OK;
    if (!x || !output || !selected_experts || !mixture_weights || !latent_routed_aggregate || !workspace)
        return fail(LMOE_ERR_INVALID_ARG, "NULL tensor pointer");
    if (T * h->cfg.k > 0x7fffffffLL) return fail(LMOE_ERR_UNSUPPORTED, "T * k exceeds 2^31 - 1");
    const Layout L = plan(h, T);
    if (ws_bytes < L.total) return fail(LMOE_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
    if ((uintptr_t)workspace % 256) return fail(LMOE_ERR_WORKSPACE, "workspace not 256-byte aligned");

    if (h->tc && (((uintptr_t)x | (uintptr_t)output) & 15u))
        return fail(LMOE_ERR_UNSUPPORTED, "x and output must be 16-byte aligned for the tensor-core path");
    const lmoe_config &c = h->cfg;
    cudaStream_t s = (cudaStream_t)stream;
    char *ws = (char *)workspace;
    float *r32 = (float *)(ws + L.r32);
    float *p32 = (float *)(ws + L.p32);
    int32_t *blockhist = (int32_t *)(ws + L.blockhist);
    int32_t *base = (int32_t *)(ws + L.base);
    int32_t *counts = (int32_t *)(ws + L.counts);
    int32_t *offsets = (int32_t *)(ws + L.offsets);
    int32_t *tile_off = (int32_t *)(ws + L.tile_off);
    int32_t *slot_of = (int32_t *)(ws + L.slot_of);
    int32_t *perm_tok = (int32_t *)(ws + L.perm_tok);
    float *perm_w = (float *)(ws + L.perm_w);
    void *z = ws + L.z, *Zp = ws + L.Zp, *H = ws + L.H, *HS = ws + L.HS;
    void *Yp = ws + L.Yp;
    int32_t *status = (int32_t *)(ws + L.status);

    const int64_t S = T * c.k;
    const int nb = (int)((T + ROUTE_TPB - 1) / ROUTE_TPB);
    const int tk = c.dtype == LMOE_BF16 ? 1 : 0;
    const int64_t ld_hs = hs_cols(c);
    // Tensor-core tiles: 256-row tiles on CTA pairs where rows are plentiful
    // (grouped: at least ~192 slot rows per expert on average), else 128.
    const int cg_grouped = (h->tc && S >= 192LL * c.E) ? 2 : 1;
    const int cg_dense = (h->tc && T >= 256) ? 2 : 1;
    const int bm = h->tc ? TC_BM * cg_grouped : SIMT_BM;
    const int max_mtiles = (int)((S + bm - 1) / bm + c.E);

    // control words: the status word (kept across the chunks of one host call),
    // the routing ticket and the touched count
    if (reset_status) LMOE_CUDA(cudaMemsetAsync(status, 0, 3 * sizeof(int32_t), s));
    else LMOE_CUDA(cudaMemsetAsync(status + CTL_TICKET, 0, 2 * sizeof(int32_t), s));
    int32_t *touched = (int32_t *)(ws + L.touched);
    // the top-k kernel's per-block expert counts start at zero (cleared here,
    // so that the router GEMM and the top-k kernel follow each other directly)
    if (!small_route(h, T)) LMOE_CUDA(cudaMemsetAsync(blockhist, 0, sizeof(int32_t) * (size_t)nb * c.E, s));
    const SplitPlan sp = plan_splits(h, T);
    float *partial = (float *)(ws + L.partial);             // router, final
    float *partial_side = (float *)(ws + L.partial_side);   // down, shared gate/up
    const bool small = small_route(h, T);
    const bool gemv_routed = gemv_experts(h, T);
    const bool fused_router = sp.fused_router;
    const bool router_partial = h->tc && !small && !fused_router && sp.router > 1;

    // ---- the stages, each launched on stream `q`
    auto st_router = [&](cudaStream_t q) -> lmoe_status {   // r = sigmoid(x W_r^T)
        GemmArgs g = {};
        g.A = x; g.lda = c.d; g.M = (int)T; g.N = c.E; g.K = c.d;
        g.epi.out = r32; g.epi.ldo = c.E;
        if (small) {   // the whole routing (stages 1-4) in one launch
            SmallRouteArgs a = {};
            a.x = (const bf16 *)x; a.Wr = h->Wr; a.bias = h->b; a.T = (int)T; a.E = c.E; a.d = c.d; a.k = c.k;
            a.bm = bm; a.r = r32; a.sel = selected_experts; a.p32 = p32; a.p_out = mixture_weights;
            a.cutoff = (float *)(ws + L.cutoff); a.counts = counts; a.offsets = offsets; a.tile_off = tile_off;
            a.slot_of = slot_of; a.perm_tok = perm_tok; a.perm_w = perm_w; a.touched = touched;
            a.n_touched = status + CTL_NTOUCHED; a.ticket = status + CTL_TICKET;
            LMOE_CUDA(launch_route_small(a, tk, q));
        } else if (fused_router) {   // router, sigmoid, top-k and p in one launch
            LMOE_CUDA(tc_router_topk((const bf16 *)x, h->Wr3, h->b, T, c.E, c.d, c.k, r32, selected_experts,
                                     p32, mixture_weights, tk, (float *)(ws + L.cutoff), blockhist, status, q));
        } else if (router_partial) {
            // raw logits in split-K slabs; the top-k kernel sums them and applies the sigmoid
            GemmArgs gp = g;
            gp.epi.out = partial;
            gp.epi.ldo = c.E;
            LMOE_CUDA(tc_gemm_router(h->Wr3, gp, router_cg(T), status, q, sp.router));
        } else if (h->tc) {
            LMOE_CUDA(tc_gemm_router(h->Wr3, g, router_cg(T), status, q));
        } else {
            g.B = h->Wr; g.ldb = c.d;
            LMOE_CUDA(launch_simt_gemm(EPI_SIGMOID, tk, 0, 0, g, 0, q));
        }
        return LMOE_OK;
    };
    auto st_topk = [&](cudaStream_t q) -> lmoe_status {
        if (small || fused_router) return LMOE_OK;
        LMOE_CUDA(launch_topk(router_partial ? partial : r32, router_partial ? sp.router : 0, r32, h->b, T, c.E, c.k,
                              selected_experts, p32, mixture_weights, tk, blockhist, (float *)(ws + L.cutoff), q));
        return LMOE_OK;
    };
    auto st_scan = [&](cudaStream_t q) -> lmoe_status {
        if (small) return LMOE_OK;
        LMOE_CUDA(launch_scan(blockhist, nb, c.E, counts, base, q));
        return LMOE_OK;
    };
    auto st_dispatch = [&](cudaStream_t q) -> lmoe_status {
        if (small) return LMOE_OK;
        LMOE_CUDA(launch_dispatch(selected_experts, p32, base, counts, T, c.E, c.k, bm, offsets, tile_off, slot_of,
                                  perm_tok, perm_w, q));
        return LMOE_OK;
    };

    // z = x W_down^T, once per token
    GemmArgs gd = {};
    gd.A = x; gd.lda = c.d; gd.B = h->Wdown; gd.ldb = c.d; gd.M = (int)T; gd.N = c.l; gd.K = c.d;
    gd.epi.out = z; gd.epi.ldo = c.l;
    // per expert h = act(G z, U z) on the slot rows Zp[m] = z[perm_tok[m]]
    GemmArgs gu = {};
    gu.A = Zp; gu.lda = c.l; gu.B = h->Wgu; gu.ldb = c.l; gu.b_group_stride = 2 * (int64_t)c.f * c.l;
    gu.M = (int)S; gu.N = 2 * c.f; gu.K = c.l; gu.offsets = offsets; gu.tile_off = tile_off; gu.E = c.E;
    gu.epi.out = H; gu.epi.ldo = c.f; gu.epi.act = c.act; gu.epi.gate_cap = c.gate_cap; gu.epi.up_cap = c.up_cap;
    gu.epi.ib = h->ib;
    // per expert Y = p (h D^T)
    GemmArgs gc = {};
    gc.A = H; gc.lda = c.f; gc.B = h->D; gc.ldb = c.f; gc.b_group_stride = (int64_t)c.l * c.f;
    gc.M = (int)S; gc.N = c.l; gc.K = c.f; gc.offsets = offsets; gc.tile_off = tile_off; gc.E = c.E;
    gc.epi.out = Yp; gc.epi.ldo = c.l; gc.epi.row_w = perm_w;
    // shared experts' hidden, both as one expert of width 2 f_s
    GemmArgs gs = {};
    gs.A = x; gs.lda = c.d; gs.B = h->Wgu_s; gs.ldb = c.d; gs.M = (int)T; gs.N = 4 * c.f_shared; gs.K = c.d;
    gs.epi.out = HS; gs.epi.ldo = ld_hs; gs.epi.act = c.act; gs.epi.gate_cap = c.gate_cap;
    gs.epi.up_cap = c.up_cap; gs.epi.ib = h->ib;
    // From 256 tokens on, the shared GEMM follows the down GEMM on the side
    // stream without launching early: launched early, its CTAs sit on the SMs
    // the down GEMM leaves free, waiting for it, and the router (on the
    // caller's stream, as big per CTA) can start only after the whole shared
    // GEMM; this way the router runs first and the routing kernels run beside
    // the shared GEMM (measured on B200: large_d4096 15.9 -> 15.4 ms per
    // forward, the others within 0.5 %).
    gs.no_early_launch = (h->tc && T >= 256) ? 1 : 0;
    // y = [h_s | n] [D_s1 | D_s2 | W_up]^T
    GemmArgs gf = {};
    gf.A = HS; gf.lda = ld_hs; gf.B = h->Wcat; gf.ldb = ld_hs; gf.M = (int)T; gf.N = c.d; gf.K = (int)ld_hs;
    gf.epi.out = output; gf.epi.ldo = c.d;
    if (c.standard) {   // y = [h_s] [D_s1 | D_s2]^T + u
        gf.epi.residual = latent_routed_aggregate;
        gf.epi.ldr = c.l;
    }

    // Dense tensor-core GEMM, split along K per the plan.
    auto dense_tc = [&](int mode, const GemmArgs &g, int ks, float *part, cudaStream_t q) -> cudaError_t {
        if (ks <= 1) return tc_gemm(mode, g, 0, cg_dense, status, q);
        GemmArgs gp = g;
        gp.epi.out = part;
        gp.epi.ldo = g.N;
        cudaError_t e = tc_gemm(EPI_STORE_F32, gp, 0, 1, status, q, ks);
        if (e != cudaSuccess) return e;
        return launch_splitk_reduce(part, ks, g.M, g.N, mode, g.epi.act, g.epi.gate_cap, g.epi.up_cap, g.epi.ib,
                                    g.epi.out, g.epi.ldo, q, g.epi.residual, g.epi.ldr);
    };
    auto st_down = [&](cudaStream_t q) -> lmoe_status {
        if (c.standard) return LMOE_OK;   // experts read x itself
        if (h->tc && T <= GEMV_MAX_T) LMOE_CUDA(launch_gemv(EPI_STORE, gd, q));
        else if (h->tc) LMOE_CUDA(dense_tc(EPI_STORE, gd, sp.down, partial_side, q));
        else LMOE_CUDA(launch_simt_gemm(EPI_STORE, tk, tk, tk, gd, 0, q));
        return LMOE_OK;
    };
    auto st_permute = [&](cudaStream_t q) -> lmoe_status {
        if (gemv_routed) return LMOE_OK;   // the routed GEMVs read z through the slot -> token map
        LMOE_CUDA(launch_permute_tokens(c.standard ? x : z, slot_of, Zp, T, c.k, c.l, (int)h->tb, q));
        return LMOE_OK;
    };
    auto st_gate_up = [&](cudaStream_t q) -> lmoe_status {
        if (gemv_routed) {
            GemmArgs g = gu;
            g.A = c.standard ? x : z;
            g.lda = c.l;
            LMOE_CUDA(launch_gemv_grouped(EPI_GLU, g, touched, status + CTL_NTOUCHED,
                                          (int)std::min<int64_t>(c.E, S), perm_tok, (int)T, q));
        } else if (h->tc) LMOE_CUDA(tc_gemm(EPI_GLU, gu, max_mtiles, cg_grouped, status, q));
        else LMOE_CUDA(launch_simt_gemm(EPI_GLU, tk, tk, tk, gu, max_mtiles, q));
        return LMOE_OK;
    };
    auto st_down_combine = [&](cudaStream_t q) -> lmoe_status {
        if (gemv_routed)
            LMOE_CUDA(launch_gemv_grouped(EPI_COMBINE, gc, touched, status + CTL_NTOUCHED,
                                          (int)std::min<int64_t>(c.E, S), nullptr, (int)T, q));
        else if (h->tc) LMOE_CUDA(tc_gemm(EPI_COMBINE, gc, max_mtiles, cg_grouped, status, q));
        else LMOE_CUDA(launch_simt_gemm(EPI_COMBINE, tk, tk, tk, gc, max_mtiles, q));
        return LMOE_OK;
    };
    auto st_combine_norm = [&](cudaStream_t q) -> lmoe_status {   // u, RMSNorm(u) after the shared hidden
        LMOE_CUDA(launch_combine_norm(Yp, slot_of, T, c.l, c.k, c.eps, latent_routed_aggregate,
                                      c.standard ? nullptr : HS, ld_hs, 2 * (int64_t)c.f_shared, tk, q));
        return LMOE_OK;
    };
    auto st_shared = [&](cudaStream_t q) -> lmoe_status {
        if (h->tc && T <= GEMV_MAX_T) LMOE_CUDA(launch_gemv(EPI_GLU, gs, q));
        else if (h->tc) LMOE_CUDA(dense_tc(EPI_GLU, gs, sp.shared, partial_side, q));
        else LMOE_CUDA(launch_simt_gemm(EPI_GLU, tk, tk, tk, gs, 0, q));
        return LMOE_OK;
    };
    // split final GEMV: [h_s] [D_s1 | D_s2]^T into fp32, then n W_up^T + that
    float *final32 = (float *)(ws + L.final32);
    const bool split_fin = split_final(h, T);
    auto st_final_shared = [&](cudaStream_t q) -> lmoe_status {
        GemmArgs g = gf;
        g.K = 2 * c.f_shared;
        g.epi.out = final32;
        g.epi.ldo = c.d;
        LMOE_CUDA(launch_gemv(EPI_STORE_F32, g, q));
        return LMOE_OK;
    };
    auto st_final = [&](cudaStream_t q) -> lmoe_status {
        if (split_fin) {
            GemmArgs g = gf;
            g.A = (const char *)HS + h->tb * 2 * (int64_t)c.f_shared;
            g.B = (const char *)h->Wcat + h->tb * 2 * (int64_t)c.f_shared;
            g.K = c.l;
            g.epi.residual32 = final32;
            LMOE_CUDA(launch_gemv(EPI_STORE, g, q));
        } else if (h->tc && T <= GEMV_MAX_T) LMOE_CUDA(launch_gemv(EPI_STORE, gf, q));
        else if (h->tc) LMOE_CUDA(dense_tc(EPI_STORE, gf, sp.final_, partial, q));
        else LMOE_CUDA(launch_simt_gemm(EPI_STORE, tk, tk, tk, gf, 0, q));
        return LMOE_OK;
    };
#define RUN(call)                                                                                \
    do {                                                                                         \
        const lmoe_status st_ = (call);                                                          \
        if (st_ != LMOE_OK) return st_;                                                          \
    } while (0)

    if (!use_side_stream(h)) {
        // One stream, in the order of the stage names; with stage events set,
        // event i is recorded before stage i and event LMOE_NUM_STAGES after the last.
#define STAGE(i)                                                                                 \
    if (h->stage_events) LMOE_CUDA(cudaEventRecord((cudaEvent_t)h->stage_events[i], s))
        STAGE(0); RUN(st_router(s));
        STAGE(1); RUN(st_topk(s));
        STAGE(2); RUN(st_scan(s));
        STAGE(3); RUN(st_dispatch(s));
        STAGE(4); RUN(st_down(s));
        STAGE(5); RUN(st_permute(s));
        STAGE(6); RUN(st_gate_up(s));
        STAGE(7); RUN(st_down_combine(s));
        STAGE(8); RUN(st_combine_norm(s));
        STAGE(9); RUN(st_shared(s));
        STAGE(10);
        if (split_fin) RUN(st_final_shared(s));
        RUN(st_final(s));
        STAGE(LMOE_NUM_STAGES);
#undef STAGE
        return LMOE_OK;
    }

    // Two streams: the down-projection and the shared experts' gate/up GEMM
    // need only x, so they run on the handle's side stream (the down GEMM
    // first, beside the router GEMM, neither of which fills the GPU alone)
    // while the caller's stream does the router and the latency-bound routing
    // steps (top-k, scan, dispatch, permute), whose blocks fit beside the GEMM
    // blocks on the same SMs.  The caller's stream waits for z before the
    // permute, and for the shared GEMM before the routed gate/up GEMM: the
    // routed GEMMs then start with every SM free, as their static tile
    // schedule wants (with a few tokens, before the final GEMV instead).  (A down-projection that writes z straight into the k
    // slot rows from its epilogue, after the dispatch, was measured 5x slower
    // than this GEMM plus the row-contiguous permute.)
    {
        // record + wait as one step, so that a forward from another host thread
        // cannot slip its own record in between
        std::lock_guard<std::mutex> lock(h->fork_mutex);
        LMOE_CUDA(cudaEventRecord(h->ev_fork, s));
        LMOE_CUDA(cudaStreamWaitEvent(h->side, h->ev_fork, 0));
        RUN(st_down(h->side));
        LMOE_CUDA(cudaEventRecord(h->ev_z, h->side));
        RUN(st_shared(h->side));
        if (split_fin) RUN(st_final_shared(h->side));
        LMOE_CUDA(cudaEventRecord(h->ev_join, h->side));
    }
    RUN(st_router(s));
    RUN(st_topk(s));
    RUN(st_scan(s));
    RUN(st_dispatch(s));
    // a later record on the in-order side stream covers this forward's GEMMs too
    LMOE_CUDA(cudaStreamWaitEvent(s, h->ev_z, 0));
    RUN(st_permute(s));
    // Weight-streaming GEMVs (a few tokens) share HBM, not SMs: the routed
    // ones start as soon as z and the routing are ready, and only the final
    // GEMV, which reads the shared experts' output, waits for the side stream.
    const bool join_late = gemv_experts(h, T);
    if (!join_late) LMOE_CUDA(cudaStreamWaitEvent(s, h->ev_join, 0));
    RUN(st_gate_up(s));
    RUN(st_down_combine(s));
    RUN(st_combine_norm(s));
    if (join_late) LMOE_CUDA(cudaStreamWaitEvent(s, h->ev_join, 0));
    RUN(st_final(s));
#undef RUN
    return LMOE_OK;
}

lmoe_status lmoe_forward(lmoe_handle *h, const void *x, int64_t T, void *output, int32_t *selected_experts,
                         void *mixture_weights, void *latent_routed_aggregate, void *workspace, size_t ws_bytes,
                         void *stream)
{
    g_err.clear();
    return forward_body(h, x, T, output, selected_experts, mixture_weights, latent_routed_aggregate, workspace,
                        ws_bytes, stream, true);
}

// Bytes of the device staging of x and the four outputs in front of the
// forward workspace inside an lmoe_forward_host workspace.
static size_t host_staging_bytes(const lmoe_handle *h, int64_t T)
{
    const lmoe_config &c = h->cfg;
    size_t o = 0;
    o = align_up(o + h->tb * T * c.d, 256);          // x
    o = align_up(o + h->tb * T * c.d, 256);          // output
    o = align_up(o + sizeof(int32_t) * T * c.k, 256);
    o = align_up(o + h->tb * T * c.k, 256);
    o = align_up(o + h->tb * T * c.l, 256);
    return o;
}

lmoe_status lmoe_host_workspace_size(const lmoe_handle *h, int64_t T, size_t *bytes)
{
    g_err.clear();
    if (!h || !bytes) return fail(LMOE_ERR_INVALID_ARG, "NULL argument");
    if (T < 0) return fail(LMOE_ERR_INVALID_ARG, "T < 0");
    if (T == 0) { *bytes = 0; return LMOE_OK; }
    const lmoe_config &c = h->cfg;
    const size_t o = host_staging_bytes(h, T);
    int64_t Tc = T;
    const int nc = host_chunks(c, T, &Tc);
    size_t fw = plan(h, Tc).total;                       // the chunks' forward workspace
    if (nc > 1) fw = std::max(fw, plan(h, T - (int64_t)(nc - 1) * Tc).total);
    *bytes = o + fw;
    return LMOE_OK;
}

lmoe_status lmoe_forward_host(lmoe_handle *h, const void *x_host, int64_t T, void *output_host,
                              int32_t *selected_experts_host, void *mixture_weights_host,
                              void *latent_routed_aggregate_host, void *workspace, size_t ws_bytes, void *stream)
{
    g_err.clear();
    if (!h) return fail(LMOE_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0) return fail(LMOE_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return LMOE_OK;
    if (!x_host || !output_host || !selected_experts_host || !mixture_weights_host || !latent_routed_aggregate_host ||
        !workspace)
        return fail(LMOE_ERR_INVALID_ARG, "NULL pointer");
    size_t need = 0;
    lmoe_host_workspace_size(h, T, &need);
    if (ws_bytes < need) return fail(LMOE_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
    if ((uintptr_t)workspace % 256) return fail(LMOE_ERR_WORKSPACE, "workspace not 256-byte aligned");
    const lmoe_config &c = h->cfg;
    cudaStream_t s = (cudaStream_t)stream;
    char *ws = (char *)workspace;
    size_t o = 0;
    const size_t bx = h->tb * T * c.d, bs = sizeof(int32_t) * T * c.k, bp = h->tb * T * c.k, bu = h->tb * T * c.l;
    char *dx = ws + o; o = align_up(o + bx, 256);
    char *dy = ws + o; o = align_up(o + bx, 256);
    char *dsel = ws + o; o = align_up(o + bs, 256);
    char *dp = ws + o; o = align_up(o + bp, 256);
    char *du = ws + o; o = align_up(o + bu, 256);
    char *fws = ws + o;
    const size_t fbytes = ws_bytes - o;
    int64_t Tc = T;
    const int nc = host_chunks(c, T, &Tc);
    if (nc == 1) {
        LMOE_CUDA(cudaMemcpyAsync(dx, x_host, bx, cudaMemcpyHostToDevice, s));
        lmoe_status st = forward_body(h, dx, T, dy, (int32_t *)dsel, dp, du, fws, fbytes, stream, true);
        if (st != LMOE_OK) return st;
        LMOE_CUDA(cudaMemcpyAsync(output_host, dy, bx, cudaMemcpyDeviceToHost, s));
        LMOE_CUDA(cudaMemcpyAsync(selected_experts_host, dsel, bs, cudaMemcpyDeviceToHost, s));
        LMOE_CUDA(cudaMemcpyAsync(mixture_weights_host, dp, bp, cudaMemcpyDeviceToHost, s));
        LMOE_CUDA(cudaMemcpyAsync(latent_routed_aggregate_host, du, bu, cudaMemcpyDeviceToHost, s));
        return LMOE_OK;
    }
    // Pipeline: chunk j's input on copy_in, its forward on `stream` (after its
    // input), its outputs on copy_out (after its forward); the caller's stream
    // waits for the last copy.  One status word for the whole call.
    std::lock_guard<std::mutex> lock(h->host_mutex);
    cudaEvent_t *ev = h->ev_host;   // [0] start, [1] all out, [2 + j] chunk j in, [2 + 8 + j] chunk j done
    const size_t rx = h->tb * c.d, rs = sizeof(int32_t) * c.k, rp = h->tb * c.k, ru = h->tb * c.l;
    LMOE_CUDA(cudaMemsetAsync(fws + plan(h, Tc).status, 0, sizeof(int32_t), s));
    LMOE_CUDA(cudaEventRecord(ev[0], s));
    LMOE_CUDA(cudaStreamWaitEvent(h->copy_in, ev[0], 0));
    LMOE_CUDA(cudaStreamWaitEvent(h->copy_out, ev[0], 0));
    for (int j = 0; j < nc; ++j) {
        const int64_t t0 = (int64_t)j * Tc;
        const int64_t tj = std::min(Tc, T - t0);
        LMOE_CUDA(cudaMemcpyAsync(dx + t0 * rx, (const char *)x_host + t0 * rx, tj * rx, cudaMemcpyHostToDevice,
                                  h->copy_in));
        LMOE_CUDA(cudaEventRecord(ev[2 + j], h->copy_in));
        LMOE_CUDA(cudaStreamWaitEvent(s, ev[2 + j], 0));
        const lmoe_status st = forward_body(h, dx + t0 * rx, tj, dy + t0 * rx, (int32_t *)(dsel + t0 * rs),
                                            dp + t0 * rp, du + t0 * ru, fws, fbytes, stream, false);
        if (st != LMOE_OK) return st;
        LMOE_CUDA(cudaEventRecord(ev[2 + HOST_MAX_CHUNKS + j], s));
        LMOE_CUDA(cudaStreamWaitEvent(h->copy_out, ev[2 + HOST_MAX_CHUNKS + j], 0));
        LMOE_CUDA(cudaMemcpyAsync((char *)output_host + t0 * rx, dy + t0 * rx, tj * rx, cudaMemcpyDeviceToHost,
                                  h->copy_out));
        LMOE_CUDA(cudaMemcpyAsync((char *)selected_experts_host + t0 * rs, dsel + t0 * rs, tj * rs,
                                  cudaMemcpyDeviceToHost, h->copy_out));
        LMOE_CUDA(cudaMemcpyAsync((char *)mixture_weights_host + t0 * rp, dp + t0 * rp, tj * rp,
                                  cudaMemcpyDeviceToHost, h->copy_out));
        LMOE_CUDA(cudaMemcpyAsync((char *)latent_routed_aggregate_host + t0 * ru, du + t0 * ru, tj * ru,
                                  cudaMemcpyDeviceToHost, h->copy_out));
    }
    LMOE_CUDA(cudaEventRecord(ev[1], h->copy_out));
    LMOE_CUDA(cudaStreamWaitEvent(s, ev[1], 0));
    return LMOE_OK;
}

// Read and clear the device status word at `word`.
static lmoe_status check_status_word(char *word, cudaStream_t s)
{
    int32_t v = 0;
    LMOE_CUDA(cudaMemcpyAsync(&v, word, sizeof v, cudaMemcpyDeviceToHost, s));
    LMOE_CUDA(cudaStreamSynchronize(s));
    if (v != 0) {
        LMOE_CUDA(cudaMemsetAsync(word, 0, sizeof(int32_t), s));
        LMOE_CUDA(cudaStreamSynchronize(s));
        return fail(LMOE_ERR_DEVICE_TIMEOUT, "a kernel's bounded wait gave up (status word 0x%x)", v);
    }
    return LMOE_OK;
}

lmoe_status lmoe_check_device(lmoe_handle *h, int64_t T, void *workspace, void *stream)
{
    g_err.clear();
    if (!h) return fail(LMOE_ERR_INVALID_ARG, "NULL argument");
    if (T < 1) return LMOE_OK;
    if (!workspace) {   // the built-in area of lmoe_forward_noalloc
        size_t area_bytes = 0;
        const lmoe_status st = noalloc_area_for(h, &workspace, &area_bytes);
        if (st != LMOE_OK) return st;
    }
    return check_status_word((char *)workspace + plan(h, T).status, (cudaStream_t)stream);
}

lmoe_status lmoe_check_device_host(lmoe_handle *h, int64_t T, void *workspace, void *stream)
{
    g_err.clear();
    if (!h || !workspace) return fail(LMOE_ERR_INVALID_ARG, "NULL argument");
    if (T < 1) return LMOE_OK;
    // the forward workspace follows the staging of x and the four outputs; its
    // status word is first in every chunk's layout
    return check_status_word((char *)workspace + host_staging_bytes(h, T) + plan(h, 1).status,
                             (cudaStream_t)stream);
}

}  // extern "C"
