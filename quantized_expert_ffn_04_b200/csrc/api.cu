// C ABI of the Strata MoE layer library: handle lifetime, weight upload and
// repack, and the per-call orchestration of the kernels on the caller's
// stream.  Every step of the layer runs in this library's kernels; there is no
// host fallback.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <string>
#include <vector>

#include "../../include/strata_moe.h"
#include "common.cuh"
#include "internal.h"

using namespace strata;

namespace {

thread_local std::string g_err;

strata_status fail(strata_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
strata_status fail(strata_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

strata_status cuda_fail(cudaError_t e, const char *what) {
    return fail(STRATA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Switch to a device for the duration of a call.
struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) ok = cudaSetDevice(dev) == cudaSuccess;
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---- every allocation of the library goes through these wrappers: they
// count the live blocks and can be told to fail the n-th allocation from now
// (a host-side fault injector for the out-of-memory paths; it never touches
// the device beyond refusing to allocate).
std::atomic<long long> g_alloc_seq{0};   // allocations attempted so far
std::atomic<long long> g_fail_at{-1};    // sequence number that fails, -1: none
std::atomic<long long> g_live{0};        // device + pinned blocks alive

bool injected_failure() {
    const long long seq = g_alloc_seq.fetch_add(1);
    return g_fail_at.load() == seq;
}
cudaError_t dev_malloc(void **p, size_t n) {
    *p = nullptr;
    if (injected_failure()) return cudaErrorMemoryAllocation;
    const cudaError_t e = cudaMalloc(p, n);
    if (e != cudaSuccess) {
        *p = nullptr;
        cudaGetLastError();  // the failure is reported, not left sticky
        return e;
    }
    if (*p) g_live.fetch_add(1);
    return cudaSuccess;
}
template <class T>
cudaError_t dev_malloc(T **p, size_t n) {
    void *v = nullptr;
    const cudaError_t e = dev_malloc(&v, n);
    *p = static_cast<T *>(v);
    return e;
}
void dev_free(void *p) {
    if (!p) return;
    cudaFree(p);
    g_live.fetch_sub(1);
}
cudaError_t pinned_malloc(int **p) {
    *p = nullptr;
    if (injected_failure()) return cudaErrorMemoryAllocation;
    void *v = nullptr;
    const cudaError_t e = cudaMallocHost(&v, sizeof(int));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return e;
    }
    *p = static_cast<int *>(v);
    g_live.fetch_add(1);
    return cudaSuccess;
}
void pinned_free(int *p) {
    if (!p) return;
    cudaFreeHost(p);
    g_live.fetch_sub(1);
}

constexpr long long kDefaultBudget = 4000000000ll;  // ~2 s at the top SM clock

}  // namespace

struct strata_moe {
    int device = 0;
    strata_moe_config cfg{};
    Geometry geo{};
    uint8_t *wq = nullptr;        // (E + 1) experts; the shared expert last
    float *router_wp = nullptr;   // [E][H/128][32][4]
    float *router_b = nullptr;    // [E] or null
    __half *router_split = nullptr;  // [router_rows][H]: fp16(W) rows, then fp16(W - fp16(W))
    int router_rows = 0;             // 2E rounded up to 128
    float screen_gam = 0.f, screen_wmax = 0.f, screen_bmax = 0.f;
    // token prescale bound: the largest gate/up row L2 norm times
    // sqrt(max(1, sqrt(I) * (largest down row L2 norm) / 2)), padded 0.1 %
    float w2eff = 0.f;
    void *ws = nullptr;
    size_t ws_bytes = 0;
    // workspace views
    float *logits = nullptr;
    int32_t *idx = nullptr, *slot = nullptr, *list = nullptr, *cnt = nullptr, *off = nullptr;
    float *wts = nullptr;
    DispatchScratch ds{};
    int4 *units = nullptr;
    int *n_units = nullptr;
    void *a = nullptr;            // fp16 [slots][Ip]
    void *Y = nullptr;            // fp32 (decode) / fp16 (prefill) [slots][H]
    int *err = nullptr;
    int *err_host = nullptr;  // pinned copy of the error word (one sync per host forward)
    void *xio = nullptr, *yio = nullptr, *xn = nullptr;  // bf16 [max_tokens][H]
    // fp16 token operand of the tensor-core path, [max_tokens * k + max_tokens][H]:
    // routed token rows in slot order, then (at row T * k) the fp16 copy of x
    void *xs = nullptr;
    float *dsplit = nullptr;  // [max_tokens][router_rows] screening GEMM output (T > 256)
    // fused decode layer: grid barrier counter (monotonic), two counter sets
    // (finished gate/up slabs per unit, finished down blocks per (token, row
    // block)) used by alternate launches, token prescale exponents
    unsigned long long *fused_bar = nullptr;
    int *fused_cnt = nullptr;
    int fused_stride = 0, fused_tok = 0;
    int *xex = nullptr;
    int *slot_ex = nullptr;       // [slots] prefill: the token exponent of every slot
    float *fcorr = nullptr;  // [min(max_tokens, 64)][H / 32] block corrections of the fused layer
    cudaEvent_t probe_begin[6] = {}, probe_end[6] = {};
    // options
    int path = 0;
    long long budget = kDefaultBudget;
    int decode_max_t = 64;
};

namespace {

strata_status validate_config(const strata_moe_config *c) {
    if (!c) return fail(STRATA_ERR_INVALID_ARG, "config is NULL");
    if (c->hidden <= 0 || c->n_experts <= 0 || c->top_k <= 0 || c->inter <= 0 ||
        c->max_tokens <= 0 || c->block <= 0)
        return fail(STRATA_ERR_INVALID_ARG, "config fields must be positive");
    if (c->block != 32) return fail(STRATA_ERR_UNSUPPORTED, "block must be 32 (got %d)", c->block);
    if (c->quant_bits < 1 || c->quant_bits > 3)
        return fail(STRATA_ERR_UNSUPPORTED, "quant_bits must be 1, 2 or 3 (got %d)", c->quant_bits);
    if (c->hidden % 128 || c->hidden > 6144)
        return fail(STRATA_ERR_UNSUPPORTED, "hidden must be a multiple of 128 and <= 6144 (got %d)",
                    c->hidden);
    if (c->inter % 32 || c->inter > 4096)
        return fail(STRATA_ERR_UNSUPPORTED, "inter must be a multiple of 32 and <= 4096 (got %d)",
                    c->inter);
    if (c->n_experts > 1024)
        return fail(STRATA_ERR_UNSUPPORTED, "n_experts must be <= 1024 (got %d)", c->n_experts);
    if (c->top_k > c->n_experts || c->top_k > 32)
        return fail(STRATA_ERR_UNSUPPORTED, "top_k must be <= min(n_experts, 32) (got %d)",
                    c->top_k);
    if (c->max_tokens > 65536)
        return fail(STRATA_ERR_UNSUPPORTED, "max_tokens must be <= 65536 (got %d)",
                    c->max_tokens);
    return STRATA_OK;
}

Geometry make_geometry(const strata_moe_config &c) {
    Geometry g{};
    g.H = c.hidden;
    g.E = c.n_experts;
    g.k = c.top_k;
    g.I = c.inter;
    g.Ip = (c.inter + 127) / 128 * 128;
    g.bits = c.quant_bits;
    g.nseg_h = g.H / kSegCols;
    g.nseg_i = g.Ip / kSegCols;
    g.ub = unit_bytes(g.bits);
    g.mat_bytes = (size_t)(g.Ip / kSlabRows) * g.nseg_h * g.ub;
    g.expert_bytes = 3 * g.mat_bytes;
    return g;
}

// Carve the workspace; with base == nullptr only computes the size.
size_t carve_workspace(strata_moe *h, char *base) {
    const Geometry &g = h->geo;
    const size_t T = (size_t)h->cfg.max_tokens, k = g.k, E = g.E, H = g.H;
    const size_t slots = T * k + T;
    const size_t y_bytes = slots * H * 4;  // fp32 staging of every (slot, column)
    int units = max_units((int)T, (int)k, (int)E, 8);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + bytes, 256);
        return base ? base + o : nullptr;
    };
    h->logits = (float *)take(T * E * 4);
    h->idx = (int32_t *)take(T * k * 4);
    h->wts = (float *)take(T * k * 4);
    h->slot = (int32_t *)take(T * k * 4);
    h->list = (int32_t *)take(T * k * 4);
    h->cnt = (int32_t *)take(E * 4);
    h->off = (int32_t *)take((E + 1) * 4);
    char *dsb = take(dispatch_scratch_bytes((int)T, (int)E));
    if (base) dispatch_scratch_carve(dsb, (int)T, (int)E, &h->ds);
    h->units = (int4 *)take((size_t)units * 16);
    h->n_units = (int *)take(4);
    h->err = (int *)take(4);
    h->a = take(slots * g.Ip * 2);
    h->Y = take(y_bytes);
    h->xio = take(T * H * 2);
    h->yio = take(T * H * 2);
    h->xn = take(T * H * 2);
    h->xs = take(slots * H * 2);
    h->dsplit = (float *)take(T > (size_t)kSmallMaxT ? T * (size_t)h->router_rows * 4 : 0);
    h->fused_tok = max_units(64, (int)k, (int)E, 8);
    // + 1: the launch's item claim counter (last entry of each set)
    h->fused_stride = h->fused_tok + 64 * (int)(H / 128) + 1;
    h->fused_bar = (unsigned long long *)take(8);
    h->fused_cnt = (int *)take((size_t)2 * h->fused_stride * 4);
    h->xex = (int *)take(T * 4);
    h->slot_ex = (int *)take(slots * 4);
    h->fcorr = (float *)take((T < 64 ? T : 64) * (H / 32) * 4);
    return off;
}

void free_handle(strata_moe *h) {
    if (!h) return;
    dev_free(h->wq);
    dev_free(h->router_wp);
    dev_free(h->router_b);
    dev_free(h->router_split);
    dev_free(h->ws);
    pinned_free(h->err_host);
    delete h;
}

strata_status check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, what);
    return STRATA_OK;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const char *pa = (const char *)a, *pb = (const char *)b;
    return pa < pb + nb && pb < pa + na;
}

strata_status check_tokens(strata_moe_t h, int T) {
    if (!h) return fail(STRATA_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0) return fail(STRATA_ERR_INVALID_ARG, "T must be >= 0 (got %d)", T);
    if (T > h->cfg.max_tokens)
        return fail(STRATA_ERR_INVALID_ARG, "T = %d exceeds max_tokens = %d", T,
                    h->cfg.max_tokens);
    return STRATA_OK;
}

enum { kStRouter, kStTopk, kStDispatch, kStGateUp, kStDown, kStCombine };

// Stage names of the NVTX ranges (one range per stage's launches on the
// host timeline; a profiler lines them up with the kernels).
const char *const kStageName[] = {"strata router", "strata top-k + dispatch", "strata dispatch",
                                  "strata gate/up", "strata down", "strata combine"};

void probe(strata_moe_t h, int stage, bool begin, cudaStream_t s) {
    if (begin)
        nvtxRangePushA(kStageName[stage]);
    else
        nvtxRangePop();
    cudaEvent_t e = begin ? h->probe_begin[stage] : h->probe_end[stage];
    if (!e) return;
    // inside a stream capture the record must become an event node of the graph
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(s, &cs);
    if (cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
    else
        cudaEventRecord(e, s);
}

// The fp16 copy of x inside the token operand (after the T * k routed rows).
__half *x16_of(strata_moe_t h, int T) {
    return reinterpret_cast<__half *>(h->xs) + (size_t)T * h->geo.k * h->geo.H;
}

// Router + top-k + dispatch into the handle's workspace.  Above kSmallMaxT
// tokens the router runs on the tensor cores (screening GEMM on the fp16 copy
// of x, which the prefill experts reuse) followed by the exact recompute of
// the candidates.
strata_status run_route(strata_moe_t h, const void *x, int T, int tile, cudaStream_t s) {
    const Geometry &g = h->geo;
    probe(h, kStRouter, true, s);
    if (T > kSmallMaxT) {
        launch_to_half(x, x16_of(h, T), (size_t)T * g.H, s);
        cudaError_t ce = launch_umma_plain(h->router_split, h->router_rows, x16_of(h, T), T,
                                           g.H, h->dsplit, h->err, h->budget, s);
        if (ce != cudaSuccess)
            return fail(STRATA_ERR_CUDA, "router screening GEMM: %s", cudaGetErrorString(ce));
        launch_screen_topk(h->dsplit, h->router_rows, x, T, g.H, h->router_wp, h->router_b, g.E,
                           g.k, h->screen_gam, h->screen_wmax, h->screen_bmax, h->idx, h->wts, s);
    } else {
        launch_router(x, T, g.H, h->router_wp, h->router_b, g.E, h->logits, s);
    }
    probe(h, kStRouter, false, s);
    if (T > kSmallMaxT) {
        probe(h, kStDispatch, true, s);
        launch_dispatch(h->idx, T, g.k, g.E, h->cnt, h->off, h->list, h->slot, h->ds, h->units,
                        h->n_units, tile, s, h->err);
        probe(h, kStDispatch, false, s);
    } else {
        // top-k and dispatch fused in one CTA (the top-k probe brackets both)
        probe(h, kStTopk, true, s);
        launch_route_small(h->logits, T, g.E, g.k, h->idx, h->wts, h->cnt, h->off, h->list,
                           h->slot, h->units, h->n_units, tile, s, h->err);
        probe(h, kStTopk, false, s);
    }
    return check_launch("routing kernels");
}

bool use_decode_path(strata_moe_t h, int T) {
    if (h->path == 1 || h->path == 3) return true;
    if (h->path == 2) return false;
    return T <= h->decode_max_t;
}

// The fused decode kernel: forced (path 3), or in auto mode for every decode
// batch it supports.
bool use_fused_path(strata_moe_t h, int T) {
    if (h->path == 3) return true;
    return h->path == 0 && T <= h->decode_max_t && fused_decode_supported(h->geo, T);
}

// The whole layer in one launch (router, top-k, dispatch, experts, combine).
strata_status run_forward_fused(strata_moe_t h, const void *x, int T, void *y, bool residual,
                                cudaStream_t s) {
    const Geometry &g = h->geo;
    if (!fused_decode_supported(g, T))
        return fail(STRATA_ERR_INVALID_ARG, "the fused decode kernel does not support T=%d", T);
    ExpertWeights w{h->wq, h->wq + (size_t)g.E * g.expert_bytes};
    FusedArgs fa{};
    fa.x = x;
    fa.router_wp = h->router_wp;
    fa.router_b = h->router_b;
    fa.w2 = h->w2eff;
    fa.logits = h->logits;
    fa.idx = h->idx;
    fa.wts = h->wts;
    fa.x16 = x16_of(h, T);
    fa.xex = h->xex;
    fa.corr = h->fcorr;
    fa.a = h->a;
    fa.Y = (float *)h->Y;
    fa.out = y;
    fa.residual = residual;
    fa.bar = h->fused_bar;
    fa.cnt = h->fused_cnt;
    fa.cnt_stride = h->fused_stride;
    fa.cnt_tok = h->fused_tok;
    fa.err = h->err;
    fa.budget = h->budget;
    probe(h, kStGateUp, true, s);
    cudaError_t ce = launch_fused_decode(g, w, fa, T, s);
    probe(h, kStGateUp, false, s);
    if (ce != cudaSuccess)
        return fail(STRATA_ERR_CUDA, "fused decode kernel: %s", cudaGetErrorString(ce));
    return check_launch("fused decode kernel");
}

strata_status run_forward(strata_moe_t h, const void *x, int T, void *y, bool residual,
                          cudaStream_t s) {
    if (use_fused_path(h, T)) return run_forward_fused(h, x, T, y, residual, s);
    const Geometry &g = h->geo;
    const bool decode = use_decode_path(h, T);
    const int tile = decode ? 8 : kUmmaTile;
    // the decode chain's token exponents: a plain launch ahead of the router,
    // so every later kernel starts after it completed
    if (decode) launch_prescale(x, T, g.H, h->w2eff, h->xex, nullptr, s);
    strata_status st = run_route(h, x, T, tile, s);
    if (st != STRATA_OK) return st;
    ExpertWeights w{h->wq, h->wq + (size_t)g.E * g.expert_bytes};
    int umax = max_units(T, g.k, g.E, tile);
    if (decode) {
        probe(h, kStGateUp, true, s);
        launch_gemv_gateup(g, w, h->units, h->n_units, umax, h->list, T * g.k, T, x, h->xex,
                           h->a, h->err, h->budget, s);
        probe(h, kStGateUp, false, s);
        probe(h, kStDown, true, s);
        launch_gemv_down(g, w, h->units, h->n_units, umax, T, h->a, (float *)h->Y, h->err,
                         h->budget, s);
        probe(h, kStDown, false, s);
    } else {
        // the gate/up probe brackets the gate/up GEMM (and, for T <= kSmallMaxT,
        // the fp16 token copy, which larger batches make in the router stage)
        probe(h, kStGateUp, true, s);
        // the prescaled fp16 token operand (above kSmallMaxT it replaces the
        // unscaled copy the router's screening GEMM read)
        launch_prescale(x, T, g.H, h->w2eff, h->xex, x16_of(h, T), s);
        launch_gather_rows(h->list, T * g.k, x16_of(h, T), h->xs, g.H, s, T, h->err, h->xex,
                           h->slot_ex);
        cudaError_t ce = launch_umma_gateup(g, w, h->units, h->n_units, umax, T * g.k + T, h->xs,
                                            h->slot_ex, h->a, h->err, h->budget, s);
        if (ce != cudaSuccess)
            return fail(STRATA_ERR_CUDA, "gate/up GEMM: %s", cudaGetErrorString(ce));
        probe(h, kStGateUp, false, s);
        probe(h, kStDown, true, s);
        ce = launch_umma_down(g, w, h->units, h->n_units, umax, T * g.k + T, h->a, h->Y, h->err,
                              h->budget, s);
        if (ce != cudaSuccess)
            return fail(STRATA_ERR_CUDA, "down GEMM: %s", cudaGetErrorString(ce));
        probe(h, kStDown, false, s);
    }
    probe(h, kStCombine, true, s);
    launch_combine(h->Y, !decode, h->idx, h->wts, h->slot, T, g.k, g.H, y, residual, s, h->err,
                   h->xex);
    probe(h, kStCombine, false, s);
    return check_launch("expert kernels");
}

}  // namespace

void strata::set_error_message(const char *msg) { g_err = msg; }

extern "C" {

const char *strata_moe_last_error(void) { return g_err.c_str(); }

const char *strata_moe_version(void) { return "strata-moe-b200 0.1 (sm_100a)"; }

strata_status strata_moe_set_probe(strata_moe_t h, int stage, void *ev_begin, void *ev_end) {
    if (!h) return fail(STRATA_ERR_INVALID_ARG, "handle is NULL");
    if (stage < 0 || stage > 5) return fail(STRATA_ERR_INVALID_ARG, "stage must be 0..5");
    h->probe_begin[stage] = (cudaEvent_t)ev_begin;
    h->probe_end[stage] = (cudaEvent_t)ev_end;
    return STRATA_OK;
}

int strata_moe_launch_count(strata_moe_t h, int T) {
    if (!h || T < 0 || T > h->cfg.max_tokens) return 0;
    if (T == 0) return 0;
    // up to kSmallMaxT tokens: router, fused top-k + dispatch; above: fp16 token
    // copy, screening GEMM, screened top-k, 3 dispatch kernels.  Then the token
    // prescale, gate/up + down (the tensor-core path adds the slot-order row
    // gather), and the combine.
    if (use_fused_path(h, T)) return 1;  // the fused layer kernel
    const bool decode = use_decode_path(h, T);
    if (T <= kSmallMaxT) return 2 + 1 + (decode ? 2 : 3) + 1;
    return 6 + 1 + 3 + 1;
}

strata_status strata_moe_create(const strata_moe_config *cfg, const strata_moe_weights *wts,
                                int device, strata_moe_t *out) {
    if (!out) return fail(STRATA_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    strata_status st = validate_config(cfg);
    if (st != STRATA_OK) return st;
    if (!wts || !wts->codes || !wts->scales || !wts->router_w || !wts->shared_codes ||
        !wts->shared_scales || (cfg->has_router_bias && !wts->router_b))
        return fail(STRATA_ERR_INVALID_ARG, "a required weight pointer is NULL");
    int ndev = 0;
    cudaError_t ce = cudaGetDeviceCount(&ndev);
    if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDeviceCount");
    if (device < 0 || device >= ndev)
        return fail(STRATA_ERR_INVALID_ARG, "device %d out of range (%d devices)", device, ndev);
    DeviceGuard guard(device);
    if (!guard.ok) return fail(STRATA_ERR_CUDA, "cudaSetDevice(%d) failed", device);

    if ((ce = init_kernel_attributes()) != cudaSuccess)
        return cuda_fail(ce, "kernel attribute setup");
    strata_moe *h = new strata_moe();
    h->device = device;
    h->cfg = *cfg;
    h->geo = make_geometry(*cfg);
    h->router_rows = (2 * cfg->n_experts + 127) / 128 * 128;
    const Geometry &g = h->geo;
    const size_t H = g.H, E = g.E;

    // ---- allocations
    size_t ws_bytes = carve_workspace(h, nullptr);
    if (dev_malloc(&h->wq, (E + 1) * g.expert_bytes) != cudaSuccess ||
        dev_malloc(&h->router_wp, E * H * 4) != cudaSuccess ||
        (cfg->has_router_bias && dev_malloc(&h->router_b, E * 4) != cudaSuccess) ||
        dev_malloc(&h->ws, ws_bytes) != cudaSuccess) {
        size_t wbytes = (E + 1) * g.expert_bytes;
        free_handle(h);
        return fail(STRATA_ERR_OOM, "device allocation failed (weights %zu B, workspace %zu B)",
                    wbytes, ws_bytes);
    }
    h->ws_bytes = ws_bytes;
    carve_workspace(h, (char *)h->ws);
    if (pinned_malloc(&h->err_host) != cudaSuccess) {
        free_handle(h);
        return fail(STRATA_ERR_OOM, "pinned host allocation (error word) failed");
    }
    *h->err_host = 0;
    if ((ce = cudaMemset(h->ws, 0, ws_bytes)) != cudaSuccess) {
        free_handle(h);
        return cuda_fail(ce, "cudaMemset(workspace)");
    }

    // ---- router: lane-interleaved copy of W (Wp[e][s4][l][j] = W[e][128 s4 + 32 j + l])
    {
        std::vector<float> wp(E * H);
        for (size_t e = 0; e < E; e++)
            for (size_t i = 0; i < H; i++) {
                size_t s4 = i / 128, j = (i / 32) % 4, l = i % 32;
                wp[((e * (H / 128) + s4) * 32 + l) * 4 + j] = wts->router_w[e * H + i];
            }
        ce = cudaMemcpy(h->router_wp, wp.data(), E * H * 4, cudaMemcpyHostToDevice);
        // screening split W = fp16(W) + fp16(W - fp16(W)) and the bound's constants
        const size_t R = (size_t)h->router_rows;
        std::vector<__half> split(R * H, __float2half_rn(0.0f));
        double wmax = 0.0, bmax = 0.0;
        for (size_t e = 0; e < E; e++) {
            double n2 = 0.0;
            for (size_t i = 0; i < H; i++) {
                float w = wts->router_w[e * H + i];
                __half hi = __float2half_rn(w);
                split[e * H + i] = hi;
                split[(E + e) * H + i] = __float2half_rn(w - __half2float(hi));
                n2 += (double)w * w;
            }
            wmax = std::max(wmax, std::sqrt(n2));
            if (cfg->has_router_bias) bmax = std::max(bmax, (double)std::fabs(wts->router_b[e]));
        }
        h->screen_wmax = (float)(wmax * (1.0 + 1e-6));
        h->screen_bmax = (float)(bmax * (1.0 + 1e-6));
        h->screen_gam = (float)(H * std::ldexp(1.0, -23) + std::ldexp(1.0, -22) +
                                (H / 32.0 + 10.0) * std::ldexp(1.0, -24));
        if (ce == cudaSuccess) {
            if (dev_malloc(&h->router_split, R * H * 2) != cudaSuccess) {
                free_handle(h);
                return fail(STRATA_ERR_OOM, "router split allocation failed");
            }
            ce = cudaMemcpy(h->router_split, split.data(), R * H * 2, cudaMemcpyHostToDevice);
        }
        if (ce == cudaSuccess && cfg->has_router_bias)
            ce = cudaMemcpy(h->router_b, wts->router_b, E * 4, cudaMemcpyHostToDevice);
        if (ce != cudaSuccess) {
            free_handle(h);
            return cuda_fail(ce, "router upload");
        }
    }

    // ---- experts: upload the canonical format in batches, repack on the device
    {
        const size_t mat_codes = H * g.I * g.bits / 8, mat_scales = H * g.I / 32;
        const size_t ex_codes = 3 * mat_codes, ex_scales = 3 * mat_scales;
        const size_t batch = 32;
        uint8_t *tc = nullptr;
        uint16_t *ts = nullptr;
        unsigned *nrm = nullptr;  // [0] gate/up rows, [1] down rows: largest L2 norm (float bits)
        if (dev_malloc(&tc, batch * ex_codes) != cudaSuccess ||
            dev_malloc(&ts, batch * ex_scales * 2) != cudaSuccess ||
            dev_malloc(&nrm, 2 * sizeof(unsigned)) != cudaSuccess) {
            dev_free(tc);
            dev_free(ts);
            free_handle(h);
            return fail(STRATA_ERR_OOM, "staging allocation failed");
        }
        ce = cudaMemset(nrm, 0, 2 * sizeof(unsigned));
        for (size_t e0 = 0; e0 <= E && ce == cudaSuccess; e0 += batch) {
            size_t nb = (E + 1 - e0) < batch ? (E + 1 - e0) : batch;  // expert E = shared
            for (size_t i = 0; i < nb && ce == cudaSuccess; i++) {
                size_t e = e0 + i;
                const uint8_t *src_c = e < E ? wts->codes + e * ex_codes : wts->shared_codes;
                const uint16_t *src_s = e < E ? wts->scales + e * ex_scales : wts->shared_scales;
                ce = cudaMemcpy(tc + i * ex_codes, src_c, ex_codes, cudaMemcpyHostToDevice);
                if (ce == cudaSuccess)
                    ce = cudaMemcpy(ts + i * ex_scales, src_s, ex_scales * 2,
                                    cudaMemcpyHostToDevice);
            }
            for (size_t i = 0; i < nb && ce == cudaSuccess; i++) {
                uint8_t *dst = h->wq + (e0 + i) * g.expert_bytes;
                for (int m = 0; m < 3; m++) {
                    const uint8_t *c = tc + i * ex_codes + m * mat_codes;
                    const uint16_t *s = ts + i * ex_scales + m * mat_scales;
                    if (m < 2) {
                        launch_repack_matrix(c, s, g.bits, g.I, g.H, g.Ip, g.H,
                                             dst + m * g.mat_bytes, 0);
                        launch_row_norm_max(c, s, g.bits, g.I, g.H, nrm, 0);
                    } else {
                        launch_repack_matrix(c, s, g.bits, g.H, g.I, g.H, g.Ip,
                                             dst + m * g.mat_bytes, 0);
                        launch_row_norm_max(c, s, g.bits, g.H, g.I, nrm + 1, 0);
                    }
                }
                ce = cudaGetLastError();
            }
            if (ce == cudaSuccess) ce = cudaDeviceSynchronize();
        }
        unsigned nb[2] = {0u, 0u};
        if (ce == cudaSuccess) ce = cudaMemcpy(nb, nrm, sizeof nb, cudaMemcpyDeviceToHost);
        dev_free(tc);
        dev_free(ts);
        dev_free(nrm);
        if (ce != cudaSuccess) {
            free_handle(h);
            return cuda_fail(ce, "expert upload / repack");
        }
        float w2, wd2;
        memcpy(&w2, &nb[0], 4);
        memcpy(&wd2, &nb[1], 4);
        const double c = std::max(1.0, std::sqrt((double)g.I) * wd2 / 2.0);
        h->w2eff = (float)(w2 * std::sqrt(c) * 1.001);
    }
    *out = h;
    return STRATA_OK;
}

void strata_moe_destroy(strata_moe_t h) {
    if (!h) return;
    DeviceGuard guard(h->device);
    cudaDeviceSynchronize();
    free_handle(h);
}

strata_status strata_moe_set_option(strata_moe_t h, int option, int64_t value) {
    if (!h) return fail(STRATA_ERR_INVALID_ARG, "handle is NULL");
    switch (option) {
    case STRATA_OPT_PATH:
        if (value < 0 || value > 3)
            return fail(STRATA_ERR_INVALID_ARG, "path must be 0, 1, 2 or 3");
        h->path = (int)value;
        return STRATA_OK;
    case STRATA_OPT_WAIT_BUDGET:
        if (value < 0) return fail(STRATA_ERR_INVALID_ARG, "wait budget must be >= 0");
        h->budget = value;
        return STRATA_OK;
    case STRATA_OPT_DECODE_MAX_T:
        if (value < 0) return fail(STRATA_ERR_INVALID_ARG, "decode max T must be >= 0");
        h->decode_max_t = (int)value;
        return STRATA_OK;
    default:
        return fail(STRATA_ERR_INVALID_ARG, "unknown option %d", option);
    }
}

strata_status strata_moe_route(strata_moe_t h, const void *x_dev, int T, int32_t *idx_dev,
                               float *w_dev, int32_t *offsets_dev, int32_t *list_dev,
                               void *stream) {
    strata_status st = check_tokens(h, T);
    if (st != STRATA_OK) return st;
    if (T == 0) return STRATA_OK;
    if (!x_dev || !idx_dev || !w_dev) return fail(STRATA_ERR_INVALID_ARG, "NULL device pointer");
    if (((uintptr_t)x_dev) & 15) return fail(STRATA_ERR_INVALID_ARG, "x must be 16-byte aligned");
    DeviceGuard guard(h->device);
    cudaStream_t s = (cudaStream_t)stream;
    const Geometry &g = h->geo;
    st = run_route(h, x_dev, T, 8, s);
    if (st != STRATA_OK) return st;
    cudaError_t ce;
    size_t tk = (size_t)T * g.k;
    if ((ce = cudaMemcpyAsync(idx_dev, h->idx, tk * 4, cudaMemcpyDeviceToDevice, s)) ||
        (ce = cudaMemcpyAsync(w_dev, h->wts, tk * 4, cudaMemcpyDeviceToDevice, s)) ||
        (offsets_dev &&
         (ce = cudaMemcpyAsync(offsets_dev, h->off, (g.E + 1) * 4, cudaMemcpyDeviceToDevice, s))) ||
        (list_dev && (ce = cudaMemcpyAsync(list_dev, h->list, tk * 4, cudaMemcpyDeviceToDevice, s))))
        return cuda_fail(ce, "route output copy");
    return STRATA_OK;
}

strata_status strata_moe_forward(strata_moe_t h, const void *x_dev, int T, void *y_dev,
                                 void *stream) {
    strata_status st = check_tokens(h, T);
    if (st != STRATA_OK) return st;
    if (T == 0) return STRATA_OK;
    if (!x_dev || !y_dev) return fail(STRATA_ERR_INVALID_ARG, "NULL device pointer");
    size_t bytes = (size_t)T * h->geo.H * 2;
    if (overlaps(x_dev, bytes, y_dev, bytes))
        return fail(STRATA_ERR_INVALID_ARG, "x and y overlap");
    if ((((uintptr_t)x_dev) | ((uintptr_t)y_dev)) & 15)
        return fail(STRATA_ERR_INVALID_ARG, "x and y must be 16-byte aligned");
    DeviceGuard guard(h->device);
    return run_forward(h, x_dev, T, y_dev, false, (cudaStream_t)stream);
}

strata_status strata_moe_sync_status(strata_moe_t h, void *stream) {
    if (!h) return fail(STRATA_ERR_INVALID_ARG, "handle is NULL");
    DeviceGuard guard(h->device);
    cudaStream_t s = (cudaStream_t)stream;
    // the error word rides on the stream after the work it reports on, so one
    // synchronisation covers both
    cudaError_t ce = cudaMemcpyAsync(h->err_host, h->err, 4, cudaMemcpyDeviceToHost, s);
    if (ce != cudaSuccess) return cuda_fail(ce, "error word read");
    ce = cudaStreamSynchronize(s);
    if (ce != cudaSuccess) return cuda_fail(ce, "stream synchronize");
    const int e = *h->err_host;
    if (e) {
        *h->err_host = 0;
        cudaMemsetAsync(h->err, 0, 4, s);
        // a launch that gave up may leave the fused layer's barrier counter and
        // per-launch counters mid-count: start them over
        cudaMemsetAsync(h->fused_bar, 0, 8, s);
        cudaMemsetAsync(h->fused_cnt, 0, (size_t)2 * h->fused_stride * 4, s);
        cudaStreamSynchronize(s);
        if (e == kErrBounds)
            return fail(STRATA_ERR_BOUNDS, "a device-side index check failed (checked build)");
        return fail(STRATA_ERR_TIMEOUT, "a device-side wait gave up (code %d)", e);
    }
    return STRATA_OK;
}

strata_status strata_moe_forward_host(strata_moe_t h, const void *x_host, int T, void *y_host,
                                      void *stream) {
    strata_status st = check_tokens(h, T);
    if (st != STRATA_OK) return st;
    if (T == 0) return STRATA_OK;
    if (!x_host || !y_host) return fail(STRATA_ERR_INVALID_ARG, "NULL host pointer");
    DeviceGuard guard(h->device);
    cudaStream_t s = (cudaStream_t)stream;
    size_t bytes = (size_t)T * h->geo.H * 2;
    cudaError_t ce = cudaMemcpyAsync(h->xio, x_host, bytes, cudaMemcpyHostToDevice, s);
    if (ce != cudaSuccess) return cuda_fail(ce, "host to device copy");
    st = run_forward(h, h->xio, T, h->yio, false, s);
    if (st != STRATA_OK) return st;
    ce = cudaMemcpyAsync(y_host, h->yio, bytes, cudaMemcpyDeviceToHost, s);
    if (ce != cudaSuccess) return cuda_fail(ce, "device to host copy");
    return strata_moe_sync_status(h, stream);
}

strata_status strata_moe_rmsnorm(const void *h_dev, void *xn_dev, int T, int H, void *stream) {
    if (T < 0 || H <= 0 || H % 32) return fail(STRATA_ERR_INVALID_ARG, "bad T or H");
    if (T == 0) return STRATA_OK;
    if (!h_dev || !xn_dev) return fail(STRATA_ERR_INVALID_ARG, "NULL device pointer");
    if (overlaps(h_dev, (size_t)T * H * 2, xn_dev, (size_t)T * H * 2))
        return fail(STRATA_ERR_INVALID_ARG, "h and xn overlap");
    launch_rmsnorm(h_dev, xn_dev, T, H, (cudaStream_t)stream);
    return check_launch("rmsnorm");
}

strata_status strata_moe_stack_forward(const strata_moe_t *layers, int n_layers, void *h_dev,
                                       int T, void *h_trace_dev, void *stream) {
    if (!layers || n_layers <= 0) return fail(STRATA_ERR_INVALID_ARG, "no layers");
    strata_moe_t l0 = layers[0];
    strata_status st = check_tokens(l0, T);
    if (st != STRATA_OK) return st;
    if (T == 0) return STRATA_OK;
    if (!h_dev) return fail(STRATA_ERR_INVALID_ARG, "h is NULL");
    for (int l = 0; l < n_layers; l++) {
        strata_moe_t L = layers[l];
        if (!L || L->device != l0->device || L->cfg.hidden != l0->cfg.hidden ||
            L->cfg.n_experts != l0->cfg.n_experts || L->cfg.top_k != l0->cfg.top_k ||
            L->cfg.inter != l0->cfg.inter || L->cfg.quant_bits != l0->cfg.quant_bits)
            return fail(STRATA_ERR_INVALID_ARG, "layer %d does not match layer 0", l);
    }
    DeviceGuard guard(l0->device);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t bytes = (size_t)T * l0->geo.H * 2;
    for (int l = 0; l < n_layers; l++) {
        strata_moe_t L = layers[l];
        if (h_trace_dev) {
            cudaError_t ce = cudaMemcpyAsync((char *)h_trace_dev + l * bytes, h_dev, bytes,
                                             cudaMemcpyDeviceToDevice, s);
            if (ce != cudaSuccess) return cuda_fail(ce, "trace copy");
        }
        launch_rmsnorm(h_dev, l0->xn, T, l0->geo.H, s);
        // run layer L's weights (everything create() derived from them) in
        // layer 0's workspace
        strata_moe view = *l0;
        view.wq = L->wq;
        view.router_wp = L->router_wp;
        view.router_b = L->router_b;
        view.router_split = L->router_split;
        view.screen_gam = L->screen_gam;
        view.screen_wmax = L->screen_wmax;
        view.screen_bmax = L->screen_bmax;
        view.cfg.has_router_bias = L->cfg.has_router_bias;
        st = run_forward(&view, l0->xn, T, h_dev, true, s);
        if (st != STRATA_OK) return st;
    }
    return STRATA_OK;
}

strata_status strata_moe_debug_dequant(strata_moe_t h, int expert, int mat, int row0, int nrows,
                                       int kind, float *out_host) {
    if (!h || !out_host) return fail(STRATA_ERR_INVALID_ARG, "NULL argument");
    const Geometry &g = h->geo;
    if (expert < -1 || expert >= g.E || mat < 0 || mat > 2 || (kind != 0 && kind != 1))
        return fail(STRATA_ERR_INVALID_ARG, "bad expert, mat or kind");
    int rows = mat < 2 ? g.I : g.H, cols = mat < 2 ? g.H : g.I, Kp = mat < 2 ? g.H : g.Ip;
    if (row0 < 0 || nrows <= 0 || row0 + nrows > rows)
        return fail(STRATA_ERR_INVALID_ARG, "row range out of bounds");
    DeviceGuard guard(h->device);
    size_t e = expert < 0 ? (size_t)g.E : (size_t)expert;
    const uint8_t *m = h->wq + e * g.expert_bytes + mat * g.mat_bytes;
    float *d = nullptr;
    size_t n = (size_t)nrows * cols;
    cudaError_t ce = dev_malloc(&d, n * 4);
    if (ce != cudaSuccess) return fail(STRATA_ERR_OOM, "debug buffer");
    launch_debug_dequant(m, g.bits, Kp, row0, nrows, cols, kind, d, 0);
    ce = cudaGetLastError();
    if (ce == cudaSuccess) ce = cudaMemcpy(out_host, d, n * 4, cudaMemcpyDeviceToHost);
    dev_free(d);
    if (ce != cudaSuccess) return cuda_fail(ce, "debug dequant");
    return STRATA_OK;
}

strata_status strata_moe_selftest_wait(int device, int64_t budget_cycles) {
    int ndev = 0;
    cudaError_t ce = cudaGetDeviceCount(&ndev);
    if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDeviceCount");
    if (device < 0 || device >= ndev) return fail(STRATA_ERR_INVALID_ARG, "bad device");
    DeviceGuard guard(device);
    int *err = nullptr;
    if (dev_malloc(&err, 4) != cudaSuccess) return fail(STRATA_ERR_OOM, "selftest buffer");
    cudaMemset(err, 0, 4);
    launch_selftest_wait(err, budget_cycles, 0);
    int e = 0;
    ce = cudaGetLastError();
    if (ce == cudaSuccess) ce = cudaMemcpy(&e, err, 4, cudaMemcpyDeviceToHost);
    dev_free(err);
    if (ce != cudaSuccess) return cuda_fail(ce, "selftest");
    if (e) return fail(STRATA_ERR_TIMEOUT, "the bounded wait gave up as designed");
    return STRATA_OK;
}

strata_status strata_moe_expert_rows(strata_moe_t h, const void *x_dev, const int32_t *ids_dev,
                                     int n, int n_shared, int prefill, void *y_dev,
                                     void *yshared_dev, void *stream) {
    if (!h) return fail(STRATA_ERR_INVALID_ARG, "handle is NULL");
    if (n < 0 || n > h->cfg.max_tokens || n_shared < 0 || n_shared > n)
        return fail(STRATA_ERR_INVALID_ARG, "n=%d / n_shared=%d out of range (max_tokens %d)", n,
                    n_shared, h->cfg.max_tokens);
    if (n == 0) return STRATA_OK;
    if (!x_dev || !ids_dev || !y_dev || (n_shared > 0 && !yshared_dev))
        return fail(STRATA_ERR_INVALID_ARG, "NULL buffer");
    if ((((uintptr_t)x_dev) | ((uintptr_t)y_dev) | ((uintptr_t)yshared_dev)) & 15)
        return fail(STRATA_ERR_INVALID_ARG, "x and y must be 16-byte aligned");
    DeviceGuard guard(h->device);
    cudaStream_t s = (cudaStream_t)stream;
    const Geometry &g = h->geo;
    const int tile = prefill ? kUmmaTile : 8;
    ExpertWeights w{h->wq, h->wq + (size_t)g.E * g.expert_bytes};
    const int umax = max_units(n, 1, g.E, tile);
    // rows = tokens with one routed pick each (k = 1); slots: picks in
    // dispatch order, then the shared expert's rows at n + t
    __half *x16 = prefill ? reinterpret_cast<__half *>(h->xs) + (size_t)n * g.H : nullptr;
    launch_prescale(x_dev, n, g.H, h->w2eff, h->xex, x16, s);
    launch_dispatch(ids_dev, n, 1, g.E, h->cnt, h->off, h->list, h->slot, h->ds, h->units,
                    h->n_units, tile, s, h->err, n_shared);
    if (!prefill) {
        launch_gemv_gateup(g, w, h->units, h->n_units, umax, h->list, n, n, x_dev, h->xex, h->a,
                           h->err, h->budget, s, n_shared);
        launch_gemv_down(g, w, h->units, h->n_units, umax, n, h->a, (float *)h->Y, h->err,
                         h->budget, s);
    } else {
        launch_gather_rows(h->list, n, x16, h->xs, g.H, s, n, h->err, h->xex, h->slot_ex);
        cudaError_t ce = launch_umma_gateup(g, w, h->units, h->n_units, umax, 2 * n, h->xs,
                                            h->slot_ex, h->a, h->err, h->budget, s);
        if (ce == cudaSuccess)
            ce = launch_umma_down(g, w, h->units, h->n_units, umax, 2 * n, h->a, h->Y, h->err,
                                  h->budget, s);
        if (ce != cudaSuccess)
            return fail(STRATA_ERR_CUDA, "expert GEMM: %s", cudaGetErrorString(ce));
    }
    const int eb = prefill ? 2 : 4, rb = g.H * eb;
    launch_gather_rows_bytes(h->Y, h->slot, n, n, rb, y_dev, h->err, s, ids_dev);
    if (n_shared > 0) {
        cudaError_t ce = cudaMemcpyAsync(yshared_dev, (const char *)h->Y + (size_t)n * rb,
                                         (size_t)n_shared * rb, cudaMemcpyDeviceToDevice, s);
        if (ce != cudaSuccess) return cuda_fail(ce, "shared rows copy");
    }
    return check_launch("expert rows");
}

strata_status strata_moe_combine_rows(strata_moe_t h, const void *x_dev, int T,
                                      const int32_t *idx_dev, const float *w_dev,
                                      const int32_t *slot_dev, const void *y_dev, int prefill,
                                      void *out_dev, void *stream) {
    if (!h) return fail(STRATA_ERR_INVALID_ARG, "handle is NULL");
    strata_status st = check_tokens(h, T);
    if (st != STRATA_OK) return st;
    if (T == 0) return STRATA_OK;
    if (!x_dev || !idx_dev || !w_dev || !slot_dev || !y_dev || !out_dev)
        return fail(STRATA_ERR_INVALID_ARG, "NULL buffer");
    if ((((uintptr_t)x_dev) | ((uintptr_t)y_dev) | ((uintptr_t)out_dev)) & 15)
        return fail(STRATA_ERR_INVALID_ARG, "x, y and out must be 16-byte aligned");
    DeviceGuard guard(h->device);
    cudaStream_t s = (cudaStream_t)stream;
    const Geometry &g = h->geo;
    launch_prescale(x_dev, T, g.H, h->w2eff, h->xex, nullptr, s);
    launch_combine(y_dev, prefill != 0, idx_dev, w_dev, slot_dev, T, g.k, g.H, out_dev, false, s,
                   h->err, h->xex);
    return check_launch("combine rows");
}

strata_status strata_moe_debug_screen(strata_moe_t h, const void *x_dev, int T, float *a_host,
                                      float *eps_host) {
    if (!h || !x_dev || !a_host || !eps_host) return fail(STRATA_ERR_INVALID_ARG, "NULL argument");
    strata_status st = check_tokens(h, T);
    if (st != STRATA_OK) return st;
    if (h->cfg.max_tokens <= kSmallMaxT)
        return fail(STRATA_ERR_UNSUPPORTED, "the screening router needs max_tokens > %d",
                    kSmallMaxT);
    if (T == 0) return STRATA_OK;
    DeviceGuard guard(h->device);
    const Geometry &g = h->geo;
    float *a = nullptr, *eps = nullptr;
    if (dev_malloc(&a, (size_t)T * g.E * 4) != cudaSuccess ||
        dev_malloc(&eps, (size_t)T * 4) != cudaSuccess) {
        dev_free(a);
        return fail(STRATA_ERR_OOM, "debug screen buffers");
    }
    launch_to_half(x_dev, x16_of(h, T), (size_t)T * g.H, 0);
    cudaError_t ce = launch_umma_plain(h->router_split, h->router_rows, x16_of(h, T), T, g.H,
                                       h->dsplit, h->err, h->budget, 0);
    if (ce == cudaSuccess) {
        launch_screen_debug(h->dsplit, h->router_rows, x_dev, T, g.H, h->router_b, g.E,
                            h->screen_gam, h->screen_wmax, h->screen_bmax, a, eps, 0);
        ce = cudaGetLastError();
    }
    if (ce == cudaSuccess) ce = cudaMemcpy(a_host, a, (size_t)T * g.E * 4, cudaMemcpyDeviceToHost);
    if (ce == cudaSuccess) ce = cudaMemcpy(eps_host, eps, (size_t)T * 4, cudaMemcpyDeviceToHost);
    dev_free(a);
    dev_free(eps);
    if (ce != cudaSuccess) return cuda_fail(ce, "debug screen");
    return strata_moe_sync_status(h, nullptr);
}

strata_status strata_moe_debug_fail_alloc(int64_t n) {
    if (n < -1) return fail(STRATA_ERR_INVALID_ARG, "n must be >= -1");
    g_fail_at.store(n < 0 ? -1 : g_alloc_seq.load() + n);
    return STRATA_OK;
}

int64_t strata_moe_debug_live_allocs(void) { return g_live.load(); }

}  // extern "C"
