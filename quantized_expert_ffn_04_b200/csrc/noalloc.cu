// Routing without any device allocation: strata_moe_route_noalloc.
//
// Some callers cannot call cudaMalloc: code that runs inside another
// framework's memory pool (every byte must come from the host framework's
// allocator, and a stray cudaMalloc bypasses its accounting and can fail once
// the pool has reserved the device), code on a hard memory budget that must
// not grow its footprint per call, and code paths that must not synchronise
// (cudaMalloc/cudaFree can implicitly synchronise the device).  This entry
// point takes the caller's buffers for inputs and outputs and keeps its own
// intermediates (logits, dispatch counters, work units) in one statically
// sized device array that every GPU loading this library holds until exit.
//
// The computation is the same routing as strata_moe_route (fixed-order fp32
// logits, top-k with the lower expert id winning a tie, renormalised weights,
// deterministic dispatch); only the router weight's layout differs: the
// caller passes the plain row-major fp32 [E][H] matrix.
#include <mutex>

#include "../../include/strata_moe.h"
#include "common.cuh"
#include "internal.h"

namespace strata {

constexpr int kNoAllocMaxT = 64;
constexpr int kNoAllocMaxE = 1024;
constexpr int kNoAllocMaxK = 32;
constexpr int kNoAllocMaxH = 6144;

// Scratch layout (bytes, each piece 256-aligned).
constexpr size_t kNaLogits = (size_t)kNoAllocMaxT * kNoAllocMaxE * 4;
constexpr size_t kNaSlot = (size_t)kNoAllocMaxT * kNoAllocMaxK * 4;
constexpr size_t kNaList = kNaSlot;
constexpr size_t kNaOff = ((size_t)kNoAllocMaxE + 1) * 4 + 252;
constexpr size_t kNaCnt = (size_t)kNoAllocMaxE * 4;
constexpr size_t kNaDisp = (size_t)kNoAllocMaxE * 4 + 8 * (size_t)kNoAllocMaxE * 4 +
                           8 * (size_t)kNoAllocMaxE * 2 + 256;  // one 256-token chunk
constexpr size_t kNaUnits = 2400 * 16;                           // >= max_units(64, 32, 1024, 8)
constexpr size_t kNaTotal = kNaLogits + kNaSlot + kNaList + kNaOff + kNaCnt + kNaDisp + kNaUnits +
                            256;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNaTotal];

// Router over the plain [E][H] weight: warp per expert, lane l accumulates
// i = l, l+32, ... in ascending order with fma (the fixed order), then the
// halving tree, then + bias.  Tokens are staged 8 at a time as bf16.
__global__ __launch_bounds__(128) void router_plain_kernel(const __nv_bfloat16 *__restrict__ x,
                                                           int T, int H,
                                                           const float *__restrict__ W,
                                                           const float *__restrict__ bias, int E,
                                                           float *__restrict__ logits) {
    extern __shared__ __align__(16) __nv_bfloat16 xs[];  // [8][H]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 4 + warp;
    for (int t0 = 0; t0 < T; t0 += 8) {
        __syncthreads();
        for (int i = threadIdx.x; i < 8 * H / 8; i += blockDim.x) {
            int tt = i / (H / 8), c = (i % (H / 8)) * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (t0 + tt < T) v = *reinterpret_cast<const uint4 *>(x + (size_t)(t0 + tt) * H + c);
            *reinterpret_cast<uint4 *>(xs + tt * H + c) = v;
        }
        __syncthreads();
        if (e >= E) continue;
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; j++) acc[j] = 0.0f;
        const float *wr = W + (size_t)e * H;
        for (int i = lane; i < H; i += 32) {
            float w = __ldg(wr + i);
#pragma unroll
            for (int j = 0; j < 8; j++) acc[j] = fmaf(__bfloat162float(xs[j * H + i]), w, acc[j]);
        }
#pragma unroll
        for (int j = 0; j < 8; j++) {
            float v = acc[j];
#pragma unroll
            for (int s = 16; s >= 1; s >>= 1) v = __fadd_rn(v, __shfl_down_sync(0xffffffffu, v, s));
            if (lane == 0 && t0 + j < T)
                logits[(size_t)(t0 + j) * E + e] = bias ? __fadd_rn(v, bias[e]) : v;
        }
    }
}

// Device address of the scratch array, looked up once per device.
static std::mutex g_na_mu;
static void *g_na_ptr[64];
static bool g_na_ready[64];

static cudaError_t noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_na_mu);
    if (!g_na_ready[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        int max_smem = 0;
        e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return e;
        e = allow_max_dyn_smem(router_plain_kernel, max_smem);
        if (e != cudaSuccess) return e;
        e = init_kernel_attributes();  // the top-k and dispatch kernels' limits
        if (e != cudaSuccess) return e;
        g_na_ptr[dev] = p;
        g_na_ready[dev] = true;
    }
    *out = g_na_ptr[dev];
    return cudaSuccess;
}

}  // namespace strata

using namespace strata;

extern "C" strata_status strata_moe_route_noalloc(const void *x_dev, int T, int H,
                                                  const float *router_w_dev,
                                                  const float *router_b_dev, int E, int k,
                                                  int32_t *idx_dev, float *w_dev,
                                                  int32_t *offsets_dev, int32_t *list_dev,
                                                  void *stream) {
    if (T < 0 || T > kNoAllocMaxT || E < 1 || E > kNoAllocMaxE || k < 1 || k > E ||
        k > kNoAllocMaxK || H < 128 || H % 128 || H > kNoAllocMaxH) {
        set_error_message(
            "strata_moe_route_noalloc: size beyond its static scratch limits (need 0 <= T <= 64, "
            "1 <= E <= 1024, 1 <= k <= min(E, 32), H a multiple of 128 in [128, 6144])");
        return STRATA_ERR_INVALID_ARG;
    }
    if (T == 0) return STRATA_OK;
    if (!x_dev || !router_w_dev || !idx_dev || !w_dev || (((uintptr_t)x_dev) & 15)) {
        set_error_message("strata_moe_route_noalloc: NULL or misaligned device pointer");
        return STRATA_ERR_INVALID_ARG;
    }
    void *base = nullptr;
    if (noalloc_scratch(&base) != cudaSuccess) {
        set_error_message("strata_moe_route_noalloc: scratch address lookup failed");
        return STRATA_ERR_CUDA;
    }
    cudaStream_t s = (cudaStream_t)stream;
    char *p = static_cast<char *>(base);
    float *logits = reinterpret_cast<float *>(p);
    p += kNaLogits;
    int32_t *slot = reinterpret_cast<int32_t *>(p);
    p += kNaSlot;
    int32_t *list = list_dev ? list_dev : reinterpret_cast<int32_t *>(p);
    p += kNaList;
    int32_t *off = offsets_dev ? offsets_dev : reinterpret_cast<int32_t *>(p);
    p += kNaOff;
    int32_t *cnt = reinterpret_cast<int32_t *>(p);
    p += kNaCnt;
    DispatchScratch ds;
    dispatch_scratch_carve(p, T, E, &ds);
    p += kNaDisp;
    int4 *units = reinterpret_cast<int4 *>(p);
    p += kNaUnits;
    int *n_units = reinterpret_cast<int *>(p);

    size_t smem = (size_t)8 * H * 2;
    router_plain_kernel<<<(E + 3) / 4, 128, smem, s>>>(
        reinterpret_cast<const __nv_bfloat16 *>(x_dev), T, H, router_w_dev, router_b_dev, E,
        logits);
    launch_topk(logits, T, E, k, idx_dev, w_dev, s);
    launch_dispatch(idx_dev, T, k, E, cnt, off, list, slot, ds, units, n_units, 8, s);
    if (cudaGetLastError() != cudaSuccess) {
        set_error_message("strata_moe_route_noalloc: kernel launch failed");
        return STRATA_ERR_CUDA;
    }
    return STRATA_OK;
}
