// Combine (fixed expert order), RMSNorm for the expert stack, and the
// timeout self-test kernel.
//
// Combine (layer specification; the pages: 10 routed + 1 shared expert per
// token, "Strata Runs 125B Qwen3.8-Flash-Next on a 12GB Gaming GPU at Up to 94
// Tokens/s", section "What it is"; reproducible output is an opt-in mode of
// the engine, section "Caveats"):
//   out[t] = Y_shared[t] + sum over the picks in ascending expert id of
//            w[t][j] * Y[slot[t][j]], in fp32, rounded once to bf16.
// Stack: h <- bf16(f32(h) + f32(out)); RMSNorm weight 1, eps 1e-6 with the
// sum of squares in the router's fixed order.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace strata {

// 8 consecutive columns of a staging row as fp32.
template <typename YT>
__device__ __forceinline__ void load8(const YT *p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<float>(const float *p, float (&v)[8]) {
    float4 a = *reinterpret_cast<const float4 *>(p);
    float4 b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__half>(const __half *p, float (&v)[8]) {
    uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        float2 f = __half22float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// grid: (T, column blocks of 512); 64 threads x 8 columns.  The k picks of the
// token are read in parallel and placed by rank of their expert id (ids of one
// token are distinct), then summed in that order.
constexpr int kCombineCols = 512;
constexpr int kCombineThreads = 64;

template <typename YT>
__global__ __launch_bounds__(kCombineThreads) void combine_kernel(
    const YT *__restrict__ Y, const int32_t *__restrict__ idx, const float *__restrict__ w,
    const int32_t *__restrict__ slot, int T, int k, int H, __nv_bfloat16 *out, int residual,
    int *err, const int *__restrict__ xex) {
    __shared__ int re[32], rs[32], ss[32];
    __shared__ float rw[32], sw[32];
    const int t = blockIdx.x;
    const int j = threadIdx.x;
    // the picks come from routing, long finished; the expert outputs need the
    // previous kernel
    if (j < k) {
        re[j] = __ldcg(idx + (size_t)t * k + j);
        rs[j] = __ldcg(slot + (size_t)t * k + j);
        rw[j] = __ldcg(w + (size_t)t * k + j);
    }
    grid_dependency_wait();
    __syncthreads();
    if (j < k) {
        int rank = 0;
        for (int i = 0; i < k; i++) rank += re[i] < re[j];
        ss[rank] = rs[j];
        sw[rank] = rw[j];
    }
    __syncthreads();
    const size_t Tk = (size_t)T * k;
    const int c = blockIdx.y * kCombineCols + threadIdx.x * 8;
    if (c >= H) return;
    float acc[8];
    load8<YT>(Y + (Tk + t) * H + c, acc);
#pragma unroll 4
    for (int i = 0; i < k; i++) {
        float v[8];
        if (!idx_ok(err, ss[i], Tk)) continue;
        load8<YT>(Y + (size_t)ss[i] * H + c, v);
        const float wi = sw[i];
#pragma unroll
        for (int q = 0; q < 8; q++) acc[q] = fmaf(wi, v[q], acc[q]);
    }
    if (xex) {  // Y in the token's prescaled units: undo 2^-2e (two steps stay in range)
        const int e = xex[t];
        if (e) {
            const float f = pow2f(e);
#pragma unroll
            for (int q = 0; q < 8; q++) acc[q] = acc[q] * f * f;
        }
    }
    __nv_bfloat16 *o = out + (size_t)t * H + c;
    uint4 hv = make_uint4(0, 0, 0, 0);
    if (residual) hv = *reinterpret_cast<const uint4 *>(o);
    const __nv_bfloat16 *hb = reinterpret_cast<const __nv_bfloat16 *>(&hv);
    __nv_bfloat16 ob[8];
#pragma unroll
    for (int q = 0; q < 8; q++) {
        __nv_bfloat16 yb = __float2bfloat16_rn(acc[q]);
        ob[q] = residual ? __float2bfloat16_rn(__fadd_rn(__bfloat162float(hb[q]), __bfloat162float(yb)))
                         : yb;
    }
    *reinterpret_cast<uint4 *>(o) = *reinterpret_cast<uint4 *>(ob);
}

void launch_combine(const void *Y, bool y_half, const int32_t *idx, const float *w,
                    const int32_t *slot, int T, int k, int H, void *out, bool residual,
                    cudaStream_t s, int *err, const int *xex) {
    auto o = reinterpret_cast<__nv_bfloat16 *>(out);
    dim3 grid(T, (H + kCombineCols - 1) / kCombineCols);
    if (y_half)
        launch_pdl(combine_kernel<__half>, grid, dim3(kCombineThreads), 0, s,
                   reinterpret_cast<const __half *>(Y), idx, w, slot, T, k, H, o,
                   residual ? 1 : 0, err, xex);
    else
        launch_pdl(combine_kernel<float>, grid, dim3(kCombineThreads), 0, s,
                   reinterpret_cast<const float *>(Y), idx, w, slot, T, k, H, o,
                   residual ? 1 : 0, err, xex);
}

// ------------------------------------------------------------------ RMSNorm
// One warp per token; lane l sums squares over i = l, l+32, ... with fma,
// then the halving tree; r = 1/sqrtf(ss/H + 1e-6f) (IEEE division and square
// root); xn = bf16(h * r).
__global__ __launch_bounds__(256) void rmsnorm_kernel(const __nv_bfloat16 *__restrict__ h,
                                                      __nv_bfloat16 *__restrict__ xn, int T,
                                                      int H) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    if (t >= T) return;
    const __nv_bfloat16 *row = h + (size_t)t * H;
    float p = 0.0f;
    for (int i = lane; i < H; i += 32) {
        float v = __bfloat162float(row[i]);
        p = fmaf(v, v, p);
    }
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) p = __fadd_rn(p, __shfl_down_sync(0xffffffffu, p, s));
    float ss = __shfl_sync(0xffffffffu, p, 0);
    float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)H), 1e-6f)));
    for (int i = lane; i < H; i += 32)
        xn[(size_t)t * H + i] = __float2bfloat16_rn(__fmul_rn(__bfloat162float(row[i]), r));
}

void launch_rmsnorm(const void *h, void *xn, int T, int H, cudaStream_t s) {
    rmsnorm_kernel<<<(T + 7) / 8, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16 *>(h),
                                               reinterpret_cast<__nv_bfloat16 *>(xn), T, H);
}

// ------------------------------------------------------------------ self-test
// A barrier that nothing completes: the bounded wait must give up and flag
// the error word.  No copy is in flight, so there is nothing to drain.
__global__ void selftest_wait_kernel(int *err, long long budget) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_wait(&bar, 0, budget, err);
    }
}

void launch_selftest_wait(int *err, long long budget, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(err, budget);
}

cudaError_t init_kernel_attributes() {
    // one set-up per device; create and the allocation-free routing may call
    // this from different host threads at once
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && done[dev]) return cudaSuccess;
    int max_smem = 0;
    e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    if ((e = route_init_attributes(max_smem)) != cudaSuccess) return e;
    if ((e = gemv_init_attributes(max_smem)) != cudaSuccess) return e;
    if ((e = umma_init_attributes(max_smem)) != cudaSuccess) return e;
    if ((e = fused_init_attributes(max_smem)) != cudaSuccess) return e;
    if (dev < 64) done[dev] = true;
    return cudaSuccess;
}

}  // namespace strata
