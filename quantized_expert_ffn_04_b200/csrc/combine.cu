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
#include "common.cuh"
#include "internal.h"

namespace strata {

template <typename YT>
__device__ __forceinline__ float4 load4(const YT *p);
template <>
__device__ __forceinline__ float4 load4<float>(const float *p) {
    return *reinterpret_cast<const float4 *>(p);
}
template <>
__device__ __forceinline__ float4 load4<__half>(const __half *p) {
    uint2 v = *reinterpret_cast<const uint2 *>(p);
    float2 a = __half22float2(*reinterpret_cast<__half2 *>(&v.x));
    float2 b = __half22float2(*reinterpret_cast<__half2 *>(&v.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

template <typename YT>
__global__ __launch_bounds__(256) void combine_kernel(const YT *__restrict__ Y,
                                                      const int32_t *__restrict__ idx,
                                                      const float *__restrict__ w,
                                                      const int32_t *__restrict__ slot, int T,
                                                      int k, int H, __nv_bfloat16 *out,
                                                      int residual) {
    __shared__ int se[32], ss[32];
    __shared__ float sw[32];
    const int t = blockIdx.x;
    if (threadIdx.x == 0) {
        // insertion sort of the k picks by expert id
        for (int j = 0; j < k; j++) {
            int e = idx[(size_t)t * k + j], s = slot[(size_t)t * k + j];
            float wj = w[(size_t)t * k + j];
            int p = j;
            while (p > 0 && se[p - 1] > e) {
                se[p] = se[p - 1];
                ss[p] = ss[p - 1];
                sw[p] = sw[p - 1];
                p--;
            }
            se[p] = e;
            ss[p] = s;
            sw[p] = wj;
        }
    }
    __syncthreads();
    const size_t Tk = (size_t)T * k;
    for (int c = threadIdx.x * 4; c < H; c += blockDim.x * 4) {
        float4 acc = load4<YT>(Y + (Tk + t) * H + c);
        for (int j = 0; j < k; j++) {
            float4 v = load4<YT>(Y + (size_t)ss[j] * H + c);
            float wj = sw[j];
            acc.x = fmaf(wj, v.x, acc.x);
            acc.y = fmaf(wj, v.y, acc.y);
            acc.z = fmaf(wj, v.z, acc.z);
            acc.w = fmaf(wj, v.w, acc.w);
        }
        __nv_bfloat16 *o = out + (size_t)t * H + c;
        float r[4] = {acc.x, acc.y, acc.z, acc.w};
        __nv_bfloat16 ob[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            __nv_bfloat16 yb = __float2bfloat16_rn(r[i]);
            if (residual)
                ob[i] = __float2bfloat16_rn(__fadd_rn(__bfloat162float(o[i]), __bfloat162float(yb)));
            else
                ob[i] = yb;
        }
        *reinterpret_cast<uint2 *>(o) = *reinterpret_cast<uint2 *>(ob);
    }
}

void launch_combine(const void *Y, bool y_half, const int32_t *idx, const float *w,
                    const int32_t *slot, int T, int k, int H, void *out, bool residual,
                    cudaStream_t s) {
    auto o = reinterpret_cast<__nv_bfloat16 *>(out);
    if (y_half)
        combine_kernel<__half><<<T, 256, 0, s>>>(reinterpret_cast<const __half *>(Y), idx, w, slot,
                                                 T, k, H, o, residual ? 1 : 0);
    else
        combine_kernel<float><<<T, 256, 0, s>>>(reinterpret_cast<const float *>(Y), idx, w, slot,
                                                T, k, H, o, residual ? 1 : 0);
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
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && done[dev]) return cudaSuccess;
    int max_smem = 0;
    e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    if ((e = route_init_attributes(max_smem)) != cudaSuccess) return e;
    if ((e = gemv_init_attributes(max_smem)) != cudaSuccess) return e;
    if ((e = umma_init_attributes(max_smem)) != cudaSuccess) return e;
    if (dev < 64) done[dev] = true;
    return cudaSuccess;
}

}  // namespace strata
