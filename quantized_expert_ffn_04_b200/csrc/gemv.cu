// Decode expert kernels (T <= 64): bandwidth-bound grouped GEMV over the
// quantised experts, gate/up with the SwiGLU epilogue, then down.
//
// Expert (layer specification): g = Wg x, u = Wu x, a = silu(g) * u,
// y = Wd a, with w = d*(q-c) from the block-32 codes.  The pages: 10 routed +
// 1 shared expert per token ("Strata Runs 125B Qwen3.8-Flash-Next on a 12GB
// Gaming GPU at Up to 94 Tokens/s", section "What it is"), 2-3 bit builds
// ("Caveats").
//
// Work unit: (expert, up to 8 tokens of that expert, 16-row slab).  One CTA =
// 4 warps.  Each warp's share of the packed weights (contiguous in the GPU
// layout) is pulled into shared memory with one or two bulk-async copies that
// are all issued at kernel start, so every byte the CTA needs is in flight at
// once.  The codes are turned into exact small odd integers 2q-(2^bits-1) in
// registers (two per 32-bit lane pair: shift, mask/or against a magic
// exponent, one packed subtract), the tensor core reduces 16x16 blocks against
// the staged token rows (mma.sync m16n8k16, fp32 accumulate), and each 32-wide
// block's partial is scaled by its fp16 scale in fp32.  The tensor core is
// used only as the in-warp reduction: products are exact (small integer x
// bf16/fp16), so the result is the exact dot product up to fp32 rounding.
#include "common.cuh"
#include "internal.h"

namespace strata {

constexpr int kTile = 8;  // tokens per unit (mma N)

__device__ __forceinline__ uint32_t comp4(const uint4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// One 32-wide block: D = A_blk(16x32) * B(32x8) with A the exact integers,
// two mma k-steps.  lo/hi: the lane's code words for this block.
template <bool kBf16, int kBits>
__device__ __forceinline__ void block_mma(float (&d)[4], uint32_t lo, uint32_t hi, int hshift,
                                          uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
    uint32_t a[4];
    const float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 4; r++) a[r] = dq_pair<kBf16, kBits>(lo, hi, r, hshift);
    if (kBf16) mma_bf16(d, a, b0, b1, z); else mma_f16(d, a, b0, b1, z);
#pragma unroll
    for (int r = 0; r < 4; r++) a[r] = dq_pair<kBf16, kBits>(lo, hi, 4 + r, hshift);
    if (kBf16) mma_bf16(d, a, b2, b3, d); else mma_f16(d, a, b2, b3, d);
}

// Accumulate one 16 x (ns*128) slab of a matrix whose units sit in smem at
// `w` against B rows staged at `xb` (row pitch `pitch` elements).
template <bool kBf16, int kBits>
__device__ __forceinline__ void slab_dot(float (&acc)[4], const uint8_t *w, int ns,
                                         const uint16_t *xb, int pitch, int lane) {
    constexpr int UB = unit_bytes(kBits);
    constexpr int SOFF = kLoBytes + (kBits == 3 ? kHiBytes : 0);
    for (int sg = 0; sg < ns; sg++) {
        const uint8_t *un = w + sg * UB;
        uint4 lo = *reinterpret_cast<const uint4 *>(un + lane * 16);
        uint2 hi = make_uint2(0, 0);
        if (kBits == 3) hi = *reinterpret_cast<const uint2 *>(un + kLoBytes + lane * 8);
        uint32_t sc = *reinterpret_cast<const uint32_t *>(un + SOFF + lane * 4);
#pragma unroll
        for (int blk = 0; blk < 4; blk++) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(b0, b1, b2, b3, xb + (lane & 7) * pitch + sg * 128 + blk * 32 + (lane >> 3) * 8);
            uint32_t s2 = __shfl_sync(0xffffffffu, sc, (lane & ~3) | blk);
            float d[4];
            block_mma<kBf16, kBits>(d, comp4(lo, blk), blk < 2 ? hi.x : hi.y, 8 * (blk & 1), b0, b1,
                                    b2, b3);
            float2 s = __half22float2(*reinterpret_cast<__half2 *>(&s2));
            acc[0] = fmaf(s.x, d[0], acc[0]);
            acc[1] = fmaf(s.x, d[1], acc[1]);
            acc[2] = fmaf(s.y, d[2], acc[2]);
            acc[3] = fmaf(s.y, d[3], acc[3]);
        }
    }
}

// ------------------------------------------------------------- gate / up
template <int kBits>
__global__ __launch_bounds__(128) void gemv_gateup_kernel(
    const uint8_t *__restrict__ routed, const uint8_t *__restrict__ shared, size_t expert_bytes,
    size_t mat_bytes, const int4 *__restrict__ units, const int *__restrict__ n_units,
    const int32_t *__restrict__ list, int Tk, int E, const __nv_bfloat16 *__restrict__ x, int H,
    int Ip, __half *__restrict__ a_out, int *err, long long budget) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ float red[4][32][8];
    constexpr int UB = unit_bytes(kBits);
    const int nslab = Ip / kSlabRows;
    const int u = blockIdx.x / nslab, slab = blockIdx.x % nslab;
    if (u >= *n_units) return;
    const int4 un = units[u];
    const int e = un.x, slot0 = un.y, n = un.z;
    const uint8_t *wg = e == E ? shared : routed + (size_t)e * expert_bytes;
    const uint8_t *wu = wg + mat_bytes;
    const int nseg = H / kSegCols;
    const int nsw = (nseg + 3) / 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sa = warp * nseg / 4, sb = (warp + 1) * nseg / 4, ns = sb - sa;
    const int wbytes = 2 * nsw * UB;
    const int pitch = nsw * kSegCols + 8;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    uint8_t *wbuf = smem + 128 + warp * (wbytes + kTile * pitch * 2);
    uint16_t *xb = reinterpret_cast<uint16_t *>(wbuf + wbytes);

    if (lane == 0) {
        mbar_init(&bars[warp], 1);
        fence_mbar_init();
        if (ns > 0) {
            uint32_t bytes = (uint32_t)(ns * UB);
            size_t off = ((size_t)slab * nseg + sa) * UB;
            mbar_arrive_expect_tx(&bars[warp], 2 * bytes);
            bulk_g2s(wbuf, wg + off, bytes, &bars[warp]);
            bulk_g2s(wbuf + nsw * UB, wu + off, bytes, &bars[warp]);
        } else {
            mbar_arrive(&bars[warp]);
        }
    }
    // stage the unit's token rows (this warp's column range), zero the rest
    for (int j = 0; j < kTile; j++) {
        uint4 *dst = reinterpret_cast<uint4 *>(xb + j * pitch);
        if (j < n) {
            int slot = slot0 + j;
            int t = slot < Tk ? list[slot] : slot - Tk;
            const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * H + sa * kSegCols);
            for (int i = lane; i < ns * 16; i += 32) dst[i] = __ldg(src + i);
        } else {
            for (int i = lane; i < ns * 16; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
        }
    }
    __syncwarp();
    float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
    if (mbar_wait(&bars[warp], 0, budget, err)) {
        slab_dot<true, kBits>(accg, wbuf, ns, xb, pitch, lane);
        slab_dot<true, kBits>(accu, wbuf + nsw * UB, ns, xb, pitch, lane);
    } else {
        mbar_drain(&bars[warp], 0);
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
        red[warp][lane][i] = accg[i];
        red[warp][lane][4 + i] = accu[i];
    }
    __syncthreads();
    if (warp == 0) {
        const int g = lane >> 2, c = lane & 3;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            float gs = ((red[0][lane][i] + red[1][lane][i]) + red[2][lane][i]) + red[3][lane][i];
            float us = ((red[0][lane][4 + i] + red[1][lane][4 + i]) + red[2][lane][4 + i]) +
                       red[3][lane][4 + i];
            gs *= 0.5f;  // the integers are 2(q - c): one factor 2 out
            us *= 0.5f;
            float a = gs / (1.0f + expf(-gs)) * us;
            int tok = 2 * c + (i & 1);
            int row = slab * kSlabRows + g + 8 * (i >> 1);
            if (tok < n) a_out[(size_t)(slot0 + tok) * Ip + row] = __float2half_rn(a);
        }
    }
}

// ------------------------------------------------------------------ down
// CTA = 4 warps x one 16-row slab each (64 output rows), full K = Ip.
template <int kBits>
__global__ __launch_bounds__(128) void gemv_down_kernel(
    const uint8_t *__restrict__ routed, const uint8_t *__restrict__ shared, size_t expert_bytes,
    size_t mat_bytes, const int4 *__restrict__ units, const int *__restrict__ n_units, int E,
    const __half *__restrict__ a, int H, int Ip, float *__restrict__ Y, int *err,
    long long budget) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int UB = unit_bytes(kBits);
    const int ngrp = H / 64;
    const int u = blockIdx.x / ngrp, grp = blockIdx.x % ngrp;
    if (u >= *n_units) return;
    const int4 un = units[u];
    const int e = un.x, slot0 = un.y, n = un.z;
    const uint8_t *wd = (e == E ? shared : routed + (size_t)e * expert_bytes) + 2 * mat_bytes;
    const int nseg = Ip / kSegCols;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slab = grp * 4 + warp;
    const int pitch = Ip + 8;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    uint8_t *wbuf = smem + 128 + warp * nseg * UB;
    uint16_t *ab = reinterpret_cast<uint16_t *>(smem + 128 + 4 * nseg * UB);

    if (lane == 0) {
        mbar_init(&bars[warp], 1);
        fence_mbar_init();
        uint32_t bytes = (uint32_t)(nseg * UB);
        mbar_arrive_expect_tx(&bars[warp], bytes);
        bulk_g2s(wbuf, wd + (size_t)slab * nseg * UB, bytes, &bars[warp]);
    }
    for (int j = 0; j < kTile; j++) {
        uint4 *dst = reinterpret_cast<uint4 *>(ab + j * pitch);
        const int nv = Ip / 8;
        if (j < n) {
            const uint4 *src = reinterpret_cast<const uint4 *>(a + (size_t)(slot0 + j) * Ip);
            for (int i = threadIdx.x; i < nv; i += blockDim.x) dst[i] = src[i];
        } else {
            for (int i = threadIdx.x; i < nv; i += blockDim.x) dst[i] = make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (mbar_wait(&bars[warp], 0, budget, err)) {
        slab_dot<false, kBits>(acc, wbuf, nseg, ab, pitch, lane);
    } else {
        mbar_drain(&bars[warp], 0);
    }
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        int tok = 2 * c + (i & 1);
        int row = slab * kSlabRows + g + 8 * (i >> 1);
        if (tok < n) Y[(size_t)(slot0 + tok) * H + row] = 0.5f * acc[i];
    }
}

static size_t gateup_smem(const Geometry &g) {
    int nseg = g.H / kSegCols, nsw = (nseg + 3) / 4;
    return 128 + 4 * (size_t)(2 * nsw * g.ub + kTile * (nsw * kSegCols + 8) * 2);
}

static size_t down_smem(const Geometry &g) {
    return 128 + 4 * (size_t)g.nseg_i * g.ub + (size_t)kTile * (g.Ip + 8) * 2;
}

void launch_gemv_gateup(const Geometry &g, const ExpertWeights &w, const int4 *units,
                        const int *n_units, int units_max, const int32_t *list, int Tk,
                        const void *x, void *a_out, int *err, long long budget, cudaStream_t s) {
    size_t smem = gateup_smem(g);
    dim3 grid((unsigned)((size_t)units_max * (g.Ip / kSlabRows)));
    auto xb = reinterpret_cast<const __nv_bfloat16 *>(x);
    auto ao = reinterpret_cast<__half *>(a_out);
    if (g.bits == 2) {
        gemv_gateup_kernel<2><<<grid, 128, smem, s>>>(w.routed, w.shared, g.expert_bytes,
                                                      g.mat_bytes, units, n_units, list, Tk, g.E,
                                                      xb, g.H, g.Ip, ao, err, budget);
    } else {
        gemv_gateup_kernel<3><<<grid, 128, smem, s>>>(w.routed, w.shared, g.expert_bytes,
                                                      g.mat_bytes, units, n_units, list, Tk, g.E,
                                                      xb, g.H, g.Ip, ao, err, budget);
    }
}

void launch_gemv_down(const Geometry &g, const ExpertWeights &w, const int4 *units,
                      const int *n_units, int units_max, const void *a, float *Y, int *err,
                      long long budget, cudaStream_t s) {
    size_t smem = down_smem(g);
    dim3 grid((unsigned)((size_t)units_max * (g.H / 64)));
    auto ap = reinterpret_cast<const __half *>(a);
    if (g.bits == 2) {
        gemv_down_kernel<2><<<grid, 128, smem, s>>>(w.routed, w.shared, g.expert_bytes,
                                                    g.mat_bytes, units, n_units, g.E, ap, g.H,
                                                    g.Ip, Y, err, budget);
    } else {
        gemv_down_kernel<3><<<grid, 128, smem, s>>>(w.routed, w.shared, g.expert_bytes,
                                                    g.mat_bytes, units, n_units, g.E, ap, g.H,
                                                    g.Ip, Y, err, budget);
    }
}

cudaError_t gemv_init_attributes(int max_smem) {
    cudaError_t e;
    if ((e = allow_max_dyn_smem(gemv_gateup_kernel<2>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(gemv_gateup_kernel<3>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(gemv_down_kernel<2>, max_smem)) != cudaSuccess) return e;
    return allow_max_dyn_smem(gemv_down_kernel<3>, max_smem);
}

}  // namespace strata
