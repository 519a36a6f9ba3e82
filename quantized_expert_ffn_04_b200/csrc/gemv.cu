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
// exponent, one packed fp16 subtract), the tensor core reduces 16x16 blocks
// against the staged token rows (mma.sync m16n8k16, fp16 operands, fp32
// accumulate), and each 32-wide block's partial is scaled by its fp16 scale in
// fp32.  The tensor core is used only as the in-warp reduction: products are
// exact (small integer x fp16), so the result is the dot product up to fp32
// rounding.  Token rows (bf16) are staged as fp16, which holds every bf16
// value of magnitude 2^-14 .. 65504 exactly; only as many rows are staged as
// the batch can put in one unit, so small batches fit more CTAs per SM.
#include "common.cuh"
#include "internal.h"

namespace strata {

constexpr int kTile = 8;  // tokens per unit (mma N)

// Accumulate one 16 x (ns*128) slab of a matrix whose units sit in smem at
// `w` against the fp16 token rows staged at `xb` (row pitch `pitch` elements,
// `xrows` rows staged; the other mma columns read row 0 and are ignored).
template <int kBits>
__device__ __forceinline__ void slab_dot(float (&acc)[4], const uint8_t *w, int ns,
                                         const uint16_t *xb, int pitch, int xrows, int lane) {
    constexpr int UB = unit_bytes(kBits);
    constexpr int SOFF = scale_off(kBits);
    const uint16_t *xrow = xb + ((lane & 7) < xrows ? (lane & 7) : 0) * pitch;
    for (int sg = 0; sg < ns; sg++) {
        const uint8_t *un = w + sg * UB;
        uint4 lo;
        if (kBits == 1) {  // two words, two blocks each (the odd block one bit higher)
            const uint2 v = *reinterpret_cast<const uint2 *>(un + lane * 8);
            lo = make_uint4(v.x, v.x >> 1, v.y, v.y >> 1);
        } else {
            lo = *reinterpret_cast<const uint4 *>(un + lane * 16);
        }
        uint2 hi = make_uint2(0, 0);
        if (kBits == 3) hi = *reinterpret_cast<const uint2 *>(un + kLoBytes + lane * 8);
        uint32_t sc = *reinterpret_cast<const uint32_t *>(un + SOFF + lane * 4);
#pragma unroll
        for (int blk = 0; blk < 4; blk++) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(b0, b1, b2, b3, xrow + sg * 128 + blk * 32 + (lane >> 3) * 8);
            uint32_t s2 = __shfl_sync(0xffffffffu, sc, (lane & ~3) | blk);
            float d[4];
            if (kBits <= 2)
                block_mma2<kBits>(d, comp4(lo, blk), b0, b1, b2, b3);
            else
                block_mma<kBits>(d, comp4(lo, blk), blk < 2 ? hi.x : hi.y, 8 * (blk & 1), b0, b1,
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
    const int32_t *__restrict__ list, int Tk, int T, int E, const __nv_bfloat16 *__restrict__ x,
    const int *__restrict__ xex, int H, int Ip, int xrows, int nsh, int srows,
    __half *__restrict__ a_out, int *err, long long budget) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ float red[4][32][8];
    constexpr int UB = unit_bytes(kBits);
    const int nslab = Ip / kSlabRows;
    const int u = blockIdx.x / nslab, slab = blockIdx.x % nslab;
    // The first nsh units are the shared expert's, fixed before routing: those
    // CTAs fetch weights and tokens while the routing kernel still runs.  The
    // others wait for routing (programmatic dependent launch).
    // Routed CTAs signal the down kernel only after their wait, i.e. once
    // routing is complete, so the down kernel may read the unit list early;
    // shared CTAs signal by exiting.
    int4 un;
    if (u < nsh) {
        const int n0 = srows - u * kTile;  // the first srows tokens take the shared expert
        un = make_int4(E, Tk + u * kTile, n0 < kTile ? n0 : kTile, 0);
    } else {
        grid_dependency_wait();
        grid_launch_dependents();
        if (u >= *n_units) return;
        un = units[u];
    }
    const int e = un.x, slot0 = un.y, n = un.z;
    // lane j < n: token row j of the unit and its prescale factor 2^-xex
    // (the exponents come from a kernel that completed before routing began)
    int my_t = 0, my_ex = 0;
    {
        const int ln = threadIdx.x & 31;
        if (ln < n) {
            const int sl = slot0 + ln;
            my_t = sl < Tk ? list[sl] : sl - Tk;
            my_ex = xex[my_t];
        }
    }
    const uint8_t *wg = e == E ? shared : routed + (size_t)e * expert_bytes;
    const uint8_t *wu = wg + mat_bytes;
    const int nseg = H / kSegCols;
    const int nsw = (nseg + 3) / 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sa = warp * nseg / 4, sb = (warp + 1) * nseg / 4, ns = sb - sa;
    const int wbytes = 2 * nsw * UB;
    const int pitch = nsw * kSegCols + 8;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    uint8_t *wbuf = smem + 128 + warp * (wbytes + xrows * pitch * 2);
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
    // stage the unit's token rows (this warp's column range) as fp16, zero the
    // rest; each lane requests a batch of 8 chunks before storing any
    {
        const int per_row = ns * 16, nchunk = xrows * per_row;
        for (int base = 0; base < nchunk; base += 8 * 32) {
            uint4 v[8];
#pragma unroll
            for (int b = 0; b < 8; b++) {
                const int idx = base + b * 32 + lane;
                const int j = idx / per_row, i = idx % per_row;
                const int t = __shfl_sync(0xffffffffu, my_t, j & 31);
                v[b] = make_uint4(0, 0, 0, 0);
                if (idx < nchunk && j < n)
                    v[b] = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)t * H +
                                                                 sa * kSegCols) + i);
            }
#pragma unroll
            for (int b = 0; b < 8; b++) {
                // every lane takes part in the shuffle (no lane leaves the
                // loop early), then only the lanes with a chunk store it
                const int idx = base + b * 32 + lane;
                const int j = idx / per_row, i = idx % per_row;
                const float sc = pow2f(-__shfl_sync(0xffffffffu, my_ex, j & 31));
                if (idx < nchunk) {
                    const __nv_bfloat162 *bb = reinterpret_cast<const __nv_bfloat162 *>(&v[b]);
                    uint4 o;
                    __half2 *h = reinterpret_cast<__half2 *>(&o);
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        const float2 f = __bfloat1622float2(bb[q]);
                        h[q] = __floats2half2_rn(f.x * sc, f.y * sc);
                    }
                    reinterpret_cast<uint4 *>(xb + j * pitch)[i] = o;
                }
            }
        }
    }
    __syncwarp();
    float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
    if (mbar_wait(&bars[warp], 0, budget, err)) {
        slab_dot<kBits>(accg, wbuf, ns, xb, pitch, xrows, lane);
        slab_dot<kBits>(accu, wbuf + nsw * UB, ns, xb, pitch, xrows, lane);
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
            int tok = 2 * c + (i & 1);
            const float a = swiglu_ps(gs, us, __shfl_sync(0xffffffffu, my_ex, tok));
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
    const __half *__restrict__ a, int H, int Ip, int xrows, float *__restrict__ Y, int *err,
    long long budget) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int UB = unit_bytes(kBits);
    const int ngrp = H / 64;
    const int u = blockIdx.x / ngrp, grp = blockIdx.x % ngrp;
    grid_launch_dependents();
    // Routing finished before the gate/up kernel let this grid start, so the
    // unit list is final; read it past L1 and fetch the weights before waiting
    // for gate/up's activations.
    if (u >= __ldcg(n_units)) return;
    const int4 un = __ldcg(units + u);
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
    grid_dependency_wait();  // gate/up's activations
    {
        const int nv = Ip / 8, nchunk = xrows * nv;
        for (int base = 0; base < nchunk; base += 8 * 128) {
            uint4 v[8];
#pragma unroll
            for (int b = 0; b < 8; b++) {
                const int idx = base + b * 128 + threadIdx.x;
                v[b] = make_uint4(0, 0, 0, 0);
                if (idx < nchunk && idx / nv < n)
                    v[b] = __ldcg(reinterpret_cast<const uint4 *>(a + (size_t)(slot0 + idx / nv) * Ip) +
                                  idx % nv);
            }
#pragma unroll
            for (int b = 0; b < 8; b++) {
                const int idx = base + b * 128 + threadIdx.x;
                if (idx >= nchunk) break;
                reinterpret_cast<uint4 *>(ab + (idx / nv) * pitch)[idx % nv] = v[b];
            }
        }
    }
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (mbar_wait(&bars[warp], 0, budget, err)) {
        slab_dot<kBits>(acc, wbuf, nseg, ab, pitch, xrows, lane);
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

static int staged_rows(int T) { return T < kTile ? (T < 1 ? 1 : T) : kTile; }

static size_t gateup_smem(const Geometry &g, int xrows) {
    int nseg = g.H / kSegCols, nsw = (nseg + 3) / 4;
    return 128 + 4 * (size_t)(2 * nsw * g.ub + xrows * (nsw * kSegCols + 8) * 2);
}

static size_t down_smem(const Geometry &g, int xrows) {
    return 128 + 4 * (size_t)g.nseg_i * g.ub + (size_t)xrows * (g.Ip + 8) * 2;
}

void launch_gemv_gateup(const Geometry &g, const ExpertWeights &w, const int4 *units,
                        const int *n_units, int units_max, const int32_t *list, int Tk, int T,
                        const void *x, const int *xex, void *a_out, int *err, long long budget,
                        cudaStream_t s, int shared_rows) {
    const int xrows = staged_rows(T);
    const int nsh = ((shared_rows < 0 ? T : shared_rows) + kTile - 1) / kTile;
    size_t smem = gateup_smem(g, xrows);
    dim3 grid((unsigned)((size_t)units_max * (g.Ip / kSlabRows)));
    auto xb = reinterpret_cast<const __nv_bfloat16 *>(x);
    auto ao = reinterpret_cast<__half *>(a_out);
    auto kern = g.bits == 1 ? gemv_gateup_kernel<1>
                : g.bits == 2 ? gemv_gateup_kernel<2> : gemv_gateup_kernel<3>;
    launch_pdl(kern, grid, dim3(128), smem, s, w.routed, w.shared, g.expert_bytes, g.mat_bytes,
               units, n_units, list, Tk, T, g.E, xb, xex, g.H, g.Ip, xrows, nsh,
               shared_rows < 0 ? T : shared_rows, ao, err, budget);
}

void launch_gemv_down(const Geometry &g, const ExpertWeights &w, const int4 *units,
                      const int *n_units, int units_max, int T, const void *a, float *Y, int *err,
                      long long budget, cudaStream_t s) {
    const int xrows = staged_rows(T);
    size_t smem = down_smem(g, xrows);
    dim3 grid((unsigned)((size_t)units_max * (g.H / 64)));
    auto ap = reinterpret_cast<const __half *>(a);
    auto kern = g.bits == 1 ? gemv_down_kernel<1>
                : g.bits == 2 ? gemv_down_kernel<2> : gemv_down_kernel<3>;
    launch_pdl(kern, grid, dim3(128), smem, s, w.routed, w.shared, g.expert_bytes, g.mat_bytes,
               units, n_units, g.E, ap, g.H, g.Ip, xrows, Y, err, budget);
}

cudaError_t gemv_init_attributes(int max_smem) {
    cudaError_t e;
    if ((e = allow_max_dyn_smem(gemv_gateup_kernel<1>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(gemv_down_kernel<1>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(gemv_gateup_kernel<2>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(gemv_gateup_kernel<3>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(gemv_down_kernel<2>, max_smem)) != cudaSuccess) return e;
    return allow_max_dyn_smem(gemv_down_kernel<3>, max_smem);
}

}  // namespace strata
