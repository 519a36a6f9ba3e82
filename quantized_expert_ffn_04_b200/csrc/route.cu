// Router logits, softmax + top-k, and the deterministic dispatch.
//
// Routing (layer specification; the pages only say the routers run on the
// GPU, "Strata Runs 125B Qwen3.8-Flash-Next on a 12GB Gaming GPU at Up to 94
// Tokens/s", section "How a 125B model fits in 12 GB", and that 10 of 512
// experts are routed per token, section "What it is"):
//   logit[t][e] = sum_i x[t][i] * W[e][i] (fp32) + b[e]
//   in the fixed order: lane partials p_l over i = l, l+32, ... with fma in
//   ascending i, then p_l += p_{l+s} for s = 16, 8, 4, 2, 1;
//   picks = the k largest logits, a tie going to the lower expert id (the same
//   picks as the k largest softmax probabilities);
//   w_j = exp(l_j - m) / sum_{picks} exp(l_i - m), m the largest logit
//   (softmax over all experts renormalised over the picks: the full softmax
//   denominator cancels).
// Dispatch: cnt[e], off = exclusive prefix sum, list[off[e] + r] = r-th token
// (ascending) that picked e, slot[t][j] = position of (t, j).
#include <float.h>

#include "common.cuh"
#include "internal.h"

namespace strata {

// ============================================================== router
// CTA: 4 warps; warp owns EE experts, lanes are the 32 residue classes of the
// fixed order; TT tokens per CTA staged in smem as fp32 in the same
// lane-interleaved layout as the weights: xs[tt][s4][lane] = float4 of
// x[128*s4 + 32*j + lane], j = 0..3.
template <int TT, int EE>
__global__ __launch_bounds__(128) void router_kernel(const __nv_bfloat16 *__restrict__ x, int T,
                                                     int H, const float4 *__restrict__ Wp,
                                                     const float *__restrict__ bias, int E,
                                                     float *__restrict__ logits) {
    extern __shared__ float4 xs[];
    const int ns4 = H / 128;
    const int t0 = blockIdx.y * TT;
    // stage TT token rows (16 bytes = 8 bf16 per step)
    for (int idx = threadIdx.x; idx < TT * H / 8; idx += blockDim.x) {
        int tt = idx / (H / 8), i0 = (idx % (H / 8)) * 8;
        int t = t0 + tt;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t < T) v = *reinterpret_cast<const uint4 *>(x + (size_t)t * H + i0);
        const __nv_bfloat16 *pv = reinterpret_cast<const __nv_bfloat16 *>(&v);
        float *xf = reinterpret_cast<float *>(xs);
#pragma unroll
        for (int q = 0; q < 8; q++) {
            int i = i0 + q;
            xf[(((size_t)tt * ns4 + (i >> 7)) * 32 + (i & 31)) * 4 + ((i >> 5) & 3)] =
                __bfloat162float(pv[q]);
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e0 = (blockIdx.x * 4 + warp) * EE;
    if (e0 >= E) return;
    float acc[TT][EE];
#pragma unroll
    for (int a = 0; a < TT; a++)
#pragma unroll
        for (int b = 0; b < EE; b++) acc[a][b] = 0.0f;

#pragma unroll 2
    for (int s4 = 0; s4 < ns4; s4++) {
        float4 wv[EE];
#pragma unroll
        for (int b = 0; b < EE; b++) {
            int e = e0 + b;
            wv[b] = e < E ? __ldg(Wp + ((size_t)e * ns4 + s4) * 32 + lane)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int a = 0; a < TT; a++) {
            float4 xv = xs[((size_t)a * ns4 + s4) * 32 + lane];
#pragma unroll
            for (int b = 0; b < EE; b++) {
                acc[a][b] = fmaf(xv.x, wv[b].x, acc[a][b]);
                acc[a][b] = fmaf(xv.y, wv[b].y, acc[a][b]);
                acc[a][b] = fmaf(xv.z, wv[b].z, acc[a][b]);
                acc[a][b] = fmaf(xv.w, wv[b].w, acc[a][b]);
            }
        }
    }
#pragma unroll
    for (int a = 0; a < TT; a++)
#pragma unroll
        for (int b = 0; b < EE; b++) {
            float v = acc[a][b];
#pragma unroll
            for (int s = 16; s >= 1; s >>= 1) v = __fadd_rn(v, __shfl_down_sync(0xffffffffu, v, s));
            acc[a][b] = v;
        }
    if (lane == 0) {
#pragma unroll
        for (int a = 0; a < TT; a++) {
            int t = t0 + a;
            if (t >= T) continue;
#pragma unroll
            for (int b = 0; b < EE; b++) {
                int e = e0 + b;
                if (e < E)
                    logits[(size_t)t * E + e] = bias ? __fadd_rn(acc[a][b], bias[e]) : acc[a][b];
            }
        }
    }
}

template <int TT, int EE>
static void run_router(const void *x, int T, int H, const float *Wp, const float *bias, int E,
                       float *logits, cudaStream_t s) {
    size_t smem = (size_t)TT * H * sizeof(float);
    auto kern = router_kernel<TT, EE>;
    dim3 grid((E + 4 * EE - 1) / (4 * EE), (T + TT - 1) / TT);
    kern<<<grid, 128, smem, s>>>(reinterpret_cast<const __nv_bfloat16 *>(x), T, H,
                                 reinterpret_cast<const float4 *>(Wp), bias, E, logits);
}

void launch_router(const void *x, int T, int H, const float *Wp, const float *bias, int E,
                   float *logits, cudaStream_t s) {
    if (T <= 1)
        run_router<1, 1>(x, T, H, Wp, bias, E, logits, s);
    else if (T <= 4)
        run_router<4, 1>(x, T, H, Wp, bias, E, logits, s);
    else if (T <= 64)
        run_router<8, 2>(x, T, H, Wp, bias, E, logits, s);
    else
        run_router<8, 8>(x, T, H, Wp, bias, E, logits, s);
}

// ============================================================== top-k
// One warp per token.  Lane l holds logits l, l+32, ...  Each of the k rounds
// takes the warp-wide best (larger logit; on equal logits the lower id).
__device__ __forceinline__ bool better(float va, int ea, float vb, int eb) {
    return va > vb || (va == vb && ea < eb);
}

__global__ __launch_bounds__(256) void topk_kernel(const float *__restrict__ logits, int T, int E,
                                                   int k, int32_t *__restrict__ idx,
                                                   float *__restrict__ wout) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    if (t >= T) return;
    const float *row = logits + (size_t)t * E;
    const int nq = (E + 31) >> 5;  // <= 32
    float v[32];
#pragma unroll
    for (int q = 0; q < 32; q++) {
        int e = q * 32 + lane;
        float lv = (q < nq && e < E) ? row[e] : -INFINITY;
        v[q] = lv != lv ? -INFINITY : lv;  // a NaN logit ranks last
    }
    uint32_t taken = 0;
    float my_v = -INFINITY;
    int my_e = -1;
    for (int j = 0; j < k; j++) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int q = 0; q < 32; q++) {
            int e = q * 32 + lane;
            if (q < nq && e < E && !((taken >> q) & 1) && better(v[q], e, bv, be)) {
                bv = v[q];
                be = e;
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (better(ov, oe, bv, be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) {
            my_v = bv;
            my_e = be;
        }
    }
    float m = __shfl_sync(0xffffffffu, my_v, 0);
    float ex = lane < k ? expf(my_v - m) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane < k) {
        idx[(size_t)t * k + lane] = my_e;
        wout[(size_t)t * k + lane] = ex / sum;
    }
}

void launch_topk(const float *logits, int T, int E, int k, int32_t *idx, float *w,
                 cudaStream_t s) {
    topk_kernel<<<(T + 7) / 8, 256, 0, s>>>(logits, T, E, k, idx, w);
}

// ============================================================== dispatch
// Chunks of 256 tokens = 8 warps x 32 tokens.  Inside a chunk, warp w builds a
// bitmap bm[w][e] of its lanes that picked e; the rank of (t, e) inside the
// chunk is (sum over earlier warps of popc(bm[w'][e])) + popc(bm[w][e] & lanes
// below t).  Chunk bases come from a scan over (e, chunk).  Every step is a
// count, so the result does not depend on scheduling.
constexpr int kChunk = 256;

static int n_chunks(int T) { return (T + kChunk - 1) / kChunk; }

size_t dispatch_scratch_bytes(int T, int E) {
    size_t nc = (size_t)n_chunks(T > 0 ? T : 1);
    return nc * E * 4 + nc * 8 * E * 4 + nc * 8 * E * 2 + 256;
}

void dispatch_scratch_carve(void *base, int T, int E, DispatchScratch *d) {
    size_t nc = (size_t)n_chunks(T > 0 ? T : 1);
    char *p = static_cast<char *>(base);
    d->hist = reinterpret_cast<int32_t *>(p);
    p += nc * E * 4;
    d->bm = reinterpret_cast<uint32_t *>(p);
    p += nc * 8 * E * 4;
    d->pre = reinterpret_cast<int16_t *>(p);
}

int max_units(int T, int k, int E, int tile) {
    long long routed = (long long)T * k;
    long long u = (routed + tile - 1) / tile + (routed < E ? routed : E);  // sum ceil(cnt/tile)
    u += (T + tile - 1) / tile;                                             // shared expert
    return (int)u;
}

// Phase A: one CTA (256 threads) per chunk.
__global__ __launch_bounds__(256) void dispatch_count_kernel(const int32_t *__restrict__ idx,
                                                             int T, int k, int E,
                                                             int32_t *__restrict__ hist,
                                                             uint32_t *__restrict__ bm_out,
                                                             int16_t *__restrict__ pre_out) {
    extern __shared__ uint32_t bm[];  // [8][E]
    const int c = blockIdx.x;
    for (int i = threadIdx.x; i < 8 * E; i += blockDim.x) bm[i] = 0;
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = c * kChunk + threadIdx.x;
    if (t < T)
        for (int j = 0; j < k; j++) {
            int e = idx[(size_t)t * k + j];
            if ((unsigned)e < (unsigned)E) atomicOr(&bm[warp * E + e], 1u << lane);
        }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int w = 0; w < 8; w++) {
            uint32_t b = bm[w * E + e];
            bm_out[((size_t)c * 8 + w) * E + e] = b;
            pre_out[((size_t)c * 8 + w) * E + e] = (int16_t)run;
            run += __popc(b);
        }
        hist[(size_t)c * E + e] = run;
    }
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 1024).
__device__ int block_exclusive_scan(int v, int *total) {
    __shared__ int warp_sums[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int s = warp_sums[lane];
        int si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, si, o);
            if (lane >= o) si += n;
        }
        warp_sums[lane] = si - s;  // exclusive prefix of the warp totals
    }
    __syncthreads();
    int base = warp_sums[warp];
    int result = base + incl - v;
    // total = last thread's inclusive value
    __shared__ int tot;
    if (threadIdx.x == blockDim.x - 1) tot = base + incl;
    __syncthreads();
    *total = tot;
    __syncthreads();
    return result;
}

// Phase B: one CTA of 1024 threads.  cnt, off, per-chunk bases (in place in
// hist), and the unit list.
__global__ __launch_bounds__(1024) void dispatch_scan_kernel(int T, int k, int E, int nchunks,
                                                             int32_t *__restrict__ hist,
                                                             int32_t *__restrict__ cnt,
                                                             int32_t *__restrict__ off,
                                                             int4 *__restrict__ units,
                                                             int *__restrict__ n_units,
                                                             int tile) {
    const int e = threadIdx.x;  // E <= 1024
    int ce = 0;
    if (e < E)
        for (int c = 0; c < nchunks; c++) ce += hist[(size_t)c * E + e];
    int total;
    int oe = block_exclusive_scan(e < E ? ce : 0, &total);
    if (e < E) {
        cnt[e] = ce;
        off[e] = oe;
        int run = oe;
        for (int c = 0; c < nchunks; c++) {
            int h = hist[(size_t)c * E + e];
            hist[(size_t)c * E + e] = run;
            run += h;
        }
    }
    if (e == 0) off[E] = total;
    // units of `tile` tokens: routed experts in ascending id, then the shared expert
    int nu = e < E ? (ce + tile - 1) / tile : 0;
    int utot;
    int us = block_exclusive_scan(nu, &utot);
    if (e < E)
        for (int i = 0; i < nu; i++) {
            int n = ce - i * tile;
            units[us + i] = make_int4(e, oe + i * tile, n < tile ? n : tile, 0);
        }
    int nsh = (T + tile - 1) / tile;
    for (int i = threadIdx.x; i < nsh; i += blockDim.x) {
        int n = T - i * tile;
        units[utot + i] = make_int4(E, T * k + i * tile, n < tile ? n : tile, 0);
    }
    if (threadIdx.x == 0) *n_units = utot + nsh;
}

// Phase C: one CTA (256 threads) per chunk.
__global__ __launch_bounds__(256) void dispatch_scatter_kernel(
    const int32_t *__restrict__ idx, int T, int k, int E, const int32_t *__restrict__ base,
    const uint32_t *__restrict__ bm, const int16_t *__restrict__ pre, int32_t *__restrict__ list,
    int32_t *__restrict__ slot) {
    const int c = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = c * kChunk + threadIdx.x;
    if (t >= T) return;
    const uint32_t below = (1u << lane) - 1u;
    for (int j = 0; j < k; j++) {
        int e = idx[(size_t)t * k + j];
        if ((unsigned)e >= (unsigned)E) continue;
        size_t wi = ((size_t)c * 8 + warp) * E + e;
        int pos = base[(size_t)c * E + e] + pre[wi] + __popc(bm[wi] & below);
        list[pos] = t;
        slot[(size_t)t * k + j] = pos;
    }
}

void launch_dispatch(const int32_t *idx, int T, int k, int E, int32_t *cnt, int32_t *off,
                     int32_t *list, int32_t *slot, const DispatchScratch &ds, int4 *units,
                     int *n_units, int tile, cudaStream_t s) {
    int nc = n_chunks(T);
    size_t smem = (size_t)8 * E * 4;
    dispatch_count_kernel<<<nc, 256, smem, s>>>(idx, T, k, E, ds.hist, ds.bm, ds.pre);
    dispatch_scan_kernel<<<1, 1024, 0, s>>>(T, k, E, nc, ds.hist, cnt, off, units, n_units,
                                            tile);
    dispatch_scatter_kernel<<<nc, 256, 0, s>>>(idx, T, k, E, ds.hist, ds.bm, ds.pre, list, slot);
}

cudaError_t route_init_attributes(int max_smem) {
    cudaError_t e;
    if ((e = allow_max_dyn_smem(router_kernel<1, 1>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(router_kernel<4, 1>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(router_kernel<8, 2>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(router_kernel<8, 8>, max_smem)) != cudaSuccess) return e;
    return allow_max_dyn_smem(dispatch_count_kernel, max_smem);
}

}  // namespace strata
