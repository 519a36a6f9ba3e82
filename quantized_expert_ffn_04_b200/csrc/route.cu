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
// CTA: NW warps; warp owns EE experts, lanes are the 32 residue classes of the
// fixed order; TT tokens per CTA staged in shared memory as bf16 in the same
// lane-interleaved layout as the weights: xs[tt][s4][lane] holds the 4 values
// x[128*s4 + 32*j + lane], j = 0..3 (8 bytes, so the staging stores and the
// LDS.64 reads are conflict-free; widening bf16 to fp32 is exact).
template <int TT, int EE, int CH, int NW>
__global__ __launch_bounds__(32 * NW) void router_kernel(const __nv_bfloat16 *__restrict__ x, int T,
                                                     int H, const float4 *__restrict__ Wp,
                                                     const float *__restrict__ bias, int E,
                                                     float *__restrict__ logits) {
    extern __shared__ uint2 xs[];
    // a dependent kernel may be scheduled now; it waits for this grid's
    // completion before reading anything written here
    grid_launch_dependents();
    const int ns4 = H / 128;
    const int t0 = blockIdx.y * TT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e0 = (blockIdx.x * NW + warp) * EE;
    // the first CH steps of this warp's weights are requested before the
    // token rows are staged, so the two latencies overlap
    float4 wv[CH][EE];
    const uint64_t pol = l2_evict_first_policy();  // the weights are read once
    auto load_w = [&](int s0) {
#pragma unroll
        for (int c = 0; c < CH; c++)
#pragma unroll
            for (int b = 0; b < EE; b++) {
                int e = e0 + b, s4 = s0 + c;
                wv[c][b] = (e < E && s4 < ns4)
                               ? ldg_f4_hint(Wp + ((size_t)e * ns4 + s4) * 32 + lane, pol)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
            }
    };
    load_w(0);
    // stage TT token rows: a thread fills slots (tt, s4, l) from four 2-byte
    // loads that are coalesced across the warp; kSB slots (all of them for
    // H = 2560 and TT <= 8) are requested per thread before any is stored,
    // so the staging costs one memory round trip
    constexpr int kSB = (TT * 20 + NW - 1) / NW < 20 ? (TT * 20 + NW - 1) / NW : 20;
    const int nslot = TT * ns4 * 32;
    const unsigned short *xu = reinterpret_cast<const unsigned short *>(x);
    for (int base = 0; base < nslot; base += kSB * blockDim.x) {
        uint32_t v[kSB][4];
#pragma unroll
        for (int b = 0; b < kSB; b++) {
            const int sl = base + b * blockDim.x + threadIdx.x;
            const int tt = sl / (ns4 * 32), r = sl % (ns4 * 32);
            const bool ok = sl < nslot && t0 + tt < T;
            const unsigned short *px = xu + (size_t)(t0 + tt) * H + (r >> 5) * 128 + (r & 31);
#pragma unroll
            for (int j = 0; j < 4; j++) v[b][j] = ok ? (uint32_t)__ldg(px + 32 * j) : 0u;
        }
#pragma unroll
        for (int b = 0; b < kSB; b++) {
            const int sl = base + b * blockDim.x + threadIdx.x;
            if (sl >= nslot) break;
            xs[sl] = make_uint2(v[b][0] | (v[b][1] << 16), v[b][2] | (v[b][3] << 16));
        }
    }
    __syncthreads();
    if (e0 >= E) return;
    float acc[TT][EE];
#pragma unroll
    for (int a = 0; a < TT; a++)
#pragma unroll
        for (int b = 0; b < EE; b++) acc[a][b] = 0.0f;

    // CH steps of weights are requested before any of them is used, so a warp
    // keeps CH x EE x 512 bytes in flight.
    for (int s0 = 0; s0 < ns4; s0 += CH) {
        if (s0 > 0) load_w(s0);
#pragma unroll
        for (int c = 0; c < CH; c++) {
            const int s4 = s0 + c;
            if (s4 >= ns4) break;
#pragma unroll
            for (int a = 0; a < TT; a++) {
                const uint2 xv = xs[((size_t)a * ns4 + s4) * 32 + lane];
                const float x0 = __uint_as_float(xv.x << 16), x1 = __uint_as_float(xv.x & 0xffff0000u);
                const float x2 = __uint_as_float(xv.y << 16), x3 = __uint_as_float(xv.y & 0xffff0000u);
#pragma unroll
                for (int b = 0; b < EE; b++) {
                    acc[a][b] = fmaf(x0, wv[c][b].x, acc[a][b]);
                    acc[a][b] = fmaf(x1, wv[c][b].y, acc[a][b]);
                    acc[a][b] = fmaf(x2, wv[c][b].z, acc[a][b]);
                    acc[a][b] = fmaf(x3, wv[c][b].w, acc[a][b]);
                }
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

template <int TT, int EE, int CH, int NW>
static void run_router(const void *x, int T, int H, const float *Wp, const float *bias, int E,
                       float *logits, cudaStream_t s) {
    size_t smem = (size_t)TT * H * sizeof(__nv_bfloat16);
    auto kern = router_kernel<TT, EE, CH, NW>;
    dim3 grid((E + NW * EE - 1) / (NW * EE), (T + TT - 1) / TT);
    kern<<<grid, 32 * NW, smem, s>>>(reinterpret_cast<const __nv_bfloat16 *>(x), T, H,
                                 reinterpret_cast<const float4 *>(Wp), bias, E, logits);
}

void launch_router(const void *x, int T, int H, const float *Wp, const float *bias, int E,
                   float *logits, cudaStream_t s) {
    if (T <= 1)
        run_router<1, 1, 20, 4>(x, T, H, Wp, bias, E, logits, s);
    else if (T <= 4)
        run_router<4, 1, 20, 4>(x, T, H, Wp, bias, E, logits, s);
    else if (T <= 64)
        run_router<8, 2, 8, 8>(x, T, H, Wp, bias, E, logits, s);
    else
        run_router<8, 8, 2, 4>(x, T, H, Wp, bias, E, logits, s);
}

// ============================================================== top-k
// One warp per token.  Lane l holds logits l, l+32, ...  Each of the k rounds
// takes the warp-wide best (larger logit; on equal logits the lower id).
__device__ __forceinline__ bool better(float va, int ea, float vb, int eb) {
    return va > vb || (va == vb && ea < eb);
}

// Top-k of one token's logits by one warp; lane j < k ends with pick j.
// Writes idx/w (global) and, when sidx != nullptr, the picks to shared memory.
__device__ __forceinline__ void topk_token(const float *__restrict__ row, int E, int k, int lane,
                                           int32_t *__restrict__ idx, float *__restrict__ wout,
                                           int *sidx) {
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
        idx[lane] = my_e;
        wout[lane] = ex / sum;
        if (sidx) sidx[lane] = my_e;
    }
}

__global__ __launch_bounds__(256) void topk_kernel(const float *__restrict__ logits, int T, int E,
                                                   int k, int32_t *__restrict__ idx,
                                                   float *__restrict__ wout) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    if (t >= T) return;
    topk_token(logits + (size_t)t * E, E, k, lane, idx + (size_t)t * k, wout + (size_t)t * k,
               nullptr);
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
                                                             int tile, int shared_rows) {
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
    // shared-expert units first (their position is known before routing), then
    // the routed experts' units in ascending expert id
    // (the first shared_rows tokens get the shared expert; every token in a
    // forward, fewer when rows are run for other ranks' tokens)
    int nsh = (shared_rows + tile - 1) / tile;
    if (e < E)
        for (int i = 0; i < nu; i++) {
            int n = ce - i * tile;
            units[nsh + us + i] = make_int4(e, oe + i * tile, n < tile ? n : tile, 0);
        }
    for (int i = threadIdx.x; i < nsh; i += blockDim.x) {
        int n = shared_rows - i * tile;
        units[i] = make_int4(E, T * k + i * tile, n < tile ? n : tile, 0);
    }
    if (threadIdx.x == 0) *n_units = utot + nsh;
}

// Phase C: one CTA (256 threads) per chunk.
__global__ __launch_bounds__(256) void dispatch_scatter_kernel(
    const int32_t *__restrict__ idx, int T, int k, int E, const int32_t *__restrict__ base,
    const uint32_t *__restrict__ bm, const int16_t *__restrict__ pre, int32_t *__restrict__ list,
    int32_t *__restrict__ slot, int *err) {
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
        if (!idx_ok(err, pos, (long long)T * k)) continue;
        list[pos] = t;
        slot[(size_t)t * k + j] = pos;
    }
}

void launch_dispatch(const int32_t *idx, int T, int k, int E, int32_t *cnt, int32_t *off,
                     int32_t *list, int32_t *slot, const DispatchScratch &ds, int4 *units,
                     int *n_units, int tile, cudaStream_t s, int *err, int shared_rows) {
    int nc = n_chunks(T);
    if (shared_rows < 0) shared_rows = T;
    size_t smem = (size_t)8 * E * 4;
    dispatch_count_kernel<<<nc, 256, smem, s>>>(idx, T, k, E, ds.hist, ds.bm, ds.pre);
    dispatch_scan_kernel<<<1, 1024, 0, s>>>(T, k, E, nc, ds.hist, cnt, off, units, n_units,
                                            tile, shared_rows);
    dispatch_scatter_kernel<<<nc, 256, 0, s>>>(idx, T, k, E, ds.hist, ds.bm, ds.pre, list, slot,
                                               err);
}

// ============================================================== screened top-k
// Large batches: the router's tensor-core screening GEMM gives approximate
// logits a_e = x . (W_hi + W_lo)_e (+ b_e), with W_hi = fp16(W) and
// W_lo = fp16(W - W_hi).  With the bound |a_e - l_e| <= eps for the exact
// fixed-order logits l_e, every expert of the exact top-k has
// a_e >= a_(k) - 2 eps (a_(k): k-th largest approximate logit; a tie at the
// boundary is included too).  Those candidates are recomputed exactly in the
// fixed order and the top-k is taken among them, so the picks and weights are
// the same bits as with the full fp32 router.
//
// eps (per token) = 2 x [ (H 2^-23 + 2^-22 + (H/32 + 10) 2^-24) ||x||_2 max_e ||W_e||_2
//                         + 2^-25 ||x||_1 + 2^-22 max_e |b_e| ]:
// tensor-core fp32 accumulation of H exact products (truncating adder assumed),
// the two-term fp16 split (relative 2^-22 plus a subnormal quantum 2^-25), the
// fixed-order fp32 sum and the bias additions, with |x|.|W_e| <= ||x|| ||W_e||;
// the leading 2 is a safety factor.  The screening GEMM reads the fp16 copy of
// x: bf16 -> fp16 is exact for 2^-14 <= |x| <= 65504 and off by at most 2^-25
// below, adding 2^-25 ||W_e||_1 <= 2^-25 sqrt(H) ||W_e||_2; a token with any
// |x| > 65504 (or a non-finite bound) keeps every expert as a candidate.

// The screening bound of one token (one warp; see above): the token row's
// L2 norm, L1 norm and largest magnitude, and eps from them.  When xs is not
// NULL the row is also stored there in the router's lane-interleaved fp32
// layout.  `finite` is false for a token the bound does not cover (a
// non-finite bound, or an entry beyond fp16's range).
__device__ float screen_eps(const __nv_bfloat16 *__restrict__ xr, int H, float gam, float wmax,
                            float bmax, int lane, float4 *xs, bool &finite) {
    const int ns4 = H / 128;
    float ss = 0.f, s1 = 0.f, xm = 0.f;
    for (int s4 = 0; s4 < ns4; s4++) {
        float v0 = __bfloat162float(xr[128 * s4 + lane]);
        float v1 = __bfloat162float(xr[128 * s4 + 32 + lane]);
        float v2 = __bfloat162float(xr[128 * s4 + 64 + lane]);
        float v3 = __bfloat162float(xr[128 * s4 + 96 + lane]);
        ss = fmaf(v0, v0, fmaf(v1, v1, fmaf(v2, v2, fmaf(v3, v3, ss))));
        s1 += fabsf(v0) + fabsf(v1) + fabsf(v2) + fabsf(v3);
        xm = fmaxf(xm, fmaxf(fmaxf(fabsf(v0), fabsf(v1)), fmaxf(fabsf(v2), fabsf(v3))));
        if (xs) xs[s4 * 32 + lane] = make_float4(v0, v1, v2, v3);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
        xm = fmaxf(xm, __shfl_xor_sync(0xffffffffu, xm, o));
    }
    __syncwarp();
    const float eps =
        2.0f * (gam * sqrtf(ss) * 1.001f * wmax + 2.9802322e-8f * s1 * 1.001f +
                2.9802322e-8f * sqrtf((float)H) * wmax + 2.3841858e-7f * bmax);
    finite = isfinite(eps) && !(xm > 65504.0f);
    return eps;
}

// Test hook: the approximate logits a[t][e] the screen compares and each
// token's eps (0 when the bound does not cover the token).  One warp per token.
__global__ void screen_debug_kernel(const float *__restrict__ D, int R,
                                    const __nv_bfloat16 *__restrict__ x, int T, int H,
                                    const float *__restrict__ bias, int E, float gam, float wmax,
                                    float bmax, float *__restrict__ a_out,
                                    float *__restrict__ eps_out) {
    const int t = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= T) return;
    bool finite;
    const float eps = screen_eps(x + (size_t)t * H, H, gam, wmax, bmax, lane, nullptr, finite);
    if (lane == 0) eps_out[t] = finite ? eps : 0.0f;
    const float *dr = D + (size_t)t * R;
    for (int e = lane; e < E; e += 32)
        a_out[(size_t)t * E + e] = (dr[e] + dr[E + e]) + (bias ? bias[e] : 0.0f);
}

void launch_screen_debug(const float *D, int R, const void *x, int T, int H, const float *bias,
                         int E, float gam, float wmax, float bmax, float *a_out, float *eps_out,
                         cudaStream_t s) {
    screen_debug_kernel<<<(T + 3) / 4, 128, 0, s>>>(
        D, R, reinterpret_cast<const __nv_bfloat16 *>(x), T, H, bias, E, gam, wmax, bmax, a_out,
        eps_out);
}

// k picks among the lanes' values v (lane l holds experts l, l+32, ...);
// experts whose bit is set in `taken` are excluded.  Lane j < k ends with pick
// j; writes idx/w.
__device__ __forceinline__ void select_topk(const float (&v)[32], uint32_t taken, int E, int k,
                                            int lane, int32_t *__restrict__ idx,
                                            float *__restrict__ wout) {
    const int nq = (E + 31) >> 5;
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
        idx[lane] = my_e;
        wout[lane] = ex / sum;
    }
}

__global__ __launch_bounds__(128) void screen_topk_kernel(
    const float *__restrict__ D, int R, const __nv_bfloat16 *__restrict__ x, int T, int H,
    const float4 *__restrict__ Wp, const float *__restrict__ bias, int E, int k, float gam,
    float wmax, float bmax, int32_t *__restrict__ idx, float *__restrict__ wout) {
    extern __shared__ float4 sm4[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 4 + warp;
    if (t >= T) return;
    const int ns4 = H / 128;
    float4 *xs = sm4 + (size_t)warp * (H / 4);
    float *exl = reinterpret_cast<float *>(sm4 + 4 * (H / 4)) + warp * 1024;
    bool finite;
    const float eps = screen_eps(x + (size_t)t * H, H, gam, wmax, bmax, lane, xs, finite);
    const int nq = (E + 31) >> 5;
    const float *dr = D + (size_t)t * R;
    float av[32];
    // unconditional loads (entries past E re-read expert 0), so the compiler
    // cannot sink them into branches and issue them one by one
#pragma unroll
    for (int q = 0; q < 32; q++) {
        const int e = q * 32 + lane, ec = e < E ? e : 0;
        float a = (dr[ec] + dr[E + ec]) + (bias ? bias[ec] : 0.0f);
        if (a != a) a = INFINITY;  // keep a NaN screening value as a candidate
        av[q] = (q < nq && e < E) ? a : -INFINITY;
    }
    // k-th largest approximate logit
    uint32_t taken = 0;
    float kth = INFINITY;
    for (int j = 0; j < k; j++) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int q = 0; q < 32; q++) {
            int e = q * 32 + lane;
            if (q < nq && e < E && !((taken >> q) & 1) && better(av[q], e, bv, be)) {
                bv = av[q];
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
        kth = bv;
    }
    const float thr = finite ? kth - 2.0f * eps : -INFINITY;
    uint32_t cand = 0;
#pragma unroll
    for (int q = 0; q < 32; q++) {
        int e = q * 32 + lane;
        if (q < nq && e < E && (!(av[q] < thr))) cand |= 1u << q;
    }
    const uint32_t cset = cand;
    // exact fixed-order logits of the candidates, one warp-wide dot product each
    for (;;) {
        const uint32_t any = __ballot_sync(0xffffffffu, cand != 0);
        if (!any) break;
        const int src = __ffs(any) - 1;
        const int q = __shfl_sync(0xffffffffu, __ffs(cand) - 1, src);
        if (lane == src) cand &= ~(1u << q);
        const int e = 32 * q + src;
        float pacc = 0.0f;
        const float4 *wr = Wp + (size_t)e * ns4 * 32 + lane;
        for (int s4 = 0; s4 < ns4; s4++) {
            const float4 w = __ldg(wr + s4 * 32);
            const float4 xv = xs[s4 * 32 + lane];
            pacc = fmaf(xv.x, w.x, pacc);
            pacc = fmaf(xv.y, w.y, pacc);
            pacc = fmaf(xv.z, w.z, pacc);
            pacc = fmaf(xv.w, w.w, pacc);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) pacc = __fadd_rn(pacc, __shfl_down_sync(0xffffffffu, pacc, o));
        if (lane == 0) exl[e] = bias ? __fadd_rn(pacc, bias[e]) : pacc;
    }
    __syncwarp();
    float v[32];
#pragma unroll
    for (int q = 0; q < 32; q++) {
        int e = q * 32 + lane;
        float lv = ((cset >> q) & 1) ? exl[e] : -INFINITY;
        v[q] = lv != lv ? -INFINITY : lv;
    }
    select_topk(v, ~cset, E, k, lane, idx + (size_t)t * k, wout + (size_t)t * k);
}

void launch_screen_topk(const float *D, int R, const void *x, int T, int H, const float *Wp,
                        const float *bias, int E, int k, float gam, float wmax, float bmax,
                        int32_t *idx, float *w, cudaStream_t s) {
    size_t smem = (size_t)4 * H * 4 + (size_t)4 * 1024 * 4;
    screen_topk_kernel<<<(T + 3) / 4, 128, smem, s>>>(
        D, R, reinterpret_cast<const __nv_bfloat16 *>(x), T, H,
        reinterpret_cast<const float4 *>(Wp), bias, E, k, gam, wmax, bmax, idx, w);
}

// ============================================================== small batches
// Top-k and dispatch of up to 256 tokens in one CTA of 1024 threads: warps
// take tokens w, w+32, ...; then the same bitmap ranking as the chunked
// kernels, all in shared memory, with one launch instead of four.
__global__ __launch_bounds__(1024) void route_small_kernel(
    const float *__restrict__ logits, int T, int E, int k, int32_t *__restrict__ idx,
    float *__restrict__ wout, int32_t *__restrict__ cnt, int32_t *__restrict__ off,
    int32_t *__restrict__ list, int32_t *__restrict__ slot, int4 *__restrict__ units,
    int *__restrict__ n_units, int tile, int *err) {
    extern __shared__ uint32_t sm[];
    grid_launch_dependents();  // the shared expert's gate/up CTAs may start now
    grid_dependency_wait();
    uint32_t *bm = sm;                                      // [8][E]
    int *pre = reinterpret_cast<int *>(bm + 8 * E);         // [8][E]
    int *soff = pre + 8 * E;                                // [E]
    int *sidx = soff + E;                                   // [T][k]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < 8 * E; i += blockDim.x) bm[i] = 0;
    for (int t = warp; t < T; t += 32)
        topk_token(logits + (size_t)t * E, E, k, lane, idx + (size_t)t * k, wout + (size_t)t * k,
                   sidx + t * k);
    __syncthreads();
    if ((int)threadIdx.x < T) {
        const int t = threadIdx.x;
        for (int j = 0; j < k; j++) atomicOr(&bm[(t >> 5) * E + sidx[t * k + j]], 1u << (t & 31));
    }
    __syncthreads();
    const int ng = (T + 31) >> 5;
    const int e = threadIdx.x;  // E <= 1024
    int ce = 0;
    if (e < E)
        for (int g = 0; g < ng; g++) {
            pre[g * E + e] = ce;
            ce += __popc(bm[g * E + e]);
        }
    int total;
    const int oe = block_exclusive_scan(e < E ? ce : 0, &total);
    if (e < E) {
        cnt[e] = ce;
        off[e] = oe;
        soff[e] = oe;
    }
    if (e == 0) off[E] = total;
    const int nu = e < E ? (ce + tile - 1) / tile : 0;
    int utot;
    const int us = block_exclusive_scan(nu, &utot);
    // shared-expert units first, then routed experts in ascending id
    const int nsh = (T + tile - 1) / tile;
    if (e < E)
        for (int i = 0; i < nu; i++) {
            int n = ce - i * tile;
            units[nsh + us + i] = make_int4(e, oe + i * tile, n < tile ? n : tile, 0);
        }
    for (int i = threadIdx.x; i < nsh; i += blockDim.x) {
        int n = T - i * tile;
        units[i] = make_int4(E, T * k + i * tile, n < tile ? n : tile, 0);
    }
    if (threadIdx.x == 0) *n_units = utot + nsh;
    __syncthreads();
    if ((int)threadIdx.x < T) {
        const int t = threadIdx.x, g = t >> 5;
        const uint32_t below = (1u << (t & 31)) - 1u;
        for (int j = 0; j < k; j++) {
            const int ej = sidx[t * k + j];
            if (!idx_ok(err, ej, E)) continue;
            const int pos = soff[ej] + pre[g * E + ej] + __popc(bm[g * E + ej] & below);
            if (!idx_ok(err, pos, (long long)T * k)) continue;
            list[pos] = t;
            slot[(size_t)t * k + j] = pos;
        }
    }
}

void launch_route_small(const float *logits, int T, int E, int k, int32_t *idx, float *w,
                        int32_t *cnt, int32_t *off, int32_t *list, int32_t *slot, int4 *units,
                        int *n_units, int tile, cudaStream_t s, int *err) {
    size_t smem = ((size_t)8 * E * 2 + E + (size_t)T * k) * 4;
    launch_pdl(route_small_kernel, dim3(1), dim3(1024), smem, s, logits, T, E, k, idx, w, cnt,
               off, list, slot, units, n_units, tile, err);
}

cudaError_t route_init_attributes(int max_smem) {
    cudaError_t e;
    if ((e = allow_max_dyn_smem(router_kernel<1, 1, 20, 4>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(router_kernel<4, 1, 20, 4>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(router_kernel<8, 2, 8, 8>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(router_kernel<8, 8, 2, 4>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(route_small_kernel, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(screen_topk_kernel, max_smem)) != cudaSuccess) return e;
    return allow_max_dyn_smem(dispatch_count_kernel, max_smem);
}

}  // namespace strata
