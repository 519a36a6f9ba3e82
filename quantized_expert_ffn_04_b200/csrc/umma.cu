// Prefill expert kernels (T > 64): persistent grouped GEMM on the sm_100
// tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// Expert (layer specification): g = Wg x, u = Wu x, a = silu(g) * u,
// y = Wd a, with w = d*(q-c) from the block-32 codes.  Prompts arrive in
// chunks of up to 8,192 tokens ("Strata Runs a 125-Billion-Parameter Qwen Model
// ...", multi-token prediction paragraph), about 160 tokens per expert at
// 10 of 512 experts, so this regime is a dense contraction per expert.
//
// Tile: 128 weight rows (MMA M) x up to 256 tokens of one expert (MMA N =
// the tile's token count rounded up to 16, so a cold expert's short tile does
// not pay for empty columns), K in stages of 64.  Operands are fp16, K-major.
// The token operand B is brought in by the tensor memory accelerator with the
// 128-byte swizzle, 64 consecutive rows per box: gate/up reads the fp16 token
// rows in slot order (each expert's tokens contiguous, built once per forward
// by gather_rows_kernel), down reads a by slot, the plain GEMM reads x.  The weight
// operand A is written by the dequant warps without swizzle, in 8-row x
// 16-byte core matrices (K-adjacent core matrices 128 B apart, row groups
// 1024 B apart); the plain GEMM loads A by tensor map as well.  Warp roles:
//   warp 0      allocates tensor memory; lane 0 issues the MMAs and commits
//               them to the stage and accumulator barriers;
//   warp 1      issues the tensor-map loads of each stage, one box per lane;
//   warps 2..5  dequantise the weight tile into the A operand: codes -> exact
//               odd integers -> one packed multiply by d/2, i.e. the fp16 value
//               of d*(q-c) rounded once to nearest even;
//   warps 6..9  read the accumulators back (tcgen05.ld) and write
//               a = silu(g) u (gate/up), y (down) as fp16, or D (plain) as fp32.
// Down and plain keep two accumulators in tensor memory, so the epilogue of a
// tile overlaps the MMAs of the next; gate/up uses both halves for g and u.
// Every wait is bounded; a wait that gives up sets the handle's error word
// and an abort flag that releases the other roles, and the CTA lets its
// copies and MMAs land before it frees tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace strata {

constexpr int kTM = 128;                // weight rows per tile
constexpr int kTN = 256;                // most tokens per tile
constexpr int kKS = 64;                 // K per stage (one 128-byte swizzle row)
constexpr int kTileA = kTM * kKS * 2;   // 16 KB
constexpr int kTileB = kTN * kKS * 2;   // 32 KB
constexpr int kBoxRows = 64;            // rows per 2-D box of the token operand (8 KB)
constexpr int kWarpMma = 0, kWarpLoad = 1, kWarpDq0 = 2, kNumDq = 4, kWarpEpi0 = 6, kNumEpi = 4;
constexpr int kUmmaThreads = 32 * 10;

// Modes: gate/up (A = dequantised Wg and Wu, SwiGLU epilogue, fp16 out),
// down (A = dequantised Wd, fp16 out), plain (A = an fp16 matrix loaded by
// tensor map, fp32 out; used by the router's screening GEMM).
constexpr int kModeGateUp = 0, kModeDown = 1, kModePlain = 2;

// Separate rings for the two operands: the dequantised weight tile (A) is
// made on the SM (three slots let the dequant run two stages ahead of the
// MMAs), while the token rows (B) arrive from L2/HBM with microseconds of
// latency and get the rest of shared memory.
// The plain GEMM loads A by tensor map as well, in the same number of slots.
template <int kMode>
struct UmmaCfg {
    static constexpr int kMats = kMode == kModeGateUp ? 2 : 1;
    static constexpr int kStagesB = kMode == kModeGateUp ? 4 : (kMode == kModeDown ? 5 : 4);
    static constexpr int kStagesA = kMode == kModePlain ? kStagesB : 3;
    static constexpr int kSlotA = kMats * kTileA;
    static constexpr int kAccBufs = kMode == kModeGateUp ? 1 : 2;
    static constexpr int kTmemCols = 512;
    // A ring + B ring + alignment slack (1024) + barriers
    static constexpr int kSmem = kStagesA * kSlotA + kStagesB * kTileB + 1024 + 2048;
};

struct UmmaParams {
    CUtensorMap tm_b;   // token operand (see the file comment)
    CUtensorMap tm_a;   // plain: A [n_rt * 128][K] fp16, boxes of 64 x 128
    const uint8_t *routed;
    const uint8_t *shared;
    size_t expert_bytes, mat_bytes, mat_off;
    const int4 *units;
    const int *n_units;
    int E;
    const int32_t *list;
    int Tk;
    int K, nseg, n_rt;
    __half *out;        // gate/up: a [slots][Ip]; down: Y [slots][H]
    const int *slot_ex; // gate/up: token prescale exponent of every slot
    float *out32;       // plain: D [T][n_rt * 128]
    int direct_T;       // plain: tiles are tokens [256u, 256u + 256) of T tokens
    int out_ld;
    int *err;
    long long budget;
};

__device__ __forceinline__ int4 tile_unit(const UmmaParams &p, int u) {
    if (p.direct_T > 0) {
        const int s0 = u * kTN, n = p.direct_T - s0;
        return make_int4(0, s0, n < kTN ? n : kTN, 0);
    }
    return p.units[u];
}

__device__ __forceinline__ bool pipe_wait(uint64_t *bar, uint32_t parity, long long budget,
                                          int *err, volatile int *abort_flag) {
    // fast path: the phase is usually complete already
    if (mbar_test_wait(bar, parity)) return true;
    if (budget <= 0) {
        atomicCAS(err, 0, kErrTimeout);
        *abort_flag = 1;
        return false;
    }
    long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > budget) {
            atomicCAS(err, 0, kErrTimeout);
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ uint32_t h2u(__half2 v) { return *reinterpret_cast<uint32_t *>(&v); }
__device__ __forceinline__ __half2 u2h(uint32_t v) { return *reinterpret_cast<__half2 *>(&v); }

// silu(g) * u of a prescaled token (g, u times 2^-ex; the sigmoid takes the
// true gate, the product stays times 2^-2ex) with the fast exponential and
// division (the output is rounded to fp16, far coarser than their error).
__device__ __forceinline__ float swiglu(float g, float u, int ex) {
    const float gt = ex ? g * pow2f(ex) : g;
    return __fdividef(g, 1.0f + __expf(-gt)) * u;
}

template <int kBits, int kMode>
__global__ void __launch_bounds__(kUmmaThreads, 1)
    umma_expert_kernel(const __grid_constant__ UmmaParams p) {
    constexpr bool kGateUp = kMode == kModeGateUp;
    constexpr bool kPlain = kMode == kModePlain;
    using Cfg = UmmaCfg<kMode>;
    constexpr int SA = Cfg::kStagesA, SBn = Cfg::kStagesB, NB = Cfg::kAccBufs;
    extern __shared__ uint8_t smem_raw[];
    // the swizzled operands need 1024-byte aligned slots
    uint8_t *ringA = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ringB = ringA + SA * Cfg::kSlotA;
    uint64_t *full_a = reinterpret_cast<uint64_t *>(ringB + SBn * kTileB);
    uint64_t *empty_a = full_a + SA;
    uint64_t *full_b = empty_a + SA;
    uint64_t *empty_b = full_b + SBn;
    uint64_t *acc_full = empty_b + SBn;  // [NB]
    uint64_t *acc_empty = acc_full + 2;  // [NB]
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; s++) {
            mbar_init(&full_a[s], kNumDq);
            mbar_init(&empty_a[s], 1);
        }
        for (int s = 0; s < SBn; s++) {
            mbar_init(&full_b[s], 1);
            mbar_init(&empty_b[s], 1);
        }
        for (int b = 0; b < NB; b++) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kNumEpi);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_tiles =
        (p.direct_T > 0 ? (p.direct_T + kTN - 1) / kTN : *p.n_units) * p.n_rt;
    const int ksteps = p.K / kKS;

    if (warp == kWarpMma) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t gs = 0;
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, it++) {
                const int n = tile_unit(p, t / p.n_rt).z;
                const uint32_t idesc = umma_idesc_f16(kTM, (n + 15) & ~15);
                const int buf = it % NB, use = it / NB;
                if (use > 0 &&
                    !pipe_wait(&acc_empty[buf], (use - 1) & 1, p.budget, p.err, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t dacc = tmem + buf * kTN;
                for (int ks = 0; ks < ksteps; ks++, gs++) {
                    const int sa = gs % SA, sb = gs % SBn;
                    if ((!kPlain && !pipe_wait(&full_a[sa], (gs / SA) & 1, p.budget, p.err,
                                               abort_flag)) ||
                        !pipe_wait(&full_b[sb], (gs / SBn) & 1, p.budget, p.err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // descriptors: the start address sits in the low bits (16-byte
                    // units), so the K steps inside a stage are plain additions
                    const uint64_t bd0 = umma_desc_sw128(smem_u32(ringB + sb * kTileB));
                    const uint32_t a0 = smem_u32(ringA + sa * Cfg::kSlotA);
                    const uint64_t ad0 = kPlain ? umma_desc_sw128(a0) : umma_desc(a0, 128, 1024);
#pragma unroll
                    for (int j = 0; j < kKS / 16; j++) {
                        const uint64_t bd = bd0 + (uint64_t)(j * 32 >> 4);
                        const uint64_t ad = ad0 + (uint64_t)((kPlain ? j * 32 : j * 256) >> 4);
                        const uint32_t acc = (ks | j) != 0;
                        umma_f16(dacc, ad, bd, idesc, acc);
                        if (kGateUp)
                            umma_f16(tmem + kTN, ad + (uint64_t)(kTileA >> 4), bd, idesc, acc);
                    }
                    umma_commit(&empty_b[sb]);
                    if (!kPlain) umma_commit(&empty_a[sa]);
                }
                if (ok) umma_commit(&acc_full[buf]);
            }
            // let every issued MMA finish before tensor memory is released
            umma_commit(drain);
            mbar_drain(drain, 0);
        }
    } else if (warp == kWarpLoad) {
        // ---------------------------------------------------------- TMA loads
        if (lane == 0) {
            prefetch_tmap(&p.tm_b);
            if (kPlain) prefetch_tmap(&p.tm_a);
        }
        uint32_t gs = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
            const int4 un = tile_unit(p, t / p.n_rt);
            const int slot0 = un.y, n = un.z;
            // whole 64-row boxes (each issue costs about as much as a box's
            // bytes take to land, so few large boxes); rows past n are never
            // read back
            const int nbox = (n + kBoxRows - 1) / kBoxRows;
            const int rt = t % p.n_rt;
            for (int ks = 0; ks < ksteps; ks++, gs++) {
                const int slot = gs % SBn;
                int okl = 1;
                if (lane == 0) {
                    if (gs >= (uint32_t)SBn && !pipe_wait(&empty_b[slot], ((gs / SBn) + 1) & 1,
                                                          p.budget, p.err, abort_flag))
                        okl = 0;
                    else
                        mbar_arrive_expect_tx(&full_b[slot], (uint32_t)(nbox * kBoxRows * 128 +
                                                                        (kPlain ? kTileA : 0)));
                }
                okl = __shfl_sync(0xffffffffu, okl, 0);
                if (!okl) {
                    ok = false;
                    break;
                }
                // the stage's boxes go out from several lanes at once
                uint8_t *sA = ringA + (gs % SA) * Cfg::kSlotA;  // plain: SA == SBn
                uint8_t *sB = ringB + slot * kTileB;
                if (lane < nbox)
                    tma_load_2d(sB + lane * kBoxRows * 128, &p.tm_b, ks * kKS,
                                slot0 + lane * kBoxRows, &full_b[slot]);
                if (kPlain && lane == nbox)
                    tma_load_2d(sA, &p.tm_a, ks * kKS, rt * kTM, &full_b[slot]);
            }
        }
        // after an abort, let the loads of the stages armed last land
        if (lane == 0 && *abort_flag) {
            for (uint32_t g2 = gs > (uint32_t)SBn ? gs - SBn : 0; g2 < gs; g2++)
                mbar_drain(&full_b[g2 % SBn], (g2 / SBn) & 1);
        }
    } else if (warp < kWarpEpi0) {
        if constexpr (!kPlain) {
            // ------------------------------------------------------ dequant
            const int dt = threadIdx.x - 32 * kWarpDq0;  // 0..127
            const int L = dt & 31, sl0 = dt >> 5;        // slabs sl0 and sl0 + 4
            const int g8 = L >> 2, c = L & 3;
            constexpr int UB = unit_bytes(kBits);
            constexpr int SOFF = scale_off(kBits);
            const __half2 half2_05 = __float2half2_rn(0.5f);
            // packed words of one stage for this thread: [matrix][slab]
            struct Raw {
                uint2 lo[Cfg::kMats][2];
                uint32_t hi[Cfg::kMats][2];
                uint2 sc[Cfg::kMats][2];
            };
            auto fetch = [&](int t, int ks, Raw &r) {
                const int rt = t % p.n_rt;
                const int e = __ldg(&p.units[t / p.n_rt].x);
                const uint8_t *wbase =
                    (e == p.E ? p.shared : p.routed + (size_t)e * p.expert_bytes) + p.mat_off;
                const int seg = ks >> 1, h = ks & 1;
#pragma unroll
                for (int m = 0; m < Cfg::kMats; m++)
#pragma unroll
                    for (int si = 0; si < 2; si++) {
                        const uint8_t *un = wbase + m * p.mat_bytes +
                                            ((size_t)(rt * 8 + sl0 + 4 * si) * p.nseg + seg) * UB;
                        if (kBits == 1) {  // blocks 2h, 2h + 1 in one word (the odd one a bit higher)
                            const uint32_t v = __ldg(reinterpret_cast<const uint32_t *>(un + L * 8 + 4 * h));
                            r.lo[m][si] = make_uint2(v, v >> 1);
                        } else {
                            r.lo[m][si] = __ldg(reinterpret_cast<const uint2 *>(un + L * 16 + 8 * h));
                        }
                        r.hi[m][si] = kBits == 3 ? __ldg(reinterpret_cast<const uint32_t *>(
                                                       un + kLoBytes + L * 8 + 4 * h))
                                                 : 0u;
                        r.sc[m][si] = __ldg(
                            reinterpret_cast<const uint2 *>(un + SOFF + (4 * g8 + 2 * h) * 4));
                    }
            };
            // Walk the (tile, stage) sequence with three register buffers: the
            // raw words of position i+3 are requested right after position i is
            // dequantised, i.e. two stages of work before they are needed.
            struct Pos {
                int t, ks;
            };
            auto advance = [&](Pos q) {
                if (++q.ks == ksteps) {
                    q.ks = 0;
                    q.t += gridDim.x;
                }
                return q;
            };
            uint32_t gs = 0;
            // returns false when the pipeline must stop (abort)
            auto step = [&](const Raw &cur) -> bool {
                const int slot = gs % SA;
                if (gs >= (uint32_t)SA &&
                    !pipe_wait(&empty_a[slot], ((gs / SA) + 1) & 1, p.budget, p.err, abort_flag))
                    return false;
                uint8_t *sA = ringA + slot * Cfg::kSlotA;
#pragma unroll
                for (int m = 0; m < Cfg::kMats; m++)
#pragma unroll
                    for (int si = 0; si < 2; si++) {
                        const int sl = sl0 + 4 * si;
#pragma unroll
                        for (int bw = 0; bw < 2; bw++) {
                            const uint32_t lw = bw ? cur.lo[m][si].y : cur.lo[m][si].x;
                            const __half2 s2 =
                                __hmul2(u2h(bw ? cur.sc[m][si].y : cur.sc[m][si].x), half2_05);
                            const __half2 s_lo = __low2half2(s2), s_hi = __high2half2(s2);
#pragma unroll
                            for (int s = 0; s < 2; s++)
#pragma unroll
                                for (int r = 0; r < 4; r++) {
                                    const uint32_t pr =
                                        kBits <= 2 ? dq2_pair<kBits == 1 ? 1 : 2>(lw, 4 * s + r)
                                                   : dq_pair<false, kBits>(lw, cur.hi[m][si],
                                                                           4 * s + r, 8 * bw);
                                    const __half2 v = __hmul2(u2h(pr), (r & 1) ? s_hi : s_lo);
                                    const int R8 = 2 * sl + (r & 1);
                                    const int kc = 4 * bw + 2 * s + (r >> 1);
                                    *reinterpret_cast<uint32_t *>(sA + m * kTileA + R8 * 1024 +
                                                                  kc * 128 + g8 * 16 + 4 * c) =
                                        h2u(v);
                                }
                        }
                    }
                fence_proxy_async_smem();
                __syncwarp();
                if (L == 0) mbar_arrive(&full_a[slot]);
                gs++;
                return true;
            };
            Raw r0, r1, r2;
            Pos p0{(int)blockIdx.x, 0}, p1 = advance(p0), p2 = advance(p1);
            if (p0.t < n_tiles) fetch(p0.t, p0.ks, r0);
            if (p1.t < n_tiles) fetch(p1.t, p1.ks, r1);
            if (p2.t < n_tiles) fetch(p2.t, p2.ks, r2);
            while (true) {
                if (p0.t >= n_tiles || !step(r0)) break;
                const Pos p3 = advance(p2);
                if (p3.t < n_tiles) fetch(p3.t, p3.ks, r0);
                if (p1.t >= n_tiles || !step(r1)) break;
                const Pos p4 = advance(p3);
                if (p4.t < n_tiles) fetch(p4.t, p4.ks, r1);
                if (p2.t >= n_tiles || !step(r2)) break;
                const Pos p5 = advance(p4);
                if (p5.t < n_tiles) fetch(p5.t, p5.ks, r2);
                p0 = p3;
                p1 = p4;
                p2 = p5;
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;  // tensor-memory lane quarter this warp may read
        const int r_in = 32 * q + lane;
        int it = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, it++) {
            const int buf = it % NB, use = it / NB;
            // the tile's unit and (gate/up) the prescale exponents of its
            // columns are requested before the wait for the accumulators, so
            // their latency hides behind the tile's MMAs: lane j holds the
            // exponent of column 32 c + j in exr[c]
            const int rt = t % p.n_rt;
            const int4 un = tile_unit(p, t / p.n_rt);
            const int slot0 = un.y, n = un.z;
            int exr[kTN / 32];
#pragma unroll
            for (int c = 0; c < kTN / 32; c++)
                exr[c] = kGateUp && 32 * c + lane < n ? __ldg(p.slot_ex + slot0 + 32 * c + lane) : 0;
            if (!pipe_wait(&acc_full[buf], use & 1, p.budget, p.err, abort_flag)) break;
            tc_fence_after();
            const int row = rt * kTM + r_in;
            const uint32_t tb = tmem + ((uint32_t)(32 * q) << 16) + buf * kTN;
            for (int nc = 0; nc * 32 < n; nc++) {
                const int cnt = n - nc * 32;  // valid columns of this chunk
                const size_t o0 = (size_t)(slot0 + nc * 32) * p.out_ld + row;
                float gv[32];
                tmem_ld32(tb + nc * 32, gv);
                if (kGateUp) {
                    float uv[32];
                    tmem_ld32(tb + kTN + nc * 32, uv);
                    // lane j holds the prescale exponent of column j of the chunk;
                    // when the chunk's columns share one (the usual case) the
                    // factor is taken once, without a shuffle per element
                    int exl = 0;
#pragma unroll
                    for (int c = 0; c < kTN / 32; c++) exl = c == nc ? exr[c] : exl;
                    const int ex0 = __shfl_sync(0xffffffffu, exl, 0);
                    if (__all_sync(0xffffffffu, lane >= cnt || exl == ex0)) {
                        const float f = pow2f(ex0);
#pragma unroll
                        for (int j = 0; j < 32; j++)
                            if (j < cnt)
                                p.out[o0 + (size_t)j * p.out_ld] = __float2half_rn(
                                    __fdividef(gv[j], 1.0f + __expf(-(gv[j] * f))) * uv[j]);
                    } else if (cnt >= 32) {
#pragma unroll
                        for (int j = 0; j < 32; j++)
                            p.out[o0 + (size_t)j * p.out_ld] = __float2half_rn(
                                swiglu(gv[j], uv[j], __shfl_sync(0xffffffffu, exl, j)));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; j++) {
                            const int ex = __shfl_sync(0xffffffffu, exl, j);
                            if (j < cnt)
                                p.out[o0 + (size_t)j * p.out_ld] =
                                    __float2half_rn(swiglu(gv[j], uv[j], ex));
                        }
                    }
                } else if (kMode == kModeDown) {
                    if (cnt >= 32) {
#pragma unroll
                        for (int j = 0; j < 32; j++)
                            p.out[o0 + (size_t)j * p.out_ld] = __float2half_rn(gv[j]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; j++)
                            if (j < cnt) p.out[o0 + (size_t)j * p.out_ld] = __float2half_rn(gv[j]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; j++)
                        if (j < cnt) p.out32[o0 + (size_t)j * p.out_ld] = gv[j];
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// x (bf16) -> fp16 copy used as the token operand of the prefill GEMM.
__global__ void to_half_kernel(const __nv_bfloat16 *__restrict__ x, __half *__restrict__ y,
                               size_t n8) {
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n8) return;
    uint4 v = reinterpret_cast<const uint4 *>(x)[i];
    const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&v);
    uint4 o;
    __half2 *h = reinterpret_cast<__half2 *>(&o);
#pragma unroll
    for (int j = 0; j < 4; j++) h[j] = __float22half2_rn(__bfloat1622float2(b[j]));
    reinterpret_cast<uint4 *>(y)[i] = o;
}

// Token prescale (see common.cuh): one warp per token computes the exponent e
// in the shared fixed order, stores it in xex[t] and, when x16 is given,
// writes the expert operand fp16(x 2^-e) of the row.
__global__ void prescale_kernel(const __nv_bfloat16 *__restrict__ x, int T, int H, float w2,
                                int *__restrict__ xex, __half *__restrict__ x16) {
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= T) return;
    const __nv_bfloat16 *row = x + (size_t)t * H;
    const int e = token_prescale_warp(row, H, w2, lane);
    if (lane == 0) xex[t] = e;
    if (!x16) return;
    const float sc = pow2f(-e);
    const uint4 *src = reinterpret_cast<const uint4 *>(row);
    uint4 *dst = reinterpret_cast<uint4 *>(x16 + (size_t)t * H);
    for (int i = lane; i < H / 8; i += 32) {
        const uint4 v = src[i];
        const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&v);
        uint4 o;
        __half2 *h = reinterpret_cast<__half2 *>(&o);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const float2 f = __bfloat1622float2(b[j]);
            h[j] = __floats2half2_rn(f.x * sc, f.y * sc);
        }
        dst[i] = o;
    }
}

void launch_prescale(const void *x, int T, int H, float w2, int *xex, void *x16, cudaStream_t s) {
    if (T <= 0) return;
    prescale_kernel<<<(unsigned)((T + 7) / 8), 256, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16 *>(x), T, H, w2, xex, reinterpret_cast<__half *>(x16));
}

// ------------------------------------------------------------------- host
static int g_num_sms = 0;

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (the library links the runtime statically and not the driver library).
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// Tensor map of an fp16 matrix [rows][cols] (row pitch cols), boxes of 64
// columns x box_rows rows, 128-byte swizzle, zero fill outside the matrix.
// base 16-byte aligned and cols a multiple of 8 (the map's own checks).
static cudaError_t encode_fp16_map(CUtensorMap *m, const void *base, int cols, int rows,
                                   int box_rows) {
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)kKS, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims,
                    strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int kBits, int kMode>
static cudaError_t run_umma(const UmmaParams &p, int max_tiles, cudaStream_t s) {
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    int grid = max_tiles < g_num_sms ? max_tiles : g_num_sms;
    if (grid <= 0) return cudaSuccess;
    umma_expert_kernel<kBits, kMode><<<grid, kUmmaThreads, UmmaCfg<kMode>::kSmem, s>>>(p);
    return cudaGetLastError();
}

// xs[slot] = x16[list[slot]] for the Tk routed slots (one warp per row,
// 16-byte copies); the shared expert's rows follow as x16 itself.
__global__ void gather_rows_kernel(const int32_t *__restrict__ list, int Tk,
                                   const uint4 *__restrict__ x16, uint4 *__restrict__ xs,
                                   int row16, int T, int *err, const int *__restrict__ xex,
                                   int *__restrict__ slot_ex) {
    const int slot = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (slot >= Tk + T) return;
    if (slot >= Tk) {  // the shared expert's slots: rows already in place after the routed ones
        if (lane == 0) slot_ex[slot] = xex[slot - Tk];
        return;
    }
    const int t = __ldg(list + slot);
    if (!idx_ok(err, t, T)) return;
    if (lane == 0) slot_ex[slot] = xex[t];
    const uint4 *src = x16 + (size_t)t * row16;
    uint4 *dst = xs + (size_t)slot * row16;
    for (int i = lane; i < row16; i += 32) dst[i] = __ldg(src + i);
}

void launch_gather_rows(const int32_t *list, int Tk, const void *x16, void *xs, int H,
                        cudaStream_t s, int T, int *err, const int *xex, int *slot_ex) {
    if (Tk + T <= 0) return;
    gather_rows_kernel<<<(unsigned)((Tk + T + 7) / 8), 256, 0, s>>>(
        list, Tk, reinterpret_cast<const uint4 *>(x16), reinterpret_cast<uint4 *>(xs), H / 8,
        T, err, xex, slot_ex);
}

void launch_to_half(const void *x, void *x16, size_t n, cudaStream_t s) {
    size_t n8 = n / 8;
    to_half_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16 *>(x), reinterpret_cast<__half *>(x16), n8);
}

static UmmaParams base_params(const Geometry &g, const ExpertWeights &w, const int4 *units,
                              const int *n_units, const int32_t *list, int Tk, int *err,
                              long long budget) {
    UmmaParams p{};
    p.routed = w.routed;
    p.shared = w.shared;
    p.expert_bytes = g.expert_bytes;
    p.mat_bytes = g.mat_bytes;
    p.units = units;
    p.n_units = n_units;
    p.E = g.E;
    p.list = list;
    p.Tk = Tk;
    p.err = err;
    p.budget = budget;
    return p;
}

cudaError_t launch_umma_gateup(const Geometry &g, const ExpertWeights &w, const int4 *units,
                               const int *n_units, int units_max, int slots, const void *xs,
                               const int *slot_ex, void *a, int *err, long long budget,
                               cudaStream_t s) {
    // A = Wg, Wu (Ip rows, K = H); B = token rows by slot
    UmmaParams p = base_params(g, w, units, n_units, nullptr, 0, err, budget);
    p.slot_ex = slot_ex;
    cudaError_t e = encode_fp16_map(&p.tm_b, xs, g.H, slots, kBoxRows);
    if (e != cudaSuccess) return e;
    p.mat_off = 0;
    p.K = g.H;
    p.nseg = g.H / kSegCols;
    p.n_rt = g.Ip / kTM;
    p.out = reinterpret_cast<__half *>(a);
    p.out_ld = g.Ip;
    return g.bits == 1   ? run_umma<1, kModeGateUp>(p, units_max * p.n_rt, s)
           : g.bits == 2 ? run_umma<2, kModeGateUp>(p, units_max * p.n_rt, s)
                         : run_umma<3, kModeGateUp>(p, units_max * p.n_rt, s);
}

cudaError_t launch_umma_down(const Geometry &g, const ExpertWeights &w, const int4 *units,
                             const int *n_units, int units_max, int slots, const void *a, void *Y,
                             int *err, long long budget, cudaStream_t s) {
    // A = Wd (H rows, K = Ip); B = a rows by slot
    UmmaParams p = base_params(g, w, units, n_units, nullptr, 0, err, budget);
    cudaError_t e = encode_fp16_map(&p.tm_b, a, g.Ip, slots, kBoxRows);
    if (e != cudaSuccess) return e;
    p.mat_off = 2 * g.mat_bytes;
    p.K = g.Ip;
    p.nseg = g.Ip / kSegCols;
    p.n_rt = g.H / kTM;
    p.out = reinterpret_cast<__half *>(Y);
    p.out_ld = g.H;
    return g.bits == 1   ? run_umma<1, kModeDown>(p, units_max * p.n_rt, s)
           : g.bits == 2 ? run_umma<2, kModeDown>(p, units_max * p.n_rt, s)
                         : run_umma<3, kModeDown>(p, units_max * p.n_rt, s);
}

cudaError_t launch_umma_plain(const __half *A, int rows, const __half *x16, int T, int K, float *D,
                              int *err, long long budget, cudaStream_t s) {
    UmmaParams p{};
    cudaError_t e = encode_fp16_map(&p.tm_b, x16, K, T, kBoxRows);
    if (e == cudaSuccess) e = encode_fp16_map(&p.tm_a, A, K, rows, kTM);
    if (e != cudaSuccess) return e;
    p.direct_T = T;
    p.K = K;
    p.nseg = K / kSegCols;
    p.n_rt = rows / kTM;
    p.out32 = D;
    p.out_ld = rows;
    p.err = err;
    p.budget = budget;
    return run_umma<2, kModePlain>(p, ((T + kTN - 1) / kTN) * p.n_rt, s);
}

cudaError_t umma_init_attributes(int max_smem) {
    // look the encoder up here, outside any stream capture
    if (!encode_fn()) return cudaErrorNotSupported;
    cudaError_t e;
    if ((e = allow_max_dyn_smem(umma_expert_kernel<1, kModeGateUp>, max_smem)) != cudaSuccess)
        return e;
    if ((e = allow_max_dyn_smem(umma_expert_kernel<1, kModeDown>, max_smem)) != cudaSuccess)
        return e;
    if ((e = allow_max_dyn_smem(umma_expert_kernel<2, kModeGateUp>, max_smem)) != cudaSuccess)
        return e;
    if ((e = allow_max_dyn_smem(umma_expert_kernel<3, kModeGateUp>, max_smem)) != cudaSuccess)
        return e;
    if ((e = allow_max_dyn_smem(umma_expert_kernel<2, kModeDown>, max_smem)) != cudaSuccess)
        return e;
    if ((e = allow_max_dyn_smem(umma_expert_kernel<3, kModeDown>, max_smem)) != cudaSuccess)
        return e;
    return allow_max_dyn_smem(umma_expert_kernel<2, kModePlain>, max_smem);
}

}  // namespace strata
