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
// not pay for empty columns), K in stages of 64.  Operands are fp16, K-major, without swizzle, in 8-row x
// 16-byte core matrices (K-adjacent core matrices 128 B apart, row groups
// 1024 B apart).  Warp roles:
//   warp 0      allocates tensor memory; lane 0 issues the MMAs and commits
//               them to the stage and accumulator barriers;
//   warp 1      gathers the tile's token rows (fp16) with cp.async;
//   warps 2..5  dequantise the weight tile into the A operand: codes -> exact
//               odd integers (shift, mask/or against a magic exponent, packed
//               subtract) -> one packed multiply by d/2, i.e. the fp16 value of
//               d*(q-c) rounded once to nearest even;
//   warps 6..9  read the accumulators back (tcgen05.ld) and write
//               a = silu(g) u (gate/up) or y (down) as fp16.
// Every wait is bounded; a wait that gives up sets the handle's error word
// and an abort flag that releases the other roles, and the CTA lets its
// copies and MMAs land before it frees tensor memory and exits.
#include "common.cuh"
#include "internal.h"

namespace strata {

constexpr int kTM = 128;                // weight rows per tile
constexpr int kTN = 256;                // most tokens per tile
constexpr int kKS = 64;                 // K per stage
constexpr int kTileA = kTM * kKS * 2;   // 16 KB
constexpr int kTileB = kTN * kKS * 2;   // 32 KB
constexpr int kWarpMma = 0, kWarpLoadB = 1, kWarpDq0 = 2, kNumDq = 4, kNumEpi = 4;  // epilogue: warps 6..9
constexpr int kUmmaThreads = 32 * 10;

template <bool kGateUp>
struct UmmaCfg {
    static constexpr int kMats = kGateUp ? 2 : 1;
    static constexpr int kStages = kGateUp ? 3 : 4;
    static constexpr int kStageBytes = kMats * kTileA + kTileB;
    static constexpr int kTmemCols = kGateUp ? 512 : 256;
    static constexpr int kSmem = kStages * kStageBytes + 2048;
};

struct UmmaParams {
    const uint8_t *routed;
    const uint8_t *shared;
    size_t expert_bytes, mat_bytes, mat_off;
    const int4 *units;
    const int *n_units;
    int E;
    const int32_t *list;
    int Tk;
    const __half *xin;  // gate/up: x as fp16 [T][K]; down: a [slots][K]
    int K, nseg, n_rt;
    __half *out;        // gate/up: a [slots][Ip]; down: Y [slots][H]
    int out_ld;
    int *err;
    long long budget;
};

__device__ __forceinline__ bool pipe_wait(uint64_t *bar, uint32_t parity, long long budget,
                                          int *err, volatile int *abort_flag) {
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

template <int kBits, bool kGateUp>
__global__ void __launch_bounds__(kUmmaThreads, 1) umma_expert_kernel(const UmmaParams p) {
    using Cfg = UmmaCfg<kGateUp>;
    constexpr int S = Cfg::kStages, SB = Cfg::kStageBytes;
    constexpr int UB = unit_bytes(kBits);
    constexpr int SOFF = kLoBytes + (kBits == 3 ? kHiBytes : 0);
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *stages = smem;
    uint64_t *full_a = reinterpret_cast<uint64_t *>(smem + S * SB);
    uint64_t *full_b = full_a + S;
    uint64_t *empty = full_b + S;
    uint64_t *acc_full = empty + S;
    uint64_t *acc_empty = acc_full + 1;
    uint64_t *drain = acc_empty + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *rowoff = reinterpret_cast<int *>(tmem_slot + 4);  // [kTN] source row offsets

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full_a[s], kNumDq);
            mbar_init(&full_b[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kNumEpi);
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
    const int n_tiles = *p.n_units * p.n_rt;
    const int ksteps = p.K / kKS;

    if (warp == kWarpMma) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t gs = 0;
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, it++) {
                const int n = p.units[t / p.n_rt].z;
                const uint32_t idesc = umma_idesc_f16(kTM, (n + 15) & ~15);
                if (it > 0 && !pipe_wait(acc_empty, (it - 1) & 1, p.budget, p.err, abort_flag)) break;
                tc_fence_after();
                for (int ks = 0; ks < ksteps; ks++, gs++) {
                    const int slot = gs % S;
                    const uint32_t ph = (gs / S) & 1;
                    if (!pipe_wait(&full_a[slot], ph, p.budget, p.err, abort_flag) ||
                        !pipe_wait(&full_b[slot], ph, p.budget, p.err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(stages + slot * SB);
                    const uint32_t b0 = a0 + Cfg::kMats * kTileA;
#pragma unroll
                    for (int j = 0; j < kKS / 16; j++) {
                        const uint64_t bd = umma_desc(b0 + j * 256, 128, 1024);
                        const uint32_t acc = (ks | j) != 0;
                        umma_f16(tmem, umma_desc(a0 + j * 256, 128, 1024), bd, idesc, acc);
                        if (kGateUp)
                            umma_f16(tmem + kTN, umma_desc(a0 + kTileA + j * 256, 128, 1024), bd,
                                     idesc, acc);
                    }
                    umma_commit(&empty[slot]);
                }
                if (ok) umma_commit(acc_full);
            }
            // let every issued MMA finish before tensor memory is released
            umma_commit(drain);
            mbar_drain(drain, 0);
        }
    } else if (warp == kWarpLoadB) {
        // ---------------------------------------------------------- token rows
        uint32_t gs = 0;
        int prev = -1;
        const int crow = lane >> 3, chunk = lane & 7;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
            const int4 un = p.units[t / p.n_rt];
            const int slot0 = un.y, n = un.z;
            const int rows = (n + 15) & ~15;
            // the previous tile's stages only read rowoff while issuing, so it
            // can be rewritten here (one warp, program order)
            __syncwarp();
            for (int r = lane; r < rows; r += 32) {
                int off = -1;
                if (r < n) {
                    const int sl = slot0 + r;
                    const int src = kGateUp ? (sl < p.Tk ? p.list[sl] : sl - p.Tk) : sl;
                    off = src * p.K;
                }
                rowoff[r] = off;
            }
            __syncwarp();
            bool ok = true;
            for (int ks = 0; ks < ksteps; ks++, gs++) {
                const int slot = gs % S;
                if (gs >= (uint32_t)S &&
                    !pipe_wait(&empty[slot], ((gs / S) + 1) & 1, p.budget, p.err, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t *sB = stages + slot * SB + Cfg::kMats * kTileA;
#pragma unroll 4
                for (int r = crow; r < rows; r += 4) {
                    uint8_t *dst = sB + (r >> 3) * 1024 + chunk * 128 + (r & 7) * 16;
                    const int off = rowoff[r];
                    const __half *src = off >= 0 ? p.xin + off + ks * kKS + chunk * 8 : p.xin;
                    cp_async16(dst, src, off >= 0 ? 16u : 0u);
                }
                cp_async_commit();
                if (prev >= 0) {
                    cp_async_wait<1>();
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full_b[prev]);
                }
                prev = slot;
            }
            if (!ok) break;
        }
        cp_async_wait<0>();
        if (prev >= 0 && !*abort_flag) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_b[prev]);
        }
    } else if (warp < kWarpDq0 + kNumDq) {
        // ---------------------------------------------------------- dequant
        const int dt = threadIdx.x - 32 * kWarpDq0;  // 0..127
        const int L = dt & 31, sl0 = dt >> 5;        // slabs sl0 and sl0 + 4
        const int g8 = L >> 2, c = L & 3;
        const __half2 half2_05 = __float2half2_rn(0.5f);
        uint32_t gs = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
            const int rt = t % p.n_rt;
            const int e = p.units[t / p.n_rt].x;
            const uint8_t *wbase =
                (e == p.E ? p.shared : p.routed + (size_t)e * p.expert_bytes) + p.mat_off;
            for (int ks = 0; ks < ksteps; ks++, gs++) {
                const int slot = gs % S;
                if (gs >= (uint32_t)S &&
                    !pipe_wait(&empty[slot], ((gs / S) + 1) & 1, p.budget, p.err, abort_flag)) {
                    ok = false;
                    break;
                }
                const int seg = ks >> 1, h = ks & 1;
                uint8_t *sA = stages + slot * SB;
#pragma unroll
                for (int m = 0; m < Cfg::kMats; m++) {
                    const uint8_t *wm = wbase + m * p.mat_bytes;
#pragma unroll
                    for (int si = 0; si < 2; si++) {
                        const int sl = sl0 + 4 * si;
                        const uint8_t *un = wm + ((size_t)(rt * 8 + sl) * p.nseg + seg) * UB;
                        const uint2 lo = __ldg(reinterpret_cast<const uint2 *>(un + L * 16 + 8 * h));
                        uint32_t hi = 0;
                        if (kBits == 3)
                            hi = __ldg(reinterpret_cast<const uint32_t *>(un + kLoBytes + L * 8 + 4 * h));
                        const uint2 sc =
                            __ldg(reinterpret_cast<const uint2 *>(un + SOFF + (4 * g8 + 2 * h) * 4));
#pragma unroll
                        for (int bw = 0; bw < 2; bw++) {
                            const uint32_t lw = bw ? lo.y : lo.x;
                            const __half2 s2 = __hmul2(u2h(bw ? sc.y : sc.x), half2_05);
                            const __half2 s_lo = __low2half2(s2), s_hi = __high2half2(s2);
#pragma unroll
                            for (int s = 0; s < 2; s++)
#pragma unroll
                                for (int r = 0; r < 4; r++) {
                                    const uint32_t pr = dq_pair<false, kBits>(lw, hi, 4 * s + r, 8 * bw);
                                    const __half2 v = __hmul2(u2h(pr), (r & 1) ? s_hi : s_lo);
                                    const int R8 = 2 * sl + (r & 1);
                                    const int kc = 4 * bw + 2 * s + (r >> 1);
                                    *reinterpret_cast<uint32_t *>(sA + m * kTileA + R8 * 1024 +
                                                                  kc * 128 + g8 * 16 + 4 * c) = h2u(v);
                                }
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (L == 0) mbar_arrive(&full_a[slot]);
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;  // tensor-memory lane quarter of this warp
        const int r_in = 32 * q + lane;
        int it = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, it++) {
            if (!pipe_wait(acc_full, it & 1, p.budget, p.err, abort_flag)) break;
            tc_fence_after();
            const int rt = t % p.n_rt;
            const int4 un = p.units[t / p.n_rt];
            const int slot0 = un.y, n = un.z;
            const int row = rt * kTM + r_in;
            for (int nc = 0; nc < kTN / 32; nc++) {
                if (nc * 32 >= n) break;  // uniform across the warp; columns past n are ignored
                float gv[32];
                tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + nc * 32, gv);
                if (kGateUp) {
                    float uv[32];
                    tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + kTN + nc * 32, uv);
#pragma unroll
                    for (int j = 0; j < 32; j++) {
                        const int tok = nc * 32 + j;
                        if (tok < n) {
                            const float a = gv[j] / (1.0f + __expf(-gv[j])) * uv[j];
                            p.out[(size_t)(slot0 + tok) * p.out_ld + row] = __float2half_rn(a);
                        }
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; j++) {
                        const int tok = nc * 32 + j;
                        if (tok < n)
                            p.out[(size_t)(slot0 + tok) * p.out_ld + row] = __float2half_rn(gv[j]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
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

static int g_num_sms = 0;

template <int kBits, bool kGateUp>
static void run_umma(const UmmaParams &p, int max_tiles, cudaStream_t s) {
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    int grid = max_tiles < g_num_sms ? max_tiles : g_num_sms;
    if (grid <= 0) return;
    umma_expert_kernel<kBits, kGateUp>
        <<<grid, kUmmaThreads, UmmaCfg<kGateUp>::kSmem, s>>>(p);
}

void launch_umma_experts(const Geometry &g, const ExpertWeights &w, const int4 *units,
                         const int *n_units, int units_max, const int32_t *list, int Tk,
                         const void *x, void *x16, void *a, void *Y, int *err, long long budget,
                         int T, cudaStream_t s) {
    size_t n8 = (size_t)T * g.H / 8;
    to_half_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16 *>(x), reinterpret_cast<__half *>(x16), n8);
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
    // gate/up: A = Wg, Wu (Ip rows, K = H); B = x rows gathered by token
    p.mat_off = 0;
    p.xin = reinterpret_cast<const __half *>(x16);
    p.K = g.H;
    p.nseg = g.H / kSegCols;
    p.n_rt = g.Ip / kTM;
    p.out = reinterpret_cast<__half *>(a);
    p.out_ld = g.Ip;
    if (g.bits == 2)
        run_umma<2, true>(p, units_max * p.n_rt, s);
    else
        run_umma<3, true>(p, units_max * p.n_rt, s);
    // down: A = Wd (H rows, K = Ip); B = a rows by slot
    p.mat_off = 2 * g.mat_bytes;
    p.xin = reinterpret_cast<const __half *>(a);
    p.K = g.Ip;
    p.nseg = g.Ip / kSegCols;
    p.n_rt = g.H / kTM;
    p.out = reinterpret_cast<__half *>(Y);
    p.out_ld = g.H;
    if (g.bits == 2)
        run_umma<2, false>(p, units_max * p.n_rt, s);
    else
        run_umma<3, false>(p, units_max * p.n_rt, s);
}

cudaError_t umma_init_attributes(int max_smem) {
    cudaError_t e;
    if ((e = allow_max_dyn_smem(umma_expert_kernel<2, true>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(umma_expert_kernel<3, true>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(umma_expert_kernel<2, false>, max_smem)) != cudaSuccess) return e;
    return allow_max_dyn_smem(umma_expert_kernel<3, false>, max_smem);
}

}  // namespace strata
