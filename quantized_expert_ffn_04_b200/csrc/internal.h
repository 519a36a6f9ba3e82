// Host-side declarations shared by the library's .cu files (not part of the ABI).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace strata {

// Geometry of one layer on the GPU.
struct Geometry {
    int H, E, k, I, Ip, bits;   // Ip: I rounded up to 128 (zero-padded rows / columns)
    int nseg_h, nseg_i;         // H/128, Ip/128
    int ub;                     // bytes of one 16x128 unit
    size_t mat_bytes;           // GPU bytes of one matrix (all three are equal)
    size_t expert_bytes;        // 3 * mat_bytes
};

// ---- repack.cu
// Canonical packed matrix [R][K/32][4*bits] + scales [R][K/32] (device copies)
// -> GPU layout with Rp rows, Kp columns (zero weights in the padding).
void launch_repack_matrix(const uint8_t *codes, const uint16_t *scales, int bits, int R, int K,
                          int Rp, int Kp, uint8_t *out, cudaStream_t s);
// ---- ep.cu
// Owner rank of expert e: floor(e n_ranks / E) (contiguous ranges).
int ep_owner(int e, int E, int n_ranks);
// dst row i = src row rows[i] (row_bytes a multiple of 16; rows outside
// [0, n_src) are reported through err and skipped; with `keep`, rows i whose
// keep[i] < 0 are skipped).
void launch_gather_rows_bytes(const void *src, const int32_t *rows, int n, int n_src,
                              int row_bytes, void *dst, int *err, cudaStream_t s,
                              const int32_t *keep = nullptr);

// Largest row L2 norm of a canonical matrix [R][K] (dequantised), max-folded
// into *out_bits as float bits (start from 0).
void launch_row_norm_max(const uint8_t *codes, const uint16_t *scales, int bits, int R, int K,
                         unsigned *out_bits, cudaStream_t s);
// Debug: dequantise rows [row0, row0+nrows) of a GPU-layout matrix with Kp
// columns.  kind 0: exact fp32, kind 1: fp16 tensor-core operand (as float).
void launch_debug_dequant(const uint8_t *mat, int bits, int Kp, int row0, int nrows, int ncols,
                          int kind, float *out, cudaStream_t s);

// ---- route.cu
// Router weight in the lane-interleaved layout: Wp[e][H/128][32 lanes][4].
void launch_router(const void *x, int T, int H, const float *Wp, const float *bias, int E,
                   float *logits, cudaStream_t s);
void launch_topk(const float *logits, int T, int E, int k, int32_t *idx, float *w,
                 cudaStream_t s);

// Dispatch scratch for T tokens (chunks of 256 tokens).
struct DispatchScratch {
    int32_t *hist;      // [nchunks][E]  per-chunk counts, then per-chunk bases
    uint32_t *bm;       // [nchunks][8][E] per-warp membership bitmaps
    int16_t *pre;       // [nchunks][8][E] per-warp exclusive prefix inside the chunk
};
size_t dispatch_scratch_bytes(int T, int E);
void dispatch_scratch_carve(void *base, int T, int E, DispatchScratch *d);

// Units: int4 {expert (E = shared), first slot, n tokens, 0}; tile = tokens per unit.
// n_units[0] receives the count.  Slots: routed 0..T*k-1 (dispatch order),
// shared T*k + t.
int max_units(int T, int k, int E, int tile);
void launch_dispatch(const int32_t *idx, int T, int k, int E, int32_t *cnt, int32_t *off,
                     int32_t *list, int32_t *slot, const DispatchScratch &ds, int4 *units,
                     int *n_units, int tile, cudaStream_t s, int *err = nullptr,
                     int shared_rows = -1);

// Top-k + dispatch for T <= kSmallMaxT tokens in a single CTA.
constexpr int kSmallMaxT = 256;
void launch_route_small(const float *logits, int T, int E, int k, int32_t *idx, float *w,
                        int32_t *cnt, int32_t *off, int32_t *list, int32_t *slot, int4 *units,
                        int *n_units, int tile, cudaStream_t s, int *err = nullptr);

// Large batches: screened top-k from the split-weight screening GEMM D
// ([T][R], hi part in columns [0, E), lo part in [E, 2E)) and exact recompute
// of the candidates (see route.cu for the bound).
void launch_screen_topk(const float *D, int R, const void *x, int T, int H, const float *Wp,
                        const float *bias, int E, int k, float gam, float wmax, float bmax,
                        int32_t *idx, float *w, cudaStream_t s);
// Test hook: the screen's approximate logits a [T][E] (the two split-GEMM
// columns plus the bias) and each token's eps (0: not covered by the bound).
void launch_screen_debug(const float *D, int R, const void *x, int T, int H, const float *bias,
                         int E, float gam, float wmax, float bmax, float *a_out, float *eps_out,
                         cudaStream_t s);

// ---- gemv.cu (decode)
struct ExpertWeights {
    const uint8_t *routed;   // expert e at routed + e * expert_bytes
    const uint8_t *shared;   // the shared expert
};
void launch_gemv_gateup(const Geometry &g, const ExpertWeights &w, const int4 *units,
                        const int *n_units, int units_max, const int32_t *list, int Tk, int T,
                        const void *x, const int *xex, void *a_out, int *err, long long budget,
                        cudaStream_t s, int shared_rows = -1);
void launch_gemv_down(const Geometry &g, const ExpertWeights &w, const int4 *units,
                      const int *n_units, int units_max, int T, const void *a, float *Y, int *err,
                      long long budget, cudaStream_t s);

// ---- umma.cu (prefill)
// x (bf16) -> x16 (fp16 prescaled copy, launch_prescale), then gate/up (a:
// fp16 [slots][Ip], prescaled units) and down (Y: fp16 [slots][H], prescaled
// units) on the tensor cores.  Units of up to 256 tokens.
// The token operand xs is fp16 [slots][H] with slots = Tk + T: the routed
// rows in slot order (launch_gather_rows), then the fp16 copy of x; a holds
// `slots` rows too.  Each returns the launch status (an error also when the
// tensor maps cannot be encoded).
constexpr int kUmmaTile = 256;
// Token prescale exponents xex[T] (common.cuh) and, when x16 is not NULL, the
// prescaled fp16 operand x16[T][H] = fp16(x 2^-xex).
void launch_prescale(const void *x, int T, int H, float w2, int *xex, void *x16, cudaStream_t s);
// T: token rows in x16 (the checked build tests every list entry against it);
// slot_ex[Tk + T] receives every slot's token exponent from xex.
void launch_gather_rows(const int32_t *list, int Tk, const void *x16, void *xs, int H,
                        cudaStream_t s, int T, int *err, const int *xex, int *slot_ex);
cudaError_t launch_umma_gateup(const Geometry &g, const ExpertWeights &w, const int4 *units,
                               const int *n_units, int units_max, int slots, const void *xs,
                               const int *slot_ex, void *a, int *err, long long budget,
                               cudaStream_t s);
cudaError_t launch_umma_down(const Geometry &g, const ExpertWeights &w, const int4 *units,
                             const int *n_units, int units_max, int slots, const void *a, void *Y,
                             int *err, long long budget, cudaStream_t s);
// Plain fp16 GEMM on the tensor cores: D[t][r] = sum_k x16[t][k] * A[r][k],
// rows a multiple of 128, K a multiple of 128; fp32 out with row stride `rows`.
cudaError_t launch_umma_plain(const __half *A, int rows, const __half *x16, int T, int K, float *D,
                              int *err, long long budget, cudaStream_t s);
void launch_to_half(const void *x, void *x16, size_t n, cudaStream_t s);
cudaError_t umma_init_attributes(int max_smem);

// ---- decode.cu (fused decode layer, T <= 64)
// The whole layer in one cooperative launch (router, top-k, dispatch,
// gate/up, down, combine); see decode.cu.
struct FusedArgs {
    const void *x;              // bf16 [T][H] layer input
    const float *router_wp;     // lane-interleaved router weight
    const float *router_b;      // [E] or null
    float w2;                   // token prescale bound (0: none)
    float *logits;              // [T][E]
    int32_t *idx;               // [T][k]
    float *wts;                 // [T][k]
    void *x16;                  // fp16 [T][H] expert token operand
    float *corr;                // [T][H / 32] its block corrections (2-bit)
    int *xex;                   // [T]
    void *a;                    // fp16 [slots][Ip]
    float *Y;                   // fp32 [slots][H]
    void *out;                  // bf16 [T][H]
    bool residual;              // out <- bf16(out + y) instead of out <- y
    unsigned long long *bar;    // grid barrier counter (zero at create, never reset)
    int *cnt;                   // 2 counter sets (zero at create)
    int cnt_stride;             // ints per set: cnt_tok + 64 * (H / 128)
    int cnt_tok;                // max_units(64, k, E, 8): per-unit counters come first
    int *err;
    long long budget;
};
int fused_decode_supported(const Geometry &g, int T);
cudaError_t launch_fused_decode(const Geometry &g, const ExpertWeights &w, const FusedArgs &a,
                                int T, cudaStream_t s);
cudaError_t fused_init_attributes(int max_smem);

// ---- combine.cu
// out[t] = Y[Tk + t] + sum_j (ascending expert id) w[t][j] * Y[slot[t][j]]; bf16.
// y_half: Y stored as fp16 (prefill) instead of fp32 (decode).  residual: h
// (bf16, in place) <- bf16(f32(h) + f32(bf16(out))) instead of writing out.
// xex: token prescale exponents (Y in prescaled units; the sum is taken
// times 2^xex twice before the rounding), or NULL for unscaled Y.
void launch_combine(const void *Y, bool y_half, const int32_t *idx, const float *w,
                    const int32_t *slot, int T, int k, int H, void *out, bool residual,
                    cudaStream_t s, int *err, const int *xex);
void launch_rmsnorm(const void *h, void *xn, int T, int H, cudaStream_t s);

// ---- selftest
void launch_selftest_wait(int *err, long long budget, cudaStream_t s);

// Launch `kernel` so that it may begin while the previous kernel of the stream
// drains (programmatic dependent launch); the kernel calls
// grid_dependency_wait() before it reads anything that kernel wrote.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Set the thread-local message returned by strata_moe_last_error().
void set_error_message(const char *msg);

// Raise every kernel's dynamic shared-memory limit to the device maximum once
// per device (outside any stream capture).
cudaError_t init_kernel_attributes();
cudaError_t route_init_attributes(int max_smem);
cudaError_t gemv_init_attributes(int max_smem);

// Allow `f` the largest dynamic shared memory the device permits next to the
// kernel's static shared memory.
template <typename F>
inline cudaError_t allow_max_dyn_smem(F *f, int max_optin) {
    cudaFuncAttributes a;
    cudaError_t e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(f));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(reinterpret_cast<const void *>(f),
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                max_optin - (int)a.sharedSizeBytes);
}

}  // namespace strata
