/*
 * strata_moe.h -- C ABI of the B200 (sm_100a) Strata MoE layer library.
 *
 * One call of strata_moe_forward runs the whole mixture-of-experts layer
 * forward on the GPU:
 *   router logits -> softmax + top-k -> dispatch -> quantised SwiGLU experts
 *   (routed + shared) -> fixed-order combine.
 *
 * Sources.  The pages describe Strata's layer as 512 experts with 10 routed and
 * 1 shared expert per token, hidden size 2,560 ("Strata Runs 125B
 * Qwen3.8-Flash-Next on a 12GB Gaming GPU at Up to 94 Tokens/s", section "What
 * it is"; "Strata ... gaming PC", spec table), with routers and shared experts
 * on the GPU ("How a 125B model fits in 12 GB") and 2-3 bit quantised builds
 * ("The numbers, measured by the author"; "Caveats").  Prompts are read in
 * chunks of up to 8,192 tokens and the MTP verify pass scores up to 4 tokens
 * at once ("Strata Runs a 125-Billion-Parameter Qwen Model ...", multi-token
 * prediction paragraph).  The quantised block format, the routing rule and the
 * combine order are the layer specification this library implements; they are
 * stated with each declaration below.
 *
 * Conventions for every entry point:
 *   - Device pointers are caller-owned CUDA device memory on the handle's
 *     device.  Host pointers are caller-owned host memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls that take a stream only enqueue work and return; they
 *     never synchronise unless stated.
 *   - A handle owns one workspace, so it serves one call in flight at a time;
 *     use one handle per concurrent stream.
 *   - Errors: every call returns a strata_status; on failure
 *     strata_moe_last_error() gives a message (thread-local, valid until the
 *     next call on that thread).  Nothing is written to caller buffers when
 *     argument validation fails.
 */
#ifndef STRATA_MOE_H
#define STRATA_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    STRATA_OK = 0,
    STRATA_ERR_INVALID_ARG = 1,  /* null pointer, T out of range, aliasing, bad value */
    STRATA_ERR_UNSUPPORTED = 2,  /* a shape or format outside the supported set */
    STRATA_ERR_OOM = 3,          /* device allocation failed (nothing leaked) */
    STRATA_ERR_CUDA = 4,         /* a CUDA call or kernel launch failed */
    STRATA_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out (see sync_status) */
    STRATA_ERR_BOUNDS = 6        /* checked build (-DSTRATA_CHECKS=1) only: a device-side
                                    gather/scatter index fell outside its buffer; the access
                                    was skipped and reported, never faulted on */
} strata_status;

typedef struct strata_moe *strata_moe_t; /* opaque, library-owned */

/* Layer shape.  Supported: hidden % 128 == 0 and 128 <= hidden <= 6144;
 * 1 <= n_experts <= 1024; 1 <= top_k <= min(n_experts, 32); inter % 32 == 0
 * and 32 <= inter <= 4096; quant_bits in {1, 2, 3}; block == 32;
 * 1 <= max_tokens <= 65536.  Anything else returns STRATA_ERR_UNSUPPORTED
 * (or INVALID_ARG for non-positive values). */
typedef struct {
    int32_t hidden;          /* H */
    int32_t n_experts;       /* E */
    int32_t top_k;           /* k routed experts per token */
    int32_t inter;           /* I, SwiGLU intermediate size */
    int32_t quant_bits;      /* 1: w = d*(q-0.5), q in 0..1;  2: w = d*(q-1.5), q in 0..3;
                                3: w = d*(q-3.5), q in 0..7 */
    int32_t block;           /* quantisation block along the input dimension: 32 */
    int32_t max_tokens;      /* largest T accepted; sizes the handle's workspace */
    int32_t has_router_bias; /* 1: router_b is read; 0: logits carry no bias */
} strata_moe_config;

/* Packed weights in the canonical host format (read during create only).
 *
 * Each expert has three matrices, in this order: 0 gate [I][H], 1 up [I][H],
 * 2 down [H][I], all row-major [out][in] and quantised along `in` in blocks of
 * 32 elements.  A block is 4*bits bytes of codes plus one fp16 scale d:
 *   1-bit: element j is bit j%8 of byte j/8 (the pages mention a 1-bit quant,
 *          "Open-Source Strata Runs a 125-Billion-Parameter Model ...", Key
 *          Facts item 4, with no layout: read as the same block-32 family);
 *   2-bit: element j in bits 2*(j%4)..2*(j%4)+1 of byte j/4;
 *   3-bit: the 12 bytes form one little-endian 96-bit integer, element j in
 *          bits 3j..3j+2.
 * Every matrix holds H*I weights, so with nb = H*I/32 blocks per matrix:
 *   codes         uint8  [E][3][nb][4*bits]   (blocks row-major within a matrix)
 *   scales        uint16 [E][3][nb]           (fp16 bit patterns)
 *   shared_codes  uint8  [3][nb][4*bits]      (the always-on shared expert)
 *   shared_scales uint16 [3][nb]
 *   router_w      float  [E][H]
 *   router_b      float  [E]  (read only when has_router_bias; may be NULL otherwise)
 */
typedef struct {
    const uint8_t *codes;
    const uint16_t *scales;
    const float *router_w;
    const float *router_b;
    const uint8_t *shared_codes;
    const uint16_t *shared_scales;
} strata_moe_weights;

/* Create a layer on CUDA device `device`: validates the shape, copies the
 * host weights to the device, repacks them into the GPU layout and allocates
 * the workspace for max_tokens.  The caller may free the host buffers once it
 * returns.  Synchronous.  On failure *out is set to NULL and nothing leaks. */
strata_status strata_moe_create(const strata_moe_config *cfg, const strata_moe_weights *weights,
                                int device, strata_moe_t *out);

/* Release a handle and all its device memory.  NULL-safe.  Synchronises the
 * device work of the handle first. */
void strata_moe_destroy(strata_moe_t h);

/* Routing only: fp32 router logits, softmax over all experts, top-k with the
 * lower expert id winning a tie, weights renormalised over the k picks.
 *   x_dev        bf16 [T][H] hidden states (device)
 *   idx_dev      int32 [T][k] out: picks in descending logit order (device)
 *   w_dev        float [T][k] out: weights of those picks, sum 1 per token
 *   offsets_dev  int32 [E+1] out or NULL: exclusive prefix sum of per-expert
 *                counts, offsets[E] = T*k
 *   list_dev     int32 [T*k] out or NULL: tokens grouped by expert, ascending
 *                token index within each expert (list[offsets[e] + r])
 * Logits are fp32 dot products in a fixed order (32 interleaved fma partial
 * sums over i = l, l+32, ..., then a halving tree, then + bias), so indices,
 * offsets and lists are reproducible bit for bit.  T == 0 is a no-op;
 * T > max_tokens returns INVALID_ARG. */
strata_status strata_moe_route(strata_moe_t h, const void *x_dev, int T, int32_t *idx_dev,
                               float *w_dev, int32_t *offsets_dev, int32_t *list_dev,
                               void *stream);

/* Layer forward: y = shared(x) + sum over the k picks in ascending expert id
 * of w_j * expert_j(x), accumulated in fp32 and rounded once to bf16, where
 * expert(x) = Wd (silu(Wg x) * (Wu x)).
 *   x_dev  bf16 [T][H] (device), y_dev bf16 [T][H] out (device); x and y must
 *          not overlap.
 * T <= 64 runs the decode kernels (bandwidth-bound grouped GEMV); larger T runs
 * the prefill kernels (tcgen05 tensor-core grouped GEMM).  T == 0 is a no-op.
 * Deterministic: the same inputs give the same bits on every call. */
strata_status strata_moe_forward(strata_moe_t h, const void *x_dev, int T, void *y_dev,
                                 void *stream);

/* End-to-end forward from host memory: copies x_host (bf16 [T][H]) to the
 * device, runs strata_moe_forward, copies the result to y_host (bf16 [T][H])
 * and synchronises `stream` before returning.  Pinned host buffers make the
 * copies asynchronous with respect to other streams.  Returns TIMEOUT if a
 * device-side wait ran out during the call. */
strata_status strata_moe_forward_host(strata_moe_t h, const void *x_host, int T, void *y_host,
                                      void *stream);

/* RMSNorm with weight 1 and eps 1e-6: xn = bf16(h * r),
 * r = 1/sqrtf(ss/H + 1e-6f), ss = fp32 sum of squares in the router's order.
 *   h_dev, xn_dev bf16 [T][H] (device); may not overlap. */
strata_status strata_moe_rmsnorm(const void *h_dev, void *xn_dev, int T, int H, void *stream);

/* 48-layer-style expert stack, in place: for each layer l in order,
 * h <- bf16(f32(h) + f32(MoE_l(RMSNorm(h)))).
 *   layers      n_layers handles of identical shape on one device
 *   h_dev       bf16 [T][H] (device), updated in place
 *   h_trace_dev bf16 [n_layers][T][H] out or NULL: the input of each layer
 * Every layer runs in layers[0]'s workspace, so layers[0] needs
 * max_tokens >= T; the other handles may be created with max_tokens = 1. */
strata_status strata_moe_stack_forward(const strata_moe_t *layers, int n_layers, void *h_dev,
                                       int T, void *h_trace_dev, void *stream);

/* Synchronise `stream`, then read and clear the handle's device error word.
 * Returns TIMEOUT if a bounded device-side wait ran out since the last check,
 * CUDA on an asynchronous CUDA error, OK otherwise. */
strata_status strata_moe_sync_status(strata_moe_t h, void *stream);

/* Message of the last failure on this thread ("" if none). */
const char *strata_moe_last_error(void);

/* Test hook: dequantised weights of rows [row0, row0+nrows) of matrix `mat`
 * (0 gate, 1 up, 2 down) of expert `expert` (-1 = the shared expert), read
 * back from the GPU layout by the device dequantiser.  kind 0: the exact value
 * d*(q-c) in fp32 (what the decode kernels use); kind 1: the fp16 tensor-core
 * operand (round to nearest even of the exact value).  out_host: float
 * [nrows][cols].  Synchronous. */
strata_status strata_moe_debug_dequant(strata_moe_t h, int expert, int mat, int row0, int nrows,
                                       int kind, float *out_host);

/* ---- Expert parallelism (experts of a layer split across ranks).
 * Rank r of N owns experts [e_begin, e_end) = [ceil(r E / N), ceil((r+1) E / N)),
 * i.e. expert e belongs to rank floor(e N / E); every rank keeps the router and
 * the shared expert.  One forward of a rank's T tokens (the Python layer
 * quantized_expert_ffn_04_b200.ep does this with torch.distributed
 * all-to-alls): route -> strata_ep_plan -> send each pick's token row and
 * expert id to the owner -> the owner runs strata_moe_expert_rows on what it
 * got -> outputs back in the same order -> strata_moe_combine_rows.  Each
 * expert output depends on one token row and one expert only, so the result
 * equals the one-GPU forward on the same kernels bit for bit (prefill =
 * T > 64; below, the decode GEMV chain, STRATA_OPT_PATH 1). */
strata_status strata_ep_expert_range(int rank, int n_ranks, int n_experts, int32_t *e_begin,
                                     int32_t *e_end);

/* Host only.  idx: int32 [T][k] picks (host).  Out (host, caller-owned):
 * send_counts [n_ranks] picks per destination rank; send_pick [T*k] the pick
 * index t*k+j of each row to send, grouped by destination rank, inside a rank
 * by expert id, then token (a stable, deterministic order); slot [T*k] the
 * position of pick t*k+j in that order.  INVALID_ARG on an id outside
 * [0, n_experts) or a bad size; nothing else can fail. */
strata_status strata_ep_plan(const int32_t *idx, int T, int k, int n_experts, int n_ranks,
                             int32_t *send_counts, int32_t *send_pick, int32_t *slot);

/* dst row i = src row rows[i] (device buffers, rows int32 [n]); row_bytes a
 * multiple of 16 and both buffers 16-byte aligned, else INVALID_ARG.  A row
 * index outside [0, n_src) is skipped.  Enqueued on `stream`. */
strata_status strata_ep_gather_rows(const void *src_dev, const int32_t *rows_dev, int n,
                                    int n_src, int row_bytes, void *dst_dev, void *stream);

/* Expert outputs of single rows: row i of x_dev (bf16 [n][H], device) goes
 * through expert ids_dev[i] (int32 [n], device; -1: none) and, for
 * i < n_shared, through the shared expert as well.
 *   y_dev        [n][H] out: row i = expert ids[i](x_i) (rows with id -1 untouched)
 *   yshared_dev  [n_shared][H] out: shared(x_i), or NULL when n_shared == 0
 * Outputs are in the row's prescaled units (times 2^-2e, e the row's token
 * prescale exponent), fp32 when prefill == 0 (the decode kernels) and fp16
 * when prefill != 0 (the tensor-core kernels): exactly the values the
 * one-GPU forward feeds its combine.  n <= max_tokens.  Enqueued on `stream`. */
strata_status strata_moe_expert_rows(strata_moe_t h, const void *x_dev, const int32_t *ids_dev,
                                     int n, int n_shared, int prefill, void *y_dev,
                                     void *yshared_dev, void *stream);

/* The layer's combine from expert outputs: out_t = shared + sum over the k
 * picks in ascending expert id of w_j * Y_j, times 2^2e (the token's
 * prescale, recomputed from x_dev), one rounding to bf16.
 *   x_dev   bf16 [T][H] the layer input (device)
 *   idx_dev int32 [T][k], w_dev float [T][k] the routing (device)
 *   slot_dev int32 [T][k]: row of y_dev holding pick (t, j)
 *   y_dev   [T*k + T][H] expert outputs, the shared expert's at row T*k + t;
 *           fp32 (prefill == 0) or fp16 (prefill != 0), as strata_moe_expert_rows
 *   out_dev bf16 [T][H] out.  Enqueued on `stream`. */
strata_status strata_moe_combine_rows(strata_moe_t h, const void *x_dev, int T,
                                      const int32_t *idx_dev, const float *w_dev,
                                      const int32_t *slot_dev, const void *y_dev, int prefill,
                                      void *out_dev, void *stream);

/* Test hook of the large-batch router (T > 256): the approximate logits
 * a[t][e] of its tensor-core screening GEMM (fp16 split of W, fp32
 * accumulation, plus the bias) and each token's error bound eps[t], so that a
 * test can measure |a - l| against eps for the exact fixed-order logits l
 * (the screen keeps every expert with a >= a_(k) - 2 eps; a token whose bound
 * is not finite or that has an entry beyond 65504 gets eps = 0 and keeps every
 * expert).  a_host float [T][E], eps_host float [T].  Needs a handle with
 * max_tokens > 256.  Synchronous. */
strata_status strata_moe_debug_screen(strata_moe_t h, const void *x_dev, int T, float *a_host,
                                      float *eps_host);

/* Test hooks for the out-of-memory paths.  Every device and pinned host
 * allocation of the library goes through one counter.
 * strata_moe_debug_fail_alloc(n), n >= 0: the n-th allocation from now (0 =
 * the next one) fails as if the device were out of memory, without
 * allocating; n = -1 switches the injection off.  Process-wide, not
 * thread-safe against concurrent creates; returns INVALID_ARG for n < -1.
 * strata_moe_debug_live_allocs(): the number of blocks the library holds now
 * (every handle's weights, workspace and pinned error word, plus any
 * transient staging buffer).  A create that fails returns with this number
 * unchanged and *out = NULL. */
strata_status strata_moe_debug_fail_alloc(int64_t n);
int64_t strata_moe_debug_live_allocs(void);

/* Options (strata_moe_set_option). */
enum {
    STRATA_OPT_PATH = 1,        /* 0 auto (default: T <= DECODE_MAX_T runs the fused decode
                                   kernel where it applies, else the decode GEMV chain; larger T
                                   the prefill GEMM), 1 force the decode GEMV kernel chain,
                                   2 force the prefill GEMM, 3 force the fused decode kernel
                                   (T <= 64, E <= 512, k <= 16, H and I multiples of 128, and
                                   its shared-memory plan must give every compute group a ring
                                   slot; auto mode takes the chain for shapes that do not fit,
                                   a forced forward fails with STRATA_ERR_INVALID_ARG) */
    STRATA_OPT_WAIT_BUDGET = 2, /* bound of every device-side wait, in SM clock cycles
                                   (default 4e9); 0 makes every wait give up at once */
    STRATA_OPT_DECODE_MAX_T = 3 /* largest T run by the decode kernels in auto mode (default 64) */
};
strata_status strata_moe_set_option(strata_moe_t h, int option, int64_t value);

/* Self-test of the timeout path: launches one kernel that waits on a barrier
 * nothing completes, bounded by `budget_cycles`, and reports the outcome the
 * way real kernels do.  Returns TIMEOUT when the bound worked.  Synchronous. */
strata_status strata_moe_selftest_wait(int device, int64_t budget_cycles);

/* Profiling hook: make every later forward of `h` record CUDA event
 * `ev_begin` (a cudaEvent_t passed as void*) on the call's stream just before
 * the kernel(s) of `stage` and `ev_end` just after them.  Stages: 0 router
 * (for T > 256: the fp16 token copy, the screening GEMM and the screened
 * top-k), 1 top-k + dispatch (T <= 256, one kernel), 2 dispatch (T > 256),
 * 3 gate/up + SwiGLU (on the prefill path with T <= 256 also the fp16 token
 * copy), 4 down, 5 combine.  NULL events
 * switch the probe off.  The events must be created by the caller on the
 * handle's device (with timing enabled); forwards captured into a CUDA graph
 * capture the event records too. */
strata_status strata_moe_set_probe(strata_moe_t h, int stage, void *ev_begin, void *ev_end);

/* Number of kernels one strata_moe_forward of T tokens launches (0 on error). */
int strata_moe_launch_count(strata_moe_t h, int T);

/* Routing for callers that cannot allocate device memory (code running inside
 * another framework's memory pool, code on a fixed memory budget, or code that
 * must not trigger the implicit synchronisation cudaMalloc/cudaFree can cause).
 * The pages have no counterpart: this is a property of the library, not of the
 * method.  Same results as strata_moe_route, without a handle:
 *   x_dev         bf16 [T][H] (device, 16-byte aligned)
 *   router_w_dev  float [E][H] plain row-major router weight (device)
 *   router_b_dev  float [E] (device) or NULL for no bias
 *   idx_dev, w_dev, offsets_dev (or NULL), list_dev (or NULL): as in
 *                 strata_moe_route
 * Limits: 1 <= T <= 64 (T == 0 is a no-op), 1 <= E <= 1024,
 * 1 <= k <= min(E, 32), H a multiple of 128 in [128, 6144]; anything else
 * returns STRATA_ERR_INVALID_ARG without launching work.
 * Intermediates live in one static device array of about 0.4 MB that every GPU
 * loading this library keeps until the process exits; the call allocates
 * nothing.  The first call on a device looks up that array's device address
 * (and sets kernel attributes), so make it before any stream capture.  Every
 * call shares the array, and nothing in it needs to start at zero: each call
 * overwrites what it reads.  Two calls that overlap on the GPU (different
 * streams, or different host threads) race on the array. */
strata_status strata_moe_route_noalloc(const void *x_dev, int T, int H,
                                       const float *router_w_dev, const float *router_b_dev,
                                       int E, int k, int32_t *idx_dev, float *w_dev,
                                       int32_t *offsets_dev, int32_t *list_dev, void *stream);

/* Library version string. */
const char *strata_moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STRATA_MOE_H */
