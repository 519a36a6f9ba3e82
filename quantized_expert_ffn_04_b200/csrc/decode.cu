// Fused decode layer (T <= 64 tokens): the whole mixture-of-experts layer in
// ONE persistent kernel, one CTA per SM: router logits, top-k, dispatch,
// gate/up + SwiGLU, down and the fixed-order combine.
//
// Layer specification (the same steps as the multi-kernel path):
//   logit[t][e] = sum_i x[t][i] W[e][i] + b[e] in fp32 in the fixed order (32
//   lane partials over i = l, l+32, ..., fma in ascending i, then a halving
//   tree); picks = the k largest logits, a tie to the lower expert id;
//   w_j = exp(l_j - m) / sum over the picks; units = (expert, up to 8 of its
//   tokens), the shared expert's units first; a = silu(Wg x) * Wu x,
//   y = Wd a with w = d (q - c) from the block-32 codes; out = y_shared + sum
//   over the picks in ascending expert id of w_j y_j (fp32), rounded once to
//   bf16.  The pages: 10 routed + 1 shared expert per token ("Strata Runs 125B
//   Qwen3.8-Flash-Next on a 12GB Gaming GPU at Up to 94 Tokens/s", section
//   "What it is"), routers and shared experts on the GPU (section "How a 125B
//   model fits in 12 GB"), decode of one token or a small multi-token-
//   prediction batch (section "The numbers, measured by the author").
//
// Why one kernel: at T = 1..4 the layer moves 20-55 MB, ~3-9 us of HBM time,
// so every dependent step costs as much as the traffic.  The structure:
//   * warp roles: 16 compute warps (4 groups of 4), a copy warp that streams
//     packed weights into a ring of shared-memory slots with 1-D bulk copies,
//     a publish warp and a fetch warp (below);
//   * prologue: the copy warp requests this CTA's slice of the router weight
//     (E / #SMs experts) and, for T <= 8, the shared expert's gate/up slabs
//     assigned to this CTA, before the previous kernel has finished
//     (programmatic dependent launch): neither depends on routing;
//   * router: each CTA computes the logits of its experts for every token;
//     one grid-wide barrier (a monotonic counter, bounded waits; the launch
//     is cooperative, so every CTA is resident) makes all logits visible;
//     meanwhile the compute groups run the shared expert's gate/up slabs;
//   * top-k and dispatch: every CTA runs them itself (identical and
//     deterministic), for T > 16 tokens the top-k is split over CTAs with a
//     second barrier;
//   * items: the list [routed gate/up slabs (unit, 16 rows)] + [down blocks
//     (unit, 128 rows)] is claimed item by item from one counter per launch
//     (two counter sets alternate by launch parity), so all CTAs work on
//     neighbouring units, a unit's gate/up slabs are all done long before
//     its down blocks come up, and a CTA that finishes early takes more;
//   * four groups of 4 compute warps take ring positions in turn; the 4
//     warps of a group each take a share of the item (a quarter of K of both
//     the gate and the up slab; two slabs of a down block, so one token
//     fragment serves both) and run independently: no barrier inside the
//     item loop, and a ring slot is free as soon as its last warp is done,
//     so most of the ring is in flight; the last warp to finish an item
//     completes it (sums the partial products in a fixed order and applies
//     SwiGLU, or stores the block's rows and counts them for the combine);
//   * the publish warp turns finished gate/up slabs into per-unit counts
//     (one gpu-scope fence per batch), and the fetch warp waits for the
//     counts a down block needs and copies that unit's activation rows in,
//     so the compute warps never wait on a fence or a remote counter;
//   * the down block that completes the last expert rows of a (token,
//     128-row block) pair combines that block of the token in the fixed order.
// The math of a block: mma.sync as the in-warp reduction with fp32 per-block
// scaling.  Gate/up (2-bit) take the magic-offset form (block_mma2m: the codes
// go into the fp16 mantissa with one mask each, and the constant offset is
// taken out through the accumulator with a precomputed per-(token, block)
// correction); the down blocks and the 3-bit weights use the exact small
// integers 2q - (2^bits - 1).  Every wait is bounded; on expiry the CTA records a timeout in the
// error word, lets its copies land and returns.
#include "common.cuh"
#include "internal.h"
#include "topk.cuh"

namespace strata {

constexpr int kFWarps = 16;                     // compute warps
constexpr bool kFExtras = false;                // shared-expert slabs before routing
constexpr int kGWarps = 4;                      // warps of a compute group (one item at a time)
constexpr int kGroups = kFWarps / kGWarps;      // the groups take ring positions in turn
constexpr int kDH = kGWarps / 4;                // K splits of a down block's slab pairs
constexpr int kFCompute = 32 * kFWarps;         // compute threads
constexpr int kWCopy = kFWarps, kWPub = kFWarps + 1, kWFetch = kFWarps + 2, kWComb = kFWarps + 3;
constexpr int kFThreads = 32 * (kFWarps + 4);
constexpr int kFTile = 8;                       // tokens per unit (mma N)
constexpr int kFMaxRing = 8;
constexpr int kDownSlabs = 8;                   // a down block: 8 slabs = 128 rows
constexpr int kFStagedMaxT = 8;                 // token rows kept in shared memory
constexpr int kFMaxT = 64;                      // most tokens per call
constexpr int kFMaxK = 16;                      // most routed experts per token
constexpr int kTopkLocalT = 16;                 // up to here every CTA runs the whole top-k
constexpr int kPubQ = 64;                       // publish queue entries
constexpr int kMaxA = 4;                        // activation buffers (one down block each)
constexpr int kRedSlot = kGWarps * 32 * 8 * 4;  // partial sums of one ring slot (bytes)

// item kinds in a ring slot's meta word
constexpr int kItemEnd = -1;
constexpr int kKindExtra = 1, kKindGU = 2, kKindDown = 3;
__host__ __device__ inline int item_kind(int m) { return (m >> 28) & 7; }

struct FusedParams {
    const __nv_bfloat16 *x;   // [T][H] layer input
    const float4 *Wp;         // router weight, [E][H/128][32 lanes] float4 (lane-interleaved)
    const float *bias;        // [E] or null
    const uint8_t *routed;
    const uint8_t *shared;
    size_t expert_bytes, mat_bytes;
    int T, E, k, H, Ip, nseg_h, nseg_i;
    int ring, item_bytes, staged, units_max, na;
    float w2;                 // bound of every gate/up row's L2 norm (token prescale), 0: none
    float *logits;            // [T][E]
    int32_t *idx;             // [T][k] picks (T > kTopkLocalT: exchanged between CTAs)
    float *wts;               // [T][k]
    __half *x16;              // [T][H] fp16 token operand (T > kFStagedMaxT)
    float *corr;              // [T][H / 32] its block corrections (T > kFStagedMaxT, 2-bit)
    int *xex;                 // [T] token prescale exponents (T > kFStagedMaxT)
    __half *a;                // [slots][Ip]
    float *Y;                 // [slots][H] (scaled by 2^(-2 ex) of the token)
    __nv_bfloat16 *out;       // [T][H]
    int residual;
    unsigned long long *bar;  // grid barrier counter, 2 arrivals per CTA per launch
    int *cnt;                 // two counter sets of cnt_stride ints, used alternately
    int cnt_stride;           // ints per set: finished gate/up slabs per unit, then
    int cnt_tok;              // (at this offset) finished down blocks per (token, row block)
    int *err;
    long long budget;
};

// Shared-memory carve (host and device agree on it).
struct FusedSmem {
    int ring, red, xs, corr, rega, sidx, sw, sslot, sord, mask, soff, units, slist, sex, misc,
        bars, total;
};

__host__ __device__ inline int align16(int v) { return (v + 15) & ~15; }
__host__ __device__ inline int imax(int a, int b) { return a > b ? a : b; }

__host__ __device__ inline FusedSmem fused_smem(int T, int E, int k, int H, int Ip, int ring,
                                                int item_bytes, int staged, int units_max,
                                                int na) {
    FusedSmem s;
    int o = 0;
    s.ring = o;  o += ring * item_bytes;
    // partial sums of the warps, per ring slot; while routing it holds the
    // lane-interleaved bf16 copy of the token rows that the router reads
    s.red = o;   o += ring * kRedSlot;
    s.xs = o;    o += staged ? align16(T * (H + 8) * 2) : 0;
    s.corr = o;  o += staged ? align16((H / 32) * kFTile * 4) : 0;
    // the raw bf16 token rows while routing, then the activation buffers
    s.rega = o;  o += imax(staged ? align16(T * H * 2) : 0, na * kFTile * (Ip + 8) * 2);
    s.sidx = o;  o += align16(T * k * 4);
    s.sw = o;    o += align16(T * k * 4);
    s.sslot = o; o += align16(T * k * 4);
    s.sord = o;  o += align16(T * k * 4);
    s.mask = o;  o += align16(E * 8);
    s.soff = o;  o += align16(E * 4);
    s.units = o; o += units_max * 16;
    s.slist = o; o += align16(T * k * 4);
    s.sex = o;   o += align16(T * 4);
    s.misc = o;  o += 256 * 4;
    s.bars = o;  o += 8 * (2 * kFMaxRing + 8 + 2 * kMaxA);
    s.total = o;
    return s;
}

// misc ints
constexpr int kMiscAbort = 0, kMiscScan = 1 /* 33 */, kMiscNUnits = 34, kMiscUtot = 35,
              kMiscPar = 36, kMiscDead = 37, kMiscCFlag = 38, kMiscTmp = 39,
              kMiscGCnt = 40 /* kFMaxRing: warps done with the item in a slot */,
              kMiscMeta = 48 /* kFMaxRing */, kMiscPubN = 56, kMiscPubSeen = 57,
              kMiscWarpsDone = 58, kMiscCombN = 59, kMiscCombSeen = 60,
              kMiscPubQ = 64 /* kPubQ */, kMiscCombQ = 128 /* kPubQ */,
              kMiscDownN = 192, kMiscDownEnd = 193, kMiscDownSeen = 194,
              kMiscDownQ = 196 /* kDownQ */;
constexpr int kDownQ = 32;  // claimed down items handed from the copy warp to the fetch warp

// Named barrier 1: the compute warps.
STRATA_DEV void compute_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kFCompute) : "memory"); }

// Exclusive scan of one int per compute thread over the compute warps.
__device__ int compute_exclusive_scan(int v, int *scratch, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) scratch[warp] = incl;
    compute_sync();
    if (warp == 0) {
        int s = lane < kFWarps ? scratch[lane] : 0, si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, si, o);
            if (lane >= o) si += n;
        }
        if (lane < kFWarps) scratch[lane] = si - s;
        if (lane == 31) scratch[32] = si;
    }
    compute_sync();
    const int r = scratch[warp] + incl - v;
    *total = scratch[32];
    compute_sync();
    return r;
}

// B fragment source of a 32-wide block at column k0 (mma m16n8k16, fp16):
// lane 4g + c needs x[token g][k0 + 8m + 2c], x[..+1] in register m = 0..3.
//   kSrcSmem:  rows staged in shared memory, fetched with one ldmatrix
//              (rowp = this lane's row for matrix row lane & 7);
//   kSrcLdg:   read-only global rows through L1 (rowp = row of token lane >> 2).
constexpr int kSrcSmem = 0, kSrcLdg = 1;

template <int kSrc>
STRATA_DEV void b_frag(const __half *rowp, int k0, int lane, uint32_t &b0, uint32_t &b1,
                       uint32_t &b2, uint32_t &b3) {
    if (kSrc == kSrcSmem) {
        ldmatrix_x4(b0, b1, b2, b3, rowp + k0 + (lane >> 3) * 8);
    } else {
        const uint32_t *p = reinterpret_cast<const uint32_t *>(rowp + k0 + 2 * (lane & 3));
        b0 = __ldg(p);
        b1 = __ldg(p + 4);
        b2 = __ldg(p + 8);
        b3 = __ldg(p + 12);
    }
}

// acc (16 rows x 8 token columns, fp32 fragment) += blocks [b0, b1) of one
// 16-row slab held in shared memory at `slab` (units of 128 columns) against
// the token rows from rowp.  kMagic: the 2-bit magic-offset form
// (block_mma2m; the token operand carries the column factors, ca/cb give the
// block corrections of the lane's two token columns, and acc comes out times
// 2^8); otherwise the exact small integers 2q - (2^bits - 1) (acc times 2).
// One block against the B fragment: dequantise (exact integers, or the
// magic-offset form with the block corrections c0 / c1) and two mma.
template <int kBits, bool kMagic>
STRATA_DEV void block_dot(float (&d)[4], uint32_t lo, uint32_t hi, int hshift, uint32_t b0,
                          uint32_t b1, uint32_t b2, uint32_t b3, float c0, float c1) {
    if (kMagic)
        block_mma2m<kBits>(d, lo, b0, b1, b2, b3, c0, c1);
    else if (kBits <= 2)
        block_mma2<kBits>(d, lo, b0, b1, b2, b3);
    else
        block_mma<kBits>(d, lo, hi, hshift, b0, b1, b2, b3);
}

// acc0 / acc1 (16 rows x 8 token columns, fp32 fragments) += blocks [b0, b1)
// of two 16-row slabs held in shared memory at s0 and s1 (units of 128
// columns) against the same token rows from rowp: one B fragment per block
// serves both slabs.  b0 is even, so every pair of blocks sits inside one
// unit; blocks go four at a time with no branch between them (eight
// independent mma chains), each pair's code words and scales coming in with
// one 8-byte load per slab (lane 4g + c holds its code words; the scales of
// rows g and g + 8).  kMagic: the 2-bit magic-offset form (block_mma2m; the
// token operand carries the column factors, ca[b] / cb[b] are the block
// corrections of the lane's two token columns, and the sums come out times
// 2^8); otherwise the exact small integers 2q - (2^bits - 1) (sums times 2).
template <int kBits, int kSrc, bool kMagic>
STRATA_DEV void slab2_blocks(float (&acc0)[4], float (&acc1)[4], const uint8_t *s0,
                             const uint8_t *s1, int b0, int b1, const __half *rowp,
                             const float *ca, const float *cb, int lane) {
    constexpr int UB = unit_bytes(kBits);
    constexpr int SOFF = scale_off(kBits);
    const int g = lane >> 2;
    int b = b0;
    for (; b + 4 <= b1; b += 4) {
        uint2 lw[2][2], kw[2][2];   // [pair][slab]: code words, scale words
        uint32_t hw[2][2];          // 3-bit: the high-bit word of each pair
#pragma unroll
        for (int pp = 0; pp < 2; pp++) {
            const int bp = b + 2 * pp;
            const int off = (bp >> 2) * UB, wo = (bp & 3) * 4;
            if (kBits == 1) {  // one word, both blocks of the pair (odd one a bit higher)
                const uint32_t v0 = *reinterpret_cast<const uint32_t *>(s0 + off + lane * 8 + wo / 2);
                const uint32_t v1 = *reinterpret_cast<const uint32_t *>(s1 + off + lane * 8 + wo / 2);
                lw[pp][0] = make_uint2(v0, v0 >> 1);
                lw[pp][1] = make_uint2(v1, v1 >> 1);
            } else {
                lw[pp][0] = *reinterpret_cast<const uint2 *>(s0 + off + lane * 16 + wo);
                lw[pp][1] = *reinterpret_cast<const uint2 *>(s1 + off + lane * 16 + wo);
            }
            kw[pp][0] = *reinterpret_cast<const uint2 *>(s0 + off + SOFF + g * 16 + wo);
            kw[pp][1] = *reinterpret_cast<const uint2 *>(s1 + off + SOFF + g * 16 + wo);
            if (kBits == 3) {
                hw[pp][0] = *reinterpret_cast<const uint32_t *>(s0 + off + kLoBytes + lane * 8 + wo / 2);
                hw[pp][1] = *reinterpret_cast<const uint32_t *>(s1 + off + kLoBytes + lane * 8 + wo / 2);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int pp = i >> 1, e = i & 1;
            uint32_t bb0, bb1, bb2, bb3;
            b_frag<kSrc>(rowp, (b + i) * 32, lane, bb0, bb1, bb2, bb3);
            const float c0 = kMagic ? ca[b + i] : 0.0f, c1 = kMagic ? cb[b + i] : 0.0f;
            float d0[4], d1[4];
            block_dot<kBits, kMagic>(d0, e ? lw[pp][0].y : lw[pp][0].x,
                                     kBits == 3 ? hw[pp][0] : 0u, 8 * e, bb0, bb1, bb2, bb3, c0,
                                     c1);
            block_dot<kBits, kMagic>(d1, e ? lw[pp][1].y : lw[pp][1].x,
                                     kBits == 3 ? hw[pp][1] : 0u, 8 * e, bb0, bb1, bb2, bb3, c0,
                                     c1);
            const uint32_t w0 = e ? kw[pp][0].y : kw[pp][0].x;
            const uint32_t w1 = e ? kw[pp][1].y : kw[pp][1].x;
            const float2 f0 = __half22float2(*reinterpret_cast<const __half2 *>(&w0));
            const float2 f1 = __half22float2(*reinterpret_cast<const __half2 *>(&w1));
            acc0[0] = fmaf(f0.x, d0[0], acc0[0]);
            acc0[1] = fmaf(f0.x, d0[1], acc0[1]);
            acc0[2] = fmaf(f0.y, d0[2], acc0[2]);
            acc0[3] = fmaf(f0.y, d0[3], acc0[3]);
            acc1[0] = fmaf(f1.x, d1[0], acc1[0]);
            acc1[1] = fmaf(f1.x, d1[1], acc1[1]);
            acc1[2] = fmaf(f1.y, d1[2], acc1[2]);
            acc1[3] = fmaf(f1.y, d1[3], acc1[3]);
        }
    }
    // the last one to three blocks, one at a time
    for (; b < b1; b++) {
        const uint8_t *u0 = s0 + (b >> 2) * UB, *u1 = s1 + (b >> 2) * UB;
        const int blk = b & 3;
        const uint32_t lw0 = unit_word<kBits>(u0, lane, blk);
        const uint32_t lw1 = unit_word<kBits>(u1, lane, blk);
        const uint32_t kw0 = *reinterpret_cast<const uint32_t *>(u0 + SOFF + g * 16 + blk * 4);
        const uint32_t kw1 = *reinterpret_cast<const uint32_t *>(u1 + SOFF + g * 16 + blk * 4);
        uint32_t hw0 = 0, hw1 = 0;
        if (kBits == 3) {
            hw0 = *reinterpret_cast<const uint32_t *>(u0 + kLoBytes + lane * 8 + (blk >> 1) * 4);
            hw1 = *reinterpret_cast<const uint32_t *>(u1 + kLoBytes + lane * 8 + (blk >> 1) * 4);
        }
        uint32_t bb0, bb1, bb2, bb3;
        b_frag<kSrc>(rowp, b * 32, lane, bb0, bb1, bb2, bb3);
        const float c0 = kMagic ? ca[b] : 0.0f, c1 = kMagic ? cb[b] : 0.0f;
        float d0[4], d1[4];
        block_dot<kBits, kMagic>(d0, lw0, hw0, 8 * (blk & 1), bb0, bb1, bb2, bb3, c0, c1);
        block_dot<kBits, kMagic>(d1, lw1, hw1, 8 * (blk & 1), bb0, bb1, bb2, bb3, c0, c1);
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2 *>(&kw0));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2 *>(&kw1));
        acc0[0] = fmaf(f0.x, d0[0], acc0[0]);
        acc0[1] = fmaf(f0.x, d0[1], acc0[1]);
        acc0[2] = fmaf(f0.y, d0[2], acc0[2]);
        acc0[3] = fmaf(f0.y, d0[3], acc0[3]);
        acc1[0] = fmaf(f1.x, d1[0], acc1[0]);
        acc1[1] = fmaf(f1.x, d1[1], acc1[1]);
        acc1[2] = fmaf(f1.y, d1[2], acc1[2]);
        acc1[3] = fmaf(f1.y, d1[3], acc1[3]);
    }
}

// Bounded wait for an mbarrier phase by one thread; false (and the error
// word set) when the budget runs out or another thread gave up already.
STRATA_DEV bool fwait(uint64_t *bar, uint32_t parity, const FusedParams &p,
                      volatile int *abort_flag) {
    long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity, 1000)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > p.budget) {
            atomicCAS(p.err, 0, kErrTimeout);
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

// The same wait for a whole warp: lane 0 waits, every lane gets its verdict.
STRATA_DEV bool warp_fwait(uint64_t *bar, uint32_t parity, const FusedParams &p,
                           volatile int *abort_flag, int lane) {
    int ok = 0;
    if (lane == 0) ok = fwait(bar, parity, p, abort_flag) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Bounded wait until a global counter reaches `target` (acquire).
STRATA_DEV bool fwait_count(const int *cnt, int target, const FusedParams &p,
                            volatile int *abort_flag) {
    long long t0 = clock64();
    while (true) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
        if (v >= target) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > p.budget) {
            atomicCAS(p.err, 0, kErrTimeout);
            *abort_flag = 1;
            return false;
        }
        __nanosleep(128);
    }
}

// Grid barrier: arrive (release), then wait (acquire, bounded) until the
// counter reaches `target`.
STRATA_DEV bool grid_barrier(unsigned long long *bar, unsigned long long target,
                             const FusedParams &p, volatile int *abort_flag) {
    asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(bar) : "memory");
    long long t0 = clock64();
    while (true) {
        unsigned long long v;
        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(bar) : "memory");
        if (v >= target) return true;
        if (clock64() - t0 > p.budget) {
            atomicCAS(p.err, 0, kErrTimeout);
            *abort_flag = 1;
            return false;
        }
        __nanosleep(32);
    }
}


// The expert token operand of column i of a token row, and the block
// correction of the magic-offset form (2-bit): B_i = fp16(x_i 2^-ex s(i mod 32)),
// corr = -sum over the block's 32 columns, in ascending order, of c(kk) B.
template <int kBits>
STRATA_DEV __half token_operand(float x, int ex, int i) {
    const float v = x * pow2f(-ex);
    return __float2half_rn(kBits <= 2 ? v * magic_col_scale(i & 31) : v);
}
// The correction of one block: the four column groups (one factor each) are
// summed in order, then combined: corr = sum over g of -c_g (sum of B in g).
template <int kBits>
STRATA_DEV float block_correction(const __nv_bfloat16 *blk, int ex) {
    float v = 0.0f;
#pragma unroll
    for (int gq = 0; gq < 4; gq++) {
        float gs = 0.0f;
#pragma unroll
        for (int kk = 8 * gq; kk < 8 * gq + 8; kk++)
            gs += __half2float(token_operand<kBits>(__bfloat162float(blk[kk]), ex, kk));
        v = fmaf(-magic_col_corr(8 * gq, kBits), gs, v);
    }
    return v;
}

// One staged block (32 columns) of a token by one thread: the expert operand
// B = fp16(x 2^-ex s(k)) written to dst, and (magic form) the block's
// correction, in the same order as block_correction.
template <int kBits>
STRATA_DEV void stage_block(const __nv_bfloat16 *src, __half *dst, int ex, float *corr) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
    const float sc = pow2f(-ex);
    float v = 0.0f;
#pragma unroll
    for (int gq = 0; gq < 4; gq++) {
        const uint4 in = s4[gq];
        const uint32_t w[4] = {in.x, in.y, in.z, in.w};
        const float f = kBits <= 2 ? magic_col_scale(8 * gq) : 1.0f;
        uint32_t o[4];
        float gs = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const __half2 h = __floats2half2_rn(bf16_lo(w[j]) * sc * f, bf16_hi(w[j]) * sc * f);
            o[j] = *reinterpret_cast<const uint32_t *>(&h);
            gs += __low2float(h);
            gs += __high2float(h);
        }
        d4[gq] = make_uint4(o[0], o[1], o[2], o[3]);
        v = fmaf(-magic_col_corr(8 * gq, kBits), gs, v);
    }
    if (kBits <= 2) *corr = v;
}


// The ring items of one compute warp: its group's positions jpos,
// jpos + kGroups, ... up to `stop`.  Returns the next position, or -1 once the end marker is
// seen or the launch aborts.  One non-inlined copy serves both calls (the
// shared expert's slabs before routing, then the routed items), so the hot
// loop exists once per kernel instantiation and stays in the instruction
// caches next to the other roles' loops.
//   gate/up slab: warp q of the group takes a quarter of K of both the gate
//   and the up slab; down block: warp q the slabs 2q and 2q + 1, all of K; the
//   last of the group's 4 warps to finish an item completes it.
template <int kBits, bool kStaged>
__device__ __noinline__ int fused_run_items(const FusedParams &p, int jpos, int stop) {
    extern __shared__ __align__(128) uint8_t sm[];
    constexpr int UB = unit_bytes(kBits);
    constexpr bool kMagic = kBits <= 2;  // magic-offset gate/up (1- and 2-bit)
    constexpr bool staged = kStaged;
    const FusedSmem L = fused_smem(p.T, p.E, p.k, p.H, p.Ip, p.ring, p.item_bytes, p.staged,
                                   p.units_max, p.na);
    uint8_t *ring = sm + L.ring;
    float *red = reinterpret_cast<float *>(sm + L.red);
    __half *xs = reinterpret_cast<__half *>(sm + L.xs);
    float *scorr = reinterpret_cast<float *>(sm + L.corr);
    __half *abuf0 = reinterpret_cast<__half *>(sm + L.rega);
    int4 *units = reinterpret_cast<int4 *>(sm + L.units);
    int *slist = reinterpret_cast<int *>(sm + L.slist);
    int *sex = reinterpret_cast<int *>(sm + L.sex);
    int *misc = reinterpret_cast<int *>(sm + L.misc);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + L.bars);
    uint64_t *empty = full + kFMaxRing;
    uint64_t *abar = empty + kFMaxRing + 8;
    uint64_t *aempty = abar + kMaxA;
    volatile int *abort_flag = misc + kMiscAbort;
    volatile int *vmisc = misc;
    const int lane = threadIdx.x & 31, q = (threadIdx.x >> 5) % kGWarps;
    const int g = lane >> 2, cq = lane & 3;
    const int T = p.T, H = p.H, Tk = T * p.k;
    const int nbh = H / 32, nbi = p.Ip / 32;
    const int nsl = p.Ip / kSlabRows;              // gate/up slabs per unit
    const int ndn = H / (kSlabRows * kDownSlabs);  // down blocks per unit
    const int nsh = (T + kFTile - 1) / kFTile;     // shared-expert units
    const size_t gu_bytes = (size_t)p.nseg_h * UB;

auto slot_exp = [&](int sl) -> int {  // the prescale exponent of a slot's token
    const int t = sl < Tk ? slist[sl] : sl - Tk;
    return staged ? sex[t] : __ldcg(p.xex + t);
};
auto slot_tok = [&](int sl) -> int { return sl < Tk ? slist[sl] : sl - Tk; };
// count this warp in for the item in `slot`; true for the last of the group
auto last_warp = [&](int slot) -> bool {
    int old = 0;
    if (lane == 0) {
        __threadfence_block();
        old = atomicAdd(misc + kMiscGCnt + slot, 1);
        if (old == kGWarps - 1) {
            misc[kMiscGCnt + slot] = 0;  // before the slot can be refilled
            __threadfence_block();
        }
    }
    const bool last = __shfl_sync(0xffffffffu, old, 0) == kGWarps - 1;
    __syncwarp();
    return last;
};
    for (; jpos < stop; jpos += kGroups) {
        const int slot = jpos % p.ring;
        if (!warp_fwait(&full[slot], (jpos / p.ring) & 1, p, abort_flag, lane)) return -1;
        const int meta = vmisc[kMiscMeta + slot];
        if (meta == kItemEnd) return -1;
        const int kind = item_kind(meta);
        int u, part, slot0, n;
        if (kind == kKindExtra) {
            const int i = meta & 0xfffffff;
            u = i / nsl;
            part = i % nsl;
            slot0 = Tk + u * kFTile;
            n = T - u * kFTile < kFTile ? T - u * kFTile : kFTile;
        } else {
            const int ug0 = kFExtras && staged ? nsh : 0;
            if (kind == kKindGU) {
                const int it = meta & 0xfffffff;
                u = ug0 + it / nsl;
                part = it % nsl;
            } else {
                const int d = meta & 0xfffff;
                u = d / ndn;
                part = d % ndn;
            }
            const int4 un = units[u];
            slot0 = un.y;
            n = un.z;
        }
        const uint8_t *w = ring + (size_t)slot * p.item_bytes;
        float *rd = red + (size_t)slot * (kRedSlot / 4);  // [warp of group][lane][8]
        float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
        if (kind != kKindDown) {
            // ---------------------------------- gate/up slab, K quarter q
            // pairs of blocks: every range starts at an even block
            const int b0 = 2 * (q * (nbh / 2) / kGWarps), b1 = 2 * ((q + 1) * (nbh / 2) / kGWarps);
            // the lane's two token columns (columns past n repeat token 0)
            const int ta = slot_tok(slot0 + (2 * cq < n ? 2 * cq : 0));
            const int tb = slot_tok(slot0 + (2 * cq + 1 < n ? 2 * cq + 1 : 0));
            if constexpr (kStaged) {
                const int r = lane & 7;
                const __half *rowp = xs + (size_t)slot_tok(slot0 + (r < n ? r : 0)) * (H + 8);
                slab2_blocks<kBits, kSrcSmem, kMagic>(a0, a1, w, w + gu_bytes, b0, b1, rowp,
                                                      scorr + ta * nbh, scorr + tb * nbh, lane);
            } else {
                const __half *rowp = p.x16 + (size_t)slot_tok(slot0 + (g < n ? g : 0)) * H;
                slab2_blocks<kBits, kSrcLdg, kMagic>(a0, a1, w, w + gu_bytes, b0, b1, rowp,
                                                     p.corr + (size_t)ta * nbh,
                                                     p.corr + (size_t)tb * nbh, lane);
            }
            float4 *rq = reinterpret_cast<float4 *>(rd + ((size_t)q * 32 + lane) * 8);
            rq[0] = make_float4(a0[0], a0[1], a0[2], a0[3]);
            rq[1] = make_float4(a1[0], a1[1], a1[2], a1[3]);
            __syncwarp();
            if (!last_warp(slot)) {
                if (lane == 0) mbar_arrive(&empty[slot]);  // weights consumed
                continue;
            }
            // the last warp: the K quarters in a fixed order, then SwiGLU
            float gs[4] = {0.f, 0.f, 0.f, 0.f}, us[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < kGWarps; j++) {
                const float4 *rj = reinterpret_cast<const float4 *>(rd + ((size_t)j * 32 + lane) * 8);
                const float4 vg = rj[0], vu = rj[1];
                gs[0] += vg.x; gs[1] += vg.y; gs[2] += vg.z; gs[3] += vg.w;
                us[0] += vu.x; us[1] += vu.y; us[2] += vu.z; us[3] += vu.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);  // weights and partials consumed
            // undo the operand factor: 2^8 (magic-offset form) or 2 (exact integers)
            const float back = kMagic ? 1.0f / 256.0f : 0.5f;
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const int tok = 2 * cq + (i & 1);
                const float gv = gs[i] * back, uv = us[i] * back;
                // silu of the true gate value; the product stays in the
                // token's prescaled units (times 2^-2ex)
                const int ex = slot_exp(slot0 + (tok < n ? tok : 0));
                const float av = swiglu_ps(gv, uv, ex);
                const int row = part * kSlabRows + g + 8 * (i >> 1);
                if (tok < n) p.a[(size_t)(slot0 + tok) * p.Ip + row] = __float2half_rn(av);
            }
            __syncwarp();
            if (lane == 0) {
                // post the slab's unit for the publish warp (CTA scope)
                __threadfence_block();
                const int idx = atomicAdd(misc + kMiscPubN, 1);
                long long t0 = clock64();
                while (idx - vmisc[kMiscPubSeen] >= kPubQ) {
                    if (*abort_flag || clock64() - t0 > p.budget) {
                        atomicCAS(p.err, 0, kErrTimeout);
                        *abort_flag = 1;
                        break;
                    }
                }
                vmisc[kMiscPubQ + idx % kPubQ] = u + 1;
            }
        } else {
            // ---- down block: slabs 2 (q / kDH) + {0, 1}, K part q % kDH of kDH
            const int kd = (meta >> 20) & 0xff, b = kd % p.na;
            if (!warp_fwait(&abar[b], (kd / p.na) & 1, p, abort_flag, lane)) return -1;
            const __half *abuf = abuf0 + (size_t)b * kFTile * (p.Ip + 8);
            const int ar = lane & 7, pr = q / kDH, h = q % kDH;
            const __half *rowp = abuf + (size_t)(ar < n ? ar : 0) * (p.Ip + 8);
            const uint8_t *s0 = w + (size_t)(2 * pr) * p.nseg_i * UB;
            slab2_blocks<kBits, kSrcSmem, false>(a0, a1, s0, s0 + (size_t)p.nseg_i * UB,
                                                 2 * (h * (nbi / 2) / kDH), 2 * ((h + 1) * (nbi / 2) / kDH), rowp, nullptr,
                                                 nullptr, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&aempty[b]);  // activation rows consumed
            float4 *rq = reinterpret_cast<float4 *>(rd + ((size_t)q * 32 + lane) * 8);
            rq[0] = make_float4(a0[0], a0[1], a0[2], a0[3]);
            rq[1] = make_float4(a1[0], a1[1], a1[2], a1[3]);
            __syncwarp();
            if (!last_warp(slot)) {
                if (lane == 0) mbar_arrive(&empty[slot]);  // weights consumed
                continue;
            }
            // the last warp: the K parts of every slab, in a fixed order
#pragma unroll
            for (int pp = 0; pp < kDownSlabs / 2; pp++) {
#pragma unroll
                for (int sl = 0; sl < 2; sl++) {
                    float yv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int hh = 0; hh < kDH; hh++) {
                        const float4 v = reinterpret_cast<const float4 *>(
                            rd + ((size_t)(kDH * pp + hh) * 32 + lane) * 8)[sl];
                        yv[0] += v.x;
                        yv[1] += v.y;
                        yv[2] += v.z;
                        yv[3] += v.w;
                    }
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const int tok = 2 * cq + (i & 1);
                        const int row = (part * kDownSlabs + 2 * pp + sl) * kSlabRows + g + 8 * (i >> 1);
                        if (tok < n) p.Y[(size_t)(slot0 + tok) * H + row] = 0.5f * yv[i];
                    }
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&empty[slot]);  // weights and partials consumed
                // all 128 rows are stored: post the block for the combine warp
                __threadfence_block();
                const int idx = atomicAdd(misc + kMiscCombN, 1);
                long long t0 = clock64();
                while (idx - vmisc[kMiscCombSeen] >= kPubQ) {
                    if (*abort_flag || clock64() - t0 > p.budget) {
                        atomicCAS(p.err, 0, kErrTimeout);
                        *abort_flag = 1;
                        break;
                    }
                }
                vmisc[kMiscCombQ + idx % kPubQ] = u * ndn + part + 1;
            }
        }
    }
    return jpos;
}
template <int kBits, bool kStaged>
__global__ void __launch_bounds__(kFThreads, 1) fused_decode_kernel(const __grid_constant__ FusedParams p) {
    extern __shared__ __align__(128) uint8_t sm[];
    constexpr int UB = unit_bytes(kBits);
    constexpr bool kMagic = kBits <= 2;  // magic-offset gate/up (1- and 2-bit)
    const FusedSmem L = fused_smem(p.T, p.E, p.k, p.H, p.Ip, p.ring, p.item_bytes, p.staged,
                                   p.units_max, p.na);
    uint8_t *ring = sm + L.ring;
    float *red = reinterpret_cast<float *>(sm + L.red);
    uint2 *xi = reinterpret_cast<uint2 *>(sm + L.red);  // while routing
    __half *xs = reinterpret_cast<__half *>(sm + L.xs);
    float *scorr = reinterpret_cast<float *>(sm + L.corr);  // [T][H / 32]
    __nv_bfloat16 *xb = reinterpret_cast<__nv_bfloat16 *>(sm + L.rega);
    __half *abuf0 = reinterpret_cast<__half *>(sm + L.rega);
    int *sidx = reinterpret_cast<int *>(sm + L.sidx);
    float *sw = reinterpret_cast<float *>(sm + L.sw);
    int *sslot = reinterpret_cast<int *>(sm + L.sslot);
    int *sord = reinterpret_cast<int *>(sm + L.sord);
    unsigned long long *mask = reinterpret_cast<unsigned long long *>(sm + L.mask);
    int *soff = reinterpret_cast<int *>(sm + L.soff);
    int4 *units = reinterpret_cast<int4 *>(sm + L.units);
    int *slist = reinterpret_cast<int *>(sm + L.slist);
    int *sex = reinterpret_cast<int *>(sm + L.sex);
    int *misc = reinterpret_cast<int *>(sm + L.misc);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + L.bars);
    uint64_t *empty = full + kFMaxRing;
    uint64_t *xbar = empty + kFMaxRing;
    uint64_t *lgbar = xbar + 1, *rdy = xbar + 2, *pickbar = xbar + 3, *rdy2 = xbar + 4,
             *dsp = xbar + 5;
    uint64_t *abar = xbar + 8;       // [kMaxA] activation rows landed
    uint64_t *aempty = abar + kMaxA; // [kMaxA] the group's warps are done with them
    volatile int *abort_flag = misc + kMiscAbort;
    volatile int *vmisc = misc;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const int T = p.T, E = p.E, k = p.k, H = p.H, Tk = T * k;
    const int ns4 = H / 128, nbh = H / 32, nbi = p.Ip / 32;
    const int nsl = p.Ip / kSlabRows;              // gate/up slabs per unit
    const int ndn = H / (kSlabRows * kDownSlabs);  // down blocks per unit
    const int nsh = (T + kFTile - 1) / kFTile;     // shared-expert units
    constexpr bool staged = kStaged;  // token rows in shared memory (T <= 8)
    const int e0 = (int)((long long)cta * E / G), e1 = (int)((long long)(cta + 1) * E / G);
    const int ne = e1 - e0;
    const int wbytes = ne * H * 4;                                 // router slice
    const int nwc = (wbytes + p.item_bytes - 1) / p.item_bytes;    // ring positions it takes
    const int nxs = kFExtras && staged ? nsh * nsl : 0;            // extras over the grid
    const int nx = cta < nxs ? (nxs - 1 - cta) / G + 1 : 0;        // this CTA's extras
    const size_t gu_bytes = (size_t)p.nseg_h * UB, dn_bytes = (size_t)kDownSlabs * p.nseg_i * UB;

    for (int i = tid; i < 256; i += blockDim.x) misc[i] = 0;
    __syncthreads();
    if (tid == 0) {
        for (int s = 0; s < p.ring; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kGWarps);  // the warps of the group
        }
        mbar_init(xbar, 1);
        mbar_init(lgbar, kFWarps);
        mbar_init(rdy, 1);
        mbar_init(pickbar, 1);
        mbar_init(rdy2, 1);
        mbar_init(dsp, 1);
        for (int b = 0; b < p.na; b++) {
            mbar_init(&abar[b], 1);
            mbar_init(&aempty[b], kGWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    // the routed item list, once dispatch has run (same in every role)
    auto item_counts = [&](int &Ng, int &N2, int &ug0) {
        const int n_units = vmisc[kMiscNUnits];
        ug0 = kFExtras && staged ? nsh : 0;  // with extras, the shared units' slabs are done already
        Ng = (n_units - ug0) * nsl;
        N2 = n_units * ndn;
    };

    // =========================================================== copy warp
    if (warp == kWCopy) {
        if (lane != 0) return;
        const uint64_t pol = l2_evict_first_policy();  // weights: read once per forward
        int pos = 0;
        bool ok = true;
        auto acquire = [&](int ps) {  // wait until ring position ps may be filled
            return ps < p.ring || fwait(&empty[ps % p.ring], ((ps / p.ring) - 1) & 1, p, abort_flag);
        };
        auto issue_gu = [&](int slot, int e, int slab) {
            const uint8_t *wg = (e == E ? p.shared : p.routed + (size_t)e * p.expert_bytes) +
                                (size_t)slab * gu_bytes;
            uint8_t *dst = ring + (size_t)slot * p.item_bytes;
            mbar_arrive_expect_tx(&full[slot], (uint32_t)(2 * gu_bytes));
            bulk_g2s_hint(dst, wg, (uint32_t)gu_bytes, &full[slot], pol);
            bulk_g2s_hint(dst + gu_bytes, wg + p.mat_bytes, (uint32_t)gu_bytes, &full[slot], pol);
        };
        // router slice: constant, requested before the previous kernel ends
        const uint8_t *wsrc = reinterpret_cast<const uint8_t *>(p.Wp) + (size_t)e0 * H * 4;
        for (int i = 0; i < nwc; i++, pos++) {
            const int bytes = wbytes - i * p.item_bytes < p.item_bytes ? wbytes - i * p.item_bytes
                                                                       : p.item_bytes;
            mbar_arrive_expect_tx(&full[pos], (uint32_t)bytes);
            bulk_g2s_hint(ring + (size_t)pos * p.item_bytes, wsrc + (size_t)i * p.item_bytes,
                          (uint32_t)bytes, &full[pos], pol);
        }
        grid_dependency_wait();  // the token rows are the previous kernel's output
        if (staged) {
            mbar_arrive_expect_tx(xbar, (uint32_t)(T * H * 2));
            for (int t = 0; t < T; t++)
                bulk_g2s(xb + (size_t)t * H, p.x + (size_t)t * H, (uint32_t)(H * 2), xbar);
        }
        // the shared expert's gate/up slabs of this CTA (no routing needed)
        int mx = 0;
        for (; mx < nx && ok; mx++) {
            const int ps = pos + mx, slot = ps % p.ring, i = cta + mx * G;
            ok = acquire(ps);
            if (!ok) break;
            vmisc[kMiscMeta + slot] = (kKindExtra << 28) | i;
            issue_gu(slot, E, i % nsl);
        }
        pos += mx;  // positions issued so far
        if (ok) ok = fwait(dsp, 0, p, abort_flag);
        if (ok) {
            int Ng, N2, ug0;
            item_counts(Ng, N2, ug0);
            const int W = Ng + N2;
            int kd = 0;
            // items are claimed from one counter per launch, in ascending
            // order: gate/up slabs first, then down blocks, so within a CTA
            // every gate/up item precedes every down item (every down wait
            // ends) and a CTA that finishes early takes more work; the next
            // claim is requested while this item's copies go out
            unsigned long long b0;
            asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(b0) : "l"(p.bar) : "memory");
            int *claim = p.cnt + (size_t)((b0 / (2ull * (unsigned long long)G)) & 1ull) * p.cnt_stride +
                         p.cnt_stride - 1;
            int nxt = atomicAdd(claim, 1);
            for (; nxt < W && ok; pos++) {
                const int it = nxt;
                ok = acquire(pos);
                if (!ok) break;
                nxt = atomicAdd(claim, 1);
                const int slot = pos % p.ring;
                if (it < Ng) {
                    const int u = ug0 + it / nsl;
                    vmisc[kMiscMeta + slot] = (kKindGU << 28) | it;
                    issue_gu(slot, units[u].x, it % nsl);
                } else {
                    const int d = it - Ng, u = d / ndn, e = units[u].x;
                    // (kd mod 2 na keeps the buffer and its phase parity in 8 bits)
                    vmisc[kMiscMeta + slot] = (kKindDown << 28) | ((kd % (2 * p.na)) << 20) | d;
                    // hand the down block to the fetch warp (its activation rows)
                    long long t0 = clock64();
                    while (kd - vmisc[kMiscDownSeen] >= kDownQ) {
                        if (*abort_flag || clock64() - t0 > p.budget) {
                            atomicCAS(p.err, 0, kErrTimeout);
                            *abort_flag = 1;
                            ok = false;
                            break;
                        }
                    }
                    if (!ok) break;
                    vmisc[kMiscDownQ + kd % kDownQ] = d;
                    __threadfence_block();
                    vmisc[kMiscDownN] = kd + 1;
                    kd++;
                    const uint8_t *wd = (e == E ? p.shared : p.routed + (size_t)e * p.expert_bytes) +
                                        2 * p.mat_bytes + (size_t)(d % ndn) * dn_bytes;
                    mbar_arrive_expect_tx(&full[slot], (uint32_t)dn_bytes);
                    bulk_g2s_hint(ring + (size_t)slot * p.item_bytes, wd, (uint32_t)dn_bytes,
                                  &full[slot], pol);
                }
            }
            __threadfence_block();
            vmisc[kMiscDownEnd] = 1;  // no more down blocks for the fetch warp
            // one end marker per group (completes its slot without bytes)
            for (int gq = 0; gq < kGroups && ok; gq++) {
                ok = acquire(pos);
                if (!ok) break;
                vmisc[kMiscMeta + pos % p.ring] = kItemEnd;
                mbar_arrive(&full[pos % p.ring]);
                pos++;
            }
        }
        // the CTA must not exit with copies in flight (abort path)
        for (int i = pos > p.ring ? pos - p.ring : 0; i < pos; i++)
            mbar_drain(&full[i % p.ring], (i / p.ring) & 1);
        if (staged) mbar_drain(xbar, 0);
        return;
    }

    // ====================================================== publish warp
    // Finished gate/up slabs -> per-unit counts: the warp that completes a
    // slab posts its unit in a shared-memory queue (CTA scope); this warp makes
    // each batch visible at gpu scope with one fence and then counts it.
    if (warp == kWPub) {
        if (lane != 0) return;
        grid_dependency_wait();
        unsigned long long b0;
        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(b0) : "l"(p.bar) : "memory");
        const int par = (int)((b0 / (2ull * (unsigned long long)G)) & 1ull);
        int *done_gu = p.cnt + (size_t)par * p.cnt_stride;
        int seen = 0;
        long long t_idle = clock64();
        while (!*abort_flag) {
            const int done = vmisc[kMiscWarpsDone];
            __threadfence_block();
            int n = 0;
            while (n < kPubQ && vmisc[kMiscPubQ + (seen + n) % kPubQ] != 0) n++;
            if (n > 0) {
                __threadfence_block();
                asm volatile("fence.acq_rel.gpu;" ::: "memory");
                for (int i = 0; i < n; i++) {
                    const int s = kMiscPubQ + (seen + i) % kPubQ;
                    asm volatile("red.relaxed.gpu.global.add.s32 [%0], 1;" ::"l"(
                                     done_gu + vmisc[s] - 1)
                                 : "memory");
                    vmisc[s] = 0;
                }
                seen += n;
                __threadfence_block();
                vmisc[kMiscPubSeen] = seen;
                t_idle = clock64();
            } else {
                if (done == kFWarps && vmisc[kMiscPubN] == seen) break;  // all posted and counted
                if (clock64() - t_idle > p.budget) {
                    atomicCAS(p.err, 0, kErrTimeout);
                    *abort_flag = 1;
                    break;
                }
                __nanosleep(200);
            }
        }
        return;
    }

    // ======================================================== fetch warp
    // Grid barrier(s), then the activation rows of this CTA's down blocks.
    if (warp == kWFetch) {
        grid_dependency_wait();
        if (lane != 0) return;
        unsigned long long b0;
        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(b0) : "l"(p.bar) : "memory");
        const unsigned long long gg = (unsigned long long)G, ep = b0 / (2ull * gg);
        const int par = (int)(ep & 1ull);
        int *done_gu = p.cnt + (size_t)par * p.cnt_stride;
        // the other counter set is the next launch's: zero this CTA's share
        int *other = p.cnt + (size_t)(1 - par) * p.cnt_stride;
        for (int i = (int)((long long)cta * p.cnt_stride / G);
             i < (int)((long long)(cta + 1) * p.cnt_stride / G); i++)
            other[i] = 0;
        bool ok = fwait(lgbar, 0, p, abort_flag);  // this CTA's logits are stored
        // every CTA arrives, also after a failed wait, so the count stays whole
        ok = grid_barrier(p.bar, 2ull * gg * ep + gg, p, abort_flag) && ok;
        if (ok) mbar_arrive(rdy);
        if (T > kTopkLocalT) {
            if (ok) ok = fwait(pickbar, 0, p, abort_flag);
            ok = grid_barrier(p.bar, 2ull * gg * (ep + 1), p, abort_flag) && ok;
            if (ok) mbar_arrive(rdy2);
        } else {
            asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(p.bar) : "memory");
        }
        if (ok) ok = fwait(dsp, 0, p, abort_flag);
        int issued = 0;
        if (ok) {
            // this CTA's down blocks in the order the copy warp claimed them
            for (;; issued++) {
                int d = -1;
                long long t0 = clock64();
                while (true) {
                    if (issued < vmisc[kMiscDownN]) {
                        d = vmisc[kMiscDownQ + issued % kDownQ];
                        break;
                    }
                    if (vmisc[kMiscDownEnd] && issued >= vmisc[kMiscDownN]) break;
                    if (*abort_flag || clock64() - t0 > p.budget) {
                        atomicCAS(p.err, 0, kErrTimeout);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    __nanosleep(32);
                }
                if (d < 0) break;
                __threadfence_block();
                vmisc[kMiscDownSeen] = issued + 1;  // the entry may be reused
                const int u = d / ndn, kd = issued, b = kd % p.na;
                const int4 un = units[u];
                // buffer b is free once the group's warps are done with its last block
                if (kd >= p.na && !(ok = fwait(&aempty[b], ((kd / p.na) - 1) & 1, p, abort_flag)))
                    break;
                ok = fwait_count(done_gu + u, nsl, p, abort_flag);
                if (!ok) break;
                asm volatile("fence.proxy.async.global;" ::: "memory");
                __half *dst = abuf0 + (size_t)b * kFTile * (p.Ip + 8);
                mbar_arrive_expect_tx(&abar[b], (uint32_t)(un.z * p.Ip * 2));
                for (int r = 0; r < un.z; r++)
                    bulk_g2s(dst + (size_t)r * (p.Ip + 8), p.a + (size_t)(un.y + r) * p.Ip,
                             (uint32_t)(p.Ip * 2), &abar[b]);
            }
        }
        // no exit with copies in flight
        for (int i = issued > p.na ? issued - p.na : 0; i < issued; i++)
            mbar_drain(&abar[i % p.na], (i / p.na) & 1);
        return;
    }

    // ====================================================== combine warp
    // Finished down blocks: count every token's finished (token, 128-row
    // block) pairs (one gpu-scope fence per batch) and combine each pair that
    // is complete: y = Y_shared + sum over the picks in ascending expert id of
    // w Y, in fp32, the token's prescale off, one rounding to bf16 (with the
    // residual added in the stack).
    if (warp == kWComb) {
        grid_dependency_wait();
        unsigned long long b0;
        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(b0) : "l"(p.bar) : "memory");
        const int par = (int)((b0 / (2ull * (unsigned long long)G)) & 1ull);
        int *done_tok = p.cnt + (size_t)par * p.cnt_stride + p.cnt_tok;
        const int per_blk = k + 1;  // down blocks that write one (token, row block)
        int seen = 0;
        long long t_idle = clock64();
        while (true) {
            int n = 0, fin = 0, stop = 0;
            if (lane == 0) {
                stop = *abort_flag;
                fin = vmisc[kMiscWarpsDone] == kFWarps;
                __threadfence_block();
                while (n < kPubQ && vmisc[kMiscCombQ + (seen + n) % kPubQ] != 0) n++;
                if (n == 0 && fin && vmisc[kMiscCombN] != seen) fin = 0;
            }
            n = __shfl_sync(0xffffffffu, n, 0);
            fin = __shfl_sync(0xffffffffu, fin, 0);
            stop = __shfl_sync(0xffffffffu, stop, 0);
            if (stop) break;
            if (n == 0) {
                if (fin) break;  // every block is posted and combined
                int late = 0;
                if (lane == 0 && clock64() - t_idle > p.budget) {
                    atomicCAS(p.err, 0, kErrTimeout);
                    *abort_flag = 1;
                    late = 1;
                }
                if (__shfl_sync(0xffffffffu, late, 0)) break;
                __nanosleep(100);
                continue;
            }
            __syncwarp();
            __threadfence();  // the posted blocks' rows, at gpu scope, before the counts
            for (int i = 0; i < n; i++) {
                const int v = vmisc[kMiscCombQ + (seen + i) % kPubQ] - 1;
                const int u = v / ndn, part = v % ndn;
                const int4 un = units[u];
                int t = 0, c = 0;
                if (lane < un.z) {
                    const int sl = un.y + lane;
                    t = sl < Tk ? slist[sl] : sl - Tk;
                    c = atomicAdd(done_tok + t * ndn + part, 1);
                }
                unsigned ready = __ballot_sync(0xffffffffu, lane < un.z && c == per_blk - 1);
                if (ready) __threadfence();  // the other blocks' rows of these tokens
                while (ready) {
                    const int j = __ffs(ready) - 1;
                    ready &= ready - 1;
                    const int tt = __shfl_sync(0xffffffffu, t, j);
                    const int ex = staged ? sex[tt] : __ldcg(p.xex + tt);
                    // lane: 4 adjacent columns of the 128-row block, every
                    // row one 16-byte load; the loads are unconditional (picks
                    // past k re-read the last one and add an exact zero with
                    // weight 0), so all k + 1 rows are in flight at once
                    const int col = part * kSlabRows * kDownSlabs + 4 * lane;
                    const int *so = sord + tt * k;
                    float4 vv[kFMaxK];
#pragma unroll
                    for (int r = 0; r < kFMaxK; r++)
                        vv[r] = __ldcg(reinterpret_cast<const float4 *>(
                            p.Y + (size_t)sslot[so[r < k ? r : k - 1]] * H + col));
                    float4 acc = __ldcg(reinterpret_cast<const float4 *>(p.Y + (size_t)(Tk + tt) * H + col));
#pragma unroll
                    for (int r = 0; r < kFMaxK; r++) {
                        const float wr = r < k ? sw[so[r]] : 0.0f;
                        acc.x = fmaf(wr, vv[r].x, acc.x);
                        acc.y = fmaf(wr, vv[r].y, acc.y);
                        acc.z = fmaf(wr, vv[r].z, acc.z);
                        acc.w = fmaf(wr, vv[r].w, acc.w);
                    }
                    if (ex) {  // the token's prescale off (2^ex twice: stays in range)
                        const float f = pow2f(ex);
                        acc.x = acc.x * f * f;
                        acc.y = acc.y * f * f;
                        acc.z = acc.z * f * f;
                        acc.w = acc.w * f * f;
                    }
                    __nv_bfloat16 *o = p.out + (size_t)tt * H + col;
                    __nv_bfloat162 y01 = __floats2bfloat162_rn(acc.x, acc.y);
                    __nv_bfloat162 y23 = __floats2bfloat162_rn(acc.z, acc.w);
                    if (p.residual) {
                        const uint2 hv = *reinterpret_cast<const uint2 *>(o);
                        const __nv_bfloat162 h01 = *reinterpret_cast<const __nv_bfloat162 *>(&hv.x);
                        const __nv_bfloat162 h23 = *reinterpret_cast<const __nv_bfloat162 *>(&hv.y);
                        y01 = __floats2bfloat162_rn(
                            __fadd_rn(__low2float(h01), __low2float(y01)),
                            __fadd_rn(__high2float(h01), __high2float(y01)));
                        y23 = __floats2bfloat162_rn(
                            __fadd_rn(__low2float(h23), __low2float(y23)),
                            __fadd_rn(__high2float(h23), __high2float(y23)));
                    }
                    uint2 ov;
                    ov.x = *reinterpret_cast<const uint32_t *>(&y01);
                    ov.y = *reinterpret_cast<const uint32_t *>(&y23);
                    *reinterpret_cast<uint2 *>(o) = ov;
                }
            }
            __syncwarp();
            if (lane == 0) {
                for (int i = 0; i < n; i++) vmisc[kMiscCombQ + (seen + i) % kPubQ] = 0;
                __threadfence_block();
                vmisc[kMiscCombSeen] = seen + n;
            }
            seen += n;
            t_idle = clock64();
        }
        return;
    }

    // ==================================================== compute warps
    const int g = lane >> 2, cq = lane & 3;
    // compute-wide verdicts go through one slot, written by thread 0 before a
    // compute barrier and read by every compute thread after it
    volatile int *cflag = misc + kMiscCFlag;
    grid_dependency_wait();
    if (tid == 0) {
        unsigned long long b0;
        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(b0) : "l"(p.bar) : "memory");
        misc[kMiscPar] = (int)((b0 / (2ull * (unsigned long long)G)) & 1ull);
    }
    for (int e = tid; e < E; e += kFCompute) mask[e] = 0ull;  // dispatch, later
    bool alive = true;

    // ---- token rows.  Staged (T <= 8): the raw rows arrive by bulk copy; one
    // pass builds the lane-interleaved bf16 copy the router reads (slot
    // (t, s, l) holds x[t][128 s + 32 j + l], j = 0..3) while warps t < T sum
    // the squares of row t in a fixed order for the token's prescale.
    if (staged) {
        if (tid == 0) *cflag = fwait(xbar, 0, p, abort_flag) ? 1 : 0;
        compute_sync();
        alive = *cflag != 0;
        if (alive) {
            const unsigned short *xu = reinterpret_cast<const unsigned short *>(xb);
            for (int i = tid; i < T * ns4 * 32; i += kFCompute) {
                const int t = i / (ns4 * 32), r = i % (ns4 * 32);
                const unsigned short *px = xu + (size_t)t * H + (r >> 5) * 128 + (r & 31);
                xi[i] = make_uint2((uint32_t)px[0] | ((uint32_t)px[32] << 16),
                                   (uint32_t)px[64] | ((uint32_t)px[96] << 16));
            }
            if (warp < T) {
                const int ex = token_prescale_warp(xb + (size_t)warp * H, H, p.w2, lane);
                if (lane == 0) sex[warp] = ex;
            }
            compute_sync();
        }
    } else {
        // this CTA writes the expert operand of tokens cta, cta + G, ... for every CTA
        for (int t = cta; t < T; t += G) {
            if (warp == 0) {
                const int ex = token_prescale_warp(p.x + (size_t)t * H, H, p.w2, lane);
                if (lane == 0) {
                    misc[kMiscTmp] = ex;
                    p.xex[t] = ex;
                }
            }
            compute_sync();
            const int ex = misc[kMiscTmp];
            for (int i = tid; i < H; i += kFCompute)
                p.x16[(size_t)t * H + i] =
                    token_operand<kBits>(__bfloat162float(p.x[(size_t)t * H + i]), ex, i);
            if (kMagic)
                for (int b = tid; b < nbh; b += kFCompute)
                    p.corr[(size_t)t * nbh + b] = block_correction<kBits>(p.x + (size_t)t * H + 32 * b, ex);
            compute_sync();
        }
    }

    // ---- router logits of this CTA's experts (fixed summation order)
    if (alive && nwc > 0) {
        if (tid == 0) {
            bool ok = true;
            for (int s = 0; s < nwc && ok; s++) ok = fwait(&full[s], 0, p, abort_flag);
            *cflag = ok ? 1 : 0;
        }
        compute_sync();
        alive = *cflag != 0;
    }
    if (alive && ne > 0 && staged) {
        // staged rows: one (token, expert) task per warp; lane l runs through
        // its columns 128 s4 + 32 j + l in order (s4, then j), the loads of
        // four steps in flight together
        const float4 *Ws = reinterpret_cast<const float4 *>(ring);  // [ne][H/128][32]
        for (int task = warp; task < T * ne; task += kFWarps) {
            const int t = task / ne, eb = task % ne;
            const float4 *wr = Ws + (size_t)eb * ns4 * 32 + lane;
            const uint2 *xr = xi + (size_t)t * ns4 * 32 + lane;
            float acc = 0.0f;
#pragma unroll 4
            for (int s4 = 0; s4 < ns4; s4++) {
                const uint2 v = xr[(size_t)s4 * 32];
                const float4 w = wr[(size_t)s4 * 32];
                acc = fmaf(__uint_as_float(v.x << 16), w.x, acc);
                acc = fmaf(__uint_as_float(v.x & 0xffff0000u), w.y, acc);
                acc = fmaf(__uint_as_float(v.y << 16), w.z, acc);
                acc = fmaf(__uint_as_float(v.y & 0xffff0000u), w.w, acc);
            }
#pragma unroll
            for (int sh = 16; sh >= 1; sh >>= 1)
                acc = __fadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, sh));
            if (lane == 0) {
                const int e = e0 + eb;
                p.logits[(size_t)t * E + e] = p.bias ? __fadd_rn(acc, p.bias[e]) : acc;
            }
        }
    } else if (alive && ne > 0) {
        // global rows: one token per warp, four of the CTA's experts at a time
        // (each row read ne / 4 times, from L1); every load unconditional
        // (a missing fourth expert repeats one and is not stored)
        const float4 *Ws = reinterpret_cast<const float4 *>(ring);  // [ne][H/128][32]
        for (int t = warp; t < T; t += kFWarps) {
            const __nv_bfloat16 *xrow = p.x + (size_t)t * H + lane;
            for (int ee = 0; ee < ne; ee += 4) {
                const int nb = ne - ee < 4 ? ne - ee : 4;
                const float4 *w0 = Ws + (size_t)ee * ns4 * 32 + lane;
                const size_t st[4] = {0, (size_t)(1 < nb ? 1 : 0) * ns4 * 32,
                                      (size_t)(2 < nb ? 2 : 0) * ns4 * 32,
                                      (size_t)(3 < nb ? 3 : 0) * ns4 * 32};
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
                for (int s4 = 0; s4 < ns4; s4++) {
                    float xv[4];
#pragma unroll
                    for (int j = 0; j < 4; j++) xv[j] = __bfloat162float(xrow[128 * s4 + 32 * j]);
#pragma unroll
                    for (int b = 0; b < 4; b++) {
                        const float4 w = w0[st[b] + (size_t)s4 * 32];
                        acc[b] = fmaf(xv[0], w.x, acc[b]);
                        acc[b] = fmaf(xv[1], w.y, acc[b]);
                        acc[b] = fmaf(xv[2], w.z, acc[b]);
                        acc[b] = fmaf(xv[3], w.w, acc[b]);
                    }
                }
#pragma unroll
                for (int b = 0; b < 4; b++) {
                    float v = acc[b];
#pragma unroll
                    for (int sh = 16; sh >= 1; sh >>= 1)
                        v = __fadd_rn(v, __shfl_down_sync(0xffffffffu, v, sh));
                    if (lane == 0 && b < nb) {
                        const int e = e0 + ee + b;
                        p.logits[(size_t)t * E + e] = p.bias ? __fadd_rn(v, p.bias[e]) : v;
                    }
                }
            }
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(lgbar);  // this warp's logits (and token rows) are stored
    compute_sync();                     // every warp is done with the router slice
    if (tid == 0)
        for (int s = 0; s < nwc; s++) mbar_arrive_cnt(&empty[s], kGWarps);  // router slice consumed

    // ring items: group gi (warps 8 gi .. 8 gi + 7) takes positions nwc + gi,
    // nwc + gi + 2, ... (fused_run_items)
    int jpos = nwc + warp / kGWarps;

    // ---- top-k (picks in descending logit order; a tie to the lower id).
    // Up to kTopkLocalT tokens every CTA picks for every token: warp t < T
    // takes token t once the grid barrier is through, while the other warps
    // build the staged tokens' expert operand and (2-bit) its block
    // corrections, which nothing reads before the first item.
    if (T <= kTopkLocalT) {
        if (warp < T) {
            int ok = alive ? 1 : 0;
            if (lane == 0 && ok) ok = fwait(rdy, 0, p, abort_flag) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (ok) {
                int pe;
                float pw;
                warp_topk(p.logits + (size_t)warp * E, E, k, lane, pe, pw);
                if (lane < k) {
                    sidx[warp * k + lane] = pe;
                    sw[warp * k + lane] = pw;
                }
            } else if (lane == 0) {
                misc[kMiscDead] = 1;
            }
        } else if (alive && staged) {
            const int t0 = tid - 32 * T, nt = kFCompute - 32 * T;
            for (int task = t0; task < T * nbh; task += nt) {
                const int t = task / nbh, b = task % nbh;
                stage_block<kBits>(xb + (size_t)t * H + 32 * b, xs + (size_t)t * (H + 8) + 32 * b,
                                   sex[t], scorr + t * nbh + b);
            }
        }
        if (!alive && lane == 0) misc[kMiscDead] = 1;
        compute_sync();
        alive = misc[kMiscDead] == 0;
    } else {
        if (tid == 0) *cflag = alive && fwait(rdy, 0, p, abort_flag) ? 1 : 0;
        compute_sync();
        alive = *cflag != 0;
        if (alive && warp == 0 && cta < T) {
            int pe;
            float pw;
            warp_topk(p.logits + (size_t)cta * E, E, k, lane, pe, pw);
            if (lane < k) {
                p.idx[(size_t)cta * k + lane] = pe;
                p.wts[(size_t)cta * k + lane] = pw;
            }
        }
        __syncwarp();
        compute_sync();
        if (tid == 0) {
            mbar_arrive(pickbar);
            *cflag = alive && fwait(rdy2, 0, p, abort_flag) ? 1 : 0;
        }
        compute_sync();
        alive = *cflag != 0;
        if (alive)
            for (int i = tid; i < Tk; i += kFCompute) {
                sidx[i] = __ldcg(p.idx + i);
                sw[i] = __ldcg(p.wts + i);
            }
    }
    compute_sync();

    // ---- dispatch, identical in every CTA
    if (alive) {
        for (int i = tid; i < Tk; i += kFCompute)
            if (idx_ok(p.err, sidx[i], E)) atomicOr(&mask[sidx[i]], 1ull << (i / k));
        compute_sync();
        // one scan of (count << 16 | units): both sums stay below 2^16 (T k <= 1024)
        const int ept = (E + kFCompute - 1) / kFCompute, eb = tid * ept;
        int local = 0;
        for (int e = eb; e < eb + ept && e < E; e++) {
            const int c = __popcll(mask[e]);
            local += (c << 16) | ((c + kFTile - 1) / kFTile);
        }
        int packed_total;
        int packed = compute_exclusive_scan(local, misc + kMiscScan, &packed_total);
        const int utot = packed_total & 0xffff;
        for (int e = eb; e < eb + ept && e < E; e++) {
            const int c = __popcll(mask[e]), nu = (c + kFTile - 1) / kFTile;
            const int off = packed >> 16, us = packed & 0xffff;
            soff[e] = off;
            for (int i = 0; i < nu; i++) {
                const int n = c - i * kFTile;
                units[nsh + us + i] = make_int4(e, off + i * kFTile, n < kFTile ? n : kFTile, 0);
            }
            packed += (c << 16) | nu;
        }
        if (tid < nsh) {
            const int n = T - tid * kFTile;
            units[tid] = make_int4(E, Tk + tid * kFTile, n < kFTile ? n : kFTile, 0);
        }
        if (tid == 0) {
            misc[kMiscNUnits] = nsh + utot;
            misc[kMiscUtot] = utot;
        }
        compute_sync();
        for (int i = tid; i < Tk; i += kFCompute) {
            const int t = i / k, ej = sidx[i];
            const int pos = soff[ej] + __popcll(mask[ej] & ((1ull << t) - 1ull));
            if (idx_ok(p.err, pos, Tk)) slist[pos] = t;
            sslot[i] = pos;
            int rank = 0;
            for (int jj = 0; jj < k; jj++) rank += sidx[t * k + jj] < ej;
            sord[t * k + rank] = i;  // combine order: ascending expert id
        }
    }
    compute_sync();
    if (tid == 0 && alive) mbar_arrive(dsp);
    // the next kernel of the stream may start its prologue once every CTA is here
    grid_launch_dependents();

    // ---- routed slabs and down blocks, then the end marker
    if (alive) fused_run_items<kBits, kStaged>(p, jpos, 1 << 30);
    __syncwarp();
    if (lane == 0) {
        __threadfence_block();
        atomicAdd(misc + kMiscWarpsDone, 1);  // the publish warp may stop once all are in
    }
}

// ------------------------------------------------------------------- host
static int g_fused_max_smem = 0;
static int g_fused_sms = 0;

size_t fused_item_bytes(const Geometry &g) {
    const int a = 2 * g.nseg_h, b = kDownSlabs * g.nseg_i;
    return (size_t)(a > b ? a : b) * g.ub;
}

int fused_grid() { return g_fused_sms; }

// Shared-memory plan of a launch: whether the token rows are staged, the
// activation buffers and the ring depth.  The groups take ring positions in
// turn and wait on a slot's barrier by phase parity, so the wait for position
// p is unambiguous only if position p - ring (the slot's previous fill) was
// waited for already, by this group: ring >= kGroups.  Likewise one activation
// buffer per group.  Returns false when the shape does not fit.
struct FusedPlan {
    int staged, na, ring, units_max, item_bytes;
};
static bool fused_plan(const Geometry &g, int T, FusedPlan &pl) {
    if (!(T >= 1 && T <= kFMaxT && g.E <= 512 && g.k <= kFMaxK && g.H % 128 == 0 &&
          g.Ip % 128 == 0 && g.H <= 8192) ||
        g_fused_max_smem == 0 || g_fused_sms == 0)
        return false;
    pl.item_bytes = (int)fused_item_bytes(g);
    pl.units_max = max_units(T, g.k, g.E, kFTile);
    auto total = [&](int ring, int staged, int na) {
        return fused_smem(T, g.E, g.k, g.H, g.Ip, ring, pl.item_bytes, staged, pl.units_max, na)
            .total;
    };
    // the router slice of the CTA with the most experts must fit the ring
    const int G = g_fused_sms;
    const int ne_max = (g.E + G - 1) / G;
    const int nwc = (ne_max * g.H * 4 + pl.item_bytes - 1) / pl.item_bytes;
    // a ring slot costs its item bytes plus the partial sums of the warps; the
    // partial-sum area also holds the router's copy of staged token rows
    const int slot_bytes = pl.item_bytes + kRedSlot;
    const int xi_slots = (align16(T * g.H * 2) + kRedSlot - 1) / kRedSlot;
    pl.na = kGroups;
    if (pl.na > kMaxA) return false;
    const int min_ring = kGroups > nwc + 1 ? kGroups : nwc + 1;
    // staging the token rows needs room for its router copy and a full ring
    const int need_staged = (xi_slots > kGroups ? xi_slots : kGroups) * slot_bytes;
    pl.staged = (T <= kFStagedMaxT && g_fused_max_smem - total(0, 1, pl.na) >= need_staged) ? 1 : 0;
    pl.ring = (g_fused_max_smem - total(0, pl.staged, pl.na)) / slot_bytes;
    if (pl.ring > kFMaxRing) pl.ring = kFMaxRing;
    if (pl.staged && pl.ring < xi_slots) return false;
    return pl.ring >= min_ring;
}

int fused_decode_supported(const Geometry &g, int T) {
    FusedPlan pl;
    return fused_plan(g, T, pl) ? 1 : 0;
}

cudaError_t launch_fused_decode(const Geometry &g, const ExpertWeights &w, const FusedArgs &fa,
                                int T, cudaStream_t s) {
    FusedPlan pl;
    if (!fused_plan(g, T, pl)) return cudaErrorInvalidValue;
    FusedParams p{};
    p.x = reinterpret_cast<const __nv_bfloat16 *>(fa.x);
    p.Wp = reinterpret_cast<const float4 *>(fa.router_wp);
    p.bias = fa.router_b;
    p.routed = w.routed;
    p.shared = w.shared;
    p.expert_bytes = g.expert_bytes;
    p.mat_bytes = g.mat_bytes;
    p.T = T;
    p.E = g.E;
    p.k = g.k;
    p.H = g.H;
    p.Ip = g.Ip;
    p.nseg_h = g.nseg_h;
    p.nseg_i = g.nseg_i;
    p.item_bytes = pl.item_bytes;
    p.units_max = pl.units_max;
    p.cnt_tok = fa.cnt_tok;
    p.w2 = fa.w2;
    p.logits = fa.logits;
    p.idx = fa.idx;
    p.wts = fa.wts;
    p.x16 = reinterpret_cast<__half *>(fa.x16);
    p.corr = fa.corr;
    p.xex = fa.xex;
    p.a = reinterpret_cast<__half *>(fa.a);
    p.Y = fa.Y;
    p.out = reinterpret_cast<__nv_bfloat16 *>(fa.out);
    p.residual = fa.residual ? 1 : 0;
    p.bar = fa.bar;
    p.cnt = fa.cnt;
    p.cnt_stride = fa.cnt_stride;
    p.err = fa.err;
    p.budget = fa.budget;
    const int G = g_fused_sms;
    p.staged = pl.staged;
    p.na = pl.na;
    p.ring = pl.ring;
    const int smem = fused_smem(T, g.E, g.k, g.H, g.Ip, p.ring, p.item_bytes, p.staged, p.units_max,
                                p.na).total;
    auto kern = g.bits == 1   ? (p.staged ? fused_decode_kernel<1, true> : fused_decode_kernel<1, false>)
                : g.bits == 2 ? (p.staged ? fused_decode_kernel<2, true> : fused_decode_kernel<2, false>)
                              : (p.staged ? fused_decode_kernel<3, true> : fused_decode_kernel<3, false>);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;  // the CTAs wait on one another
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

cudaError_t fused_init_attributes(int max_smem) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_fused_sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e;
    if ((e = allow_max_dyn_smem(fused_decode_kernel<1, true>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(fused_decode_kernel<1, false>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(fused_decode_kernel<2, true>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(fused_decode_kernel<2, false>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(fused_decode_kernel<3, true>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(fused_decode_kernel<3, false>, max_smem)) != cudaSuccess) return e;
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, reinterpret_cast<const void *>(fused_decode_kernel<2, true>))) !=
        cudaSuccess)
        return e;
    g_fused_max_smem = max_smem - (int)fa.sharedSizeBytes;
    return cudaSuccess;
}

}  // namespace strata
