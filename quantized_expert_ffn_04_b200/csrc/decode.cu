// Fused decode layer (T <= 64 tokens): top-k, dispatch, gate/up + SwiGLU,
// down and the combine in ONE persistent kernel that follows the router.
//
// Layer specification (the same steps as the multi-kernel path): the router
// kernel before it leaves the picks (the k largest logits, a tie to the lower
// expert id) and w_j = exp(l_j - m) / sum over the picks; units = (expert, up
// to 8 of its tokens), the shared
// expert's units first; a = silu(Wg x) * Wu x, y = Wd a with w = d (q - c) from
// the block-32 codes; out = y_shared + sum over the picks in ascending expert
// id of w_j y_j (fp32), rounded once to bf16.  The pages: 10 routed + 1 shared
// expert per token ("Strata Runs 125B Qwen3.8-Flash-Next on a 12GB Gaming GPU
// at Up to 94 Tokens/s", section "What it is"), decode of one token or a small
// multi-token-prediction batch (section "The numbers, measured by the author").
//
// Why one kernel: at T = 1..4 the layer moves 20-55 MB, ~3-9 us of HBM time,
// while each extra launch in a chain costs a few microseconds of ramp and
// drain.  Here:
//   * every CTA builds the dispatch tables itself (identical, deterministic)
//     from the router's T k picks, so no grid-wide barrier;
//   * each CTA owns a contiguous range of gate/up items (unit, 16-row slab)
//     and then of down items (unit, 128 rows); a copy warp streams the
//     items' packed weights through a ring of shared-memory slots with bulk
//     copies, up to `ring` items ahead, while 4 groups of 4 warps compute;
//   * a down item of unit u waits (bounded) until all gate/up slabs of u are
//     done (a counter per unit); every CTA finishes its gate/up items before
//     its down items, so the waits always end;
//   * the down item that completes the last expert's rows of a (token,
//     128-row block) pair (a counter per pair) combines that block of the
//     token, in the fixed order, so the combine is spread over the down
//     items instead of waiting for all of them.
// The counters are zeroed by the router kernel, which this kernel waits for
// (programmatic dependent launch).  The math of a block is the decode GEMV's:
// exact small integers from the codes, fp16 token rows, mma.sync as the
// in-warp reduction, fp32 per-block scaling.
#include "common.cuh"
#include "internal.h"

namespace strata {

constexpr int kFGroups = 4;                     // compute groups of 4 warps
constexpr int kFWarps = 4 * kFGroups;
constexpr int kFThreads = 32 * (kFWarps + 1);   // + the copy warp
constexpr int kFTile = 8;                       // tokens per unit (mma N)
constexpr int kFMaxRing = 6;
constexpr int kDownSlabs = 8;                   // a down item: 8 slabs = 128 rows
constexpr int kFStagedMaxT = 8;                 // token rows kept in shared memory
constexpr int kFMaxT = 64;                      // most tokens per call
constexpr int kFMaxK = 16;                      // most routed experts per token

struct FusedParams {
    const uint8_t *routed;
    const uint8_t *shared;
    size_t expert_bytes, mat_bytes;
    const int32_t *idx;    // [T][k] top-k picks (router)
    const float *wts;      // [T][k] their weights (router)
    const __half *x16;     // [T][H] fp16 copy of x (router)
    int T, E, k, H, Ip, nseg_h, nseg_i;
    int ring, item_bytes, staged, units_max;
    __half *a;             // [slots][Ip]
    float *Y;              // [slots][H]
    __nv_bfloat16 *out;    // [T][H]
    int residual;
    int *done_gu;          // [units_max] finished gate/up slabs per unit
    int *done_tok;         // [T][H / 128] finished down items per (token, row block)
    int *queue;            // [2] next gate/up item, next down item (claimed by CTAs)
    int *err;
    long long budget;
};

// Shared-memory carve (host and device agree on it).
struct FusedSmem {
    int ring, xs, abuf, red, sidx, sw, sslot, sord, mask, soff, units, slist, misc, bars, total;
};

__host__ __device__ inline int align16(int v) { return (v + 15) & ~15; }

__host__ __device__ inline FusedSmem fused_smem(int T, int E, int k, int H, int Ip, int ring,
                                                int item_bytes, int staged, int units_max) {
    FusedSmem s;
    int o = 0;
    s.ring = o;  o += ring * item_bytes;
    s.xs = o;    o += staged ? align16(T * (H + 8) * 2) : 0;
    s.abuf = o;  o += kFGroups * kFTile * (Ip + 8) * 2;  // a rows of each group's down item
    s.red = o;   o += kFGroups * 4 * 32 * 8 * 4;
    s.sidx = o;  o += align16(T * k * 4);
    s.sw = o;    o += align16(T * k * 4);
    s.sslot = o; o += align16(T * k * 4);
    s.sord = o;  o += align16(T * k * 4);
    s.mask = o;  o += align16(E * 8);
    s.soff = o;  o += align16(E * 4);
    s.units = o; o += units_max * 16;
    s.slist = o; o += align16(T * k * 4);
    s.misc = o;  o += 512;                       // flags, scan scratch, combine lists, item ids
    s.bars = o;  o += 8 * (2 * kFMaxRing + 2 + kFGroups);
    s.total = o;
    return s;
}

// Exclusive scan of one int per thread over the whole CTA (<= 32 warps).
__device__ int cta_exclusive_scan(int v, int *scratch, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int s = lane < nw ? scratch[lane] : 0, si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, si, o);
            if (lane >= o) si += n;
        }
        if (lane < nw) scratch[lane] = si - s;
        if (lane == 31) scratch[32] = si;
    }
    __syncthreads();
    const int r = scratch[warp] + incl - v;
    *total = scratch[32];
    __syncthreads();
    return r;
}

// B fragment source of a 32-wide block at column k0 (mma m16n8k16, fp16):
// lane 4g + c needs x[token g][k0 + 8m + 2c], x[..+1] in register m = 0..3.
//   kSrcSmem:  the token rows staged in shared memory, fetched with one
//              ldmatrix (rowp = this lane's row for matrix row lane & 7);
//   kSrcLdg:   read-only global rows through L1 (rowp = row of token lane >> 2);
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

// acc0/acc1 (16 rows x 8 tokens fragments) += two slabs' segments [0, ns),
// held in shared memory at w0 and w1, against the same token rows from rowp
// starting at column col0: one B fragment per block serves both slabs, and
// the two mma chains are independent.  Each lane reads its rows' four block
// scales with one 16-byte load (lane 4g + c: scales of rows g and g + 8).
template <int kBits, int kSrc>
STRATA_DEV void fused_slab2(float (&acc0)[4], float (&acc1)[4], const uint8_t *w0,
                            const uint8_t *w1, int ns, const __half *rowp, int col0, int lane) {
    constexpr int UB = unit_bytes(kBits);
    constexpr int SOFF = kLoBytes + (kBits == 3 ? kHiBytes : 0);
    const int g = lane >> 2;
    for (int sg = 0; sg < ns; sg++) {
        const uint8_t *u0 = w0 + sg * UB, *u1 = w1 + sg * UB;
        const uint4 lo0 = *reinterpret_cast<const uint4 *>(u0 + lane * 16);
        const uint4 lo1 = *reinterpret_cast<const uint4 *>(u1 + lane * 16);
        uint2 hi0 = make_uint2(0, 0), hi1 = make_uint2(0, 0);
        if (kBits == 3) {
            hi0 = *reinterpret_cast<const uint2 *>(u0 + kLoBytes + lane * 8);
            hi1 = *reinterpret_cast<const uint2 *>(u1 + kLoBytes + lane * 8);
        }
        const uint4 sc0 = *reinterpret_cast<const uint4 *>(u0 + SOFF + g * 16);
        const uint4 sc1 = *reinterpret_cast<const uint4 *>(u1 + SOFF + g * 16);
#pragma unroll
        for (int blk = 0; blk < 4; blk++) {
            uint32_t b0, b1, b2, b3;
            b_frag<kSrc>(rowp, col0 + sg * 128 + blk * 32, lane, b0, b1, b2, b3);
            float d0[4], d1[4];
            if (kBits == 2) {
                block_mma2(d0, comp4(lo0, blk), b0, b1, b2, b3);
                block_mma2(d1, comp4(lo1, blk), b0, b1, b2, b3);
            } else {
                block_mma<kBits>(d0, comp4(lo0, blk), blk < 2 ? hi0.x : hi0.y, 8 * (blk & 1), b0,
                                 b1, b2, b3);
                block_mma<kBits>(d1, comp4(lo1, blk), blk < 2 ? hi1.x : hi1.y, 8 * (blk & 1), b0,
                                 b1, b2, b3);
            }
            const uint32_t s0 = comp4(sc0, blk), s1 = comp4(sc1, blk);
            const float2 f0 = __half22float2(*reinterpret_cast<const __half2 *>(&s0));
            const float2 f1 = __half22float2(*reinterpret_cast<const __half2 *>(&s1));
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
}

// Bounded wait for an mbarrier phase by one thread; false (and the error
// word set) when the budget runs out or another thread gave up already.
STRATA_DEV bool fwait(uint64_t *bar, uint32_t parity, const FusedParams &p,
                      volatile int *abort_flag) {
    long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > p.budget) {
            atomicCAS(p.err, 0, kErrTimeout);
            *abort_flag = 1;
            return false;
        }
    }
    return true;
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
        __nanosleep(256);
    }
}

STRATA_DEV void group_sync(int group) {
    asm volatile("bar.sync %0, 128;" ::"r"(group + 1) : "memory");
}

// misc ints: [1] abort flag, [2..34] scan scratch, [36 + g] and [88 + g]
// group go/stop flags, [40 + 9 g] combine list of group g (count, then up to
// 8 tokens), [80 + slot] item id of each ring slot
constexpr int kMiscAbort = 1, kMiscScan = 2, kMiscFlag = 36, kMiscComb = 40, kMiscMeta = 80,
              kMiscFlag2 = 88;
constexpr int kItemEnd = -1;  // ring slot marker: no more items for this CTA

template <int kBits>
__global__ void __launch_bounds__(kFThreads, 1) fused_decode_kernel(const FusedParams p) {
    extern __shared__ __align__(16) uint8_t sm[];
    constexpr int UB = unit_bytes(kBits);
    const FusedSmem L =
        fused_smem(p.T, p.E, p.k, p.H, p.Ip, p.ring, p.item_bytes, p.staged, p.units_max);
    uint8_t *ring = sm + L.ring;
    __half *xs = reinterpret_cast<__half *>(sm + L.xs);
    float *red = reinterpret_cast<float *>(sm + L.red);
    int *sidx = reinterpret_cast<int *>(sm + L.sidx);
    float *sw = reinterpret_cast<float *>(sm + L.sw);
    int *sslot = reinterpret_cast<int *>(sm + L.sslot);
    int *sord = reinterpret_cast<int *>(sm + L.sord);
    unsigned long long *mask = reinterpret_cast<unsigned long long *>(sm + L.mask);
    int *soff = reinterpret_cast<int *>(sm + L.soff);
    int4 *units = reinterpret_cast<int4 *>(sm + L.units);
    int *slist = reinterpret_cast<int *>(sm + L.slist);
    int *misc = reinterpret_cast<int *>(sm + L.misc);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + L.bars);
    uint64_t *empty = full + kFMaxRing;
    uint64_t *xbar = empty + kFMaxRing;
    uint64_t *abar = xbar + 2;  // [kFGroups]
    volatile int *abort_flag = misc + kMiscAbort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = p.T, E = p.E, k = p.k, H = p.H, Tk = T * k;
    if (tid == 0) {
        for (int s = 0; s < p.ring; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(xbar, 1);
        for (int i = 0; i < kFGroups; i++) mbar_init(&abar[i], 1);
        misc[kMiscAbort] = 0;
        fence_mbar_init();
    }
    for (int e = tid; e < E; e += blockDim.x) mask[e] = 0ull;
    // everything below reads what the router wrote
    grid_dependency_wait();
    __syncthreads();

    // ------------------------------------------------------------- dispatch
    for (int i = tid; i < Tk; i += blockDim.x) {
        sidx[i] = __ldcg(p.idx + i);
        sw[i] = __ldcg(p.wts + i);
    }
    __syncthreads();
    for (int i = tid; i < Tk; i += blockDim.x) atomicOr(&mask[sidx[i]], 1ull << (i / k));
    __syncthreads();
    // one scan of (count << 16 | units): both sums stay below 2^16 (T k <= 1024)
    // thread tid owns experts [tid ept, tid ept + ept) (E <= 2 blockDim.x)
    const int ept = (E + blockDim.x - 1) / blockDim.x, eb = tid * ept;
    int local = 0;
    for (int e = eb; e < eb + ept && e < E; e++) {
        const int c = __popcll(mask[e]);
        local += (c << 16) | ((c + kFTile - 1) / kFTile);
    }
    int packed_total;
    int packed = cta_exclusive_scan(local, misc + kMiscScan, &packed_total);
    const int utot = packed_total & 0xffff;
    const int nsh = (T + kFTile - 1) / kFTile;
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
    __syncthreads();
    for (int i = tid; i < Tk; i += blockDim.x) {
        const int t = i / k, ej = sidx[i];
        const int pos = soff[ej] + __popcll(mask[ej] & ((1ull << t) - 1ull));
        slist[pos] = t;
        sslot[i] = pos;
        int rank = 0;
        for (int jj = 0; jj < k; jj++) rank += sidx[t * k + jj] < ej;
        sord[t * k + rank] = i;  // combine order: ascending expert id
    }
    __syncthreads();

    // --------------------------------------------------------------- items
    const int n_units = nsh + utot;
    const int nsl = p.Ip / kSlabRows;                 // gate/up items per unit
    const int ndn = H / (kSlabRows * kDownSlabs);     // down items per unit
    const int N1 = n_units * nsl, N2 = n_units * ndn;
    // items are claimed from two global queues (gate/up first, then down):
    // a CTA that finishes early takes more, so the last CTA does not trail
    const bool staged = p.staged != 0;
    int *meta = misc + kMiscMeta;  // item id of each ring slot (or kItemEnd)
    const size_t gu_bytes = (size_t)p.nseg_h * UB, dn_bytes = (size_t)kDownSlabs * p.nseg_i * UB;

    if (warp == kFWarps) {
        // ---------------------------------------------------- copy warp
        if (lane == 0) {
            if (staged) {
                mbar_arrive_expect_tx(xbar, (uint32_t)(T * H * 2));
                for (int t = 0; t < T; t++)
                    bulk_g2s(xs + (size_t)t * (H + 8), p.x16 + (size_t)t * H, (uint32_t)(H * 2),
                             xbar);
            }
            // claim items until both queues are empty, then leave one end
            // marker per group (a marker completes its slot with no bytes)
            int j = 0, ended = 0;
            bool gu_left = true, dn_left = true;
            for (; ended < kFGroups; j++) {
                const int slot = j % p.ring;
                if (j >= p.ring && !fwait(&empty[slot], ((j / p.ring) - 1) & 1, p, abort_flag))
                    break;
                int item = kItemEnd;
                if (gu_left) {
                    const int gq = atomicAdd(p.queue, 1);
                    if (gq < N1) item = gq;
                    else gu_left = false;
                }
                if (item == kItemEnd && dn_left) {
                    const int dq = atomicAdd(p.queue + 1, 1);
                    if (dq < N2) item = N1 + dq;
                    else dn_left = false;
                }
                meta[slot] = item;  // published by the arrive below
                uint8_t *dst = ring + (size_t)slot * p.item_bytes;
                if (item == kItemEnd) {
                    mbar_arrive(&full[slot]);
                    ended++;
                } else if (item < N1) {
                    const int u = item / nsl, slab = item % nsl;
                    const int e = units[u].x;
                    const uint8_t *wg = (e == E ? p.shared : p.routed + (size_t)e * p.expert_bytes) +
                                        (size_t)slab * gu_bytes;
                    mbar_arrive_expect_tx(&full[slot], (uint32_t)(2 * gu_bytes));
                    const uint64_t pol = l2_evict_first_policy();  // weights: read once
                    bulk_g2s_hint(dst, wg, (uint32_t)gu_bytes, &full[slot], pol);
                    bulk_g2s_hint(dst + gu_bytes, wg + p.mat_bytes, (uint32_t)gu_bytes, &full[slot],
                                  pol);
                } else {
                    const int di = item - N1, u = di / ndn, rg = di % ndn;
                    const int e = units[u].x;
                    const uint8_t *wd = (e == E ? p.shared : p.routed + (size_t)e * p.expert_bytes) +
                                        2 * p.mat_bytes + (size_t)rg * dn_bytes;
                    mbar_arrive_expect_tx(&full[slot], (uint32_t)dn_bytes);
                    bulk_g2s_hint(dst, wd, (uint32_t)dn_bytes, &full[slot],
                                  l2_evict_first_policy());
                }
            }
            // the CTA must not exit with copies in flight (abort path)
            for (int i = j > p.ring ? j - p.ring : 0; i < j; i++)
                mbar_drain(&full[i % p.ring], (i / p.ring) & 1);
            if (staged) mbar_drain(xbar, 0);
        }
        return;
    }

    // ------------------------------------------------------ compute groups
    const int gi = warp >> 2, q = warp & 3, gtid = tid & 127;
    const int sa = q * p.nseg_h / 4, sb = (q + 1) * p.nseg_h / 4;
    const int g = lane >> 2, cq = lane & 3;
    const int per_blk = k + 1;  // down items that write one (token, row block)
    int *flag = misc + kMiscFlag + gi;
    int *flag2 = misc + kMiscFlag2 + gi;  // second go/stop word of a down item
    int *comb = misc + kMiscComb + 9 * gi;
    __half *abuf = reinterpret_cast<__half *>(sm + L.abuf) + (size_t)gi * kFTile * (p.Ip + 8);
    uint32_t a_uses = 0;  // phases of abar[gi] used so far (thread gtid 0)
    if (staged) {
        // one waiter per group, the answer shared through the group barrier
        if (gtid == 0) *flag = fwait(xbar, 0, p, abort_flag) ? 1 : 0;
        group_sync(gi);
        if (!*flag) return;
        group_sync(gi);
    }
    for (int j = gi;; j += kFGroups) {
        const int slot = j % p.ring;
        if (gtid == 0) *flag = fwait(&full[slot], (j / p.ring) & 1, p, abort_flag) ? 1 : 0;
        group_sync(gi);
        if (!*flag) return;  // the whole group leaves together
        const int item = meta[slot];
        if (item == kItemEnd) break;
        const bool is_gu = item < N1;
        const int u = is_gu ? item / nsl : (item - N1) / ndn;
        const int part = is_gu ? item % nsl : (item - N1) % ndn;
        const int4 un = units[u];
        const int slot0 = un.y, n = un.z;
        if (!is_gu) {
            // a down item needs every gate/up slab of its unit (other CTAs);
            // then its n activation rows come in with one bulk copy each
            if (gtid == 0) {
                bool ok = fwait_count(p.done_gu + u, nsl, p, abort_flag);
                if (ok) {
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                    mbar_arrive_expect_tx(&abar[gi], (uint32_t)(n * p.Ip * 2));
                    for (int r = 0; r < n; r++)
                        bulk_g2s(abuf + (size_t)r * (p.Ip + 8), p.a + (size_t)(slot0 + r) * p.Ip,
                                 (uint32_t)(p.Ip * 2), &abar[gi]);
                    ok = fwait(&abar[gi], a_uses & 1, p, abort_flag);
                    if (!ok) mbar_drain(&abar[gi], a_uses & 1);
                    a_uses++;
                }
                *flag2 = ok ? 1 : 0;
            }
            group_sync(gi);
            if (!*flag2) return;
        }
        const uint8_t *w = ring + (size_t)slot * p.item_bytes;
        if (is_gu) {
            // ------------------------------------------------ gate/up item
            float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
            if (staged) {
                const int r = lane & 7, sl = slot0 + (r < n ? r : 0);
                const __half *rowp = xs + (size_t)(sl < Tk ? slist[sl] : sl - Tk) * (H + 8);
                fused_slab2<kBits, kSrcSmem>(accg, accu, w + sa * UB, w + gu_bytes + sa * UB,
                                             sb - sa, rowp, sa * 128, lane);
            } else {
                const int sl = slot0 + (g < n ? g : 0);
                const __half *rowp = p.x16 + (size_t)(sl < Tk ? slist[sl] : sl - Tk) * H;
                fused_slab2<kBits, kSrcLdg>(accg, accu, w + sa * UB, w + gu_bytes + sa * UB,
                                            sb - sa, rowp, sa * 128, lane);
            }
            float *rd = red + ((gi * 4 + q) * 32 + lane) * 8;
#pragma unroll
            for (int i = 0; i < 4; i++) {
                rd[i] = accg[i];
                rd[4 + i] = accu[i];
            }
            group_sync(gi);
            if (gtid == 0) mbar_arrive(&empty[slot]);  // the weights are consumed
            if (q == 0) {
                const float *r0 = red + ((gi * 4 + 0) * 32 + lane) * 8;
                const float *r1 = r0 + 32 * 8, *r2 = r1 + 32 * 8, *r3 = r2 + 32 * 8;
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    float gs = ((r0[i] + r1[i]) + r2[i]) + r3[i];
                    float us = ((r0[4 + i] + r1[4 + i]) + r2[4 + i]) + r3[4 + i];
                    gs *= 0.5f;  // the integers are 2(q - c): one factor 2 out
                    us *= 0.5f;
                    const float av = gs / (1.0f + expf(-gs)) * us;
                    const int tok = 2 * cq + (i & 1);
                    const int row = part * kSlabRows + g + 8 * (i >> 1);
                    if (tok < n) p.a[(size_t)(slot0 + tok) * p.Ip + row] = __float2half_rn(av);
                }
                __syncwarp();
                if (lane == 0) {
                    __threadfence();  // the warp's stores, then the count
                    atomicAdd(p.done_gu + u, 1);
                }
            }
            group_sync(gi);  // the reduction scratch is free again
        } else {
            // --------------------------------------------------- down item
            const int ar = lane & 7;
            const __half *rowp = abuf + (size_t)(ar < n ? ar : 0) * (p.Ip + 8);
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            const uint8_t *w0 = w + (size_t)(2 * q) * p.nseg_i * UB;  // slabs 2q, 2q + 1
            fused_slab2<kBits, kSrcSmem>(acc[0], acc[1], w0, w0 + (size_t)p.nseg_i * UB, p.nseg_i,
                                         rowp, 0, lane);
#pragma unroll
            for (int s = 0; s < 2; s++)
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int tok = 2 * cq + (i & 1);
                    const int row = (part * kDownSlabs + 2 * q + s) * kSlabRows + g + 8 * (i >> 1);
                    if (tok < n) p.Y[(size_t)(slot0 + tok) * H + row] = 0.5f * acc[s][i];
                }
            __threadfence();
            group_sync(gi);
            if (gtid == 0) {
                mbar_arrive(&empty[slot]);
                int nc = 0;
                for (int i = 0; i < n; i++) {
                    const int sl = slot0 + i;
                    const int t = sl < Tk ? slist[sl] : sl - Tk;
                    if (atomicAdd(p.done_tok + t * ndn + part, 1) == per_blk - 1)
                        comb[1 + nc++] = t;
                }
                comb[0] = nc;
                __threadfence();
            }
            group_sync(gi);
            // this item finished the last expert rows of these (token, block)
            // pairs: y = Y_shared + sum over the picks in ascending expert id
            // of w Y, one column per thread, every row requested up front
            for (int ci = 0; ci < comb[0]; ci++) {
                const int t = comb[1 + ci];
                const int col = part * kSlabRows * kDownSlabs + gtid;
                float v[kFMaxK];
#pragma unroll
                for (int r = 0; r < kFMaxK; r++)
                    v[r] = r < k ? __ldcg(p.Y + (size_t)sslot[sord[t * k + r]] * H + col) : 0.0f;
                float acc = __ldcg(p.Y + (size_t)(Tk + t) * H + col);
#pragma unroll
                for (int r = 0; r < kFMaxK; r++)
                    if (r < k) acc = fmaf(sw[sord[t * k + r]], v[r], acc);
                __nv_bfloat16 *o = p.out + (size_t)t * H + col;
                const __nv_bfloat16 yb = __float2bfloat16_rn(acc);
                *o = p.residual ? __float2bfloat16_rn(__fadd_rn(__bfloat162float(*o),
                                                                __bfloat162float(yb)))
                                : yb;
            }
        }
    }
}

// ------------------------------------------------------------------- host
static int g_fused_max_smem = 0;
static int g_fused_sms = 0;

int fused_decode_supported(const Geometry &g, int T) {
    return T >= 1 && T <= kFMaxT && g.E <= 512 && g.E <= 2 * kFThreads && g.k <= kFMaxK &&
           g.H % 128 == 0 && g.Ip % 128 == 0 && g.H <= 8192;
}

size_t fused_item_bytes(const Geometry &g) {
    const int a = 2 * g.nseg_h, b = kDownSlabs * g.nseg_i;
    return (size_t)(a > b ? a : b) * g.ub;
}

cudaError_t launch_fused_decode(const Geometry &g, const ExpertWeights &w, const int32_t *idx,
                                const float *wts, const void *x16, int T, int units_max, void *a,
                                float *Y,
                                void *out, bool residual, int *done_gu, int *done_tok, int *queue,
                                int *err, long long budget, cudaStream_t s) {
    if (!fused_decode_supported(g, T) || g_fused_max_smem == 0) return cudaErrorInvalidValue;
    FusedParams p{};
    p.routed = w.routed;
    p.shared = w.shared;
    p.expert_bytes = g.expert_bytes;
    p.mat_bytes = g.mat_bytes;
    p.idx = idx;
    p.wts = wts;
    p.x16 = reinterpret_cast<const __half *>(x16);
    p.T = T;
    p.E = g.E;
    p.k = g.k;
    p.H = g.H;
    p.Ip = g.Ip;
    p.nseg_h = g.nseg_h;
    p.nseg_i = g.nseg_i;
    p.item_bytes = (int)fused_item_bytes(g);
    p.units_max = units_max;
    p.a = reinterpret_cast<__half *>(a);
    p.Y = Y;
    p.out = reinterpret_cast<__nv_bfloat16 *>(out);
    p.residual = residual ? 1 : 0;
    p.done_gu = done_gu;
    p.done_tok = done_tok;
    p.queue = queue;
    p.err = err;
    p.budget = budget;
    // ring depth and token staging from the shared memory left over
    const int fixed_nost =
        fused_smem(T, g.E, g.k, g.H, g.Ip, 0, p.item_bytes, 0, units_max).total;
    const int xs_bytes = align16(T * (g.H + 8) * 2);
    p.staged = (T <= kFStagedMaxT && g_fused_max_smem - fixed_nost - xs_bytes >= 4 * p.item_bytes)
                   ? 1 : 0;
    const int room = g_fused_max_smem - fixed_nost - (p.staged ? xs_bytes : 0);
    p.ring = room / p.item_bytes;
    if (p.ring > kFMaxRing) p.ring = kFMaxRing;
    if (p.ring < 2) return cudaErrorInvalidValue;
    const int smem =
        fused_smem(T, g.E, g.k, g.H, g.Ip, p.ring, p.item_bytes, p.staged, units_max).total;
    auto kern = g.bits == 2 ? fused_decode_kernel<2> : fused_decode_kernel<3>;
    return launch_pdl(kern, dim3(g_fused_sms), dim3(kFThreads), (size_t)smem, s, p);
}

cudaError_t fused_init_attributes(int max_smem) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_fused_sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e;
    if ((e = allow_max_dyn_smem(fused_decode_kernel<2>, max_smem)) != cudaSuccess) return e;
    if ((e = allow_max_dyn_smem(fused_decode_kernel<3>, max_smem)) != cudaSuccess) return e;
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, reinterpret_cast<const void *>(fused_decode_kernel<2>))) !=
        cudaSuccess)
        return e;
    g_fused_max_smem = max_smem - (int)fa.sharedSizeBytes;
    return cudaSuccess;
}

}  // namespace strata

