// Device helpers shared by the library's kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define STRATA_DEV __device__ __forceinline__

namespace strata {

// ---------------------------------------------------------------- layout
// GPU weight layout of one quantised matrix [R rows][K cols]:
//   slabs of 16 rows x segments of 128 columns; unit (slab, seg) at
//   ((slab * (K/128)) + seg) * unit_bytes.  Inside a unit:
//     [0, 512)        low two bits of every code, mma-fragment order:
//                     lane L = 4g + c owns 16 bytes = 4 words, word w = block w
//                     of the segment (32 columns).  Bit positions inside word w
//                     for fragment register r' = 4s + r (s = k-step of the block,
//                     r = mma A register 0..3): half 0 at bits P..P+1, half 1 at
//                     bits 16+P..16+P+1, with P = code_pos(bits, r'):
//                       2-bit: P = 2, 10, 4, 12, 6, 14, 8, 0 for r' = 0..7:
//                              r' = 0, 2, 4, 6 come out of one mask each (the code
//                              sits in the fp16 mantissa at bit 2, 4, 6, 8),
//                              r' = 1, 3, 5 after one shift right by 8 and r' = 7
//                              after one shift left by 8, so the two registers
//                              of a k-step that share columns (r and r + 1, r
//                              even) hold their codes at the same mantissa bit
//                              (2 + 2 (r' >> 1)): columns 8h .. 8h + 7 of a block
//                              all sit at bit 2 + 2h;
//                       3-bit: P = 2r'.
//                     Register r holds (row, col) pairs of the m16n8k16 A
//                     fragment: r=0 (g, 2c|2c+1), r=1 (g+8, 2c|2c+1),
//                     r=2 (g, 2c+8|2c+9), r=3 (g+8, 2c+8|2c+9); col relative to
//                     16*s inside the block.
//   1-bit units keep the same positions with half the words: [0, 256), lane
//                     L owns 8 bytes = 2 words, word h holds block 2h's codes
//                     at the 2-bit positions P, 16 + P and block 2h+1's one
//                     bit higher (P + 1, 17 + P), so block 2h+1 decodes from
//                     the word shifted right by one.
//     [512, 768)      3-bit only: high bit of every code, lane L owns 8 bytes =
//                     2 words; word h holds blocks 2h (bits r', 16+r') and
//                     2h+1 (bits 8+r', 24+r').
//     [.., +128)      scales: lane L = 4g + c owns {d[g][c], d[g+8][c]} (fp16).
constexpr int kSlabRows = 16;
constexpr int kSegCols = 128;
constexpr int kLoBytes = 512;
constexpr int kHiBytes = 256;
constexpr int kScaleBytes = 128;

__host__ __device__ constexpr int code_pos(int bits, int rp) {
    return bits == 2 ? ((rp & 1) ? (rp == 7 ? 0 : 2 * (rp >> 1) + 10) : 2 * (rp >> 1) + 2)
                     : 2 * rp;
}

// Code bytes of a unit below the 3-bit high bits and the scales.
__host__ __device__ constexpr int lo_bytes(int bits) { return bits == 1 ? kLoBytes / 2 : kLoBytes; }
// Offset of the scales inside a unit.
__host__ __device__ constexpr int scale_off(int bits) {
    return lo_bytes(bits) + (bits == 3 ? kHiBytes : 0);
}
__host__ __device__ constexpr int unit_bytes(int bits) {
    return scale_off(bits) + kScaleBytes;
}
// The code word of block b (0..3) of a unit for this lane, in the 2-bit
// positions (1-bit: the shared word, shifted for the odd block).
template <int kBits>
__device__ __forceinline__ uint32_t unit_word(const uint8_t *unit, int lane, int b) {
    if (kBits == 1)
        return *reinterpret_cast<const uint32_t *>(unit + lane * 8 + (b >> 1) * 4) >> (b & 1);
    return *reinterpret_cast<const uint32_t *>(unit + lane * 16 + b * 4);
}

// ---------------------------------------------------------------- errors
// Device error word codes (handle workspace).
constexpr int kErrTimeout = 1;
constexpr int kErrBounds = 2;  // checked build: a gather/scatter index was out of range

// Index check of the checked build (compiled with -DSTRATA_CHECKS=1): true
// when 0 <= i < n; otherwise the error word (if any) gets kErrBounds and the
// caller skips the access.  In the normal build it is constant true and
// compiles away.  It never traps: a bad index is reported, not faulted on.
#ifndef STRATA_CHECKS
#define STRATA_CHECKS 0
#endif
__device__ __forceinline__ bool idx_ok(int *err, long long i, long long n) {
#if STRATA_CHECKS
    if (i >= 0 && i < n) return true;
    if (err) atomicCAS(err, 0, kErrBounds);
    return false;
#else
    (void)err, (void)i, (void)n;
    return true;
#endif
}

// ---------------------------------------------------------------- smem / PTX
STRATA_DEV uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

STRATA_DEV void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

STRATA_DEV void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

STRATA_DEV void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

STRATA_DEV void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

STRATA_DEV void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// `count` arrivals at once.
STRATA_DEV void mbar_arrive_cnt(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

STRATA_DEV bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that lets the thread sleep until the phase completes or about
// `ns` nanoseconds pass (a waiting thread then issues no instructions that the
// SM's other warps could use).
STRATA_DEV bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Non-blocking test of phase `parity` (never suspends the thread).
STRATA_DEV bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar`, giving up after `budget` SM cycles.  On
// give-up the handle's error word gets kErrTimeout and false is returned.
STRATA_DEV bool mbar_wait(uint64_t *bar, uint32_t parity, long long budget, int *err) {
    if (budget <= 0) {
        if (err) atomicCAS(err, 0, kErrTimeout);
        return false;
    }
    long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > budget) {
            if (err) atomicCAS(err, 0, kErrTimeout);
            return false;
        }
    }
    return true;
}

// After a wait gave up: let the copies this barrier tracks land before the
// CTA exits (bounded by a fixed, generous limit).
constexpr long long kDrainCycles = 1ll << 31;
STRATA_DEV void mbar_drain(uint64_t *bar, uint32_t parity) {
    long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kDrainCycles) return;
    }
}

// 1-D bulk copy global -> shared (no multicast), completes tx on `bar`.
// dst, src 16-byte aligned, bytes a multiple of 16.
STRATA_DEV void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// L2 policy for data read once per forward (expert and router weights):
// evict first, so the weight streams do not push the kernels' code, the
// routing data and the activations out of L2 between launches.
STRATA_DEV uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
STRATA_DEV void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                              uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
        "[%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
// Read-only 16-byte load with an L2 cache policy (data constant for the kernel).
STRATA_DEV float4 ldg_f4_hint(const float4 *p, uint64_t pol) {
    float4 v;
    asm("ld.global.nc.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
        : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
        : "l"(p), "l"(pol));
    return v;
}

// Programmatic dependent launch: block until the preceding kernel in the
// stream has completed and its memory is visible (a no-op when the kernel was
// launched without the programmatic-serialization attribute).
// gpu-scope add with acquire-release ordering (PTX memory model): its
// release half is cumulative over the stores a preceding barrier ordered
// first, its acquire half covers the loads a following barrier orders after.
STRATA_DEV int atom_add_acq_rel_gpu(int *p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
STRATA_DEV void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the next kernel of the stream start launching once every CTA of this
// grid has called this (or exited).
STRATA_DEV void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

STRATA_DEV void ldmatrix_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                            const void *smem_row) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(smem_row)));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + C, fp32 accumulate.
STRATA_DEV void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                         const float (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
          "f"(c[2]), "f"(c[3]));
}

STRATA_DEV void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                        const float (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
          "f"(c[2]), "f"(c[3]));
}

// ---------------------------------------------------------------- dequant
// Exact integer operand 2q - (2^bits - 1) in a 16-bit float lane pair, from the
// GPU layout's code words.  The magic exponent leaves an ulp of 1, so OR-ing
// 2q into the mantissa gives M + 2q exactly; subtracting M + 2^bits - 1 (exact)
// leaves the odd integer 2q - (2^bits - 1) in {-3..3} or {-7..7}.
//   bf16: M = 128 (0x4300), fp16: M = 1024 (0x6400).
template <bool kBf16>
struct Magic;
template <>
struct Magic<true> {
    static constexpr uint32_t kBits = 0x43004300u;
    STRATA_DEV static uint32_t sub(uint32_t v, int bits) {
        // v - (128 + 2^bits - 1) in bf16x2; 131 = 0x4303, 135 = 0x4307
        __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&v);
        uint32_t cb = bits == 2 ? 0x43034303u : 0x43074307u;
        __nv_bfloat162 c = *reinterpret_cast<__nv_bfloat162 *>(&cb);
        __nv_bfloat162 r = __hsub2(a, c);
        return *reinterpret_cast<uint32_t *>(&r);
    }
};
template <>
struct Magic<false> {
    static constexpr uint32_t kBits = 0x64006400u;
    STRATA_DEV static uint32_t sub(uint32_t v, int bits) {
        // v - (1024 + 2^bits - 1) in fp16x2; 1027 = 0x6403, 1031 = 0x6407
        __half2 a = *reinterpret_cast<__half2 *>(&v);
        uint32_t cb = bits == 2 ? 0x64036403u : 0x64076407u;
        __half2 c = *reinterpret_cast<__half2 *>(&cb);
        __half2 r = __hsub2(a, c);
        return *reinterpret_cast<uint32_t *>(&r);
    }
};

// Register r' (0..7) of block word `lo` (and high-bit word `hi` for 3-bit):
// a lane pair holding 2q - (2^bits - 1) for the two codes of that register.
template <bool kBf16, int kBits>
STRATA_DEV uint32_t dq_pair(uint32_t lo, uint32_t hi, int rp, int hshift) {
    uint32_t t = rp == 0 ? (lo << 1) : (lo >> (2 * rp - 1));
    uint32_t v = (t & 0x00060006u) | Magic<kBf16>::kBits;
    if (kBits == 3) {
        // high bit of half 0 sits at bit (hshift + rp), of half 1 at bit 16 + hshift + rp;
        // move both to bit 3 / 19 (the 8s place of 2q).
        int sh = hshift + rp - 3;
        uint32_t u = sh >= 0 ? (hi >> sh) : (hi << (-sh));
        v |= u & 0x00080008u;
    }
    return Magic<kBf16>::sub(v, kBits);
}

}  // namespace strata

// ---------------------------------------------------------------- tcgen05
namespace strata {

// Tensor memory allocation (one full warp executes these).
STRATA_DEV void tmem_alloc(uint32_t *smem_dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(smem_dst)),
                 "r"(ncols)
                 : "memory");
}
STRATA_DEV void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
STRATA_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// Shared-memory matrix descriptor, K-major without swizzle: core matrices of
// 8 rows x 16 bytes; `lbo` = byte distance between core matrices adjacent in
// K, `sbo` = between core matrices adjacent in M/N.
STRATA_DEV uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3fff);
    d |= (uint64_t)((lbo >> 4) & 0x3fff) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3fff) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100
    // base offset 0, legacy LBO mode, layout type 0 = no swizzle
    return d;
}

// Instruction descriptor, kind::f16: fp16 A and B (both K-major), fp32 D.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N) {
    return (1u << 4)                         // D format: fp32
           | (0u << 7) | (0u << 10)          // A, B format: fp16
           | ((uint32_t)(N >> 3) << 17)      // N / 8
           | ((uint32_t)(M >> 4) << 24);     // M / 16
}

STRATA_DEV void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05.mma this thread issued so far completes.
STRATA_DEV void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

STRATA_DEV void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
STRATA_DEV void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
STRATA_DEV void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor, K-major with the 128-byte swizzle: rows of
// 128 bytes (64 fp16 of K), 8-row groups 1024 bytes apart, the group base
// 1024-byte aligned.  Steps along K inside the 128-byte row add to the start
// address (the swizzle is a function of the address bits).
STRATA_DEV uint64_t umma_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3fff);
    d |= (uint64_t)1 << 16;              // leading offset: not used by swizzled K-major
    d |= (uint64_t)(1024 >> 4) << 32;    // 8-row groups
    d |= (uint64_t)1 << 46;              // descriptor version for sm_100
    d |= (uint64_t)2 << 61;              // 128-byte swizzle
    return d;
}

// Tensor-map (TMA) loads into this CTA's shared memory, completing bytes on
// `bar`; no multicast.  `map` is the generic address of a CUtensorMap kernel
// parameter; x (the column) must make x * 2 bytes a multiple of 16.
STRATA_DEV void tma_load_2d(void *dst, const void *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
STRATA_DEV void prefetch_tmap(const void *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// 16-byte cp.async global -> shared; bytes beyond `src_bytes` (0 or 16) are zero.
STRATA_DEV void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
STRATA_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
STRATA_DEV void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace strata

// ---------------------------------------------------------------- 2-bit fast path
namespace strata {

// A code q at mantissa bit pe of the fp16 value M = 1024 (0x6400, ulp 1) gives
// h = 1024 + q 2^pe exactly; fma(h, 2^(1-pe), -(1024 2^(1-pe) + 3)) is the
// exact small integer 2q - 3 (one rounding of an exact value).  Multipliers
// and offsets for pe = 2, 4, 6, 8 as fp16 pairs:
STRATA_DEV uint32_t dq2_mul(int j) {
    return j == 0 ? 0x38003800u : j == 1 ? 0x30003000u : j == 2 ? 0x28002800u : 0x20002000u;
}
STRATA_DEV uint32_t dq2_off(int j) {
    return j == 0 ? 0xE006E006u : j == 1 ? 0xD818D818u : j == 2 ? 0xD060D060u : 0xC980C980u;
}
// 1-bit: -(2^(11 - P) + 1), so h 2^(1 - P) + off = 2q - 1 (P = 2 + 2j).
STRATA_DEV uint32_t dq1_off(int j) {
    return j == 0 ? 0xE002E002u : j == 1 ? 0xD808D808u : j == 2 ? 0xD020D020u : 0xC880C880u;
}
// The code mask of column group j at mantissa bit P = 2 + 2j: two bits
// (2-bit) or one (1-bit), in both halves.
template <int kBits>
__host__ __device__ constexpr uint32_t dq_mask(int j) {
    return (kBits == 2 ? 3u : 1u) * ((1u << (2 + 2 * j)) | (1u << (18 + 2 * j)));
}

// ---------------------------------------------------------- token prescale
// The expert kernels take the token operand in fp16, whose range (largest
// 65504, smallest normal 2^-14) is far narrower than bf16's.  Every token row
// x is therefore scaled by an exact power of two, x' = x 2^-e, with e the
// smallest integer such that
//   max_i |x'_i| <= 2^9   (the 2-bit magic-offset operand x' 2^6 stays < 2^15), and
//   ||x'||_2 w2 <= 2^7    where w2 bounds the L2 norm of every gate/up row of
//                         the layer (times the down-row factor folded in on
//                         the host), so by Cauchy-Schwarz |gate'|, |up'| <= 2^7,
//                         the SwiGLU output a'' = silu(g) u 2^-2e <= 2^14 and
//                         every down output row stays below 2^15.
// The gate is unscaled for the sigmoid, a'' and the down outputs stay in
// prescaled units, and the combine multiplies by 2^e twice.  Small rows get
// e < 0 (scaled up), so their operand does not underflow.  e is clamped to
// [-120, 120]; an all-zero or non-finite row takes e = 0.

// ceil(log2 v) for finite v > 0, subnormals included.
STRATA_DEV int ceil_log2f(float v) {
    const int bits = __float_as_int(v), b = (bits >> 23) & 0xff, mant = bits & 0x7fffff;
    if (b == 0) return (32 - __clz(mant - 1)) - 149;
    return b - 127 + (mant ? 1 : 0);
}
STRATA_DEV float pow2f(int e) { return __int_as_float((127 + e) << 23); }  // -126 <= e <= 127

// First step: the exponent from the row's largest magnitude m alone.
STRATA_DEV int prescale_emax(float m) {
    if (!(m > 0.0f) || m > 3.0e38f) return 0;
    const int e = ceil_log2f(m) - 9;
    return e < -120 ? -120 : (e > 120 ? 120 : e);
}
// Final exponent: em from prescale_emax, ss = sum over the row of (x_i 2^-em)^2
// (in fp32: every term is at most 2^18, so no overflow), w2 the layer bound
// (0: no bound, em alone).
STRATA_DEV int prescale_final(int em, float ss, float w2) {
    if (!(w2 > 0.0f)) return em;
    const float v = sqrtf(ss) * w2 * 1.001f;
    const int d = (v > 128.0f && v < 3.0e38f) ? ceil_log2f(v) - 7 : 0;
    const int e = em + d;
    return e > 120 ? 120 : e;
}
// The prescale exponent of one bf16 row of length H (a multiple of 8, the row
// 16-byte aligned), computed by one warp in one fixed order: lane l takes the
// 8-element groups l, l + 32, ... (16-byte loads, four in flight), each group
// in ascending order with fma, then a halving tree.  Every kernel that needs
// e calls this, so they all get the same e.  All lanes return e.
STRATA_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
STRATA_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
STRATA_DEV int token_prescale_warp(const __nv_bfloat16 *row, int H, float w2, int lane) {
    const uint4 *r4 = reinterpret_cast<const uint4 *>(row);
    const int n8 = H >> 3;
    float m = 0.0f;
#pragma unroll 4
    for (int i = lane; i < n8; i += 32) {
        const uint4 v = r4[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; j++)
            m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int em = prescale_emax(m);
    const float sc = pow2f(-em);
    float ss = 0.0f;
#pragma unroll 4
    for (int i = lane; i < n8; i += 32) {
        const uint4 v = r4[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const float a = bf16_lo(w[j]) * sc, b = bf16_hi(w[j]) * sc;
            ss = fmaf(a, a, ss);
            ss = fmaf(b, b, ss);
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    return prescale_final(em, ss, w2);
}
// SwiGLU of a prescaled token (g, u are gate and up times 2^-ex): silu of the
// true gate, the product left in prescaled units (times 2^-2ex).
STRATA_DEV float swiglu_ps(float g, float u, int ex) {
    const float gt = ex ? g * pow2f(ex) : g;
    return g / (1.0f + expf(-gt)) * u;
}

STRATA_DEV uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Register r' (0..7) of a 2-bit (1-bit) block word: fp16 pair of 2q - 3
// (2q - 1).
template <int kBits = 2>
STRATA_DEV uint32_t dq2_pair(uint32_t w, int rp) {
    const uint32_t src = (rp & 1) ? (rp == 7 ? (w << 8) : (w >> 8)) : w;
    const int j = rp >> 1;  // the code sits at mantissa bit 2 j + 2
    return hfma2_u32((src & dq_mask<kBits>(j)) | 0x64006400u, dq2_mul(j),
                     kBits == 2 ? dq2_off(j) : dq1_off(j));
}

// One 32-wide block of a 2-bit matrix against 8 token columns, fp16
// operands, fp32 result d (fresh): the 8 fragment registers are extracted from
// word w (2 shifts, 8 mask/or, 8 packed fma) and fed to two m16n8k16 mma in
// one asm block so they land directly in the operand registers.
template <int kBits = 2>
STRATA_DEV void block_mma2(float (&d)[4], uint32_t w, uint32_t b0, uint32_t b1, uint32_t b2,
                           uint32_t b3) {
    // pure register arithmetic (not volatile): the compiler may schedule the
    // blocks of a loop around one another
    asm(
        "{\n\t"
        ".reg .b32 s8, s2, h0, h1, h2, h3, h4, h5, h6, h7;\n\t"
        ".reg .f32 z;\n\t"
        "mov.f32 z, 0f00000000;\n\t"
        "shr.b32 s8, %4, 8;\n\t"
        "shl.b32 s2, %4, 8;\n\t"
        "lop3.b32 h0, %4, %17, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h1, s8, %17, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h2, %4, %18, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h3, s8, %18, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h4, %4, %19, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h5, s8, %19, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h6, %4, %20, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h7, s2, %20, 0x64006400, 0xEA;\n\t"
        "fma.rn.f16x2 h0, h0, %9, %13;\n\t"
        "fma.rn.f16x2 h1, h1, %9, %13;\n\t"
        "fma.rn.f16x2 h2, h2, %10, %14;\n\t"
        "fma.rn.f16x2 h3, h3, %10, %14;\n\t"
        "fma.rn.f16x2 h4, h4, %11, %15;\n\t"
        "fma.rn.f16x2 h5, h5, %11, %15;\n\t"
        "fma.rn.f16x2 h6, h6, %12, %16;\n\t"
        "fma.rn.f16x2 h7, h7, %12, %16;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {h0,h1,h2,h3}, "
        "{%5,%6}, {z,z,z,z};\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {h4,h5,h6,h7}, "
        "{%7,%8}, {%0,%1,%2,%3};\n\t"
        "}\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(w), "r"(b0), "r"(b1), "r"(b2), "r"(b3), "r"(0x38003800u), "r"(0x30003000u),
          "r"(0x28002800u), "r"(0x20002000u), "r"(kBits == 2 ? 0xE006E006u : 0xE002E002u),
          "r"(kBits == 2 ? 0xD818D818u : 0xD808D808u), "r"(kBits == 2 ? 0xD060D060u : 0xD020D020u),
          "r"(kBits == 2 ? 0xC980C980u : 0xC880C880u), "n"(dq_mask<kBits>(0)),
          "n"(dq_mask<kBits>(1)), "n"(dq_mask<kBits>(2)), "n"(dq_mask<kBits>(3)));
}

// The same block without normalising the codes: each fragment register holds
// h = 1024 + q 2^P (the code at mantissa bit P = 2 + 2 (r' >> 1), exact), and
// the token operand carries the column group's factor: B_k = x_k 2^(8 - P_k)
// for column k of the block (P_k = 2 + 2 ((k mod 32) >> 3)).  Then
//   sum_k h_k B_k = sum_k 1024 B_k + 2^8 sum_k q_k x_k,
// so with the accumulator started at c = -sum_k (1024 + 1.5 2^P_k) B_k (one
// value per token column: c0 for column 2 (lane & 3), c1 for the next) the
// result is 2^8 sum_k (q_k - 1.5) x_k, the block's dot product with the
// dequantised weights over its scale, times 2^8.  Two shifts and 8 mask/or
// per block, no packed fma.
template <int kBits = 2>
STRATA_DEV void block_mma2m(float (&d)[4], uint32_t w, uint32_t b0, uint32_t b1, uint32_t b2,
                            uint32_t b3, float c0, float c1) {
    asm(
        "{\n\t"
        ".reg .b32 s8, s2, h0, h1, h2, h3, h4, h5, h6, h7;\n\t"
        "shr.b32 s8, %4, 8;\n\t"
        "shl.b32 s2, %4, 8;\n\t"
        "lop3.b32 h0, %4, %11, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h1, s8, %11, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h2, %4, %12, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h3, s8, %12, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h4, %4, %13, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h5, s8, %13, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h6, %4, %14, 0x64006400, 0xEA;\n\t"
        "lop3.b32 h7, s2, %14, 0x64006400, 0xEA;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {h0,h1,h2,h3}, "
        "{%5,%6}, {%9,%10,%9,%10};\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {h4,h5,h6,h7}, "
        "{%7,%8}, {%0,%1,%2,%3};\n\t"
        "}\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(w), "r"(b0), "r"(b1), "r"(b2), "r"(b3), "f"(c0), "f"(c1), "n"(dq_mask<kBits>(0)),
          "n"(dq_mask<kBits>(1)), "n"(dq_mask<kBits>(2)), "n"(dq_mask<kBits>(3)));
}

// Column factor of the magic-offset token operand and the correction weight
// of column k of a block (see block_mma2m), kk = k mod 32:
// B_k = x_k * magic_col_scale(kk) = x_k 2^(8 - P_k), c_k = 1024 + centre 2^P_k.
__host__ __device__ inline float magic_col_scale(int kk) {  // kk = k mod 32
    return (float)(1 << (6 - 2 * (kk >> 3)));
}
__host__ __device__ inline float magic_col_corr(int kk, int bits = 2) {
    // 1024 + centre 2^P_k, centre = (2^bits - 1) / 2 (1.5 for 2-bit, 0.5 for 1-bit)
    return 1024.0f + 0.5f * (float)((1 << bits) - 1) * (float)(1 << (2 + 2 * (kk >> 3)));
}

// ---------------------------------------------------------------- GEMV blocks
STRATA_DEV uint32_t comp4(const uint4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// One 32-wide block: D = A_blk(16x32) * B(32x8) with A the exact integers,
// two mma k-steps.  lo/hi: the lane's code words for this block.
template <int kBits>
STRATA_DEV void block_mma(float (&d)[4], uint32_t lo, uint32_t hi, int hshift, uint32_t b0,
                          uint32_t b1, uint32_t b2, uint32_t b3) {
    uint32_t a[4];
    const float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 4; r++) a[r] = dq_pair<false, kBits>(lo, hi, r, hshift);
    mma_f16(d, a, b0, b1, z);
#pragma unroll
    for (int r = 0; r < 4; r++) a[r] = dq_pair<false, kBits>(lo, hi, 4 + r, hshift);
    mma_f16(d, a, b2, b3, d);
}

}  // namespace strata
