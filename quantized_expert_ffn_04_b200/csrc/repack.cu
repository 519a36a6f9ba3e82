// Weight repack (canonical packed format -> GPU fragment layout) and the debug
// dequantiser that reads the GPU layout back.
//
// Format (layer specification): blocks of 32 weights along the input dimension,
// 2-bit w = d*(q-1.5) or 3-bit w = d*(q-3.5), one fp16 scale d per block.  The
// pages name the 2-3 bit builds only ("Strata Runs 125B Qwen3.8-Flash-Next on a
// 12GB Gaming GPU at Up to 94 Tokens/s", sections "The numbers, measured by the
// author" and "Caveats").
#include "common.cuh"
#include "internal.h"

namespace strata {

// Code of (row, col) of a canonical matrix with K columns.
__device__ __forceinline__ int canon_code(const uint8_t *codes, int bits, int K, int row,
                                          int col) {
    size_t blk = (size_t)row * (K / 32) + col / 32;
    const uint8_t *b = codes + blk * (size_t)(4 * bits);
    int bit = bits * (col & 31);
    uint32_t two = b[bit >> 3] | ((bit >> 3) + 1 < 4 * bits ? (uint32_t)b[(bit >> 3) + 1] << 8 : 0u);
    return (two >> (bit & 7)) & ((1 << bits) - 1);
}

// One thread per (unit, lane).
__global__ void repack_kernel(const uint8_t *__restrict__ codes,
                              const uint16_t *__restrict__ scales, int bits, int R, int K, int Rp,
                              int Kp, uint8_t *__restrict__ out) {
    int nseg = Kp / kSegCols;
    long long n_units = (long long)(Rp / kSlabRows) * nseg;
    long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= n_units * 32) return;
    int lane = (int)(gid & 31);
    long long unit = gid >> 5;
    int slab = (int)(unit / nseg), seg = (int)(unit % nseg);
    int g = lane >> 2, c = lane & 3;
    int ub = unit_bytes(bits);
    uint8_t *u = out + unit * ub;

    uint32_t lo[4] = {0, 0, 0, 0}, hi[2] = {0, 0};
    for (int w = 0; w < 4; w++) {
        for (int rp = 0; rp < 8; rp++) {
            int s = rp >> 2, r = rp & 3;
            int row = slab * kSlabRows + g + 8 * (r & 1);
            int col0 = seg * kSegCols + 32 * w + 16 * s + 2 * c + 8 * (r >> 1);
            for (int half = 0; half < 2; half++) {
                int col = col0 + half;
                int q = (row < R && col < K) ? canon_code(codes, bits, K, row, col) : 0;
                lo[w] |= (uint32_t)(q & 3) << (code_pos(bits == 1 ? 2 : bits, rp) + 16 * half);
                if (bits == 3)
                    hi[w >> 1] |= (uint32_t)((q >> 2) & 1) << (rp + 8 * (w & 1) + 16 * half);
            }
        }
    }
    uint16_t sc[2];
    for (int h = 0; h < 2; h++) {
        int row = slab * kSlabRows + g + 8 * h;
        int blkcol = seg * 4 + c;
        sc[h] = (row < R && blkcol * 32 < K) ? scales[(size_t)row * (K / 32) + blkcol] : 0;
    }
    if (bits == 1)  // blocks 2h and 2h + 1 share word h, the odd one a bit higher
        reinterpret_cast<uint2 *>(u)[lane] = make_uint2(lo[0] | (lo[1] << 1), lo[2] | (lo[3] << 1));
    else
        reinterpret_cast<uint4 *>(u)[lane] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    int off = lo_bytes(bits);
    if (bits == 3) {
        reinterpret_cast<uint2 *>(u + off)[lane] = make_uint2(hi[0], hi[1]);
        off += kHiBytes;
    }
    reinterpret_cast<uint32_t *>(u + off)[lane] = (uint32_t)sc[0] | ((uint32_t)sc[1] << 16);
}

void launch_repack_matrix(const uint8_t *codes, const uint16_t *scales, int bits, int R, int K,
                          int Rp, int Kp, uint8_t *out, cudaStream_t s) {
    long long threads = (long long)(Rp / kSlabRows) * (Kp / kSegCols) * 32;
    int bs = 256;
    long long grid = (threads + bs - 1) / bs;
    repack_kernel<<<(unsigned)grid, bs, 0, s>>>(codes, scales, bits, R, K, Rp, Kp, out);
}

// ---- row norms for the token prescale: the largest L2 norm over the rows of
// a canonical matrix [R][K] of dequantised weights d (q - c), folded into
// *out_bits with an integer max (a non-negative float's bits order like the
// float).  One warp per row.  The prescale only needs a bound, and it pads
// this one by 0.1 %, far more than the rounding of the fp32 sum.
__global__ void row_norm_max_kernel(const uint8_t *__restrict__ codes,
                                    const uint16_t *__restrict__ scales, int bits, int R, int K,
                                    unsigned *__restrict__ out_bits) {
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (row >= R) return;
    const float c = bits == 2 ? 1.5f : 3.5f;
    float ss = 0.0f;
    for (int col = lane; col < K; col += 32) {
        const float d = __half2float(__ushort_as_half(scales[(size_t)row * (K / 32) + col / 32]));
        const float w = d * ((float)canon_code(codes, bits, K, row, col) - c);
        ss = fmaf(w, w, ss);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) atomicMax(out_bits, __float_as_uint(sqrtf(ss)));
}

void launch_row_norm_max(const uint8_t *codes, const uint16_t *scales, int bits, int R, int K,
                         unsigned *out_bits, cudaStream_t s) {
    row_norm_max_kernel<<<(unsigned)((R + 7) / 8), 256, 0, s>>>(codes, scales, bits, R, K,
                                                                 out_bits);
}

// ---- debug dequant: decode single weights from the GPU layout with the same
// device routines the kernels use.
template <int kBits>
__device__ float debug_weight(const uint8_t *mat, int Kp, int row, int col, int kind) {
    int nseg = Kp / kSegCols;
    int slab = row / kSlabRows, seg = col / kSegCols;
    const uint8_t *u = mat + ((size_t)slab * nseg + seg) * unit_bytes(kBits);
    int rr = row % kSlabRows, cc = col % kSegCols;
    int w = cc / 32, j = cc % 32;
    int s = j / 16, kk = j % 16;
    int g = rr & 7;
    int r = (rr >= 8 ? 1 : 0) + (kk >= 8 ? 2 : 0);
    int c = (kk & 7) >> 1, half = kk & 1;
    int lane = 4 * g + c;
    int rp = 4 * s + r;
    uint32_t lo = unit_word<kBits>(u, lane, w);
    uint32_t hi = 0;
    int off = lo_bytes(kBits);
    if (kBits == 3) {
        hi = reinterpret_cast<const uint32_t *>(u + off)[lane * 2 + (w >> 1)];
        off += kHiBytes;
    }
    // scale of (row, block w): stored by lane 4*(row&7) + w
    uint32_t sw = reinterpret_cast<const uint32_t *>(u + off)[4 * g + w];
    uint16_t dbits = (uint16_t)(rr >= 8 ? (sw >> 16) : (sw & 0xffff));
    __half d = __ushort_as_half(dbits);
    if (kind == 0) {
        // the code read straight from its bit position, then 2q - (2^bits - 1)
        int q = (lo >> (code_pos(kBits == 1 ? 2 : kBits, rp) + 16 * half)) & (kBits == 1 ? 1 : 3);
        if (kBits == 3) q |= ((hi >> (rp + 8 * (w & 1) + 16 * half)) & 1) << 2;
        const float q2 = (float)(2 * q - ((1 << kBits) - 1));
        return q2 * (__half2float(d) * 0.5f);  // exact in fp32
    } else {
        // the tensor-core operand, computed by the prefill kernels' routine
        uint32_t p = kBits <= 2 ? dq2_pair<kBits == 1 ? 1 : 2>(lo, rp)
                                : dq_pair<false, kBits>(lo, hi, rp, 8 * (w & 1));
        __half2 v = *reinterpret_cast<__half2 *>(&p);
        __half dh = __hmul(d, __float2half(0.5f));
        __half2 wv = __hmul2(v, __half2half2(dh));
        return __half2float(half ? __high2half(wv) : __low2half(wv));
    }
}

__global__ void debug_dequant_kernel(const uint8_t *mat, int bits, int Kp, int row0, int nrows,
                                     int ncols, int kind, float *out) {
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)nrows * ncols) return;
    int r = (int)(i / ncols), c = (int)(i % ncols);
    out[i] = bits == 1   ? debug_weight<1>(mat, Kp, row0 + r, c, kind)
             : bits == 2 ? debug_weight<2>(mat, Kp, row0 + r, c, kind)
                         : debug_weight<3>(mat, Kp, row0 + r, c, kind);
}

void launch_debug_dequant(const uint8_t *mat, int bits, int Kp, int row0, int nrows, int ncols,
                          int kind, float *out, cudaStream_t s) {
    long long n = (long long)nrows * ncols;
    debug_dequant_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(mat, bits, Kp, row0, nrows,
                                                                      ncols, kind, out);
}

}  // namespace strata
