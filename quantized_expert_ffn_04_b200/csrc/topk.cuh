// Warp-level top-k of one token's logits (shared by the router kernels and
// the fused decode layer).  Routing rule (layer specification): the k largest
// logits, a tie going to the lower expert id, weights exp(l_j - m) / sum over
// the picks.
#pragma once

#include "common.cuh"

namespace strata {

// ============================================================== warp top-k
// Order-preserving 32-bit key of a logit: larger float <=> larger key; -0 is
// read as +0 (equal floats, equal keys) and a NaN as -inf (it ranks last).
// Key 0 is below every logit and marks a taken or missing entry.
__device__ __forceinline__ uint32_t logit_key(float f) {
    if (f != f) f = -INFINITY;
    if (f == 0.0f) f = 0.0f;
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_logit(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Best of a lane's 16 entries: the largest key, and on equal keys the lowest
// q.  A pairwise tree over adjacent entries: the left operand of every
// comparison holds the lower q's, so ">=" keeps ties on the lower q.
__device__ __forceinline__ void lane_best(const uint32_t (&key)[16], uint32_t &bk, int &bq) {
    uint32_t k8[8], k4[4], k2[2];
    int q8[8], q4[4], q2[2];
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const bool l = key[2 * i] >= key[2 * i + 1];
        k8[i] = l ? key[2 * i] : key[2 * i + 1];
        q8[i] = l ? 2 * i : 2 * i + 1;
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const bool l = k8[2 * i] >= k8[2 * i + 1];
        k4[i] = l ? k8[2 * i] : k8[2 * i + 1];
        q4[i] = l ? q8[2 * i] : q8[2 * i + 1];
    }
#pragma unroll
    for (int i = 0; i < 2; i++) {
        const bool l = k4[2 * i] >= k4[2 * i + 1];
        k2[i] = l ? k4[2 * i] : k4[2 * i + 1];
        q2[i] = l ? q4[2 * i] : q4[2 * i + 1];
    }
    const bool l = k2[0] >= k2[1];
    bk = l ? k2[0] : k2[1];
    bq = l ? q2[0] : q2[1];
}

// Top-k of one token by one warp (E <= 512: lane l holds the logits of
// experts 16 l .. 16 l + 15, read with four 16-byte loads when E is a multiple
// of 4).  Each round takes the largest key over the warp (redux.sync max) and,
// among the lanes holding it, the lowest expert id (redux.sync min), i.e. the
// larger logit and on equal logits the lower id; the winning lane drops that
// entry and finds its next best.  Lane j < k ends with pick j and its weight
// exp(l_j - m) / sum.
static __device__ __noinline__ void warp_topk(const float *__restrict__ row, int E, int k, int lane,
                                              int &pick_e, float &pick_w) {
    uint32_t key[16];
    const int e0 = 16 * lane;
    // every load is unconditional (entries past E re-read valid ones) and its
    // value is used unconditionally (masked), so no load waits for another
    if ((E & 3) == 0) {
        const float4 *r4 = reinterpret_cast<const float4 *>(row);
        float4 v[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int e = e0 + 4 * i;
            v[i] = __ldcg(r4 + ((e < E ? e : E - 4) >> 2));
        }
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float f[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int j = 0; j < 4; j++)
                key[4 * i + j] = logit_key(f[j]) & (0u - (uint32_t)(e0 + 4 * i + j < E));
        }
    } else {
#pragma unroll
        for (int q = 0; q < 16; q++) {
            const int e = e0 + q;
            const float v = __ldcg(row + (e < E ? e : E - 1));
            key[q] = logit_key(v) & (0u - (uint32_t)(e < E));
        }
    }
    uint32_t bk;
    int bq;
    lane_best(key, bk, bq);
    uint32_t my_k = 0u;
    int my_e = -1;
    for (int j = 0; j < k; j++) {
        const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t cand = (bk == wk && bk != 0u) ? (uint32_t)(e0 + bq) : 0xffffffffu;
        const uint32_t we = __reduce_min_sync(0xffffffffu, cand);
        if (lane == j) {
            my_k = wk;
            my_e = (int)we;
        }
        if ((int)(we >> 4) == lane) {
            const int wq = (int)(we & 15u);
#pragma unroll
            for (int q = 0; q < 16; q++) key[q] = q == wq ? 0u : key[q];
            lane_best(key, bk, bq);
        }
    }
    const float my_v = key_logit(my_k);
    const float m = __shfl_sync(0xffffffffu, my_v, 0);
    const float ex = lane < k ? expf(my_v - m) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    pick_e = my_e;
    pick_w = ex / sum;
}

}  // namespace strata
