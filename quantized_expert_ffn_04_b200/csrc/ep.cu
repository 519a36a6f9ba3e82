// Expert parallelism: the exchange plan of one rank's routing picks (host
// code) and the row gather the exchange needs (device).
//
// The pages run the model on one card or split it layer by layer across two
// or three cards, and serve several conversations at once ("Strata Runs a
// 125-Billion-Parameter Qwen Model on a 12 GB Gaming GPU ...", multi-GPU
// paragraph; "Strata ... gaming PC", usage paragraph).  Here the experts of
// one layer are split across ranks instead: rank r owns the contiguous expert
// range [ceil(r E / N), ceil((r + 1) E / N)) (expert e goes to rank
// floor(e N / E)); every rank keeps the router and
// the shared expert.  One forward of a rank's T tokens:
//   route locally -> plan (this file) -> all-to-all of the picked token rows
//   and their expert ids -> the owners run their experts on the rows they got
//   -> all-to-all of the outputs back, in the same order -> the home rank runs
//   the shared expert and combines in the layer's fixed order.
// Each expert output is a function of one token row and one expert only, so
// the result is the same bits as on one GPU on the same kernels, whatever the
// batch around it.
#include <cuda_runtime.h>

#include <vector>

#include "../../include/strata_moe.h"
#include "common.cuh"
#include "internal.h"

namespace strata {

int ep_owner(int e, int E, int n_ranks) { return (int)(((long long)e * n_ranks) / E); }

// rows[i] of src (row_bytes each, a multiple of 16) -> row i of dst; rows
// whose `keep` entry is negative (when keep is given) are left alone.
__global__ void gather_rows_bytes_kernel(const uint4 *__restrict__ src,
                                         const int32_t *__restrict__ rows, int n, int n_src,
                                         int row16, uint4 *__restrict__ dst,
                                         const int32_t *__restrict__ keep, int *err) {
    const int i = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (i >= n) return;
    if (keep && keep[i] < 0) return;
    const int r = rows[i];
    if ((unsigned)r >= (unsigned)n_src) {  // reported, never read out of bounds
        if (lane == 0 && err) atomicCAS(err, 0, kErrBounds);
        return;
    }
    const uint4 *s = src + (size_t)r * row16;
    uint4 *d = dst + (size_t)i * row16;
    for (int c = lane; c < row16; c += 32) d[c] = s[c];
}

void launch_gather_rows_bytes(const void *src, const int32_t *rows, int n, int n_src,
                              int row_bytes, void *dst, int *err, cudaStream_t s,
                              const int32_t *keep) {
    if (n <= 0) return;
    gather_rows_bytes_kernel<<<(unsigned)((n + 7) / 8), 256, 0, s>>>(
        reinterpret_cast<const uint4 *>(src), rows, n, n_src, row_bytes / 16,
        reinterpret_cast<uint4 *>(dst), keep, err);
}

}  // namespace strata

using namespace strata;

extern "C" {

strata_status strata_ep_expert_range(int rank, int n_ranks, int n_experts, int32_t *e_begin,
                                     int32_t *e_end) {
    if (n_ranks < 1 || rank < 0 || rank >= n_ranks || n_experts < 1 || !e_begin || !e_end)
        return STRATA_ERR_INVALID_ARG;
    // the smallest e with owner(e) == rank, and the same for rank + 1
    *e_begin = (int32_t)(((long long)rank * n_experts + n_ranks - 1) / n_ranks);
    *e_end = (int32_t)(((long long)(rank + 1) * n_experts + n_ranks - 1) / n_ranks);
    return STRATA_OK;
}

strata_status strata_ep_plan(const int32_t *idx, int T, int k, int n_experts, int n_ranks,
                             int32_t *send_counts, int32_t *send_pick, int32_t *slot) {
    if (T < 0 || k < 1 || n_experts < 1 || n_ranks < 1 || !send_counts ||
        (T > 0 && (!idx || !send_pick || !slot)))
        return STRATA_ERR_INVALID_ARG;
    const long long Tk = (long long)T * k;
    for (long long i = 0; i < Tk; i++)
        if (idx[i] < 0 || idx[i] >= n_experts) return STRATA_ERR_INVALID_ARG;
    // counting sort of the picks by expert id (stable: ascending pick index
    // t k + j, so ascending token inside an expert); the expert ranges of the
    // ranks are contiguous and ascending, so this is also grouped by rank
    std::vector<int64_t> cnt((size_t)n_experts + 1, 0);
    for (long long i = 0; i < Tk; i++) cnt[(size_t)idx[i] + 1]++;
    for (int e = 0; e < n_experts; e++) cnt[(size_t)e + 1] += cnt[(size_t)e];
    for (int r = 0; r < n_ranks; r++) send_counts[r] = 0;
    for (long long i = 0; i < Tk; i++) {
        const int e = idx[i];
        const int64_t p = cnt[(size_t)e]++;
        send_pick[p] = (int32_t)i;
        slot[i] = (int32_t)p;
        send_counts[ep_owner(e, n_experts, n_ranks)]++;
    }
    return STRATA_OK;
}

strata_status strata_ep_gather_rows(const void *src_dev, const int32_t *rows_dev, int n,
                                    int n_src, int row_bytes, void *dst_dev, void *stream) {
    if (n < 0 || n_src < 0 || row_bytes <= 0 || row_bytes % 16 != 0 ||
        (n > 0 && (!src_dev || !rows_dev || !dst_dev)))
        return STRATA_ERR_INVALID_ARG;
    if (((uintptr_t)src_dev | (uintptr_t)dst_dev) & 15) return STRATA_ERR_INVALID_ARG;
    launch_gather_rows_bytes(src_dev, rows_dev, n, n_src, row_bytes, dst_dev, nullptr,
                             (cudaStream_t)stream);
    return cudaGetLastError() == cudaSuccess ? STRATA_OK : STRATA_ERR_CUDA;
}

}  // extern "C"
