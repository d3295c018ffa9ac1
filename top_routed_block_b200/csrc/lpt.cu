// lpt.cu -- longest-first ordering of the work items (CSR rows).
//
// FVAttn review, §1 "RLB" and §3: once the sparse mask is fixed, the per-head
// work is known and is balanced at run time (there by moving heads between
// GPUs).  On one GPU the same idea becomes a longest-processing-time-first
// queue: rows sorted by selected-block count descending, equal counts by
// ascending row id, consumed by a persistent grid.
//
// A stable counting sort in three kernels:
//   lpt_rank_kernel     per chunk of 1024 rows: a per-chunk histogram of the
//                       counts and each row's rank among earlier rows of the
//                       chunk with the same count (warps in turn, so the rank
//                       follows row order).
//   lpt_offsets_kernel  one CTA: bucket starts in descending count order, then
//                       per (chunk, count) starting offsets.
//   lpt_scatter_kernel  order[offset(chunk, count) + rank] = row.
#include <cstdint>

#include "common.cuh"
#include "lpt.cuh"

namespace fvattn {

namespace {

constexpr int kChunk = 1024;

__device__ __forceinline__ int row_count(const int32_t *row_ptr, int64_t r, int max_count, int32_t *dev_status) {
    int c = row_ptr[r + 1] - row_ptr[r];
    if (c < 0 || c > max_count) {
        record_error(dev_status, FVATTN_ERR_BAD_CSR);
        c = c < 0 ? 0 : max_count;
    }
    return c;
}

__global__ void __launch_bounds__(kChunk) lpt_rank_kernel(const int32_t *__restrict__ row_ptr, int64_t rows,
                                                          int max_count, int32_t *__restrict__ hist,
                                                          int32_t *__restrict__ rank, int32_t *dev_status) {
    extern __shared__ int32_t counters[];  // [max_count + 1]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int k = tid; k <= max_count; k += kChunk) counters[k] = 0;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * kChunk + tid;
    const bool valid = r < rows;
    const int key = valid ? row_count(row_ptr, r, max_count, dev_status) : -1;
    __syncthreads();
    for (int w = 0; w < kChunk / 32; ++w) {
        if (warp == w) {
            const unsigned peers = __match_any_sync(0xffffffffu, key);
            const int leader = __ffs(peers) - 1;
            int base = 0;
            if (valid && lane == leader) {
                base = counters[key];
                counters[key] = base + __popc(peers);
            }
            base = __shfl_sync(0xffffffffu, base, leader);
            if (valid) rank[r] = base + __popc(peers & ((1u << lane) - 1u));
        }
        __syncthreads();
    }
    int32_t *h = hist + static_cast<int64_t>(blockIdx.x) * (max_count + 1);
    for (int k = tid; k <= max_count; k += kChunk) h[k] = counters[k];
}

__global__ void __launch_bounds__(1024) lpt_offsets_kernel(int32_t *__restrict__ hist, int64_t nchunks,
                                                           int max_count) {
    // hist[chunk][k] -> first output position of (chunk, k); keys descending.
    __shared__ long long wsum[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = max_count + 1;
    long long carry = 0;
    // process keys in descending order, 1024 keys per pass
    for (int pass = 0; pass * 1024 < K; ++pass) {
        const int k = max_count - (pass * 1024 + tid);  // descending
        long long tot = 0;
        if (k >= 0)
            for (int64_t c = 0; c < nchunks; ++c) tot += hist[c * K + k];
        long long inc = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long t = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += t;
        }
        if (lane == 31) wsum[warp] = inc;
        __syncthreads();
        long long wpre = 0;
        for (int w = 0; w < warp; ++w) wpre += wsum[w];
        long long start = carry + wpre + inc - tot;
        if (k >= 0)
            for (int64_t c = 0; c < nchunks; ++c) {
                const long long h = hist[c * K + k];
                hist[c * K + k] = static_cast<int32_t>(start);
                start += h;
            }
        long long block_total = 0;
        for (int w = 0; w < 32; ++w) block_total += wsum[w];
        carry += block_total;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(256) lpt_scatter_kernel(const int32_t *__restrict__ row_ptr, int64_t rows,
                                                          int max_count, const int32_t *__restrict__ hist,
                                                          const int32_t *__restrict__ rank,
                                                          int32_t *__restrict__ order) {
    const int64_t r = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
    if (r >= rows) return;
    int c = row_ptr[r + 1] - row_ptr[r];
    c = c < 0 ? 0 : (c > max_count ? max_count : c);
    const int64_t chunk = r / kChunk;
    order[hist[chunk * (max_count + 1) + c] + rank[r]] = static_cast<int32_t>(r);
}

}  // namespace

LptWorkspace lpt_workspace_layout(int64_t rows, int max_count) {
    LptWorkspace w{};
    Carver c;
    const int64_t nchunks = ceil_div(rows > 0 ? rows : 1, kChunk);
    w.rank = c.take<int32_t>(static_cast<size_t>(rows > 0 ? rows : 1));
    w.hist = c.take<int32_t>(static_cast<size_t>(nchunks) * (max_count + 1));
    w.total = align_up(c.off, 256);
    return w;
}

cudaError_t launch_lpt_order(const int32_t *row_ptr, int64_t rows, int max_count, int32_t *order, void *workspace,
                             int32_t *dev_status, cudaStream_t stream) {
    if (rows <= 0) return cudaSuccess;
    const LptWorkspace w = lpt_workspace_layout(rows, max_count);
    char *ws = static_cast<char *>(workspace);
    int32_t *rank = reinterpret_cast<int32_t *>(ws + w.rank);
    int32_t *hist = reinterpret_cast<int32_t *>(ws + w.hist);
    const int64_t nchunks = ceil_div(rows, kChunk);
    const size_t smem = sizeof(int32_t) * (max_count + 1);
    lpt_rank_kernel<<<static_cast<unsigned>(nchunks), kChunk, smem, stream>>>(row_ptr, rows, max_count, hist, rank,
                                                                            dev_status);
    lpt_offsets_kernel<<<1, 1024, 0, stream>>>(hist, nchunks, max_count);
    lpt_scatter_kernel<<<static_cast<unsigned>(ceil_div(rows, 256)), 256, 0, stream>>>(row_ptr, rows, max_count,
                                                                                       hist, rank, order);
    return cudaGetLastError();
}

}  // namespace fvattn
