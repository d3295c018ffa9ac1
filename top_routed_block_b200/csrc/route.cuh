// route.cuh -- internal interface of the routing kernels (route.cu).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace fvattn {

// Byte offsets of the routing workspace regions.
struct RouteWorkspace {
    size_t qbar, kbarT, counts, bitmap, total;
    int W;  // 32-bit words per row bitmap
};

RouteWorkspace route_workspace_layout(int64_t BH, int nb, int d);
size_t route_select_smem_bytes(int d, int nb);

// Key blocks past the cut reported per row for the slack-aware augmentation.
constexpr int kSasaCandidates = 8;

// Enqueues pooling, selection, CSR scan and scatter on `stream`.  With cand and
// cand_p (int32 / fp64 [rows, kSasaCandidates]), also the blocks that follow each
// row's cut in the routing order (-1 past the last) and their probabilities.
cudaError_t launch_route(const void *Q, const void *K, int64_t BH, int N, int d, int bs, int nb, double p,
                         int32_t *row_ptr, int32_t *col_idx, int64_t capacity, int32_t *head_counts,
                         void *workspace, int32_t *dev_status, cudaStream_t stream, int32_t *cand = nullptr,
                         double *cand_p = nullptr);

// row_ptr = exclusive scan of counts (one CTA; capacity overflow recorded in dev_status)
// and per-head sums of the counts of nb consecutive rows.
cudaError_t launch_csr_scan(const int32_t *counts, int64_t rows, int nb, int64_t BH, int32_t *row_ptr,
                            int64_t capacity, int32_t *head_counts, int32_t *dev_status, cudaStream_t stream);

}  // namespace fvattn
