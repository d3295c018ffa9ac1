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

// Enqueues pooling, selection, CSR scan and scatter on `stream`.
cudaError_t launch_route(const void *Q, const void *K, int64_t BH, int N, int d, int bs, int nb, double p,
                         int32_t *row_ptr, int32_t *col_idx, int64_t capacity, int32_t *head_counts,
                         void *workspace, int32_t *dev_status, cudaStream_t stream);

}  // namespace fvattn
