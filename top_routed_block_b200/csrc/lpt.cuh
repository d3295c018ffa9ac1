// lpt.cuh -- internal interface of the longest-first ordering kernels (lpt.cu).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace fvattn {

struct LptWorkspace {
    size_t rank, hist, total;
};

LptWorkspace lpt_workspace_layout(int64_t rows, int max_count);

// Enqueues the three ordering kernels on `stream`; order[rows] receives the rows
// by count descending, equal counts by ascending row id.
cudaError_t launch_lpt_order(const int32_t *row_ptr, int64_t rows, int max_count, int32_t *order, void *workspace,
                             int32_t *dev_status, cudaStream_t stream);

}  // namespace fvattn
