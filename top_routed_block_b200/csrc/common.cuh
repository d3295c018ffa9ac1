// common.cuh -- status codes, device-status helpers and small utilities shared
// by the routing, ordering and attention kernels of libfvattn.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "fvattn.h"

namespace fvattn {

// First device error wins: the status word holds 0 until some thread records
// an error, after which it is never overwritten.
__device__ __forceinline__ void record_error(int32_t *dev_status, int32_t code) {
    if (dev_status) atomicCAS(reinterpret_cast<int *>(dev_status), 0, code);
}

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Host side: records the reason of the calling thread's latest FVATTN_ERR_CUDA (a
// static string), read back through fvattn_last_error().
void set_last_error(const char *what);
__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace carving: every region starts on a 256-byte boundary.
struct Carver {
    size_t off = 0;
    template <class T>
    size_t take(size_t count) {
        size_t at = align_up(off, 256);
        off = at + count * sizeof(T);
        return at;
    }
};

constexpr int kMaxRouteBlocks = 1024;   // routing keeps one row's scores in shared memory
constexpr int kMaxCount = 4096;         // largest key-block count a row may hold
constexpr int kMaxHeads = 4096;         // largest B*H of the attention call (head ordering in one CTA)

}  // namespace fvattn
