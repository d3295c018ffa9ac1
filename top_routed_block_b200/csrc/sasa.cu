// sasa.cu -- slack-aware augmentation of a routed block mask (FVAttn review, §1
// Key Terms "SASA" and §3: once the work is balanced, the ranks that would sit
// idle before the slowest one finishes compute extra high-value key blocks).
//
// On one GPU the ranks are the SMs of the persistent attention grid.  The plan:
//   1. schedule: the rows, in the attention's queue order, each go to the machine
//      with the least load so far (the lowest machine on equal loads), a row's
//      load being its selected-block count; the makespan T is the largest load;
//   2. augmentation: each machine m walks its rows in the order they were
//      assigned, round after round, giving each row its next candidate (the key
//      blocks past the row's cut in the routing order, at most kSasaCandidates),
//      one block each, until its slack T - load_m is used up or no row of m has a
//      candidate left;
//   3. the augmented CSR: each row's blocks plus its added ones, ascending.
// The plan is integer arithmetic on the routed mask; it does not depend on how
// the attention kernel's dynamic queue then runs.
//
// Kernels:
//   sasa_plan_kernel     one CTA: warp 0 runs the list schedule with the machine
//                        loads in registers (warp argmin per row; the rows' counts
//                        fetched 32 at a time, one per lane); then every thread
//                        collects one machine's rows (machine ids as bytes, read
//                        through L1) and fills its slack.
//   sasa_counts_kernel   augmented row counts (then the CSR scan of route.cu).
//   sasa_scatter_kernel  one thread per row: the row's blocks merged with its
//                        added ones.
#include <climits>
#include <cstdint>

#include "common.cuh"
#include "route.cuh"
#include "sasa.cuh"

namespace fvattn {

namespace {

constexpr int kPlanThreads = kSasaMaxMachines;
constexpr int kMPL = kSasaMaxMachines / 32;  // machines per lane of the schedule warp

__global__ void __launch_bounds__(kPlanThreads)
    sasa_plan_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ order, int64_t rows,
                     int machines, const int32_t *__restrict__ cand, const double *__restrict__ cand_p,
                     uint8_t *mach_of_item, int32_t *__restrict__ lists, int32_t *__restrict__ list_off,
                     int32_t *__restrict__ added, double *__restrict__ added_mass) {
    __shared__ long long load_s[kSasaMaxMachines];
    __shared__ int rows_s[kSasaMaxMachines];
    __shared__ long long makespan;
    const int tid = threadIdx.x, lane = tid & 31;
    for (int64_t r = tid; r < rows; r += kPlanThreads) {
        added[r] = 0;
        added_mass[r] = 0.0;
    }
    if (tid < 32) {
        // 1. list schedule; lane l holds machines l, l + 32, ... (absent machines never win)
        long long ld[kMPL];
        int nr[kMPL];
#pragma unroll
        for (int q = 0; q < kMPL; ++q) {
            ld[q] = (lane + 32 * q < machines) ? 0 : LLONG_MAX;
            nr[q] = 0;
        }
        // A machine's load packed with its index, (load << 8) | m, orders machines by
        // (load, index), so one warp-wide unsigned minimum picks the machine; the
        // packed form holds loads below 2^24 (otherwise the 64-bit path below).
        const bool packed = static_cast<long long>(__ldg(row_ptr + rows)) < (1LL << 24);
        for (int64_t x0 = 0; x0 < rows; x0 += 32) {
            // the next 32 rows' block counts, one per lane
            int my_c = 0;
            if (x0 + lane < rows) {
                const int32_t row = __ldg(order + x0 + lane);
                my_c = __ldg(row_ptr + row + 1) - __ldg(row_ptr + row);
            }
            const int nx = static_cast<int>(rows - x0 < 32 ? rows - x0 : 32);
            for (int j = 0; j < nx; ++j) {
                const long long c = __shfl_sync(0xffffffffu, my_c, j);
                int bi;
                if (packed) {
                    uint32_t key = 0xffffffffu;
#pragma unroll
                    for (int q = 0; q < kMPL; ++q)
                        if (lane + 32 * q < machines)
                            key = min(key, (static_cast<uint32_t>(ld[q]) << 8) | static_cast<uint32_t>(lane + 32 * q));
                    bi = static_cast<int>(__reduce_min_sync(0xffffffffu, key) & 0xffu);
                } else {
                    long long best = ld[0];
                    bi = lane;
#pragma unroll
                    for (int q = 1; q < kMPL; ++q)
                        if (ld[q] < best) {
                            best = ld[q];
                            bi = lane + 32 * q;
                        }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        const long long ob = __shfl_xor_sync(0xffffffffu, best, o);
                        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                        if (ob < best || (ob == best && oi < bi)) {
                            best = ob;
                            bi = oi;
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < kMPL; ++q)
                    if (lane + 32 * q == bi) {
                        ld[q] += c;
                        ++nr[q];
                    }
                if (lane == 0) mach_of_item[x0 + j] = static_cast<uint8_t>(bi);
            }
        }
#pragma unroll
        for (int q = 0; q < kMPL; ++q) {
            load_s[lane + 32 * q] = ld[q];
            rows_s[lane + 32 * q] = nr[q];
        }
    }
    __syncthreads();
    if (tid == 0) {
        long long t = 0;
        int off = 0;
        for (int m = 0; m < machines; ++m) {
            if (load_s[m] > t) t = load_s[m];
            list_off[m] = off;
            off += rows_s[m];
        }
        list_off[machines] = off;
        makespan = t;
    }
    __syncthreads();
    if (tid >= machines) return;
    // each machine's rows, in the order they were assigned
    const int base = list_off[tid];
    int n = 0;
    // (plain loads: mach_of_item was written by warp 0 of this CTA, visible after the barrier)
    for (int64_t x = 0; x < rows; ++x)
        if (mach_of_item[x] == tid) lists[base + n++] = __ldg(order + x);
    // 2. fill the slack, round robin over the machine's rows
    long long slack = makespan - load_s[tid];
    while (slack > 0) {
        bool progress = false;
        for (int i = 0; i < n && slack > 0; ++i) {
            const int32_t row = lists[base + i];
            const int e = added[row];
            if (e < kSasaCandidates && cand[static_cast<int64_t>(row) * kSasaCandidates + e] >= 0) {
                added_mass[row] = added_mass[row] + cand_p[static_cast<int64_t>(row) * kSasaCandidates + e];
                added[row] = e + 1;
                --slack;
                progress = true;
            }
        }
        if (!progress) break;
    }
}

__global__ void sasa_counts_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ added,
                                   int64_t rows, int32_t *__restrict__ counts) {
    for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < rows;
         r += static_cast<int64_t>(gridDim.x) * blockDim.x)
        counts[r] = row_ptr[r + 1] - row_ptr[r] + added[r];
}

__global__ void sasa_scatter_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                                    const int32_t *__restrict__ cand, const int32_t *__restrict__ added,
                                    int64_t rows, const int32_t *__restrict__ row_ptr_out,
                                    int32_t *__restrict__ col_idx_out, int64_t capacity) {
    for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < rows;
         r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (row_ptr_out[r + 1] > capacity) continue;  // capacity error recorded by the scan
        int x[kSasaCandidates];
        const int na = added[r];
#pragma unroll
        for (int e = 0; e < kSasaCandidates; ++e) x[e] = (e < na) ? cand[r * kSasaCandidates + e] : INT_MAX;
        // the added blocks ascending (at most kSasaCandidates: insertion sort)
#pragma unroll
        for (int a = 1; a < kSasaCandidates; ++a)
#pragma unroll
            for (int b = a; b > 0; --b)
                if (x[b - 1] > x[b]) {
                    const int t = x[b - 1];
                    x[b - 1] = x[b];
                    x[b] = t;
                }
        int32_t *dst = col_idx_out + row_ptr_out[r];
        int32_t i = row_ptr[r];
        const int32_t end = row_ptr[r + 1];
        int k = 0;
        while (i < end || k < na) {
            int take;
            if (k >= na || (i < end && col_idx[i] < x[k])) {
                take = col_idx[i++];
            } else {
                take = x[k++];
            }
            *dst++ = take;
        }
    }
}

}  // namespace

cudaError_t launch_sasa(const int32_t *row_ptr, const int32_t *col_idx, const int32_t *order, int64_t rows, int nb,
                        int64_t BH, int machines, const int32_t *cand, const double *cand_p, uint8_t *mach_of_item,
                        int32_t *lists, int32_t *list_off, int32_t *counts, int32_t *added, double *added_mass,
                        int32_t *row_ptr_out, int32_t *col_idx_out, int64_t capacity, int32_t *head_counts,
                        int32_t *dev_status, cudaStream_t stream) {
    sasa_plan_kernel<<<1, kPlanThreads, 0, stream>>>(row_ptr, order, rows, machines, cand, cand_p, mach_of_item,
                                                     lists, list_off, added, added_mass);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int grid = static_cast<int>(rows / 256 + 1 < 1024 ? rows / 256 + 1 : 1024);
    sasa_counts_kernel<<<grid, 256, 0, stream>>>(row_ptr, added, rows, counts);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_csr_scan(counts, rows, nb, BH, row_ptr_out, capacity, head_counts, dev_status, stream)) !=
        cudaSuccess)
        return e;
    sasa_scatter_kernel<<<grid, 256, 0, stream>>>(row_ptr, col_idx, cand, added, rows, row_ptr_out, col_idx_out,
                                                  capacity);
    return cudaGetLastError();
}

}  // namespace fvattn
