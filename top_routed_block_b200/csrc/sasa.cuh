// sasa.cuh -- internal interface of the slack-aware augmentation (sasa.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fvattn {

constexpr int kSasaMaxMachines = 256;  // machines (SMs) the schedule can model

// Plans the augmentation of the routed mask (row_ptr, col_idx; the rows taken in
// `order`) over `machines` machines and writes the augmented CSR.  cand / cand_p:
// [rows, kSasaCandidates] routing candidates.  Scratch: mach_of_item [rows] (bytes),
// lists [rows], list_off [machines + 1], counts [rows].  Outputs: added [rows],
// added_mass [rows], row_ptr_out [rows + 1], col_idx_out [capacity], head_counts [BH].
cudaError_t launch_sasa(const int32_t *row_ptr, const int32_t *col_idx, const int32_t *order, int64_t rows, int nb,
                        int64_t BH, int machines, const int32_t *cand, const double *cand_p, uint8_t *mach_of_item,
                        int32_t *lists, int32_t *list_off, int32_t *counts, int32_t *added, double *added_mass,
                        int32_t *row_ptr_out, int32_t *col_idx_out, int64_t capacity, int32_t *head_counts,
                        int32_t *dev_status, cudaStream_t stream);

}  // namespace fvattn
