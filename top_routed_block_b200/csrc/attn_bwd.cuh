// attn_bwd.cuh -- internal interface of the attention gradient kernels (attn_bwd.cu).
#pragma once

#include <cuda.h>
#include <cstdint>
#include <cuda_runtime.h>

namespace fvattn {

struct BwdLaunch {
    const CUtensorMap *tmap_q, *tmap_k, *tmap_v, *tmap_do;  // host copies, passed by value
    const void *Q, *dO;                                      // bf16 [B,H,N,d], read row by row by dq_kernel
    const float *LSE, *D;                                    // fp32 [B,H,N]
    const int32_t *row_ptr, *col_idx, *col_ptr, *csc_idx;    // the mask and its transpose
    const int32_t *order_q, *order_k;                        // work queues (rows, key blocks)
    int n_items;                                             // B*H*nb (both kernels)
    int *counters;                                           // [2], zeroed before the launches
    int N, nb, causal;
    float scale;                                             // 1/sqrt(d)
    void *dQ, *dK, *dV;                                      // bf16 [B,H,N,d] out
    int32_t *dev_status;
    int grid;
};

int bwd_dq_smem_bytes(int d);
int bwd_dkdv_smem_bytes(int d);
// D[t] = dO[t] . O[t] over `tokens` rows of d bf16.
cudaError_t launch_bwd_rowdot(const void *O, const void *dO, int64_t tokens, int d, float *D, cudaStream_t stream);
// Transpose of the block mask: col_ptr[B*H*nb + 1], csc_idx[nnz] (query blocks, ascending); nb <= 4096.
cudaError_t launch_csc(const int32_t *row_ptr, const int32_t *col_idx, int64_t BH, int nb, int32_t *col_ptr,
                       int32_t *csc_idx, int32_t *dev_status, cudaStream_t stream);
cudaError_t launch_bwd_dq(const BwdLaunch &a, int d, cudaStream_t stream);
cudaError_t launch_bwd_dkdv(const BwdLaunch &a, int d, cudaStream_t stream);

}  // namespace fvattn
