// attn_fwd.cuh -- internal interface of the sparse attention kernel (attn_fwd.cu).
#pragma once

#include <cuda.h>
#include <cstdint>
#include <cuda_runtime.h>

namespace fvattn {

struct AttnLaunch {
    const CUtensorMap *tmap_k, *tmap_v;  // host copies, passed by value as kernel parameters
    const void *Q;                       // [B,H,N,d] bf16 or e4m3 codes, read row by row into tensor memory
    // order: work items, head-major, longest first; an item is a CSR row at block 128,
    // a pair of neighbouring rows (query blocks 2i, 2i+1; item id bh * ceil(nb/2) + i)
    // at block 64
    const int32_t *row_ptr, *col_idx, *order;
    int n_items;
    int *work_counter;  // zeroed before the launch
    int N, nb, causal;
    float scale_log2;   // log2(e) / sqrt(d)
    void *O;
    float *LSE;
    int32_t *dev_status;
    int sms;            // multiprocessors of the device; the launcher sizes the persistent grid
    int *grid_out;      // receives the number of CTAs launched, or null
    int test_stall;     // nonzero only from the test hook: one bounded wait runs out
    long long *cta_busy_ns;  // per-CTA busy time (global timer, ns), or null
    // e4m3 operands only: power-of-two scale exponents per (head, block), int32 [B*H, nb]
    const int32_t *q_exp, *k_exp, *v_exp;
};

int attn_smem_bytes(int d, int bs);
// Work items of the attention kernel: the CSR rows (query blocks of every head) at
// block 128, the pairs of neighbouring rows at block 64.
int64_t attn_num_items(int64_t BH, int nb, int bs);
// Block 64: counts[bh * ceil(nb/2) + i] = size of the union of the key-block lists of
// rows 2i and 2i+1 of head bh; a malformed row records FVATTN_ERR_BAD_CSR.
cudaError_t launch_pair_counts(const int32_t *row_ptr, const int32_t *col_idx, int64_t BH, int nb, int32_t *counts,
                               int32_t *dev_status, cudaStream_t stream);
// order[] = rows head-major, longest first (heads by total selected blocks, rows of
// a head by block count); head_rank[BH] is scratch.  B*H <= 4096, nb <= 4096.
cudaError_t launch_item_order(const int32_t *row_ptr, int64_t BH, int nb, int32_t *head_rank, int32_t *order,
                              cudaStream_t stream);
// order[i] = i: rows in index order (the comparison point for the load balance).
cudaError_t launch_natural_order(int64_t n, int32_t *order, cudaStream_t stream);
int attn_ctas_per_sm();  // resident CTAs per SM the launch grid is sized for
cudaError_t launch_sparse_attn(const AttnLaunch &a, int d, int bs, cudaStream_t stream);
// e4m3 operands (tmap_* over uint8 codes), d = 128, bs in {64, 128}.
cudaError_t launch_sparse_attn_fp8(const AttnLaunch &a, int bs, cudaStream_t stream);

}  // namespace fvattn
