/*
 * fvattn.h -- C ABI of libfvattn.so: top-p routed block-sparse attention
 * forward for NVIDIA B200 (sm_100a).
 *
 * What it computes (page title, section):
 *   - FVAttn review ("[논문리뷰] FVAttn: Adaptive Sparse Attention with Runtime
 *     Load Balancing for Video Generation"), §1 Key Terms "Top-p routing":
 *     every query block keeps key blocks, most important first, until their
 *     cumulative probability reaches p.  §1 "RLB" and §3: the per-head amount
 *     of work is known once the mask is fixed and is balanced at run time.
 *   - FlashAttention review ("FlashAttention - Fast and Memory-Efficient Exact
 *     Attention with IO-Awareness"), §Background "Motivation" (S = QK^T,
 *     P = softmax(S), O = PV) and §Model (one fused kernel, tiled matmul,
 *     "Tiling Softmax"): exact attention computed tile by tile without writing
 *     S or P to memory.
 * The pages name the routing score without defining it; this library fixes
 * it as: mean of each block of `block` tokens of Q and of K (over the tokens
 * that exist), score = qbar . kbar / sqrt(d), softmax over all key blocks,
 * and keep the shortest prefix of key blocks sorted by descending score
 * (equal scores: lower index first) whose mass is >= p; p = 1 keeps all.
 *
 * Conventions shared by every call:
 *   - Tensors Q, K, V, O are bf16, contiguous [B, H, N, d] (d fastest).
 *     LSE is fp32 [B, H, N], natural logarithm.
 *   - nb = ceil(N / block); a "row" is one (b, h, query block i), numbered
 *     r = (b*H + h)*nb + i.  The CSR block mask is row_ptr int32[rows + 1]
 *     and col_idx int32[row_ptr[rows]] with strictly ascending key-block
 *     indices inside a row.
 *   - The caller owns and allocates every buffer (device memory unless a
 *     parameter says "host").  The library allocates nothing and keeps no
 *     state between calls apart from cached device attributes; calls on
 *     different streams with disjoint buffers may run concurrently.
 *   - Every device call is asynchronous on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream) and never synchronises the host, except
 *     fvattn_attention_host, which synchronises before returning.
 *   - Errors: the return value reports argument and launch errors found on
 *     the host (fvattn_status, negative).  Errors found on the device (a
 *     column index out of range or not ascending, CSR capacity exceeded, a
 *     bounded wait that timed out) are written to *dev_status (int32 in
 *     device memory; the call sets it to 0 first).  Read it after the stream
 *     has completed.  The first device error wins.
 *   - Supported: d in {64, 128}; block in {64, 128}; 0 < p <= 1; 1 <= N;
 *     nb <= 4096 (nb <= 1024 for fvattn_route); B*H*nb < 2^31.  Tensor and
 *     workspace pointers 16-byte aligned, int32/fp32 arrays 4-byte aligned.
 */
#ifndef FVATTN_H
#define FVATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FVATTN_API __attribute__((visibility("default")))
#else
#define FVATTN_API
#endif

typedef struct CUstream_st *fvattn_stream_t; /* identical to cudaStream_t */

typedef enum {
    FVATTN_OK = 0,
    FVATTN_ERR_INVALID_ARG = -1,    /* null pointer, bad size, p outside (0, 1] */
    FVATTN_ERR_UNSUPPORTED = -2,    /* d or block not supported, no sm_100 device */
    FVATTN_ERR_ALIGNMENT = -3,      /* a pointer is not 16-byte aligned */
    FVATTN_ERR_CAPACITY = -4,       /* workspace or col_idx capacity too small */
    FVATTN_ERR_CUDA = -5,           /* a CUDA runtime/driver call failed */
    FVATTN_ERR_BAD_CSR = -6,        /* device: index out of range, not ascending, count > nb */
    FVATTN_ERR_DEVICE_TIMEOUT = -7  /* device: a bounded wait gave up */
} fvattn_status;

/* Human-readable name of a status code (static string, never NULL). */
FVATTN_API const char *fvattn_status_string(int status);

/*
 * The reason for the calling host thread's most recent FVATTN_ERR_CUDA: the CUDA
 * error name of the failing call, or a description of the launch check that
 * refused it.  A static string ("" if there was none); not cleared by successful
 * calls.
 */
FVATTN_API const char *fvattn_last_error(void);

/* Number of rows B*H*ceil(N/block) (0 on bad arguments). */
FVATTN_API int64_t fvattn_num_rows(int B, int H, int N, int block);

/* Largest possible nnz of a routing CSR: B*H*nb*nb (0 on bad arguments). */
FVATTN_API int64_t fvattn_route_max_nnz(int B, int H, int N, int block);

/* Device workspace fvattn_route needs, in bytes (0 on bad arguments). */
FVATTN_API size_t fvattn_route_workspace_bytes(int B, int H, int N, int d, int block);

/*
 * fvattn_route -- top-p routing (FVAttn review §1 "Top-p routing"), then the
 * CSR block mask and per-head selected-block counts.
 *
 *   Q, K          bf16 [B,H,N,d], read only.
 *   p             threshold in (0, 1]; p = 1 selects every block.
 *   row_ptr       out, int32[rows + 1].
 *   col_idx       out, int32[col_capacity]; row_ptr[rows] entries are written,
 *                 ascending within each row.  If the selection needs more than
 *                 col_capacity entries, *dev_status = FVATTN_ERR_CAPACITY and
 *                 col_idx is left incomplete (row_ptr is still complete).
 *                 col_capacity >= fvattn_route_max_nnz() never overflows.
 *   head_counts   out, int32[B*H]: selected blocks of each head (its work).
 *   workspace     device scratch of ws_bytes >= fvattn_route_workspace_bytes().
 *   dev_status    device int32, see above.
 * Steps: mean pooling (fp64 accumulation of the bf16 inputs), fp64 scores and
 * softmax, sort by (score desc, index asc), prefix sum to p, CSR emission.
 */
FVATTN_API int fvattn_route(const void *Q, const void *K, int B, int H, int N, int d, int block, double p,
                 int32_t *row_ptr, int32_t *col_idx, int64_t col_capacity, int32_t *head_counts,
                 void *workspace, size_t ws_bytes, int32_t *dev_status, fvattn_stream_t stream);

/* Device workspace fvattn_sparse_fwd needs, in bytes (0 on bad arguments). */
FVATTN_API size_t fvattn_fwd_workspace_bytes(int B, int H, int N, int block);

/* Device workspace fvattn_lpt_order needs for `rows` rows with counts <= max_count. */
FVATTN_API size_t fvattn_lpt_workspace_bytes(int64_t rows, int max_count);

/*
 * fvattn_lpt_order -- longest-first order of the rows of a CSR block mask:
 * rows sorted by selected-block count descending, equal counts by ascending
 * row id.  This is the single-GPU counterpart of FVAttn's run-time balancing
 * of per-head work (§1 "RLB", §3): the attention kernel hands rows to SMs in
 * this order.
 *
 *   row_ptr     int32[rows + 1], read only; counts must lie in [0, max_count].
 *   max_count   largest allowed count (nb for a routing mask), <= 4096.
 *   order       out, int32[rows].
 *   workspace   >= fvattn_lpt_workspace_bytes(rows, max_count) bytes.
 * A count outside [0, max_count] sets *dev_status = FVATTN_ERR_BAD_CSR and is
 * clamped.
 */
FVATTN_API int fvattn_lpt_order(const int32_t *row_ptr, int64_t rows, int max_count, int32_t *order, void *workspace,
                     size_t ws_bytes, int32_t *dev_status, fvattn_stream_t stream);

/*
 * fvattn_quant_e4m3 -- bf16 -> FP8 (e4m3) block quantization, the input step of
 * the FP8 attention variant.  "Accelerating HunyuanVideo inference with
 * ParaAttention" (WaveSpeed), § "FP8 dynamic quantization", quantizes weights and
 * activations to FP8 at run time to use the 8-bit tensor cores, without naming a
 * format or a scaling; the reading taken: OCP E4M3FN values -- exponent bias 7,
 * 3 mantissa bits, subnormals m * 2^-9, largest finite 448 -- with scales
 * computed from the data (dynamic), one per block.
 *   X          device bf16 [B,H,N,d], 16-byte aligned.
 *   out        device uint8 [B,H,N,d], 16-byte aligned: the e4m3 codes.
 *   scale_exp  device int32 [B,H,ceil(N/block)]: per (batch, head, block of
 *              `block` tokens) the exponent e of the power-of-two scale 2^e, the
 *              smallest e with (block max |x|) * 2^-e <= 448 (0 for an all-zero
 *              block or one holding inf).
 * Each code is x * 2^-e rounded to the nearest e4m3 value, ties to the even
 * code, magnitudes above 448 saturated to 448, NaN kept as NaN (0x7F / 0xFF);
 * value = e4m3 value * 2^e.  d in {64, 128}, block in {64, 128}.  Asynchronous
 * on `stream`; allocates nothing.  Returns FVATTN_OK or a host-side error.
 */
FVATTN_API int fvattn_quant_e4m3(const void *X, int B, int H, int N, int d, int block, uint8_t *out,
                                 int32_t *scale_exp, fvattn_stream_t stream);

/*
 * fvattn_sparse_fwd -- exact attention restricted to the CSR block mask
 * (FlashAttention review §Model: one fused kernel, tiled matmuls, tiled
 * online softmax; FVAttn review §1: only the selected key blocks are read).
 *
 * For every query token t of row r = (b,h,i):
 *   keys(t) = { u : u in block j for some j in col_idx[row_ptr[r]..row_ptr[r+1]),
 *               u < N, and u <= t if causal }
 *   O[t]   = sum_{u in keys(t)} softmax_u(q_t.k_u/sqrt(d)) v_u      (bf16 out)
 *   LSE[t] = ln sum_{u in keys(t)} exp(q_t.k_u/sqrt(d))            (fp32 out)
 * An empty keys(t) gives O[t] = 0 and LSE[t] = -inf.
 *
 *   Q, K, V     bf16 [B,H,N,d], read only.
 *   row_ptr, col_idx  CSR as above (e.g. from fvattn_route), read only.  The
 *               library reads col_idx[row_ptr[r] .. row_ptr[r+1]) for every row and
 *               cannot check that this lies inside the caller's col_idx buffer:
 *               row_ptr[B*H*nb] must not exceed its length (a row with a negative
 *               count is reported as FVATTN_ERR_BAD_CSR and read as empty).
 *   causal      0 or 1.
 *   O           out, bf16 [B,H,N,d].   LSE  out, fp32 [B,H,N].
 *   workspace   >= fvattn_fwd_workspace_bytes(B,H,N,block).
 * Matmuls run on the tensor cores in bf16 with fp32 accumulation; softmax in
 * fp32.  A work item is 128 query tokens of one head: one CSR row at block 128;
 * at block 64 the pair of rows 2i and 2i+1 (query blocks of the same head),
 * which walks the union of the two rows' key blocks, each row masking the blocks
 * it did not select (item size = the union's size; see fvattn_attn_work_order).
 * A persistent grid takes the items from a queue ordered head-major and
 * longest-first: heads by total work descending, the items of a head by size
 * descending (ties by lower index), so that the SMs share one head's K and V in
 * L2 at a time and finish on the shortest items.  B*H <= 4096 and
 * ceil(N/block) <= 4096, else FVATTN_ERR_UNSUPPORTED (before any device work).
 * Malformed rows (a negative count, column indices out of range or not
 * ascending) set *dev_status = FVATTN_ERR_BAD_CSR; at block 128 the offending
 * indices are skipped (an index not above the one before it), at block 64 each
 * row uses the set of its in-range indices.
 */
FVATTN_API int fvattn_sparse_fwd(const void *Q, const void *K, const void *V, const int32_t *row_ptr,
                      const int32_t *col_idx, int B, int H, int N, int d, int block, int causal, void *O,
                      float *LSE, void *workspace, size_t ws_bytes, int32_t *dev_status,
                      fvattn_stream_t stream);

/*
 * fvattn_attention_host -- the whole path from host memory: copies Q, K, V
 * (host, ideally pinned) to the device buffers dQ, dK, dV, routes with p,
 * runs the sparse forward, and copies O (bf16) and LSE (fp32) back to the
 * host buffers hO, hLSE; synchronises `stream` before returning.
 *   hQ, hK, hV    host bf16 [B,H,N,d];  hO host bf16 [B,H,N,d];  hLSE host fp32 [B,H,N].
 *   dQ, dK, dV, dO, dLSE, row_ptr, col_idx (capacity col_capacity), head_counts,
 *   route_ws (route_ws_bytes), fwd_ws (fwd_ws_bytes): device buffers as for
 *   fvattn_route / fvattn_sparse_fwd.  dev_status: device int32[3] (scratch for
 *   routing and attention, then the first error over the whole call).
 * The heads are processed in chunks of about 64 MB per tensor: the copies in of
 * one chunk, the compute of the previous one (on `stream`) and the copies out of
 * the one before run concurrently, on two streams the call creates and destroys
 * (host buffers must be pinned for the copies to overlap).  Once two chunks or
 * fewer remain, the chunks halve in size down to one head, so that little
 * compute and copying out follows the last copy in.  Work already queued on
 * `stream` completes before the first copy starts.
 * Returns the first host error, else the first nonzero device status read
 * after the sync.
 */
FVATTN_API int fvattn_attention_host(const void *hQ, const void *hK, const void *hV, int B, int H, int N, int d, int block,
                          double p, int causal, void *hO, float *hLSE, void *dQ, void *dK, void *dV, void *dO,
                          float *dLSE, int32_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                          int32_t *head_counts, void *route_ws, size_t route_ws_bytes, void *fwd_ws,
                          size_t fwd_ws_bytes, int32_t *dev_status, fvattn_stream_t stream);

/* Size of the library-owned device scratch used by fvattn_sparse_fwd_noalloc. */
#define FVATTN_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * fvattn_sparse_fwd_noalloc -- fvattn_sparse_fwd without a caller workspace.
 * The pages have no counterpart to this call; it exists for callers that cannot
 * allocate device memory when they call the library: a host that hands the
 * library a stream and its tensors but owns every allocation itself (plugin-style
 * enqueue functions, fixed memory pools), or code that must not pay for the device
 * synchronisation that cudaMalloc/cudaFree imply in the middle of a step.
 *
 * Arguments and results are those of fvattn_sparse_fwd minus workspace/ws_bytes;
 * the caller still provides Q, K, V, the CSR, O, LSE and dev_status.  The scratch
 * the call needs (fvattn_fwd_workspace_bytes(B,H,N,block) bytes) comes from one
 * file-scope device array of FVATTN_NOALLOC_SCRATCH_BYTES (4 MiB) inside the
 * library, which every device that loads the library keeps until the process
 * exits.  Shapes that need more return FVATTN_ERR_CAPACITY without launching
 * anything (rows B*H*ceil(N/block) up to about 1M at block 128, about 700k at
 * block 64, whose pairs also keep their union sizes and a scan of them).
 *
 * Each call made outside stream capture looks up the array's device address
 * (cudaGetSymbolAddress, with the call's device current; a lookup allocates
 * nothing) and keeps it per device; a call made while `stream` is capturing uses
 * the address kept by the last call outside capture, so the first call on each
 * device must come before any stream capture, and a call after a device reset
 * must also come before capture.  The call allocates nothing: no cudaMalloc,
 * cudaFree or allocating library routine.  All calls on a device share the one
 * array, which keeps the previous call's contents (the parts that must start at
 * zero are cleared on the stream by each call), so calls whose executions overlap
 * on the GPU -- on different streams, or from different host threads -- race on it
 * and must be serialised by the caller.
 */
FVATTN_API int fvattn_sparse_fwd_noalloc(const void *Q, const void *K, const void *V, const int32_t *row_ptr,
                                         const int32_t *col_idx, int B, int H, int N, int d, int block, int causal,
                                         void *O, float *LSE, int32_t *dev_status, fvattn_stream_t stream);

/*
 * fvattn_test_sparse_fwd_stall -- test hook for failure detection, not for
 * production use.  Same arguments as fvattn_sparse_fwd; the pipeline that takes
 * the first work item of the queue never reports that item's Q as loaded, so one
 * of its bounded waits runs out (after about one second) and the call ends with
 * *dev_status = FVATTN_ERR_DEVICE_TIMEOUT, the rest of the grid finishing its
 * items.  No fault, trap or hang: the CUDA context stays usable.
 */
FVATTN_API int fvattn_test_sparse_fwd_stall(const void *Q, const void *K, const void *V, const int32_t *row_ptr,
                                            const int32_t *col_idx, int B, int H, int N, int d, int block,
                                            int causal, void *O, float *LSE, void *workspace, size_t ws_bytes,
                                            int32_t *dev_status, fvattn_stream_t stream);

/* Device workspace fvattn_sparse_bwd needs, in bytes (0 on bad arguments). */
FVATTN_API size_t fvattn_bwd_workspace_bytes(int B, int H, int N, int block);

/*
 * fvattn_sparse_bwd -- gradients of the block-sparse attention of
 * fvattn_sparse_fwd.  The FlashAttention review measures training with the
 * fused kernel (§Experiments 1 "Training Efficiency") without printing the
 * backward pass; these are the plain derivatives of L = sum(dO * O) with P
 * recomputed from the LSE the forward returned:
 *   D_t = dO_t . O_t,  P = exp(S - LSE),  dS = P * (dO V^T - D),
 *   dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d),  dV = P^T dO,
 * every sum restricted to the key tokens the CSR mask allows (u < N, u <= t if
 * causal), exactly as in the forward.
 *
 *   Q, K, V, O, dO  bf16 [B,H,N,d], read only (O and LSE from fvattn_sparse_fwd).
 *   LSE             fp32 [B,H,N], read only.
 *   row_ptr, col_idx  the CSR block mask of the forward (ascending columns).
 *   dQ, dK, dV      out, bf16 [B,H,N,d] (fp32 accumulation in tensor memory).
 *   workspace       >= fvattn_bwd_workspace_bytes(B,H,N,block).
 * block must be 128 and d 64 or 128 (else FVATTN_ERR_UNSUPPORTED); B*H <= 4096 and
 * ceil(N/block) <= 4096 (else FVATTN_ERR_UNSUPPORTED, before any device work).
 * Work: D; the transpose of the mask (key block -> the query blocks that
 * selected it); a dQ pass over the CSR rows and a dK/dV pass over the key
 * blocks, both on tcgen05 with accumulators in tensor memory and longest-first
 * persistent grids.  A malformed CSR sets *dev_status = FVATTN_ERR_BAD_CSR and
 * leaves the gradients unspecified.  Asynchronous on `stream`.
 */
FVATTN_API int fvattn_sparse_bwd(const void *Q, const void *K, const void *V, const void *O, const float *LSE,
                                 const void *dO, const int32_t *row_ptr, const int32_t *col_idx, int B, int H, int N,
                                 int d, int block, int causal, void *dQ, void *dK, void *dV, void *workspace,
                                 size_t ws_bytes, int32_t *dev_status, fvattn_stream_t stream);

/*
 * fvattn_sparse_fwd_profiled -- fvattn_sparse_fwd that also reports how busy
 * each CTA of its persistent grid was, for the load-imbalance factor
 * LIF = max / mean busy time over the SMs (FVAttn review §3 reports the LIF of
 * its run-time balancing, 1.34 -> 1.08 across GPUs; here the SMs of one GPU).
 * A diagnostic entry point: results equal those of fvattn_sparse_fwd.
 *   order_mode   0: the head-major longest-first work queue fvattn_sparse_fwd uses;
 *                1: rows in index order, the comparison point.
 *   cta_busy_ns  device int64[number of SMs], 8-byte aligned: entry c receives the
 *                global-timer nanoseconds from CTA c's start to the end of its last
 *                work item (entries past *grid are left untouched).  The persistent
 *                grid runs one CTA per SM, each with two work items in flight.
 *   grid         out (host): number of CTAs launched (at most the number of SMs).
 * Other arguments, layouts and errors as fvattn_sparse_fwd; order_mode outside
 * {0,1} or a null cta_busy_ns / grid is FVATTN_ERR_INVALID_ARG.
 */
FVATTN_API int fvattn_sparse_fwd_profiled(const void *Q, const void *K, const void *V, const int32_t *row_ptr,
                                          const int32_t *col_idx, int B, int H, int N, int d, int block, int causal,
                                          void *O, float *LSE, void *workspace, size_t ws_bytes, int32_t *dev_status,
                                          int order_mode, int64_t *cta_busy_ns, int *grid, fvattn_stream_t stream);

/*
 * fvattn_sparse_fwd_fp8 -- the block-sparse attention forward of fvattn_sparse_fwd
 * on FP8 operands ("Accelerating HunyuanVideo inference with ParaAttention"
 * (WaveSpeed), § "FP8 dynamic quantization": attention computed on activations
 * quantized to FP8 at run time).  Q, K, V are given as fvattn_quant_e4m3 returns
 * them: e4m3 codes (OCP E4M3FN) with one power-of-two scale per (head, block), the
 * value of a code being its e4m3 value times 2^exponent.  Both GEMMs run on the
 * tensor cores as e4m3 x e4m3 with fp32 accumulation; P is rounded to e4m3 before
 * P V (an approximation: about 2^-4 relative per probability), the row sums use
 * the unrounded P.
 *   Q8, K8, V8          device uint8 [B,H,N,d] e4m3 codes, 16-byte aligned.
 *   q_exp, k_exp, v_exp device int32 [B,H,ceil(N/block)] block exponents.
 *   Other arguments, layouts, outputs (O bf16, LSE fp32 natural log), workspace
 *   (fvattn_fwd_workspace_bytes) and errors as fvattn_sparse_fwd.
 * Supported: d = 128 (an e4m3 row fills one 128-byte swizzle span), block 64 or
 * 128; other d give FVATTN_ERR_UNSUPPORTED.
 */
FVATTN_API int fvattn_sparse_fwd_fp8(const void *Q8, const void *K8, const void *V8, const int32_t *q_exp,
                                     const int32_t *k_exp, const int32_t *v_exp, const int32_t *row_ptr,
                                     const int32_t *col_idx, int B, int H, int N, int d, int block, int causal,
                                     void *O, float *LSE, void *workspace, size_t ws_bytes, int32_t *dev_status,
                                     fvattn_stream_t stream);

/* Device workspace fvattn_route_sasa needs, in bytes (0 on bad arguments). */
FVATTN_API size_t fvattn_sasa_workspace_bytes(int B, int H, int N, int d, int block);

/*
 * fvattn_route_sasa -- top-p routing followed by slack-aware augmentation (FVAttn
 * review, §1 Key Terms "SASA" and §3: after the work is balanced, the ranks that
 * would idle before the slowest one finishes compute extra high-value key
 * blocks).  On one GPU the ranks are the SMs of the persistent attention grid:
 *   1. the routed rows, head-major and longest first (the attention's queue order
 *      at block 128, fvattn_attn_work_order; at block 64 the attention takes pairs
 *      of rows, and the plan still schedules single rows, a model of that queue),
 *      are list-scheduled onto `machines` machines: each row to the machine with
 *      the least load so far, the lowest machine on equal loads, a row's load
 *      being its selected-block count; the makespan T is the largest load;
 *   2. each machine walks its rows in the order they were assigned, round after
 *      round, giving each row its next unselected key block in the routing order
 *      (score descending, index ascending; at most 8 per row), one block each,
 *      until T - (its load) blocks are added or no row has a candidate left;
 *   3. the augmented mask is written as a CSR with ascending columns.
 * The output is a mask for fvattn_sparse_fwd (a superset of fvattn_route's).
 *   machines      1..256; the attention kernel runs one CTA per SM, so the SM count
 *                 of the device is the natural choice.
 *   row_ptr, col_idx, col_capacity, head_counts   as fvattn_route, for the
 *                 augmented mask (col_capacity >= routed blocks + 8 per row is
 *                 always enough; B*H*ceil(N/block)^2 too).
 *   added         device int32[rows] (out): blocks added to each row.
 *   added_mass    device fp64[rows] (out), 8-byte aligned: their routing probability.
 *   cand, cand_p  optional (null: not written) device int32 / fp64 [rows, 8] (out):
 *                 the routing candidates of every row (the key blocks past the cut
 *                 in the routing order, -1 past the last) and their probabilities.
 *   workspace     fvattn_sasa_workspace_bytes(B,H,N,d,block) bytes, 16-byte aligned.
 * Other arguments and errors as fvattn_route; machines outside 1..256 give
 * FVATTN_ERR_UNSUPPORTED.  Asynchronous on `stream`.
 */
FVATTN_API int fvattn_route_sasa(const void *Q, const void *K, int B, int H, int N, int d, int block, double p,
                                 int machines, int32_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                                 int32_t *head_counts, int32_t *added, double *added_mass, int32_t *cand,
                                 double *cand_p, void *workspace, size_t ws_bytes, int32_t *dev_status,
                                 fvattn_stream_t stream);

/*
 * fvattn_rlb_plan -- the head moves of run-time load balancing across ranks
 * (FVAttn review, §1 Key Terms "RLB" and §3: once routing has fixed every head's
 * amount of work, heads move between GPUs over P2P so the critical path shortens).
 * Host code; no device work.
 *   work       host int64[ranks * units]: work[r * units + i] = selected blocks of
 *              unit i (a (batch, head) pair) that rank r holds; >= 0.
 *   moves out  move_unit[k] = the unit's home index r * units + i, move_src[k] and
 *              move_dst[k] its ranks, for k < *n_moves, in the order decided.
 * Rule: while the most loaded rank holds a unit whose work lies strictly between 0
 * and its gap to the least loaded rank, it hands the largest such unit (the lowest
 * home index among equal works) to that rank; ranks tie by lower index.  Every
 * move lowers the sum of squared loads, so the plan ends; a unit may move again.
 * Errors: FVATTN_ERR_INVALID_ARG on null pointers or negative sizes or work;
 * FVATTN_ERR_CAPACITY when the plan needs more than max_moves moves (the first
 * max_moves are written).
 */
FVATTN_API int fvattn_rlb_plan(const int64_t *work, int ranks, int units, int max_moves, int32_t *move_unit,
                               int32_t *move_src, int32_t *move_dst, int32_t *n_moves);

/* Work items of fvattn_sparse_fwd: B*H*nb at block 128, B*H*ceil(nb/2) at block
 * 64 (nb = ceil(N/block)); 0 on bad arguments. */
FVATTN_API int64_t fvattn_attn_num_items(int B, int H, int N, int block);

/*
 * fvattn_attn_work_order -- the order in which fvattn_sparse_fwd takes its work
 * items, written to order[0 .. items), items = fvattn_attn_num_items(B,H,N,block).
 * An item is 128 query tokens of one head: at block 128 one CSR row (item id =
 * row id (b*H+h)*nb + i, size = its block count); at block 64 the pair of rows 2i
 * and 2i+1 of head (b,h) (item id (b*H+h)*ceil(nb/2) + i, size = the number of
 * key blocks either row selects; with nb odd the last pair has row 2i only).
 * FVAttn review §1 "RLB" balances per-head work at run time once the mask is
 * known; on one GPU the SMs pop the items from this queue: heads by their total
 * item size (descending, equal totals by lower head index), and inside a head its
 * items by size (descending, equal sizes by lower item id).  The same kernels run
 * inside fvattn_sparse_fwd; this call exposes their result (for checks and
 * diagnostics).
 *   row_ptr    device int32[B*H*nb + 1], the CSR of fvattn_route (or a caller's mask).
 *   col_idx    device int32, its column indices: read at block 64 (the pairs'
 *              unions), ignored (may be null) at block 128.
 *   order      device int32[items] (out): item ids.
 *   workspace  device, fvattn_fwd_workspace_bytes(B,H,N,block) bytes, 16-byte aligned.
 *   dev_status device int32[1]: at block 64 cleared, then FVATTN_ERR_BAD_CSR for a
 *              malformed row; ignored (may be null) at block 128.
 * Asynchronous on `stream`.  Errors: bad sizes or null pointers
 * FVATTN_ERR_INVALID_ARG; B*H > 4096 or ceil(N/block) > 4096
 * FVATTN_ERR_UNSUPPORTED; short workspace FVATTN_ERR_CAPACITY.
 */
FVATTN_API int fvattn_attn_work_order(const int32_t *row_ptr, const int32_t *col_idx, int B, int H, int N, int block,
                                      int32_t *order, void *workspace, size_t ws_bytes, int32_t *dev_status,
                                      fvattn_stream_t stream);

/* Compiled-in build description (architecture, version), static string. */
FVATTN_API const char *fvattn_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* FVATTN_H */
