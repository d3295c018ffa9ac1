// abi.cu -- the extern "C" surface of libfvattn.so (declared in include/fvattn.h):
// argument checks, workspace carving, TMA descriptor encoding and launches.
// All compute runs in the kernels of route.cu, lpt.cu and attn_fwd.cu.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fvattn.h"
#include "attn_bwd.cuh"
#include "attn_fwd.cuh"
#include "common.cuh"
#include "lpt.cuh"
#include "quant.cuh"
#include "route.cuh"
#include "sasa.cuh"

using namespace fvattn;

namespace {
thread_local const char *t_last_error = "";
}  // namespace

void fvattn::set_last_error(const char *what) { t_last_error = what ? what : ""; }

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

struct DeviceInfo {
    int sms = 0;
    int major = 0;
    bool ok = false;
};

// Cached per device: multiprocessor count and compute capability.
bool device_info(DeviceInfo *out) {
    static std::mutex mu;
    static DeviceInfo cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> g(mu);
    if (!cache[dev].ok) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
        if (cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
        d.ok = true;
        cache[dev] = d;
    }
    *out = cache[dev];
    return true;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int B, int H, int N, int d, int block) {
    if (B < 1 || H < 1 || N < 1) return FVATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FVATTN_ERR_UNSUPPORTED;
    if (block != 64 && block != 128) return FVATTN_ERR_UNSUPPORTED;
    const int64_t nb = ceil_div(N, block);
    if (nb > kMaxCount) return FVATTN_ERR_UNSUPPORTED;
    const int64_t rows = static_cast<int64_t>(B) * H * nb;
    if (rows >= (1LL << 31)) return FVATTN_ERR_UNSUPPORTED;
    return FVATTN_OK;
}

int check_device() {
    DeviceInfo info;
    if (!device_info(&info)) return FVATTN_ERR_CUDA;
    if (info.major != 10) return FVATTN_ERR_UNSUPPORTED;
    return FVATTN_OK;
}

// 3-D map over a contiguous [B*H, N, d] tensor of bf16 (elem_bytes 2) or of 8-bit
// codes (elem_bytes 1); box = 128 bytes of columns (the swizzle width) x `rows`
// tokens x 1 head; out-of-range rows read as zero.
bool make_map(CUtensorMap *m, const void *base, int64_t BH, int N, int d, int rows, int elem_bytes = 2) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t eb = static_cast<cuuint64_t>(elem_bytes);
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * eb, static_cast<cuuint64_t>(N) * d * eb};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
               const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return FVATTN_OK;
    set_last_error(cudaGetErrorName(e));
    return FVATTN_ERR_CUDA;
}

struct FwdWorkspace {
    size_t order, head_rank, counter, pair_count, pair_ptr, pair_head, total;
};

// The forward's scratch for BH heads of nb query blocks at block bs: the queue order
// of the work items, the ordering kernels' head ranks and the queue counter; at block
// 64 also the pairs' union sizes, their scan and per-head sums.
FwdWorkspace fwd_layout(int64_t BH, int nb, int bs) {
    FwdWorkspace w{};
    Carver c;
    const int64_t items = attn_num_items(BH, nb, bs);
    w.order = c.take<int32_t>(static_cast<size_t>(items));
    w.head_rank = c.take<int32_t>(static_cast<size_t>(BH));
    w.counter = c.take<int32_t>(64);
    if (bs == 64) {
        w.pair_count = c.take<int32_t>(static_cast<size_t>(items));
        w.pair_ptr = c.take<int32_t>(static_cast<size_t>(items) + 1);
        w.pair_head = c.take<int32_t>(static_cast<size_t>(BH));
    }
    w.total = align_up(c.off, 256);
    return w;
}

// The queue order of the forward's work items into ws + w.order (head-major, longest
// first; order_mode 1: items by index).  Block 64 first sizes the pairs (their key-block
// unions, which also checks the CSR) and orders them by those sizes.
int enqueue_work_order(const int32_t *row_ptr, const int32_t *col_idx, int64_t BH, int nb, int bs, int order_mode,
                       char *ws, const FwdWorkspace &w, int32_t *dev_status, cudaStream_t s) {
    const int64_t items = attn_num_items(BH, nb, bs);
    auto i32 = [&](size_t off) { return reinterpret_cast<int32_t *>(ws + off); };
    const int32_t *item_ptr = row_ptr;
    int per_head = nb;
    if (bs == 64) {
        const int np = (nb + 1) / 2;
        cudaError_t e = launch_pair_counts(row_ptr, col_idx, BH, nb, i32(w.pair_count), dev_status, s);
        if (e == cudaSuccess)
            e = launch_csr_scan(i32(w.pair_count), items, np, BH, i32(w.pair_ptr), items * nb, i32(w.pair_head),
                                dev_status, s);
        if (e != cudaSuccess) return from_cuda(e);
        item_ptr = i32(w.pair_ptr);
        per_head = np;
    }
    return from_cuda(order_mode == 1 ? launch_natural_order(items, i32(w.order), s)
                                     : launch_item_order(item_ptr, BH, per_head, i32(w.head_rank), i32(w.order), s));
}

struct BwdWorkspace {
    size_t D, col_ptr, csc_idx, order_q, order_k, head_rank, counters, total;
};

// rows = B*H*nb CSR rows (= key-block columns); csc capacity = the worst case B*H*nb^2.
BwdWorkspace bwd_layout(int64_t BH, int N, int nb) {
    BwdWorkspace w{};
    Carver c;
    const int64_t rows = BH * nb;
    w.D = c.take<float>(static_cast<size_t>(BH) * N);
    w.col_ptr = c.take<int32_t>(static_cast<size_t>(rows) + 1);
    w.csc_idx = c.take<int32_t>(static_cast<size_t>(rows) * nb);
    w.order_q = c.take<int32_t>(static_cast<size_t>(rows));
    w.order_k = c.take<int32_t>(static_cast<size_t>(rows));
    w.head_rank = c.take<int32_t>(static_cast<size_t>(BH));
    w.counters = c.take<int32_t>(64);
    w.total = align_up(c.off, 256);
    return w;
}

// st[2] keeps the first error of st[0] (routing) and st[1] (attention) over successive calls.
__global__ void status_merge_kernel(int32_t *st) {
    if (st[2] == 0) st[2] = st[0] != 0 ? st[0] : st[1];
}

}  // namespace

extern "C" {

const char *fvattn_status_string(int status) {
    switch (status) {
        case FVATTN_OK: return "ok";
        case FVATTN_ERR_INVALID_ARG: return "invalid argument";
        case FVATTN_ERR_UNSUPPORTED: return "unsupported configuration or device";
        case FVATTN_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case FVATTN_ERR_CAPACITY: return "workspace or output capacity too small";
        case FVATTN_ERR_CUDA: return "CUDA error";
        case FVATTN_ERR_BAD_CSR: return "malformed CSR block mask";
        case FVATTN_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        default: return "unknown status";
    }
}

const char *fvattn_build_info(void) { return "libfvattn 0.2 sm_100a (tcgen05/TMA/TMEM)"; }

const char *fvattn_last_error(void) { return t_last_error; }

int64_t fvattn_num_rows(int B, int H, int N, int block) {
    if (B < 1 || H < 1 || N < 1 || block < 1) return 0;
    return static_cast<int64_t>(B) * H * ceil_div(N, block);
}

int64_t fvattn_route_max_nnz(int B, int H, int N, int block) {
    if (B < 1 || H < 1 || N < 1 || block < 1) return 0;
    const int64_t nb = ceil_div(N, block);
    return static_cast<int64_t>(B) * H * nb * nb;
}

size_t fvattn_route_workspace_bytes(int B, int H, int N, int d, int block) {
    if (check_shape(B, H, N, d, block) != FVATTN_OK) return 0;
    const int nb = static_cast<int>(ceil_div(N, block));
    return route_workspace_layout(static_cast<int64_t>(B) * H, nb, d).total;
}

size_t fvattn_lpt_workspace_bytes(int64_t rows, int max_count) {
    if (rows < 0 || max_count < 0 || max_count > kMaxCount) return 0;
    return lpt_workspace_layout(rows, max_count).total;
}

size_t fvattn_fwd_workspace_bytes(int B, int H, int N, int block) {
    if (B < 1 || H < 1 || N < 1 || (block != 64 && block != 128)) return 0;
    const int64_t nb = ceil_div(N, block);
    if (nb > kMaxCount) return 0;
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (BH > kMaxHeads) return 0;
    return fwd_layout(BH, static_cast<int>(nb), block).total;
}

int fvattn_route(const void *Q, const void *K, int B, int H, int N, int d, int block, double p, int32_t *row_ptr,
                 int32_t *col_idx, int64_t col_capacity, int32_t *head_counts, void *workspace, size_t ws_bytes,
                 int32_t *dev_status, fvattn_stream_t stream) {
    int rc = check_shape(B, H, N, d, block);
    if (rc != FVATTN_OK) return rc;
    if (!Q || !K || !row_ptr || !col_idx || !head_counts || !workspace || !dev_status) return FVATTN_ERR_INVALID_ARG;
    if (!(p > 0.0) || p > 1.0 || std::isnan(p)) return FVATTN_ERR_INVALID_ARG;
    if (col_capacity < 0) return FVATTN_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(workspace)) return FVATTN_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(row_ptr) | reinterpret_cast<uintptr_t>(col_idx) |
         reinterpret_cast<uintptr_t>(head_counts) | reinterpret_cast<uintptr_t>(dev_status)) & 3u)
        return FVATTN_ERR_ALIGNMENT;
    const int nb = static_cast<int>(ceil_div(N, block));
    if (nb > kMaxRouteBlocks) return FVATTN_ERR_UNSUPPORTED;
    if (ws_bytes < fvattn_route_workspace_bytes(B, H, N, d, block)) return FVATTN_ERR_CAPACITY;
    if ((rc = check_device()) != FVATTN_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = from_cuda(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s))) != FVATTN_OK) return rc;
    return from_cuda(launch_route(Q, K, static_cast<int64_t>(B) * H, N, d, block, nb, p, row_ptr, col_idx,
                                  col_capacity, head_counts, workspace, dev_status, s));
}

int fvattn_lpt_order(const int32_t *row_ptr, int64_t rows, int max_count, int32_t *order, void *workspace,
                     size_t ws_bytes, int32_t *dev_status, fvattn_stream_t stream) {
    if (!row_ptr || !order || !workspace || !dev_status || rows < 0 || rows >= (1LL << 31))
        return FVATTN_ERR_INVALID_ARG;
    if (max_count < 0 || max_count > kMaxCount) return FVATTN_ERR_UNSUPPORTED;
    if (!aligned16(workspace)) return FVATTN_ERR_ALIGNMENT;
    if (ws_bytes < fvattn_lpt_workspace_bytes(rows, max_count)) return FVATTN_ERR_CAPACITY;
    int rc = check_device();
    if (rc != FVATTN_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = from_cuda(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s))) != FVATTN_OK) return rc;
    return from_cuda(launch_lpt_order(row_ptr, rows, max_count, order, workspace, dev_status, s));
}

int fvattn_quant_e4m3(const void *X, int B, int H, int N, int d, int block, uint8_t *out, int32_t *scale_exp,
                      fvattn_stream_t stream) {
    int rc = check_shape(B, H, N, d, block);
    if (rc != FVATTN_OK) return rc;
    if (!X || !out || !scale_exp) return FVATTN_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(out) || (reinterpret_cast<uintptr_t>(scale_exp) & 3u)) return FVATTN_ERR_ALIGNMENT;
    if ((rc = check_device()) != FVATTN_OK) return rc;
    return from_cuda(launch_quant_e4m3(X, static_cast<int64_t>(B) * H, N, d, block, out, scale_exp,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

// exps: e4m3 operands (Q, K, V are codes) with their block exponents {q, k, v}, or null for bf16.
static int sparse_fwd_impl(const void *Q, const void *K, const void *V, const int32_t *row_ptr,
                           const int32_t *col_idx, int B, int H, int N, int d, int block, int causal, void *O,
                           float *LSE, void *workspace, size_t ws_bytes, int32_t *dev_status, fvattn_stream_t stream,
                           int test_stall, int order_mode = 0, int64_t *cta_busy_ns = nullptr,
                           int *grid_out = nullptr, const int32_t *const *exps = nullptr) {
    int rc = check_shape(B, H, N, d, block);
    if (rc != FVATTN_OK) return rc;
    const bool fp8 = exps != nullptr;
    if (fp8 && d != 128) return FVATTN_ERR_UNSUPPORTED;
    if (fp8 && (!exps[0] || !exps[1] || !exps[2])) return FVATTN_ERR_INVALID_ARG;
    if (fp8 && ((reinterpret_cast<uintptr_t>(exps[0]) | reinterpret_cast<uintptr_t>(exps[1]) |
                 reinterpret_cast<uintptr_t>(exps[2])) & 3u))
        return FVATTN_ERR_ALIGNMENT;
    if (!Q || !K || !V || !row_ptr || !col_idx || !O || !LSE || !workspace || !dev_status)
        return FVATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FVATTN_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(workspace))
        return FVATTN_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(row_ptr) | reinterpret_cast<uintptr_t>(col_idx) |
         reinterpret_cast<uintptr_t>(LSE) | reinterpret_cast<uintptr_t>(dev_status)) & 3u)
        return FVATTN_ERR_ALIGNMENT;
    // at most kMaxCount query blocks per sequence (the ordering kernels' shared arrays, and
    // at block 64 the pairs' bitmaps and union slots); the workspace query returns 0 beyond
    if (ceil_div(N, block) > kMaxCount || static_cast<int64_t>(B) * H > kMaxHeads) return FVATTN_ERR_UNSUPPORTED;
    if (ws_bytes < fvattn_fwd_workspace_bytes(B, H, N, block)) return FVATTN_ERR_CAPACITY;
    if ((rc = check_device()) != FVATTN_OK) return rc;
    DeviceInfo info;
    if (!device_info(&info)) return FVATTN_ERR_CUDA;
    const int64_t BH = static_cast<int64_t>(B) * H;
    const int nb = static_cast<int>(ceil_div(N, block));
    if (BH > kMaxHeads) return FVATTN_ERR_UNSUPPORTED;
    const int64_t items = attn_num_items(BH, nb, block);
    const FwdWorkspace w = fwd_layout(BH, nb, block);
    char *ws = static_cast<char *>(workspace);
    int32_t *order = reinterpret_cast<int32_t *>(ws + w.order);
    int *counter = reinterpret_cast<int *>(ws + w.counter);

    // K and V are read one key block per TMA box
    CUtensorMap mk, mv;
    const int eb = fp8 ? 1 : 2;
    if (!make_map(&mk, K, BH, N, d, block, eb) || !make_map(&mv, V, BH, N, d, block, eb)) return FVATTN_ERR_CUDA;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = from_cuda(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s))) != FVATTN_OK) return rc;
    // work items (rows, or pairs of rows at block 64): head-major, longest first (or by
    // index, for comparison)
    if ((rc = enqueue_work_order(row_ptr, col_idx, BH, nb, block, order_mode, ws, w, dev_status, s)) != FVATTN_OK)
        return rc;
    if ((rc = from_cuda(cudaMemsetAsync(counter, 0, sizeof(int), s))) != FVATTN_OK) return rc;

    AttnLaunch a{};
    a.Q = Q;
    a.tmap_k = &mk;
    a.tmap_v = &mv;
    a.row_ptr = row_ptr;
    a.col_idx = col_idx;
    a.order = order;
    a.n_items = static_cast<int>(items);
    a.work_counter = counter;
    a.N = N;
    a.nb = nb;
    a.causal = causal;
    a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
    a.O = O;
    a.LSE = LSE;
    a.dev_status = dev_status;
    a.sms = info.sms;
    a.grid_out = grid_out;
    a.test_stall = test_stall;
    a.cta_busy_ns = reinterpret_cast<long long *>(cta_busy_ns);
    if (fp8) {
        a.q_exp = exps[0];
        a.k_exp = exps[1];
        a.v_exp = exps[2];
    }
    return from_cuda(fp8 ? launch_sparse_attn_fp8(a, block, s) : launch_sparse_attn(a, d, block, s));
}

int fvattn_sparse_fwd_fp8(const void *Q8, const void *K8, const void *V8, const int32_t *q_exp, const int32_t *k_exp,
                          const int32_t *v_exp, const int32_t *row_ptr, const int32_t *col_idx, int B, int H, int N,
                          int d, int block, int causal, void *O, float *LSE, void *workspace, size_t ws_bytes,
                          int32_t *dev_status, fvattn_stream_t stream) {
    const int32_t *exps[3] = {q_exp, k_exp, v_exp};
    return sparse_fwd_impl(Q8, K8, V8, row_ptr, col_idx, B, H, N, d, block, causal, O, LSE, workspace, ws_bytes,
                           dev_status, stream, 0, 0, nullptr, nullptr, exps);
}

int fvattn_sparse_fwd(const void *Q, const void *K, const void *V, const int32_t *row_ptr, const int32_t *col_idx,
                      int B, int H, int N, int d, int block, int causal, void *O, float *LSE, void *workspace,
                      size_t ws_bytes, int32_t *dev_status, fvattn_stream_t stream) {
    return sparse_fwd_impl(Q, K, V, row_ptr, col_idx, B, H, N, d, block, causal, O, LSE, workspace, ws_bytes,
                           dev_status, stream, 0);
}

int fvattn_test_sparse_fwd_stall(const void *Q, const void *K, const void *V, const int32_t *row_ptr,
                                 const int32_t *col_idx, int B, int H, int N, int d, int block, int causal, void *O,
                                 float *LSE, void *workspace, size_t ws_bytes, int32_t *dev_status,
                                 fvattn_stream_t stream) {
    return sparse_fwd_impl(Q, K, V, row_ptr, col_idx, B, H, N, d, block, causal, O, LSE, workspace, ws_bytes,
                           dev_status, stream, 1);
}

int fvattn_sparse_fwd_profiled(const void *Q, const void *K, const void *V, const int32_t *row_ptr,
                               const int32_t *col_idx, int B, int H, int N, int d, int block, int causal, void *O,
                               float *LSE, void *workspace, size_t ws_bytes, int32_t *dev_status, int order_mode,
                               int64_t *cta_busy_ns, int *grid, fvattn_stream_t stream) {
    if (order_mode != 0 && order_mode != 1) return FVATTN_ERR_INVALID_ARG;
    if (!cta_busy_ns || !grid) return FVATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(cta_busy_ns) & 7u) return FVATTN_ERR_ALIGNMENT;
    return sparse_fwd_impl(Q, K, V, row_ptr, col_idx, B, H, N, d, block, causal, O, LSE, workspace, ws_bytes,
                           dev_status, stream, 0, order_mode, cta_busy_ns, grid);
}

int64_t fvattn_attn_num_items(int B, int H, int N, int block) {
    if (B < 1 || H < 1 || N < 1 || (block != 64 && block != 128)) return 0;
    return attn_num_items(static_cast<int64_t>(B) * H, static_cast<int>(ceil_div(N, block)), block);
}

int fvattn_attn_work_order(const int32_t *row_ptr, const int32_t *col_idx, int B, int H, int N, int block,
                           int32_t *order, void *workspace, size_t ws_bytes, int32_t *dev_status,
                           fvattn_stream_t stream) {
    if (B < 1 || H < 1 || N < 1 || !row_ptr || !order || !workspace) return FVATTN_ERR_INVALID_ARG;
    if (block != 64 && block != 128) return FVATTN_ERR_UNSUPPORTED;
    if (block == 64 && (!col_idx || !dev_status)) return FVATTN_ERR_INVALID_ARG;
    const int64_t BH = static_cast<int64_t>(B) * H;
    const int64_t nb = ceil_div(N, block);
    if (BH > kMaxHeads || nb > kMaxCount) return FVATTN_ERR_UNSUPPORTED;
    if (!aligned16(workspace)) return FVATTN_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(row_ptr) | reinterpret_cast<uintptr_t>(order) |
         reinterpret_cast<uintptr_t>(col_idx) | reinterpret_cast<uintptr_t>(dev_status)) & 3u)
        return FVATTN_ERR_ALIGNMENT;
    if (ws_bytes < fvattn_fwd_workspace_bytes(B, H, N, block)) return FVATTN_ERR_CAPACITY;
    int rc = check_device();
    if (rc != FVATTN_OK) return rc;
    const FwdWorkspace w = fwd_layout(BH, static_cast<int>(nb), block);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (dev_status && (rc = from_cuda(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s))) != FVATTN_OK) return rc;
    char *ws = static_cast<char *>(workspace);
    if ((rc = enqueue_work_order(row_ptr, col_idx, BH, static_cast<int>(nb), block, 0, ws, w, dev_status, s)) !=
        FVATTN_OK)
        return rc;
    const int64_t items = attn_num_items(BH, static_cast<int>(nb), block);
    return from_cuda(cudaMemcpyAsync(order, ws + w.order, sizeof(int32_t) * items, cudaMemcpyDeviceToDevice, s));
}

namespace {
struct SasaWorkspace {
    size_t route, row_ptr, col_idx, head_counts, cand, cand_p, order, head_rank, mach, lists, list_off, counts, total;
};
SasaWorkspace sasa_layout(int64_t BH, int nb, int d) {
    SasaWorkspace w{};
    Carver c;
    const int64_t rows = BH * nb;
    w.route = c.take<char>(route_workspace_layout(BH, nb, d).total);
    w.row_ptr = c.take<int32_t>(static_cast<size_t>(rows) + 1);
    w.col_idx = c.take<int32_t>(static_cast<size_t>(rows) * nb);
    w.head_counts = c.take<int32_t>(static_cast<size_t>(BH));
    w.cand = c.take<int32_t>(static_cast<size_t>(rows) * kSasaCandidates);
    w.cand_p = c.take<double>(static_cast<size_t>(rows) * kSasaCandidates);
    w.order = c.take<int32_t>(static_cast<size_t>(rows));
    w.head_rank = c.take<int32_t>(static_cast<size_t>(BH));
    w.mach = c.take<uint8_t>(static_cast<size_t>(rows));
    w.lists = c.take<int32_t>(static_cast<size_t>(rows));
    w.list_off = c.take<int32_t>(kSasaMaxMachines + 1);
    w.counts = c.take<int32_t>(static_cast<size_t>(rows));
    w.total = align_up(c.off, 256);
    return w;
}
}  // namespace

size_t fvattn_sasa_workspace_bytes(int B, int H, int N, int d, int block) {
    if (check_shape(B, H, N, d, block) != FVATTN_OK) return 0;
    const int64_t nb = ceil_div(N, block);
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (nb > kMaxRouteBlocks || BH > kMaxHeads) return 0;
    return sasa_layout(BH, static_cast<int>(nb), d).total;
}

int fvattn_route_sasa(const void *Q, const void *K, int B, int H, int N, int d, int block, double p, int machines,
                      int32_t *row_ptr, int32_t *col_idx, int64_t col_capacity, int32_t *head_counts,
                      int32_t *added, double *added_mass, int32_t *cand, double *cand_p, void *workspace,
                      size_t ws_bytes, int32_t *dev_status, fvattn_stream_t stream) {
    int rc = check_shape(B, H, N, d, block);
    if (rc != FVATTN_OK) return rc;
    if (machines < 1 || machines > kSasaMaxMachines) return FVATTN_ERR_UNSUPPORTED;
    if (!Q || !K || !row_ptr || !col_idx || !head_counts || !added || !added_mass || !workspace || !dev_status)
        return FVATTN_ERR_INVALID_ARG;
    if (!(p > 0.0) || p > 1.0 || std::isnan(p) || col_capacity < 0) return FVATTN_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(workspace)) return FVATTN_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(row_ptr) | reinterpret_cast<uintptr_t>(col_idx) |
         reinterpret_cast<uintptr_t>(head_counts) | reinterpret_cast<uintptr_t>(added) |
         reinterpret_cast<uintptr_t>(dev_status) | reinterpret_cast<uintptr_t>(cand)) & 3u ||
        ((reinterpret_cast<uintptr_t>(added_mass) | reinterpret_cast<uintptr_t>(cand_p)) & 7u))
        return FVATTN_ERR_ALIGNMENT;
    const int nb = static_cast<int>(ceil_div(N, block));
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (nb > kMaxRouteBlocks || BH > kMaxHeads) return FVATTN_ERR_UNSUPPORTED;
    if (ws_bytes < fvattn_sasa_workspace_bytes(B, H, N, d, block)) return FVATTN_ERR_CAPACITY;
    if ((rc = check_device()) != FVATTN_OK) return rc;
    const SasaWorkspace w = sasa_layout(BH, nb, d);
    char *ws = static_cast<char *>(workspace);
    auto i32 = [&](size_t off) { return reinterpret_cast<int32_t *>(ws + off); };
    const int64_t rows = BH * nb;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = from_cuda(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s))) != FVATTN_OK) return rc;
    // the routed mask and its candidates, the attention's queue order, then the plan
    rc = from_cuda(launch_route(Q, K, BH, N, d, block, nb, p, i32(w.row_ptr), i32(w.col_idx), rows * nb,
                                i32(w.head_counts), ws + w.route, dev_status, s, i32(w.cand),
                                reinterpret_cast<double *>(ws + w.cand_p)));
    if (rc != FVATTN_OK) return rc;
    if ((rc = from_cuda(launch_item_order(i32(w.row_ptr), BH, nb, i32(w.head_rank), i32(w.order), s))) != FVATTN_OK)
        return rc;
    rc = from_cuda(launch_sasa(i32(w.row_ptr), i32(w.col_idx), i32(w.order), rows, nb, BH, machines, i32(w.cand),
                               reinterpret_cast<const double *>(ws + w.cand_p),
                               reinterpret_cast<uint8_t *>(ws + w.mach), i32(w.lists),
                               i32(w.list_off), i32(w.counts), added, added_mass, row_ptr, col_idx, col_capacity,
                               head_counts, dev_status, s));
    if (rc == FVATTN_OK && cand)
        rc = from_cuda(cudaMemcpyAsync(cand, ws + w.cand, sizeof(int32_t) * rows * kSasaCandidates,
                                       cudaMemcpyDeviceToDevice, s));
    if (rc == FVATTN_OK && cand_p)
        rc = from_cuda(cudaMemcpyAsync(cand_p, ws + w.cand_p, sizeof(double) * rows * kSasaCandidates,
                                       cudaMemcpyDeviceToDevice, s));
    return rc;
}

size_t fvattn_bwd_workspace_bytes(int B, int H, int N, int block) {
    if (B < 1 || H < 1 || N < 1 || block != 128) return 0;
    const int64_t nb = ceil_div(N, block);
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (nb > kMaxCount || BH > kMaxHeads) return 0;
    return bwd_layout(BH, N, static_cast<int>(nb)).total;
}

int fvattn_sparse_bwd(const void *Q, const void *K, const void *V, const void *O, const float *LSE, const void *dO,
                      const int32_t *row_ptr, const int32_t *col_idx, int B, int H, int N, int d, int block,
                      int causal, void *dQ, void *dK, void *dV, void *workspace, size_t ws_bytes,
                      int32_t *dev_status, fvattn_stream_t stream) {
    int rc = check_shape(B, H, N, d, block);
    if (rc != FVATTN_OK) return rc;
    if (block != 128) return FVATTN_ERR_UNSUPPORTED;
    if (!Q || !K || !V || !O || !LSE || !dO || !row_ptr || !col_idx || !dQ || !dK || !dV || !workspace ||
        !dev_status)
        return FVATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FVATTN_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) || !aligned16(dQ) ||
        !aligned16(dK) || !aligned16(dV) || !aligned16(workspace))
        return FVATTN_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(row_ptr) | reinterpret_cast<uintptr_t>(col_idx) |
         reinterpret_cast<uintptr_t>(LSE) | reinterpret_cast<uintptr_t>(dev_status)) & 3u)
        return FVATTN_ERR_ALIGNMENT;
    const int64_t BH = static_cast<int64_t>(B) * H;
    if (BH > kMaxHeads) return FVATTN_ERR_UNSUPPORTED;
    // at most kMaxCount blocks per sequence (the workspace query returns 0 beyond)
    if (ceil_div(N, block) > kMaxCount) return FVATTN_ERR_UNSUPPORTED;
    const int nb = static_cast<int>(ceil_div(N, block));
    if (ws_bytes < fvattn_bwd_workspace_bytes(B, H, N, block)) return FVATTN_ERR_CAPACITY;
    if ((rc = check_device()) != FVATTN_OK) return rc;
    DeviceInfo info;
    if (!device_info(&info)) return FVATTN_ERR_CUDA;
    const int64_t rows = BH * nb;
    const BwdWorkspace w = bwd_layout(BH, N, nb);
    char *ws = static_cast<char *>(workspace);
    float *Dv = reinterpret_cast<float *>(ws + w.D);
    int32_t *col_ptr = reinterpret_cast<int32_t *>(ws + w.col_ptr);
    int32_t *csc_idx = reinterpret_cast<int32_t *>(ws + w.csc_idx);
    int32_t *order_q = reinterpret_cast<int32_t *>(ws + w.order_q);
    int32_t *order_k = reinterpret_cast<int32_t *>(ws + w.order_k);
    int32_t *head_rank = reinterpret_cast<int32_t *>(ws + w.head_rank);
    int *counters = reinterpret_cast<int *>(ws + w.counters);

    CUtensorMap mq, mk, mv, mdo;
    if (!make_map(&mq, Q, BH, N, d, block) || !make_map(&mk, K, BH, N, d, block) ||
        !make_map(&mv, V, BH, N, d, block) || !make_map(&mdo, dO, BH, N, d, block))
        return FVATTN_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = from_cuda(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s))) != FVATTN_OK) return rc;
    if ((rc = from_cuda(cudaMemsetAsync(counters, 0, 2 * sizeof(int), s))) != FVATTN_OK) return rc;
    if ((rc = from_cuda(launch_bwd_rowdot(O, dO, BH * N, d, Dv, s))) != FVATTN_OK) return rc;
    if ((rc = from_cuda(launch_csc(row_ptr, col_idx, BH, nb, col_ptr, csc_idx, dev_status, s))) != FVATTN_OK)
        return rc;
    // both queues head-major, longest first: rows by selected blocks, key blocks by selecting rows
    if ((rc = from_cuda(launch_item_order(row_ptr, BH, nb, head_rank, order_q, s))) != FVATTN_OK) return rc;
    if ((rc = from_cuda(launch_item_order(col_ptr, BH, nb, head_rank, order_k, s))) != FVATTN_OK) return rc;

    BwdLaunch a{};
    a.tmap_q = &mq;
    a.tmap_k = &mk;
    a.tmap_v = &mv;
    a.tmap_do = &mdo;
    a.Q = Q;
    a.dO = dO;
    a.LSE = LSE;
    a.D = Dv;
    a.row_ptr = row_ptr;
    a.col_idx = col_idx;
    a.col_ptr = col_ptr;
    a.csc_idx = csc_idx;
    a.order_q = order_q;
    a.order_k = order_k;
    a.n_items = static_cast<int>(rows);
    a.counters = counters;
    a.N = N;
    a.nb = nb;
    a.causal = causal;
    a.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
    a.dQ = dQ;
    a.dK = dK;
    a.dV = dV;
    a.dev_status = dev_status;
    a.grid = static_cast<int>(rows < info.sms ? rows : info.sms);
    if ((rc = from_cuda(launch_bwd_dq(a, d, s))) != FVATTN_OK) return rc;
    return from_cuda(launch_bwd_dkdv(a, d, s));
}

int fvattn_attention_host(const void *hQ, const void *hK, const void *hV, int B, int H, int N, int d, int block,
                          double p, int causal, void *hO, float *hLSE, void *dQ, void *dK, void *dV, void *dO,
                          float *dLSE, int32_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                          int32_t *head_counts, void *route_ws, size_t route_ws_bytes, void *fwd_ws,
                          size_t fwd_ws_bytes, int32_t *dev_status, fvattn_stream_t stream) {
    int rc = check_shape(B, H, N, d, block);
    if (rc != FVATTN_OK) return rc;
    if (!hQ || !hK || !hV || !hO || !hLSE || !dQ || !dK || !dV || !dO || !dLSE || !dev_status)
        return FVATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(dev_status) & 3u) return FVATTN_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t BH = static_cast<int64_t>(B) * H;
    const size_t head_bytes = static_cast<size_t>(N) * d * 2;
    // Heads are independent for routing and attention: split B*H into chunks of about
    // 64 MB per tensor so that copies in, compute and copies out of different chunks
    // overlap (two extra streams for the copies, the caller's stream for compute).  The
    // copies in are the bottleneck; what follows the last one (that chunk's compute and
    // copy out) is not hidden, so the last chunks halve in size down to one head.
    const int64_t hc = std::max<int64_t>(1, std::min<int64_t>(BH, (64ll << 20) / static_cast<int64_t>(head_bytes)));
    auto chunk_heads = [&](int64_t remaining) {
        return remaining > 2 * hc ? hc : std::max<int64_t>(1, std::min<int64_t>(hc, (remaining + 1) / 2));
    };
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev_in = nullptr, ev_out = nullptr;
    auto cleanup = [&]() {
        if (ev_in) cudaEventDestroy(ev_in);
        if (ev_out) cudaEventDestroy(ev_out);
        if (s_in) cudaStreamDestroy(s_in);
        if (s_out) cudaStreamDestroy(s_out);
    };
    if (cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ev_in, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ev_out, cudaEventDisableTiming) != cudaSuccess) {
        cleanup();
        return FVATTN_ERR_CUDA;
    }
    // dev_status: [0] routing of the current chunk, [1] attention of the current chunk,
    // [2] first error over all chunks.  The copy streams start after everything already
    // queued on the caller's stream.
    rc = from_cuda(cudaMemsetAsync(dev_status + 2, 0, sizeof(int32_t), s));
    if (rc == FVATTN_OK) rc = from_cuda(cudaEventRecord(ev_out, s));
    if (rc == FVATTN_OK) rc = from_cuda(cudaStreamWaitEvent(s_in, ev_out, 0));
    int hn = 0;
    for (int64_t off = 0; off < BH && rc == FVATTN_OK; off += hn) {
        hn = static_cast<int>(chunk_heads(BH - off));
        const size_t o = static_cast<size_t>(off) * head_bytes, nbytes = static_cast<size_t>(hn) * head_bytes;
        const size_t lo = static_cast<size_t>(off) * N * sizeof(float), lbytes = static_cast<size_t>(hn) * N * sizeof(float);
        auto dptr = [&](void *base) { return static_cast<char *>(base) + o; };
        auto hptr = [&](const void *base) { return static_cast<const char *>(base) + o; };
        if ((rc = from_cuda(cudaMemcpyAsync(dptr(dQ), hptr(hQ), nbytes, cudaMemcpyHostToDevice, s_in))) ||
            (rc = from_cuda(cudaMemcpyAsync(dptr(dK), hptr(hK), nbytes, cudaMemcpyHostToDevice, s_in))) ||
            (rc = from_cuda(cudaMemcpyAsync(dptr(dV), hptr(hV), nbytes, cudaMemcpyHostToDevice, s_in))) ||
            (rc = from_cuda(cudaEventRecord(ev_in, s_in))) || (rc = from_cuda(cudaStreamWaitEvent(s, ev_in, 0))))
            break;
        rc = fvattn_route(dptr(dQ), dptr(dK), 1, hn, N, d, block, p, row_ptr, col_idx, col_capacity,
                          head_counts + off, route_ws, route_ws_bytes, dev_status, stream);
        if (rc != FVATTN_OK) break;
        rc = fvattn_sparse_fwd(dptr(dQ), dptr(dK), dptr(dV), row_ptr, col_idx, 1, hn, N, d, block, causal,
                               dptr(dO), reinterpret_cast<float *>(reinterpret_cast<char *>(dLSE) + lo), fwd_ws,
                               fwd_ws_bytes, dev_status + 1, stream);
        if (rc != FVATTN_OK) break;
        status_merge_kernel<<<1, 1, 0, s>>>(dev_status);
        if ((rc = from_cuda(cudaGetLastError())) || (rc = from_cuda(cudaEventRecord(ev_out, s))) ||
            (rc = from_cuda(cudaStreamWaitEvent(s_out, ev_out, 0))) ||
            (rc = from_cuda(cudaMemcpyAsync(static_cast<char *>(hO) + o, dptr(dO), nbytes, cudaMemcpyDeviceToHost,
                                            s_out))) ||
            (rc = from_cuda(cudaMemcpyAsync(reinterpret_cast<char *>(hLSE) + lo,
                                            reinterpret_cast<char *>(dLSE) + lo, lbytes, cudaMemcpyDeviceToHost,
                                            s_out))))
            break;
    }
    int32_t st = 0;
    if (rc == FVATTN_OK) rc = from_cuda(cudaMemcpyAsync(&st, dev_status + 2, sizeof(st), cudaMemcpyDeviceToHost, s));
    const int rs1 = from_cuda(cudaStreamSynchronize(s_in));
    const int rs2 = from_cuda(cudaStreamSynchronize(s_out));
    const int rs3 = from_cuda(cudaStreamSynchronize(s));
    cleanup();
    if (rc != FVATTN_OK) return rc;
    if (rs1 != FVATTN_OK || rs2 != FVATTN_OK || rs3 != FVATTN_OK) return FVATTN_ERR_CUDA;
    return st;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------
// fvattn_sparse_fwd_noalloc: the sparse forward for callers that cannot allocate device memory
// when they call it.  Its scratch (the longest-first order, the ordering kernels' counters and
// the work-queue counter) lives in one statically sized device array that the library owns;
// every device that loads the library keeps FVATTN_NOALLOC_SCRATCH_BYTES of it until exit.

namespace {

__device__ __align__(256) unsigned char g_fwd_scratch[FVATTN_NOALLOC_SCRATCH_BYTES];

// Device address of g_fwd_scratch on the current device.  In host code the symbol
// g_fwd_scratch is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress (with that device current).  The lookup allocates nothing; it
// is repeated on every call made outside stream capture, so the address follows the
// module if the device was reset and the library's module reloaded.  During capture
// the address of the last call outside capture is used (the first call on a device
// must therefore come before any capture).
int static_scratch(cudaStream_t stream, void **out) {
    static std::mutex mu;
    static void *addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FVATTN_ERR_CUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return FVATTN_ERR_CUDA;
    std::lock_guard<std::mutex> g(mu);
    if (addr[dev] == nullptr || cap == cudaStreamCaptureStatusNone) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fwd_scratch) != cudaSuccess || p == nullptr) return FVATTN_ERR_CUDA;
        addr[dev] = p;
    }
    *out = addr[dev];
    return FVATTN_OK;
}

}  // namespace

extern "C" int fvattn_sparse_fwd_noalloc(const void *Q, const void *K, const void *V, const int32_t *row_ptr,
                                         const int32_t *col_idx, int B, int H, int N, int d, int block, int causal,
                                         void *O, float *LSE, int32_t *dev_status, fvattn_stream_t stream) {
    int rc = check_shape(B, H, N, d, block);
    if (rc != FVATTN_OK) return rc;
    const size_t need = fvattn_fwd_workspace_bytes(B, H, N, block);
    if (need == 0) return FVATTN_ERR_INVALID_ARG;
    if (need > FVATTN_NOALLOC_SCRATCH_BYTES) return FVATTN_ERR_CAPACITY;
    void *scratch = nullptr;
    if ((rc = static_scratch(reinterpret_cast<cudaStream_t>(stream), &scratch)) != FVATTN_OK) return rc;
    // Same launches as fvattn_sparse_fwd; the work-queue counter in the scratch is
    // cleared there on the stream before the attention kernel starts, and every other
    // scratch word is written before it is read, so stale contents never matter.
    return fvattn_sparse_fwd(Q, K, V, row_ptr, col_idx, B, H, N, d, block, causal, O, LSE, scratch,
                             FVATTN_NOALLOC_SCRATCH_BYTES, dev_status, stream);
}
