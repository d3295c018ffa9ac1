// route.cu -- top-p routing kernels (FVAttn review, §1 Key Terms "Top-p routing").
//
// The pages name the importance score without defining it; this library fixes
// it as: the mean of every block of `bs` tokens of Q and of K (over the tokens
// that exist), score s_ij = qbar_i . kbar_j / sqrt(d), a softmax over all key
// blocks, and the shortest prefix of key blocks in (score desc, index asc)
// order whose probability mass is >= p (p >= 1 keeps every block).
//
// The whole chain after the bf16 loads runs in fp64, with the pooled sums and
// the dot products accumulated in index order with separate multiply and add
// roundings, so every score is bit-identical to a plain sequential fp64
// evaluation of the definition; the sort key is the score itself.
//
// Kernels:
//   pool_kernel           HBM-bound: reads Q and K once, writes fp64 block means
//                         (Q means row-major [BH,nb,d], K means transposed [BH,d,nb]).
//   route_select_kernel   per (head, 8 query blocks): fp64 scores, softmax, a bitonic
//                         sort of (score, index), prefix sum to p, a row bitmap.
//   csr_scan_kernel       row_ptr = exclusive scan of the row counts; head counts.
//   csr_scatter_kernel    col_idx from the row bitmaps, ascending.
#include <cstdint>
#include <math_constants.h>

#include "common.cuh"
#include "route.cuh"

namespace fvattn {

namespace {

__device__ __forceinline__ double bf16_lo(uint32_t w) { return static_cast<double>(__uint_as_float(w << 16)); }
__device__ __forceinline__ double bf16_hi(uint32_t w) {
    return static_cast<double>(__uint_as_float(w & 0xFFFF0000u));
}

// ------------------------------------------------------------------ pooling

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K,
                                                   int64_t BH, int N, int bs, int nb, double *__restrict__ qbar,
                                                   double *__restrict__ kbarT) {
    constexpr int TPU = D / 8;         // threads per block of tokens (8 channels each)
    constexpr int UPC = 256 / TPU;     // token blocks per CTA
    const uint16_t *X = (blockIdx.y == 0) ? Q : K;
    const int64_t unit = static_cast<int64_t>(blockIdx.x) * UPC + threadIdx.x / TPU;
    if (unit >= BH * nb) return;
    const int c0 = (threadIdx.x % TPU) * 8;
    const int64_t bh = unit / nb;
    const int i = static_cast<int>(unit % nb);
    const int64_t t0 = static_cast<int64_t>(i) * bs;
    const int n = static_cast<int>(min(static_cast<int64_t>(N), t0 + bs) - t0);
    const uint4 *src = reinterpret_cast<const uint4 *>(X + ((bh * N + t0) * D + c0));
    double acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.0;
    for (int t = 0; t < n; t += 8) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (t + u < n) v[u] = __ldg(src + static_cast<int64_t>(t + u) * (D / 8));
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (t + u < n) {
                // tokens strictly in order: acc = acc + x
                acc[0] = __dadd_rn(acc[0], bf16_lo(v[u].x));
                acc[1] = __dadd_rn(acc[1], bf16_hi(v[u].x));
                acc[2] = __dadd_rn(acc[2], bf16_lo(v[u].y));
                acc[3] = __dadd_rn(acc[3], bf16_hi(v[u].y));
                acc[4] = __dadd_rn(acc[4], bf16_lo(v[u].z));
                acc[5] = __dadd_rn(acc[5], bf16_hi(v[u].z));
                acc[6] = __dadd_rn(acc[6], bf16_lo(v[u].w));
                acc[7] = __dadd_rn(acc[7], bf16_hi(v[u].w));
            }
        }
    }
    const double cnt = static_cast<double>(n);
    if (blockIdx.y == 0) {
        double2 *dst = reinterpret_cast<double2 *>(qbar + unit * D + c0);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_double2(__ddiv_rn(acc[2 * q], cnt), __ddiv_rn(acc[2 * q + 1], cnt));
    } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) kbarT[(bh * D + c0 + q) * nb + i] = __ddiv_rn(acc[q], cnt);
    }
}

// ------------------------------------------------------ scores and selection

constexpr int kSelThreads = 256;
constexpr int kSelRows = 8;  // query blocks per CTA (they share the K-mean loads)

__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Block-wide reductions over kSelThreads threads; `red` holds 32 doubles.
__device__ __forceinline__ double block_max(double v, double *red) {
    v = warp_max(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    double r = (l < kSelThreads / 32) ? red[l] : -CUDART_INF;
    return warp_max(r);
}
__device__ __forceinline__ double block_sum(double v, double *red) {
    v = warp_sum(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    double r = (l < kSelThreads / 32) ? red[l] : 0.0;
    return warp_sum(r);
}

// "x comes after y" in the selection order: score descending, index ascending.
__device__ __forceinline__ bool after(double kx, int ix, double ky, int iy) {
    return (kx < ky) || (kx == ky && ix > iy);
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) route_select_kernel(const double *__restrict__ qbar,
                                                                   const double *__restrict__ kbarT, int nb, int np2,
                                                                   double p, double scale,
                                                                   int32_t *__restrict__ counts,
                                                                   uint32_t *__restrict__ bitmap, int W) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    double *sq = reinterpret_cast<double *>(smem_raw);          // [kSelRows][D]
    double *ss = sq + kSelRows * D;                             // [kSelRows][nb] scores
    double *pe = ss + kSelRows * nb;                            // [nb] probabilities by index
    double *sk = pe + nb;                                       // [np2] sort keys, then cumulative mass
    double *red = sk + np2;                                     // [32]
    int *si = reinterpret_cast<int *>(red + 32);                // [np2] sort indices
    uint32_t *bm = reinterpret_cast<uint32_t *>(si + np2);      // [32] row bitmap
    int *kfirst = reinterpret_cast<int *>(bm + 32);             // [1]

    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.y;
    const int i0 = blockIdx.x * kSelRows;
    const int nrows = min(kSelRows, nb - i0);

    for (int e = tid; e < kSelRows * D; e += kSelThreads) {
        const int r = e / D;
        sq[e] = (r < nrows) ? qbar[(bh * nb + i0) * D + e] : 0.0;
    }
    __syncthreads();

    // s_ij = (sum_c qbar_i[c] * kbar_j[c]) * scale, c in index order, no fused multiply-add
    constexpr int MJ = kMaxRouteBlocks / kSelThreads;
    double acc[kSelRows][MJ];
#pragma unroll
    for (int r = 0; r < kSelRows; ++r)
#pragma unroll
        for (int m = 0; m < MJ; ++m) acc[r][m] = 0.0;
    const double *kt = kbarT + bh * D * nb;
    for (int c = 0; c < D; ++c) {
        double kv[MJ];
#pragma unroll
        for (int m = 0; m < MJ; ++m) {
            const int j = tid + m * kSelThreads;
            kv[m] = (j < nb) ? __ldg(kt + static_cast<int64_t>(c) * nb + j) : 0.0;
        }
#pragma unroll
        for (int r = 0; r < kSelRows; ++r) {
            const double qv = sq[r * D + c];
#pragma unroll
            for (int m = 0; m < MJ; ++m) acc[r][m] = __dadd_rn(acc[r][m], __dmul_rn(qv, kv[m]));
        }
    }
#pragma unroll
    for (int r = 0; r < kSelRows; ++r)
#pragma unroll
        for (int m = 0; m < MJ; ++m) {
            const int j = tid + m * kSelThreads;
            if (j < nb && r < nrows) ss[r * nb + j] = __dmul_rn(acc[r][m], scale);
        }
    __syncthreads();

    const int ept = (np2 >= kSelThreads) ? np2 / kSelThreads : 1;  // scan items per thread
    for (int r = 0; r < nrows; ++r) {
        const double *s = ss + r * nb;
        const int64_t row = bh * nb + i0 + r;
        // softmax over key blocks
        double mx = -CUDART_INF;
        for (int j = tid; j < nb; j += kSelThreads) mx = fmax(mx, s[j]);
        mx = block_max(mx, red);
        double z = 0.0;
        for (int j = tid; j < nb; j += kSelThreads) {
            const double e = exp(__dsub_rn(s[j], mx));
            pe[j] = e;
            z = __dadd_rn(z, e);
        }
        z = block_sum(z, red);
        for (int j = tid; j < nb; j += kSelThreads) pe[j] = __ddiv_rn(pe[j], z);
        if (tid < 32) bm[tid] = 0u;
        if (tid == 0) *kfirst = np2;
        __syncthreads();

        int count;
        if (p >= 1.0) {
            count = nb;
            for (int j = tid; j < nb; j += kSelThreads) atomicOr(&bm[j >> 5], 1u << (j & 31));
        } else {
            for (int e = tid; e < np2; e += kSelThreads) {
                sk[e] = (e < nb) ? s[e] : -CUDART_INF;
                si[e] = (e < nb) ? e : 0x7fffffff;
            }
            __syncthreads();
            // bitonic network: ascending in the "after" relation
            for (int k = 2; k <= np2; k <<= 1) {
                for (int jj = k >> 1; jj > 0; jj >>= 1) {
                    for (int e = tid; e < (np2 >> 1); e += kSelThreads) {
                        const int a = (e / jj) * 2 * jj + (e % jj);
                        const int b = a + jj;
                        const double ka = sk[a], kb = sk[b];
                        const int ia = si[a], ib = si[b];
                        const bool up = (a & k) == 0;
                        const bool swap = up ? after(ka, ia, kb, ib) : after(kb, ib, ka, ia);
                        if (swap) {
                            sk[a] = kb;
                            sk[b] = ka;
                            si[a] = ib;
                            si[b] = ia;
                        }
                    }
                    __syncthreads();
                }
            }
            // inclusive prefix sum of the probabilities in sorted order
            const int e0 = tid * ept;
            double loc[kMaxRouteBlocks / kSelThreads];
            double run = 0.0;
#pragma unroll
            for (int q = 0; q < kMaxRouteBlocks / kSelThreads; ++q) {
                const int e = e0 + q;
                const double v = (q < ept && e < nb) ? pe[si[e]] : 0.0;
                run = __dadd_rn(run, v);
                loc[q] = run;
            }
            // exclusive scan of the per-thread totals
            const int lane = tid & 31, warp = tid >> 5;
            double inc = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double t = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc = __dadd_rn(inc, t);
            }
            double exc = __shfl_up_sync(0xffffffffu, inc, 1);
            if (lane == 0) exc = 0.0;
            __syncthreads();
            if (lane == 31) red[warp] = inc;
            __syncthreads();
            double wpre = 0.0;
            for (int w = 0; w < warp; ++w) wpre = __dadd_rn(wpre, red[w]);
            const double pre = __dadd_rn(wpre, exc);
#pragma unroll
            for (int q = 0; q < kMaxRouteBlocks / kSelThreads; ++q) {
                const int e = e0 + q;
                if (q < ept && e < nb && __dadd_rn(pre, loc[q]) >= p) {
                    atomicMin(kfirst, e);
                    break;
                }
            }
            __syncthreads();
            const int kcut = (*kfirst < nb) ? *kfirst : nb - 1;
            count = kcut + 1;
            for (int e = tid; e <= kcut; e += kSelThreads) atomicOr(&bm[si[e] >> 5], 1u << (si[e] & 31));
        }
        __syncthreads();
        if (tid < W) bitmap[row * W + tid] = bm[tid];
        if (tid == 0) counts[row] = count;
        __syncthreads();
    }
}

// -------------------------------------------------------------------- CSR

constexpr int kScanThreads = 1024;
constexpr int kScanItems = 8;

__global__ void __launch_bounds__(kScanThreads) csr_scan_kernel(const int32_t *__restrict__ counts, int64_t rows,
                                                               int nb, int64_t BH, int32_t *__restrict__ row_ptr,
                                                               int64_t capacity, int32_t *__restrict__ head_counts,
                                                               int32_t *dev_status) {
    __shared__ long long wsum[32];
    __shared__ long long carry_s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry_s = 0;
    __syncthreads();
    for (int64_t base = 0; base < rows; base += static_cast<int64_t>(kScanThreads) * kScanItems) {
        long long loc[kScanItems];
        long long run = 0;
        const int64_t i0 = base + static_cast<int64_t>(tid) * kScanItems;
#pragma unroll
        for (int q = 0; q < kScanItems; ++q) {
            loc[q] = run;  // exclusive within the thread
            run += (i0 + q < rows) ? counts[i0 + q] : 0;
        }
        long long inc = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long t = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += t;
        }
        if (lane == 31) wsum[warp] = inc;
        __syncthreads();
        long long wpre = 0;
        for (int w = 0; w < warp; ++w) wpre += wsum[w];
        const long long carry = carry_s;
        const long long pre = carry + wpre + inc - run;
#pragma unroll
        for (int q = 0; q < kScanItems; ++q) {
            if (i0 + q < rows) {
                const long long v = pre + loc[q];
                if (v > 0x7fffffffLL) record_error(dev_status, FVATTN_ERR_CAPACITY);
                row_ptr[i0 + q] = static_cast<int32_t>(v);
            }
        }
        __syncthreads();
        if (tid == kScanThreads - 1) carry_s = pre + run;
        __syncthreads();
    }
    if (tid == 0) {
        const long long total = carry_s;
        if (total > 0x7fffffffLL || total > capacity) record_error(dev_status, FVATTN_ERR_CAPACITY);
        row_ptr[rows] = static_cast<int32_t>(total > 0x7fffffffLL ? 0x7fffffffLL : total);
    }
    __syncthreads();
    for (int64_t bh = tid; bh < BH; bh += kScanThreads)
        head_counts[bh] = row_ptr[(bh + 1) * nb] - row_ptr[bh * nb];
}

__global__ void __launch_bounds__(256) csr_scatter_kernel(const uint32_t *__restrict__ bitmap,
                                                          const int32_t *__restrict__ row_ptr, int64_t rows, int W,
                                                          int32_t *__restrict__ col_idx, int64_t capacity) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const int64_t base = row_ptr[row];
    const int64_t end = row_ptr[row + 1];
    if (end > capacity) return;  // capacity error already recorded by the scan
    uint32_t word = (lane < W) ? bitmap[row * W + lane] : 0u;
    const int pc = __popc(word);
    int inc = pc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
    }
    int64_t off = base + inc - pc;
    while (word) {
        const int b = __ffs(word) - 1;
        col_idx[off++] = lane * 32 + b;
        word &= word - 1;
    }
}

}  // namespace

// ---------------------------------------------------------------- launcher

size_t route_select_smem_bytes(int d, int nb) {
    int np2 = 1;
    while (np2 < nb) np2 <<= 1;
    return sizeof(double) * (kSelRows * d + kSelRows * nb + nb + np2 + 32) + sizeof(int) * np2 +
           sizeof(uint32_t) * 32 + sizeof(int) * 4;
}

RouteWorkspace route_workspace_layout(int64_t BH, int nb, int d) {
    RouteWorkspace w{};
    Carver c;
    const int64_t rows = BH * nb;
    w.W = static_cast<int>(ceil_div(nb, 32));
    w.qbar = c.take<double>(static_cast<size_t>(rows) * d);
    w.kbarT = c.take<double>(static_cast<size_t>(rows) * d);
    w.counts = c.take<int32_t>(static_cast<size_t>(rows));
    w.bitmap = c.take<uint32_t>(static_cast<size_t>(rows) * w.W);
    w.total = align_up(c.off, 256);
    return w;
}

cudaError_t launch_route(const void *Q, const void *K, int64_t BH, int N, int d, int bs, int nb, double p,
                         int32_t *row_ptr, int32_t *col_idx, int64_t capacity, int32_t *head_counts,
                         void *workspace, int32_t *dev_status, cudaStream_t stream) {
    const RouteWorkspace w = route_workspace_layout(BH, nb, d);
    char *ws = static_cast<char *>(workspace);
    double *qbar = reinterpret_cast<double *>(ws + w.qbar);
    double *kbarT = reinterpret_cast<double *>(ws + w.kbarT);
    int32_t *counts = reinterpret_cast<int32_t *>(ws + w.counts);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(ws + w.bitmap);
    const int64_t rows = BH * nb;
    const double scale = 1.0 / sqrt(static_cast<double>(d));
    int np2 = 1;
    while (np2 < nb) np2 <<= 1;
    const size_t sel_smem = route_select_smem_bytes(d, nb);
    const dim3 sel_grid(static_cast<unsigned>(ceil_div(nb, kSelRows)), static_cast<unsigned>(BH));
    const auto *q16 = static_cast<const uint16_t *>(Q);
    const auto *k16 = static_cast<const uint16_t *>(K);
    if (d == 128) {
        const dim3 grid(static_cast<unsigned>(ceil_div(rows, 256 / 16)), 2);
        pool_kernel<128><<<grid, 256, 0, stream>>>(q16, k16, BH, N, bs, nb, qbar, kbarT);
        cudaError_t e = cudaFuncSetAttribute(route_select_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(sel_smem));
        if (e != cudaSuccess) return e;
        route_select_kernel<128><<<sel_grid, kSelThreads, sel_smem, stream>>>(qbar, kbarT, nb, np2, p, scale, counts,
                                                                              bitmap, w.W);
    } else {
        const dim3 grid(static_cast<unsigned>(ceil_div(rows, 256 / 8)), 2);
        pool_kernel<64><<<grid, 256, 0, stream>>>(q16, k16, BH, N, bs, nb, qbar, kbarT);
        cudaError_t e = cudaFuncSetAttribute(route_select_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(sel_smem));
        if (e != cudaSuccess) return e;
        route_select_kernel<64><<<sel_grid, kSelThreads, sel_smem, stream>>>(qbar, kbarT, nb, np2, p, scale, counts,
                                                                             bitmap, w.W);
    }
    csr_scan_kernel<<<1, kScanThreads, 0, stream>>>(counts, rows, nb, BH, row_ptr, capacity, head_counts,
                                                    dev_status);
    csr_scatter_kernel<<<static_cast<unsigned>(ceil_div(rows, 8)), 256, 0, stream>>>(bitmap, row_ptr, rows, w.W,
                                                                                     col_idx, capacity);
    return cudaGetLastError();
}

}  // namespace fvattn
