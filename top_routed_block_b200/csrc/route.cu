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
//   route_select_kernel   per (head, 8 query blocks): fp64 scores for the 8 rows, then
//                         one warp per row: softmax, a bitonic sort of (score, index) in
//                         registers, prefix sum to p, a row bitmap.
//   csr_scan_kernel       row_ptr = exclusive scan of the row counts; head counts.
//   csr_scatter_kernel    col_idx from the row bitmaps, ascending.
// With candidate outputs (the slack-aware augmentation of sasa.cu), the select
// kernel also writes, per row, the kSasaCandidates key blocks that follow the cut
// in the routing order and their probabilities.
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
//
// One CTA per (head, kSelRows consecutive query blocks), one warp per query
// block.  The score phase is shared by the CTA: thread t owns key blocks
// j = t + m*kSelThreads and accumulates all kSelRows rows for them, so every K
// mean is loaded once per CTA.  After one block barrier each warp finishes its
// row alone (softmax, a bitonic sort held in registers, the prefix sum to p,
// the row bitmap), with warp shuffles and no further block barrier.

constexpr int kSelRows = 8;                  // query blocks (and warps) per CTA
constexpr int kSelThreads = 32 * kSelRows;

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

// x precedes y in the selection order: score descending, then index ascending.
__device__ __forceinline__ bool precedes(double sx, int ix, double sy, int iy) {
    return (sx > sy) || (sx == sy && ix < iy);
}

// MJ: key blocks per thread in the score phase (nb <= MJ * kSelThreads).
// EPL: sorted positions per lane (nb <= 32 * EPL); lane l holds positions
// l*EPL .. l*EPL+EPL-1, so a bitonic stage of partner distance j < EPL stays in
// one lane's registers and a stage of distance j >= EPL pairs lane l with lane
// l ^ (j / EPL).
template <int D, int MJ, int EPL>
__global__ void __launch_bounds__(kSelThreads) route_select_kernel(const double *__restrict__ qbar,
                                                                   const double *__restrict__ kbarT, int nb, double p,
                                                                   double scale, int32_t *__restrict__ counts,
                                                                   uint32_t *__restrict__ bitmap, int W,
                                                                   int32_t *__restrict__ cand, double *__restrict__ cand_p) {
    constexpr int NP2 = 32 * EPL;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    double *sq = reinterpret_cast<double *>(smem_raw);                 // [kSelRows][D] query means
    double *ss = sq + kSelRows * D;                                    // [kSelRows][nb] scores, then probabilities
    uint32_t *bm = reinterpret_cast<uint32_t *>(ss + kSelRows * nb);   // [kSelRows][32] row bitmaps

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.y;
    const int i0 = blockIdx.x * kSelRows;
    const int nrows = min(kSelRows, nb - i0);

    for (int e = tid; e < kSelRows * D; e += kSelThreads) sq[e] = (e / D < nrows) ? qbar[(bh * nb + i0) * D + e] : 0.0;
    __syncthreads();

    // s_ij = (sum_c qbar_i[c] * kbar_j[c]) * scale, c in index order, no fused multiply-add
    {
        double acc[kSelRows][MJ];
#pragma unroll
        for (int r = 0; r < kSelRows; ++r)
#pragma unroll
            for (int m = 0; m < MJ; ++m) acc[r][m] = 0.0;
        const double *kt = kbarT + bh * D * nb;
#pragma unroll 4
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
    }
    __syncthreads();
    if (warp >= nrows) return;  // only warp-level synchronisation from here on

    double *s = ss + warp * nb;
    uint32_t *bmw = bm + warp * 32;
    const int64_t row = bh * nb + i0 + warp;
    int count;
    if (cand && lane < kSasaCandidates) {  // no candidate unless written below
        cand[row * kSasaCandidates + lane] = -1;
        cand_p[row * kSasaCandidates + lane] = 0.0;
    }
    __syncwarp();
    if (p >= 1.0) {
        count = nb;
        if (lane < W) {
            const int nbits = min(32, nb - lane * 32);
            bmw[lane] = (nbits == 32) ? 0xffffffffu : ((1u << nbits) - 1u);
        }
    } else {
        bmw[lane] = 0u;
        double key[EPL];
        int idx[EPL];
        double mx = -CUDART_INF;
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = lane * EPL + q;
            idx[q] = e;  // padding positions keep their own index and sort last
            key[q] = (e < nb) ? s[e] : -CUDART_INF;
            mx = fmax(mx, key[q]);
        }
        mx = warp_max(mx);
        // softmax over key blocks; the probabilities replace the scores in s[] (by index)
        double z = 0.0;
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = lane * EPL + q;
            if (e < nb) {
                const double v = exp(__dsub_rn(key[q], mx));
                s[e] = v;
                z = __dadd_rn(z, v);
            }
        }
        z = warp_sum(z);
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = lane * EPL + q;
            if (e < nb) s[e] = __ddiv_rn(s[e], z);
        }
        // bitonic sort of (score, index) into selection order
#pragma unroll
        for (int k = 2; k <= NP2; k <<= 1) {
#pragma unroll
            for (int j = k >> 1; j > 0; j >>= 1) {
                if (j >= EPL) {
                    const int lm = j / EPL;
                    const bool lower = ((lane * EPL) & j) == 0;
#pragma unroll
                    for (int q = 0; q < EPL; ++q) {
                        const bool up = (((lane * EPL + q) & k) == 0);
                        const double ok = __shfl_xor_sync(0xffffffffu, key[q], lm);
                        const int oi = __shfl_xor_sync(0xffffffffu, idx[q], lm);
                        // the lower position of an ascending pair keeps the preceding element
                        const bool take = (lower == up) ? precedes(ok, oi, key[q], idx[q])
                                                        : precedes(key[q], idx[q], ok, oi);
                        if (take) {
                            key[q] = ok;
                            idx[q] = oi;
                        }
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < EPL; ++q) {
                        const int q2 = q ^ j;
                        if (q2 > q) {
                            const bool up = (((lane * EPL + q) & k) == 0);
                            const bool sw = up ? precedes(key[q2], idx[q2], key[q], idx[q])
                                               : precedes(key[q], idx[q], key[q2], idx[q2]);
                            if (sw) {
                                const double tk = key[q];
                                key[q] = key[q2];
                                key[q2] = tk;
                                const int ti = idx[q];
                                idx[q] = idx[q2];
                                idx[q2] = ti;
                            }
                        }
                    }
                }
            }
        }
        __syncwarp();
        // cumulative mass in sorted order: per-lane running sums plus the lanes before
        double loc[EPL];
        double run = 0.0;
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            run = __dadd_rn(run, (idx[q] < nb) ? s[idx[q]] : 0.0);
            loc[q] = run;
        }
        double inc = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double t = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc = __dadd_rn(t, inc);
        }
        double pre = __shfl_up_sync(0xffffffffu, inc, 1);
        if (lane == 0) pre = 0.0;
        int first = NP2;
#pragma unroll
        for (int q = EPL - 1; q >= 0; --q)
            if (__dadd_rn(pre, loc[q]) >= p) first = lane * EPL + q;
        first = __reduce_min_sync(0xffffffffu, first);
        const int kcut = (first < nb) ? first : nb - 1;  // the mass never reached p: keep every block
        count = kcut + 1;
        __syncwarp();
#pragma unroll
        for (int q = 0; q < EPL; ++q)
            if (lane * EPL + q <= kcut) atomicOr(&bmw[idx[q] >> 5], 1u << (idx[q] & 31));
        if (cand) {  // the blocks right after the cut, in routing order
#pragma unroll
            for (int q = 0; q < EPL; ++q) {
                const int e = lane * EPL + q - kcut - 1;
                if (e >= 0 && e < kSasaCandidates && idx[q] < nb) {
                    cand[row * kSasaCandidates + e] = idx[q];
                    cand_p[row * kSasaCandidates + e] = s[idx[q]];
                }
            }
        }
    }
    __syncwarp();
    if (lane < W) bitmap[row * W + lane] = bmw[lane];
    if (lane == 0) counts[row] = count;
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
    return sizeof(double) * (kSelRows * d + kSelRows * nb) + sizeof(uint32_t) * kSelRows * 32;
}

namespace {

struct SelectArgs {
    const double *qbar, *kbarT;
    int nb;
    double p, scale;
    int32_t *counts;
    uint32_t *bitmap;
    int W;
    int64_t BH;
    int32_t *cand;
    double *cand_p;
};

template <int D, int MJ, int EPL>
cudaError_t launch_select(const SelectArgs &a, cudaStream_t stream) {
    const size_t smem = route_select_smem_bytes(D, a.nb);
    cudaError_t e = cudaFuncSetAttribute(route_select_kernel<D, MJ, EPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(ceil_div(a.nb, kSelRows)), static_cast<unsigned>(a.BH));
    route_select_kernel<D, MJ, EPL><<<grid, kSelThreads, smem, stream>>>(a.qbar, a.kbarT, a.nb, a.p, a.scale,
                                                                         a.counts, a.bitmap, a.W, a.cand, a.cand_p);
    return cudaGetLastError();
}

// Smallest register sort that holds nb positions (nb <= kMaxRouteBlocks = 1024).
template <int D>
cudaError_t dispatch_select(const SelectArgs &a, cudaStream_t stream) {
    static_assert(kSelThreads == 256 && kMaxRouteBlocks == 1024, "dispatch covers nb <= 1024 with 256 threads");
    if (a.nb <= 32) return launch_select<D, 1, 1>(a, stream);
    if (a.nb <= 64) return launch_select<D, 1, 2>(a, stream);
    if (a.nb <= 128) return launch_select<D, 1, 4>(a, stream);
    if (a.nb <= 256) return launch_select<D, 1, 8>(a, stream);
    if (a.nb <= 512) return launch_select<D, 2, 16>(a, stream);
    return launch_select<D, 4, 32>(a, stream);
}

}  // namespace

cudaError_t launch_csr_scan(const int32_t *counts, int64_t rows, int nb, int64_t BH, int32_t *row_ptr,
                            int64_t capacity, int32_t *head_counts, int32_t *dev_status, cudaStream_t stream) {
    csr_scan_kernel<<<1, kScanThreads, 0, stream>>>(counts, rows, nb, BH, row_ptr, capacity, head_counts,
                                                    dev_status);
    return cudaGetLastError();
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
                         void *workspace, int32_t *dev_status, cudaStream_t stream, int32_t *cand, double *cand_p) {
    const RouteWorkspace w = route_workspace_layout(BH, nb, d);
    char *ws = static_cast<char *>(workspace);
    double *qbar = reinterpret_cast<double *>(ws + w.qbar);
    double *kbarT = reinterpret_cast<double *>(ws + w.kbarT);
    int32_t *counts = reinterpret_cast<int32_t *>(ws + w.counts);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(ws + w.bitmap);
    const int64_t rows = BH * nb;
    const double scale = 1.0 / sqrt(static_cast<double>(d));
    const SelectArgs sel{qbar, kbarT, nb, p, scale, counts, bitmap, w.W, BH, cand, cand_p};
    const auto *q16 = static_cast<const uint16_t *>(Q);
    const auto *k16 = static_cast<const uint16_t *>(K);
    cudaError_t e;
    if (d == 128) {
        const dim3 grid(static_cast<unsigned>(ceil_div(rows, 256 / 16)), 2);
        pool_kernel<128><<<grid, 256, 0, stream>>>(q16, k16, BH, N, bs, nb, qbar, kbarT);
        e = dispatch_select<128>(sel, stream);
    } else {
        const dim3 grid(static_cast<unsigned>(ceil_div(rows, 256 / 8)), 2);
        pool_kernel<64><<<grid, 256, 0, stream>>>(q16, k16, BH, N, bs, nb, qbar, kbarT);
        e = dispatch_select<64>(sel, stream);
    }
    if (e != cudaSuccess) return e;
    e = launch_csr_scan(counts, rows, nb, BH, row_ptr, capacity, head_counts, dev_status, stream);
    if (e != cudaSuccess) return e;
    csr_scatter_kernel<<<static_cast<unsigned>(ceil_div(rows, 8)), 256, 0, stream>>>(bitmap, row_ptr, rows, w.W,
                                                                                     col_idx, capacity);
    return cudaGetLastError();
}

}  // namespace fvattn
