// attn_bwd.cu -- gradients of the block-sparse attention on sm_100a tensor cores.
//
// The loss gradient dO of O = softmax(Q K^T / sqrt(d)) V over each query
// block's selected key blocks (FVAttn review, §1 "Top-p routing") is taken back
// to dQ, dK and dV.  The FlashAttention review measures training with the fused
// kernel (§Experiments 1 "Training Efficiency") without printing the backward;
// these are the plain derivatives, recomputing P from the LSE the forward saved
// instead of storing it:
//   P = exp(S - LSE),  dV += P^T dO,  dP = dO V^T,  D = rowsum(dO * O),
//   dS = P * (dP - D),  dQ += dS K / sqrt(d),  dK += dS^T Q / sqrt(d).
//
// Kernels:
//   bwd_rowdot_kernel  D[t] = dO[t] . O[t] (fp32; HBM-bound).
//   csc_kernel         the transpose of the block mask per head: for every key
//                      block, the query blocks that selected it, ascending.
//   dq_kernel          one work item = one query block (CSR row): per selected
//                      key block S = Q K^T and dP = dO V^T (Q and dO from TMEM,
//                      TS MMAs), P and dS by the softmax warps, dQ += dS K
//                      accumulated in TMEM over the row's key blocks.
//   dkdv_kernel        one work item = one key block (CSC column): per query
//                      block that selected it S^T = K Q^T and dP^T = V dO^T (SS
//                      MMAs), P^T and dS^T by the softmax warps (thread = key
//                      row), dV += P^T dO and dK += dS^T Q accumulated in TMEM.
// Both gradient kernels use a persistent grid popping items longest-first from a
// head-major queue, a TMA warp streaming tiles into a ring of shared-memory
// stages and an MMA warp; every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <math_constants.h>

#include "attn_bwd.cuh"
#include "common.cuh"
#include "ptx_sm100.cuh"

namespace fvattn {

namespace {

using namespace ptx;

constexpr int kRowsM = 128;   // tile rows (tcgen05 M) = block size
constexpr int kThreads = 192;  // 4 softmax warps + TMA warp + MMA warp
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// ------------------------------------------------------------- D = rowsum(dO * O)

__global__ void __launch_bounds__(256) bwd_rowdot_kernel(const uint16_t *__restrict__ O,
                                                         const uint16_t *__restrict__ dO, int64_t tokens, int d,
                                                         float *__restrict__ D) {
    // one warp per token, 8 bf16 per lane per step
    const int64_t warp_id = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t t = warp_id; t < tokens; t += nwarps) {
        float acc = 0.0f;
        for (int c = lane * 8; c < d; c += 256) {
            const uint4 a = __ldg(reinterpret_cast<const uint4 *>(O + t * d + c));
            const uint4 b = __ldg(reinterpret_cast<const uint4 *>(dO + t * d + c));
            const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc = fmaf(__uint_as_float(av[q] << 16), __uint_as_float(bv[q] << 16), acc);
                acc = fmaf(__uint_as_float(av[q] & 0xFFFF0000u), __uint_as_float(bv[q] & 0xFFFF0000u), acc);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) D[t] = acc;
    }
}

// ------------------------------------------------------------- mask transpose

// One CTA per head.  col_ptr[bh*nb + j] = start of key block j's list; the lists
// of a head start where its CSR rows start (same number of entries).  csc_idx
// holds query-block indices, ascending within each list.
__global__ void __launch_bounds__(1024) csc_kernel(const int32_t *__restrict__ row_ptr,
                                                   const int32_t *__restrict__ col_idx, int nb,
                                                   int32_t *__restrict__ col_ptr, int32_t *__restrict__ csc_idx,
                                                   int32_t *dev_status) {
    extern __shared__ int cnt[];  // [nb] counts, then cursors
    const int64_t bh = blockIdx.x;
    const int64_t r0 = bh * nb;
    const int32_t base = row_ptr[r0], end = row_ptr[r0 + nb];
    for (int j = threadIdx.x; j < nb; j += blockDim.x) cnt[j] = 0;
    __syncthreads();
    for (int32_t e = base + threadIdx.x; e < end; e += blockDim.x) {
        const int32_t j = col_idx[e];
        if (j >= 0 && j < nb) {
            atomicAdd(&cnt[j], 1);
        } else {
            record_error(dev_status, FVATTN_ERR_BAD_CSR);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {  // exclusive scan (nb <= 4096: one thread is fast enough here)
        int32_t run = base;
        for (int j = 0; j < nb; ++j) {
            const int32_t c = cnt[j];
            cnt[j] = run;
            col_ptr[r0 + j] = run;
            run += c;
        }
        if (bh == gridDim.x - 1) col_ptr[r0 + nb] = run;
    }
    __syncthreads();
    // rows in order, so every list comes out ascending; entries of one row are distinct
    for (int i = 0; i < nb; ++i) {
        for (int32_t e = row_ptr[r0 + i] + threadIdx.x; e < row_ptr[r0 + i + 1]; e += blockDim.x) {
            const int32_t j = col_idx[e];
            if (j >= 0 && j < nb) csc_idx[cnt[j]++] = i;
        }
        __syncthreads();
    }
}

}  // namespace

namespace {

// --------------------------------------------------------------------- dQ
// TMEM columns: Q (bf16 pairs) at 0, dO at 64, S at 128, dP (then dS as bf16
// pairs) at 256, dQ (fp32) at 384.
template <int D>
struct DqCfg {
    static constexpr int KBLK = D / 64;
    static constexpr int STAGE_BYTES = KBLK * kRowsM * 128;  // one K or V tile
    static constexpr int NST = 6;
    static constexpr int TILE_BYTES = NST * STAGE_BYTES;
    static constexpr int SMEM_BYTES = TILE_BYTES + 1024 + 512;
    static constexpr uint32_t T_Q = 0, T_DO = 64, T_S = 128, T_DP = 256, T_DQ = 384;
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(kRowsM, kRowsM, 0, 0);  // S, dP: B K-major
    static constexpr uint32_t IDESC_Q = idesc_bf16_f32(kRowsM, D, 0, 1);       // dQ: B (K) MN-major
};

struct DqBarriers {
    uint64_t ring_full[6], ring_empty[6];
    uint64_t q_full, s_full, s_free, dp_full, ds_full, dq_full, dq_empty;
    uint64_t sched_full[2], sched_empty[2];
    uint64_t drain;
    int4 sched_item[2];  // {row, col start, count, valid item}
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(DqBarriers) <= 512, "barrier block exceeds its reservation");

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
              const __nv_bfloat16 *__restrict__ Qg, const __nv_bfloat16 *__restrict__ dOg,
              const float *__restrict__ LSE, const float *__restrict__ Dg, const int32_t *__restrict__ row_ptr,
              const int32_t *__restrict__ col_idx, const int32_t *__restrict__ order, int n_items,
              int *__restrict__ work_counter, int N, int nb, int causal, float scale, __nv_bfloat16 *__restrict__ dQ,
              int32_t *dev_status) {
    using C = DqCfg<D>;
    constexpr int NST = C::NST;
    constexpr int BS = kRowsM;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t base_addr = smem_addr(smem_raw);
    unsigned char *ring = smem_raw + ((1024 - (base_addr & 1023)) & 1023);
    DqBarriers *bar = reinterpret_cast<DqBarriers *>(ring + C::TILE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_flag = &bar->abort_flag;
    const float scale_log2 = scale * kLog2e;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&bar->ring_full[s], 1);
            mbar_init(&bar->ring_empty[s], 1);
        }
        mbar_init(&bar->q_full, 4);
        mbar_init(&bar->s_full, 1);
        mbar_init(&bar->s_free, 4);
        mbar_init(&bar->dp_full, 1);
        mbar_init(&bar->ds_full, 4);
        mbar_init(&bar->dq_full, 1);
        mbar_init(&bar->dq_empty, 4);
        for (int k = 0; k < 2; ++k) {
            mbar_init(&bar->sched_full[k], 1);
            mbar_init(&bar->sched_empty[k], 1 + 4);
        }
        mbar_init(&bar->drain, 1);
        bar->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&bar->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
            uint32_t it = 0, rc = 0;
            bool ok = true;
            while (ok) {
                const int idx = atomicAdd(work_counter, 1);
                const int rw = (idx < n_items) ? order[idx] : -1;
                int4 item = make_int4(-1, 0, 0, 0);
                if (rw >= 0) {
                    int c = row_ptr[rw + 1] - row_ptr[rw];
                    if (c < 0) {
                        record_error(dev_status, FVATTN_ERR_BAD_CSR);
                        c = 0;
                    }
                    item = make_int4(rw, row_ptr[rw], c, 1);
                }
                const uint32_t k = it & 1;
                if (!mbar_wait_short(&bar->sched_empty[k], ((it >> 1) & 1) ^ 1, abort_flag, dev_status)) break;
                bar->sched_item[k] = item;
                mbar_arrive(&bar->sched_full[k]);
                ++it;
                if (rw < 0) break;
                const int bh = rw / nb;
                int prev = -1;
                for (int j = 0; j < item.z && ok; ++j) {
                    int kblk = __ldg(col_idx + item.y + j);
                    if (kblk >= 0 && kblk < nb && kblk > prev) {
                        prev = kblk;
                    } else {
                        record_error(dev_status, FVATTN_ERR_BAD_CSR);
                        kblk = 0;
                    }
                    for (int kv = 0; kv < 2; ++kv) {
                        const uint32_t st = rc % NST;
                        if (!mbar_wait_short(&bar->ring_empty[st], ((rc / NST) & 1) ^ 1, abort_flag, dev_status)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bar->ring_full[st], C::STAGE_BYTES);
                        for (int kb = 0; kb < C::KBLK; ++kb)
                            tma_load_3d(ring + st * C::STAGE_BYTES + kb * BS * 128, kv == 0 ? &tmap_k : &tmap_v,
                                        &bar->ring_full[st], kb * 64, kblk * BS, bh);
                        ++rc;
                    }
                }
            }
            for (uint32_t st = 0; st < static_cast<uint32_t>(NST); ++st) {
                if (rc > st) {
                    const uint32_t times = (rc - st + NST - 1) / NST;
                    mbar_wait_teardown(&bar->ring_full[st], (times - 1) & 1);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t r0 = smem_addr(ring);
            uint32_t it = 0, rc = 0, tc = 0, qn = 0, on = 0;  // items, ring loads, tiles, Q loads, outputs
            bool ok = true;
            auto wait = [&](uint64_t *b, uint32_t parity) {
                if (ok && !mbar_wait_short(b, parity, abort_flag, dev_status)) ok = false;
                return ok;
            };
            // D[dcol] = A[acol] (TMEM, 128 x d) * B^T, B a K-major tile of ring stage st
            auto issue_nt = [&](uint32_t dcol, uint32_t acol, uint32_t st) {
                const uint64_t d0 = smem_desc_sw128(r0 + st * C::STAGE_BYTES, 16, 1024);
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    mma_ts_nc(tmem + dcol, tmem + acol + k * 8, d0 + (((k >> 2) * BS * 128 + (k & 3) * 32) >> 4),
                              C::IDESC_S, k > 0 ? 1u : 0u);
            };
            // dQ (+)= dS K, K of ring stage st read MN-major
            auto issue_dq = [&](uint32_t st, bool first) {
                const uint64_t d0 = smem_desc_sw128(r0 + st * C::STAGE_BYTES, BS * 128, 1024);
                const uint32_t acc0 = first ? 0u : 1u;
#pragma unroll
                for (int k = 0; k < BS / 16; ++k)
                    mma_ts_nc(tmem + C::T_DQ, tmem + C::T_DP + k * 8, d0 + ((k * 16 * 128) >> 4), C::IDESC_Q,
                              k > 0 ? 1u : acc0);
            };
            while (ok) {
                const uint32_t k = it & 1;
                if (!wait(&bar->sched_full[k], (it >> 1) & 1)) break;
                const int4 item = bar->sched_item[k];
                mbar_arrive(&bar->sched_empty[k]);
                ++it;
                if (!item.w) break;
                const int count = item.z;
                if (count == 0) {
                    if (!wait(&bar->dq_empty, (on & 1) ^ 1)) break;
                    mma_commit(&bar->dq_full);
                    ++on;
                    continue;
                }
                if (!wait(&bar->q_full, qn & 1)) break;
                tc_fence_after();
                // S and dP of the first key block
                if (!wait(&bar->ring_full[rc % NST], (rc / NST) & 1)) break;
                issue_nt(C::T_S, C::T_Q, rc % NST);
                mma_commit(&bar->s_full);
                if (!wait(&bar->ring_full[(rc + 1) % NST], ((rc + 1) / NST) & 1)) break;
                issue_nt(C::T_DP, C::T_DO, (rc + 1) % NST);
                mma_commit(&bar->dp_full);
                mma_commit(&bar->ring_empty[(rc + 1) % NST]);  // V read by dP
                for (int j = 0; j < count && ok; ++j) {
                    const uint32_t t = tc + j;
                    const uint32_t kst = (rc + 2 * j) % NST;
                    if (j + 1 < count) {  // S of the next block once the softmax has read this one
                        if (!wait(&bar->s_free, t & 1)) break;
                        const uint32_t ki = rc + 2 * (j + 1);
                        if (!wait(&bar->ring_full[ki % NST], (ki / NST) & 1)) break;
                        tc_fence_after();
                        issue_nt(C::T_S, C::T_Q, ki % NST);
                        mma_commit(&bar->s_full);
                    }
                    if (!wait(&bar->ds_full, t & 1)) break;
                    if (j == 0 && !wait(&bar->dq_empty, (on & 1) ^ 1)) break;
                    tc_fence_after();
                    issue_dq(kst, j == 0);
                    mma_commit(&bar->ring_empty[kst]);  // K read by S and dQ
                    if (j + 1 < count) {  // dP of the next block, after dQ has read dS
                        const uint32_t vi = rc + 2 * (j + 1) + 1;
                        if (!wait(&bar->ring_full[vi % NST], (vi / NST) & 1)) break;
                        issue_nt(C::T_DP, C::T_DO, vi % NST);
                        mma_commit(&bar->dp_full);
                        mma_commit(&bar->ring_empty[vi % NST]);
                    }
                }
                if (!ok) break;
                mma_commit(&bar->dq_full);
                ++on;
                ++qn;
                rc += 2 * static_cast<uint32_t>(count);
                tc += static_cast<uint32_t>(count);
            }
            mma_commit(&bar->drain);
            mbar_wait_teardown(&bar->drain, 0);
        }
    } else {
        // ------------------------------------------------ P, dS and the epilogue (warps 0-3)
        const int r = threadIdx.x;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        uint32_t it = 0, tc = 0, qn = 0, on = 0;
        while (true) {
            const uint32_t k = it & 1;
            if (!mbar_wait_short(&bar->sched_full[k], (it >> 1) & 1, abort_flag, dev_status)) break;
            const int4 item = bar->sched_item[k];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->sched_empty[k]);
            ++it;
            if (!item.w) break;
            const int row = item.x, start = item.y, count = item.z;
            const int64_t bh = row / nb;
            const int t_row = (row % nb) * BS + r;
            const bool row_in = t_row < N;
            const int64_t tok = bh * N + (row_in ? t_row : 0);
            bool ok = true;
            if (count > 0) {
                // Q and dO rows into TMEM (bf16 pairs), zeros past N
                const uint4 *q4 = reinterpret_cast<const uint4 *>(Qg + tok * D);
                const uint4 *g4 = reinterpret_cast<const uint4 *>(dOg + tok * D);
#pragma unroll
                for (int src = 0; src < 2; ++src) {
                    const uint4 *p4 = src ? g4 : q4;
#pragma unroll
                    for (int c0 = 0; c0 < D / 2; c0 += 32) {
                        uint32_t w[32];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const uint4 x = row_in ? __ldg(p4 + c0 / 4 + i) : make_uint4(0, 0, 0, 0);
                            w[4 * i] = x.x;
                            w[4 * i + 1] = x.y;
                            w[4 * i + 2] = x.z;
                            w[4 * i + 3] = x.w;
                        }
                        tmem_st32(tmem + lane_base + (src ? C::T_DO : C::T_Q) + c0, w);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar->q_full);
            }
            // this row's LSE (log2 units; +inf gives P = 0) and D
            const float lse = row_in ? __ldg(LSE + tok) : CUDART_INF_F;
            const float lse2 = (lse == -CUDART_INF_F) ? CUDART_INF_F : lse * kLog2e;
            const float Dt = row_in ? __ldg(Dg + tok) : 0.0f;
            int prev = -1;
            for (int j = 0; j < count; ++j) {
                const int kblk = __ldg(col_idx + start + j);
                const bool valid = kblk >= 0 && kblk < nb && kblk > prev;
                if (valid) prev = kblk;
                const int key0 = kblk * BS;
                int lim = valid ? min(BS, N - key0) : 0;
                if (causal) lim = min(lim, t_row - key0 + 1);
                if (!row_in) lim = 0;
                if (!mbar_wait_short(&bar->s_full, tc & 1, abort_flag, dev_status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // P = exp(S / sqrt(d) - LSE) in fp32, in place
                uint32_t v[BS];
#pragma unroll
                for (int c0 = 0; c0 < BS; c0 += 32)
                    tmem_ld32(tmem + lane_base + C::T_S + c0, *reinterpret_cast<uint32_t(*)[32]>(&v[c0]));
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar->s_free);  // S may be overwritten by the next block
                if (__all_sync(0xffffffffu, lim >= BS)) {
                    // scale-and-shift on fp32 pairs (one instruction per two columns)
                    const uint64_t sc2 = f32x2_pack(scale_log2, scale_log2), nl2 = f32x2_pack(-lse2, -lse2);
#pragma unroll
                    for (int c = 0; c < BS; c += 2) {
                        float x0, x1;
                        f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), sc2, nl2),
                                     x0, x1);
                        v[c] = __float_as_uint(ex2_approx(x0));
                        v[c + 1] = __float_as_uint(ex2_approx(x1));
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < BS; ++c)
                        v[c] = __float_as_uint(c < lim ? ex2_approx(fmaf(__uint_as_float(v[c]), scale_log2, -lse2))
                                                       : 0.0f);
                }
                if (!mbar_wait_short(&bar->dp_full, tc & 1, abort_flag, dev_status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // dS = P (dP - D), as bf16 pairs into the dP columns (two halves of 64 columns)
#pragma unroll
                for (int h0 = 0; h0 < BS; h0 += 64) {
                    uint32_t g[64];
                    tmem_ld32(tmem + lane_base + C::T_DP + h0, *reinterpret_cast<uint32_t(*)[32]>(&g[0]));
                    tmem_ld32(tmem + lane_base + C::T_DP + h0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&g[32]));
                    tmem_wait_ld();
                    uint32_t w[32];
                    const uint64_t d2 = f32x2_pack(Dt, Dt);
#pragma unroll
                    for (int c = 0; c < 64; c += 2) {
                        // on fp32 pairs: (dP - D) and the product with P, one instruction each per two columns
                        float y0, y1;
                        f32x2_unpack(f32x2_mul(f32x2_pack(__uint_as_float(v[h0 + c]), __uint_as_float(v[h0 + c + 1])),
                                               f32x2_sub(f32x2_pack(__uint_as_float(g[c]), __uint_as_float(g[c + 1])),
                                                         d2)),
                                     y0, y1);
                        w[c >> 1] = pack_bf16(y0, y1);
                    }
                    tmem_st32(tmem + lane_base + C::T_DP + h0 / 2, w);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar->ds_full);
                ++tc;
            }
            if (!ok) break;
            if (count > 0) ++qn;
            // epilogue: dQ = (sum over blocks of dS K) / sqrt(d)
            if (!mbar_wait_short(&bar->dq_full, on & 1, abort_flag, dev_status)) break;
            ++on;
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t v[32];
                if (count > 0) {
                    tmem_ld32(tmem + lane_base + C::T_DQ + c0, v);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) v[c] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2)
                    pk[c >> 1] = pack_bf16(__uint_as_float(v[c]) * scale, __uint_as_float(v[c + 1]) * scale);
                if (row_in && r < BS) {
                    uint4 *dst = reinterpret_cast<uint4 *>(dQ + tok * D + c0);
#pragma unroll
                    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->dq_empty);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

namespace {

// ------------------------------------------------------------------- dK, dV
// TMEM columns: S^T (then P^T as bf16 pairs) at 0, dP^T (then dS^T) at 128,
// dK at 256, dV at 384 (fp32).  Shared memory: the item's K and V tiles, then a
// ring of Q / dO tiles, then per-tile LSE and D of the query block (two copies).
template <int D>
struct KvCfg {
    static constexpr int KBLK = D / 64;
    static constexpr int STAGE_BYTES = KBLK * kRowsM * 128;  // one tile
    static constexpr int NST = 4;
    static constexpr int OFF_RING = 2 * STAGE_BYTES;         // K, V of the item first
    static constexpr int OFF_META = OFF_RING + NST * STAGE_BYTES;
    static constexpr int TILE_BYTES = OFF_META + 3 * 2 * kRowsM * 4;
    static constexpr int SMEM_BYTES = TILE_BYTES + 1024 + 512;
    static constexpr uint32_t T_S = 0, T_DP = 128, T_DK = 256, T_DV = 384;
    static constexpr uint32_t IDESC_T = idesc_bf16_f32(kRowsM, kRowsM, 0, 0);  // S^T, dP^T: both K-major
    static constexpr uint32_t IDESC_A = idesc_bf16_f32(kRowsM, D, 0, 1);       // dK, dV: B MN-major
};

struct KvBarriers {
    uint64_t ring_full[4], ring_empty[4];
    uint64_t kv_full, kv_empty, st_full, dpt_full, p_full, ds_full, meta[3], acc_full, acc_empty;
    uint64_t sched_full[2], sched_empty[2];
    uint64_t drain;
    int4 sched_item[2];  // {column (bh*nb + j), list start, count, valid item}
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(KvBarriers) <= 512, "barrier block exceeds its reservation");

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_do,
                const float *__restrict__ LSE, const float *__restrict__ Dg, const int32_t *__restrict__ col_ptr,
                const int32_t *__restrict__ csc_idx, const int32_t *__restrict__ order, int n_items,
                int *__restrict__ work_counter, int N, int nb, int causal, float scale,
                __nv_bfloat16 *__restrict__ dK, __nv_bfloat16 *__restrict__ dV, int32_t *dev_status) {
    using C = KvCfg<D>;
    constexpr int NST = C::NST;
    constexpr int BS = kRowsM;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t base_addr = smem_addr(smem_raw);
    unsigned char *smem = smem_raw + ((1024 - (base_addr & 1023)) & 1023);
    unsigned char *ring = smem + C::OFF_RING;
    float *meta = reinterpret_cast<float *>(smem + C::OFF_META);  // [3 copies][LSE 128 | D 128]
    KvBarriers *bar = reinterpret_cast<KvBarriers *>(smem + C::TILE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_flag = &bar->abort_flag;
    const float scale_log2 = scale * kLog2e;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&bar->ring_full[s], 1);
            mbar_init(&bar->ring_empty[s], 1);
        }
        mbar_init(&bar->kv_full, 1);
        mbar_init(&bar->kv_empty, 1);
        mbar_init(&bar->st_full, 1);
        mbar_init(&bar->dpt_full, 1);
        mbar_init(&bar->p_full, 4);
        mbar_init(&bar->ds_full, 4);
        for (int x = 0; x < 3; ++x) mbar_init(&bar->meta[x], 4);
        mbar_init(&bar->acc_full, 1);
        mbar_init(&bar->acc_empty, 4);
        for (int k = 0; k < 2; ++k) {
            mbar_init(&bar->sched_full[k], 1);
            mbar_init(&bar->sched_empty[k], 1 + 4);
        }
        mbar_init(&bar->drain, 1);
        bar->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&bar->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_q);
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
            prefetch_tensormap(&tmap_do);
            uint32_t it = 0, rc = 0, kn = 0;  // items published, ring loads, K/V loads
            bool ok = true;
            while (ok) {
                const int idx = atomicAdd(work_counter, 1);
                const int cl = (idx < n_items) ? order[idx] : -1;
                int4 item = make_int4(-1, 0, 0, 0);
                if (cl >= 0) item = make_int4(cl, col_ptr[cl], col_ptr[cl + 1] - col_ptr[cl], 1);
                const uint32_t k = it & 1;
                if (!mbar_wait_short(&bar->sched_empty[k], ((it >> 1) & 1) ^ 1, abort_flag, dev_status)) break;
                bar->sched_item[k] = item;
                mbar_arrive(&bar->sched_full[k]);
                ++it;
                if (cl < 0) break;
                if (item.z <= 0) continue;
                const int bh = cl / nb, kblk = cl % nb;
                // the item's K and V tiles, once the previous item's MMAs are done with them
                if (!mbar_wait_short(&bar->kv_empty, (kn & 1) ^ 1, abort_flag, dev_status)) break;
                mbar_arrive_expect_tx(&bar->kv_full, 2 * C::STAGE_BYTES);
                for (int kb = 0; kb < C::KBLK; ++kb) {
                    tma_load_3d(smem + kb * BS * 128, &tmap_k, &bar->kv_full, kb * 64, kblk * BS, bh);
                    tma_load_3d(smem + C::STAGE_BYTES + kb * BS * 128, &tmap_v, &bar->kv_full, kb * 64, kblk * BS,
                                bh);
                }
                ++kn;
                for (int j = 0; j < item.z && ok; ++j) {
                    int qblk = __ldg(csc_idx + item.y + j);
                    if (qblk < 0 || qblk >= nb) {
                        record_error(dev_status, FVATTN_ERR_BAD_CSR);
                        qblk = 0;
                    }
                    for (int kv = 0; kv < 2; ++kv) {
                        const uint32_t st = rc % NST;
                        if (!mbar_wait_short(&bar->ring_empty[st], ((rc / NST) & 1) ^ 1, abort_flag, dev_status)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bar->ring_full[st], C::STAGE_BYTES);
                        for (int kb = 0; kb < C::KBLK; ++kb)
                            tma_load_3d(ring + st * C::STAGE_BYTES + kb * BS * 128, kv == 0 ? &tmap_q : &tmap_do,
                                        &bar->ring_full[st], kb * 64, qblk * BS, bh);
                        ++rc;
                    }
                }
            }
            for (uint32_t st = 0; st < static_cast<uint32_t>(NST); ++st) {
                if (rc > st) {
                    const uint32_t times = (rc - st + NST - 1) / NST;
                    mbar_wait_teardown(&bar->ring_full[st], (times - 1) & 1);
                }
            }
            if (kn > 0) mbar_wait_teardown(&bar->kv_full, (kn - 1) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t k0 = smem_addr(smem), v0 = k0 + C::STAGE_BYTES, r0 = smem_addr(ring);
            uint32_t it = 0, rc = 0, tc = 0, kn = 0, on = 0;
            bool ok = true;
            auto wait = [&](uint64_t *b, uint32_t parity) {
                if (ok && !mbar_wait_short(b, parity, abort_flag, dev_status)) ok = false;
                return ok;
            };
            // D[dcol] = A B^T with A (the item's K or V) and B (a ring tile) both K-major
            auto issue_t = [&](uint32_t dcol, uint32_t a, uint32_t st) {
                const uint64_t a0 = smem_desc_sw128(a, 16, 1024);
                const uint64_t b0 = smem_desc_sw128(r0 + st * C::STAGE_BYTES, 16, 1024);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = ((k >> 2) * BS * 128 + (k & 3) * 32) >> 4;
                    mma_ss_nc(tmem + dcol, a0 + off, b0 + off, C::IDESC_T, k > 0 ? 1u : 0u);
                }
            };
            // acc[dcol] (+)= A[acol] (TMEM, bf16 pairs) B, B a ring tile read MN-major
            auto issue_acc = [&](uint32_t dcol, uint32_t acol, uint32_t st, bool first) {
                const uint64_t b0 = smem_desc_sw128(r0 + st * C::STAGE_BYTES, BS * 128, 1024);
                const uint32_t acc0 = first ? 0u : 1u;
#pragma unroll
                for (int k = 0; k < BS / 16; ++k)
                    mma_ts_nc(tmem + dcol, tmem + acol + k * 8, b0 + ((k * 16 * 128) >> 4), C::IDESC_A,
                              k > 0 ? 1u : acc0);
            };
            while (ok) {
                const uint32_t k = it & 1;
                if (!wait(&bar->sched_full[k], (it >> 1) & 1)) break;
                const int4 item = bar->sched_item[k];
                mbar_arrive(&bar->sched_empty[k]);
                ++it;
                if (!item.w) break;
                const int count = item.z;
                if (count <= 0) {  // a key block no query block selected: zero gradients
                    if (!wait(&bar->acc_empty, (on & 1) ^ 1)) break;
                    mma_commit(&bar->acc_full);
                    ++on;
                    continue;
                }
                if (!wait(&bar->kv_full, kn & 1)) break;
                // S^T and dP^T of the first query block
                if (!wait(&bar->ring_full[rc % NST], (rc / NST) & 1)) break;
                issue_t(C::T_S, k0, rc % NST);
                mma_commit(&bar->st_full);
                if (!wait(&bar->ring_full[(rc + 1) % NST], ((rc + 1) / NST) & 1)) break;
                issue_t(C::T_DP, v0, (rc + 1) % NST);
                mma_commit(&bar->dpt_full);
                for (int j = 0; j < count && ok; ++j) {
                    const uint32_t t = tc + j;
                    const uint32_t qst = (rc + 2 * j) % NST, gst = (rc + 2 * j + 1) % NST;
                    if (!wait(&bar->p_full, t & 1)) break;
                    if (j == 0 && !wait(&bar->acc_empty, (on & 1) ^ 1)) break;
                    tc_fence_after();
                    issue_acc(C::T_DV, C::T_S, gst, j == 0);  // dV += P^T dO
                    mma_commit(&bar->ring_empty[gst]);
                    if (j + 1 < count) {  // S^T of the next block into the columns dV has just read
                        const uint32_t qi = rc + 2 * (j + 1);
                        if (!wait(&bar->ring_full[qi % NST], (qi / NST) & 1)) break;
                        issue_t(C::T_S, k0, qi % NST);
                        mma_commit(&bar->st_full);
                    }
                    if (!wait(&bar->ds_full, t & 1)) break;
                    tc_fence_after();
                    issue_acc(C::T_DK, C::T_DP, qst, j == 0);  // dK += dS^T Q
                    mma_commit(&bar->ring_empty[qst]);
                    if (j + 1 < count) {  // dP^T of the next block after dK has read dS^T
                        const uint32_t gi = rc + 2 * (j + 1) + 1;
                        if (!wait(&bar->ring_full[gi % NST], (gi / NST) & 1)) break;
                        issue_t(C::T_DP, v0, gi % NST);
                        mma_commit(&bar->dpt_full);
                    }
                }
                if (!ok) break;
                mma_commit(&bar->kv_empty);  // K and V of this item read by every MMA above
                mma_commit(&bar->acc_full);
                ++on;
                ++kn;
                rc += 2 * static_cast<uint32_t>(count);
                tc += static_cast<uint32_t>(count);
            }
            mma_commit(&bar->drain);
            mbar_wait_teardown(&bar->drain, 0);
        }
    } else {
        // ------------------------------------------------ P^T, dS^T and the epilogue (warps 0-3)
        const int r = threadIdx.x;  // key row of the item's block
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        uint32_t it = 0, tc = 0, on = 0;
        while (true) {
            const uint32_t k = it & 1;
            if (!mbar_wait_short(&bar->sched_full[k], (it >> 1) & 1, abort_flag, dev_status)) break;
            const int4 item = bar->sched_item[k];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->sched_empty[k]);
            ++it;
            if (!item.w) break;
            const int cl = item.x, start = item.y, count = item.z > 0 ? item.z : 0;
            const int64_t bh = cl / nb;
            const int ku = (cl % nb) * BS + r;  // this thread's key token
            const bool key_in = ku < N;
            bool ok = true;
            // The negated LSE (log2 units, -inf past N) and D of the item's query block jj, the
            // CTA's tile number tt, go into shared copy tt % 3 one tile ahead, shared by
            // the four warps (three copies: a warp can run one tile ahead of the others).
            auto stage_meta = [&](int jj, uint32_t tt) {
                const int qb = __ldg(csc_idx + start + jj);
                float *mt = meta + (tt % 3) * 2 * BS;
                const int tq = qb * BS + r;
                const bool qin = qb >= 0 && qb < nb && tq < N;
                const float lse = qin ? __ldg(LSE + bh * N + tq) : CUDART_INF_F;
                mt[r] = (lse == -CUDART_INF_F) ? -CUDART_INF_F : -(lse * kLog2e);  // -LSE, log2 units
                mt[BS + r] = qin ? __ldg(Dg + bh * N + tq) : 0.0f;
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar->meta[tt % 3]);
            };
            if (count > 0) stage_meta(0, tc);
            for (int j = 0; j < count; ++j) {
                const int qblk = __ldg(csc_idx + start + j);
                const int q0 = qblk * BS;
                const float *mt = meta + (tc % 3) * 2 * BS;
                // queries of this block that exist (and, causal, come at or after the key)
                int lo = 0, hi = min(BS, N - q0);  // allowed columns: [lo, hi)
                if (causal) lo = max(0, ku - q0);
                if (!key_in || qblk < 0 || qblk >= nb) hi = 0;
                if (!mbar_wait_short(&bar->st_full, tc & 1, abort_flag, dev_status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t v[BS];
#pragma unroll
                for (int c0 = 0; c0 < BS; c0 += 32)
                    tmem_ld32(tmem + lane_base + C::T_S + c0, *reinterpret_cast<uint32_t(*)[32]>(&v[c0]));
                if (!mbar_wait_short(&bar->meta[tc % 3], (tc / 3) & 1, abort_flag, dev_status)) {
                    ok = false;
                    break;
                }
                tmem_wait_ld();
                // P^T = exp(S^T / sqrt(d) - LSE), packed in place as bf16 pairs: v[c/2] <- (p[c], p[c+1])
                if (__all_sync(0xffffffffu, lo == 0 && hi == BS)) {
                    // scale-and-shift on fp32 pairs (one instruction per two columns)
                    const uint64_t sc2 = f32x2_pack(scale_log2, scale_log2);
#pragma unroll
                    for (int c = 0; c < BS; c += 4) {
                        const float4 l4 = *reinterpret_cast<const float4 *>(mt + c);
                        float x0, x1, x2, x3;
                        f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), sc2,
                                               f32x2_pack(l4.x, l4.y)),
                                     x0, x1);
                        f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(v[c + 2]), __uint_as_float(v[c + 3])), sc2,
                                               f32x2_pack(l4.z, l4.w)),
                                     x2, x3);
                        v[c >> 1] = pack_bf16(ex2_approx(x0), ex2_approx(x1));
                        v[(c >> 1) + 1] = pack_bf16(ex2_approx(x2), ex2_approx(x3));
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < BS; c += 2) {
                        const float p0 = (c >= lo && c < hi)
                                             ? ex2_approx(fmaf(__uint_as_float(v[c]), scale_log2, mt[c])) : 0.0f;
                        const float p1 = (c + 1 >= lo && c + 1 < hi)
                                             ? ex2_approx(fmaf(__uint_as_float(v[c + 1]), scale_log2, mt[c + 1]))
                                             : 0.0f;
                        v[c >> 1] = pack_bf16(p0, p1);
                    }
                }
                // P^T into the S^T columns, for dV += P^T dO
#pragma unroll
                for (int c0 = 0; c0 < BS / 2; c0 += 32)
                    tmem_st32(tmem + lane_base + C::T_S + c0, *reinterpret_cast<const uint32_t(*)[32]>(&v[c0]));
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar->p_full);
                // the next block's LSE and D while the tensor cores work
                if (j + 1 < count) stage_meta(j + 1, tc + 1);
                if (!mbar_wait_short(&bar->dpt_full, tc & 1, abort_flag, dev_status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // dS^T = P^T (dP^T - D) with P^T in bf16, packed into the dP^T columns
                uint32_t g[BS];
#pragma unroll
                for (int c0 = 0; c0 < BS; c0 += 32)
                    tmem_ld32(tmem + lane_base + C::T_DP + c0, *reinterpret_cast<uint32_t(*)[32]>(&g[c0]));
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < BS; c += 4) {
                    // on fp32 pairs: (dP^T - D) and the product with P^T, one instruction each per two columns
                    const float4 d4 = *reinterpret_cast<const float4 *>(mt + BS + c);
                    const uint32_t pa = v[c >> 1], pb = v[(c >> 1) + 1];
                    float y0, y1, y2, y3;
                    f32x2_unpack(f32x2_mul(f32x2_pack(__uint_as_float(pa << 16), __uint_as_float(pa & 0xFFFF0000u)),
                                           f32x2_sub(f32x2_pack(__uint_as_float(g[c]), __uint_as_float(g[c + 1])),
                                                     f32x2_pack(d4.x, d4.y))),
                                 y0, y1);
                    f32x2_unpack(f32x2_mul(f32x2_pack(__uint_as_float(pb << 16), __uint_as_float(pb & 0xFFFF0000u)),
                                           f32x2_sub(f32x2_pack(__uint_as_float(g[c + 2]), __uint_as_float(g[c + 3])),
                                                     f32x2_pack(d4.z, d4.w))),
                                 y2, y3);
                    g[c >> 1] = pack_bf16(y0, y1);
                    g[(c >> 1) + 1] = pack_bf16(y2, y3);
                }
#pragma unroll
                for (int c0 = 0; c0 < BS / 2; c0 += 32)
                    tmem_st32(tmem + lane_base + C::T_DP + c0, *reinterpret_cast<const uint32_t(*)[32]>(&g[c0]));
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar->ds_full);
                ++tc;
            }
            if (!ok) break;
            // epilogue: dK = (sum of dS^T Q) / sqrt(d), dV = sum of P^T dO
            if (!mbar_wait_short(&bar->acc_full, on & 1, abort_flag, dev_status)) break;
            ++on;
            tc_fence_after();
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const float f = which == 0 ? scale : 1.0f;
                __nv_bfloat16 *dst_row = (which == 0 ? dK : dV) + (bh * N + (key_in ? ku : 0)) * D;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t v[32];
                    if (count > 0) {
                        tmem_ld32(tmem + lane_base + (which == 0 ? C::T_DK : C::T_DV) + c0, v);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c) v[c] = 0u;
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 32; c += 2)
                        pk[c >> 1] = pack_bf16(__uint_as_float(v[c]) * f, __uint_as_float(v[c + 1]) * f);
                    if (key_in) {
                        uint4 *dst = reinterpret_cast<uint4 *>(dst_row + c0);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->acc_empty);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

// ------------------------------------------------------------------ launchers

int bwd_dq_smem_bytes(int d) { return d == 128 ? DqCfg<128>::SMEM_BYTES : DqCfg<64>::SMEM_BYTES; }
int bwd_dkdv_smem_bytes(int d) { return d == 128 ? KvCfg<128>::SMEM_BYTES : KvCfg<64>::SMEM_BYTES; }

cudaError_t launch_bwd_rowdot(const void *O, const void *dO, int64_t tokens, int d, float *D, cudaStream_t stream) {
    const int64_t blocks = (tokens + 7) / 8;  // 8 warps per CTA, one token per warp
    const int grid = static_cast<int>(blocks < 8192 ? blocks : 8192);
    bwd_rowdot_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint16_t *>(O), static_cast<const uint16_t *>(dO),
                                                tokens, d, D);
    return cudaGetLastError();
}

cudaError_t launch_csc(const int32_t *row_ptr, const int32_t *col_idx, int64_t BH, int nb, int32_t *col_ptr,
                       int32_t *csc_idx, int32_t *dev_status, cudaStream_t stream) {
    csc_kernel<<<static_cast<unsigned>(BH), 1024, static_cast<size_t>(nb) * sizeof(int), stream>>>(
        row_ptr, col_idx, nb, col_ptr, csc_idx, dev_status);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_dq_t(const BwdLaunch &a, cudaStream_t stream) {
    auto kern = dq_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DqCfg<D>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<a.grid, kThreads, DqCfg<D>::SMEM_BYTES, stream>>>(
        *a.tmap_k, *a.tmap_v, static_cast<const __nv_bfloat16 *>(a.Q), static_cast<const __nv_bfloat16 *>(a.dO),
        a.LSE, a.D, a.row_ptr, a.col_idx, a.order_q, a.n_items, a.counters, a.N, a.nb, a.causal, a.scale,
        static_cast<__nv_bfloat16 *>(a.dQ), a.dev_status);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_dkdv_t(const BwdLaunch &a, cudaStream_t stream) {
    auto kern = dkdv_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, KvCfg<D>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<a.grid, kThreads, KvCfg<D>::SMEM_BYTES, stream>>>(
        *a.tmap_q, *a.tmap_k, *a.tmap_v, *a.tmap_do, a.LSE, a.D, a.col_ptr, a.csc_idx, a.order_k, a.n_items,
        a.counters + 1, a.N, a.nb, a.causal, a.scale, static_cast<__nv_bfloat16 *>(a.dK),
        static_cast<__nv_bfloat16 *>(a.dV), a.dev_status);
    return cudaGetLastError();
}

cudaError_t launch_bwd_dq(const BwdLaunch &a, int d, cudaStream_t stream) {
    return d == 128 ? launch_dq_t<128>(a, stream) : launch_dq_t<64>(a, stream);
}

cudaError_t launch_bwd_dkdv(const BwdLaunch &a, int d, cudaStream_t stream) {
    return d == 128 ? launch_dkdv_t<128>(a, stream) : launch_dkdv_t<64>(a, stream);
}

}  // namespace fvattn
