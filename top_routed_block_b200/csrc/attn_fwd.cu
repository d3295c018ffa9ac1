// attn_fwd.cu -- block-sparse exact attention forward on sm_100a tensor cores.
//
// What it computes (FlashAttention review, §Background "Motivation" and §Model):
// for every query token, softmax(q.K^T/sqrt(d)) V over the key tokens of the
// key blocks its query block selected (FVAttn review, §1 "Top-p routing"),
// without writing S or P to memory, one fused kernel, tiled matmuls and the
// tiled ("online") softmax: a running row maximum m and row sum l, with the
// partial output rescaled by exp(m_old - m_new) whenever the maximum grows.
//
// B200 design:
//   * One work item = one CSR row = one (b, h, query block).  A persistent grid
//     of 2 CTAs per SM pops items from a longest-first queue (FVAttn §1 "RLB"
//     balances per-head work at run time; here the SMs are balanced instead).
//   * Per CTA, 10 warps: warps 0-7 run the softmax, rescale and epilogue of the
//     128-row query tile, two warps per row (warp w and w+4 address the same 32
//     TMEM lanes and take the lower and upper half of the key columns; only the
//     row maximum is exchanged, through shared memory, once per tile); warp 8
//     issues TMA loads; warp 9 issues tcgen05 MMAs.
//   * Q, K, V tiles arrive by TMA (3-D tensor maps over [B*H, N, d], 128-byte
//     swizzle, out-of-range rows zero-filled).  K/V tiles are gathered by the
//     CSR's column indices.
//   * S = Q K^T accumulates in tensor memory (TMEM) in fp32 (SS MMA, M=128,
//     N=block, K=16 steps over d).  The softmax warps read S with tcgen05.ld,
//     write P as bf16 back into the first half of the S columns each of them
//     read, and O += P V runs as a TS MMA with P taken from TMEM and V from
//     shared memory (MN-major).  The next S is issued right behind the PV:
//     tcgen05 MMAs of one thread execute in issue order, so the PV has read P
//     before S overwrites those columns.
//   * O (fp32) stays in TMEM for the whole item; the epilogue divides by l,
//     converts to bf16 and stores; LSE = (m + log2 l) ln 2.
//   * Every mbarrier wait is bounded; a timeout raises the CTA abort flag and
//     records FVATTN_ERR_DEVICE_TIMEOUT; all roles then drain and exit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <math_constants.h>

#include "attn_fwd.cuh"
#include "common.cuh"
#include "ptx_sm100.cuh"

namespace fvattn {

namespace {

using namespace ptx;

constexpr int kRowsM = 128;           // query rows per tile (tcgen05 M)
constexpr int kSoftmaxWarps = 8;      // two per 32-row lane group
constexpr int kThreads = 320;         // 8 softmax warps + TMA warp + MMA warp
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 256;   // per CTA; two CTAs share an SM's 512 columns
constexpr uint32_t kTmemS = 0;        // S (fp32, block columns) / P (bf16 pairs, block/2 columns)
constexpr uint32_t kTmemO = 128;      // O (fp32, d columns)
// S_{j+1} is written into the TMEM columns that hold P_j.  tcgen05 MMAs issued by
// one thread run in issue order, so S_{j+1} may be queued right behind PV_j; with
// this set the MMA warp instead waits for PV_j to complete first.
constexpr bool kWaitPvBeforeS = false;

template <int D, int BS>
struct Cfg {
    static constexpr int KBLK = D / 64;                 // 128-byte (64 x bf16) column blocks along d
    static constexpr int Q_BYTES = KBLK * kRowsM * 128;
    static constexpr int KV_BYTES = KBLK * BS * 128;
    static constexpr int Q_LOAD_BYTES = KBLK * BS * 128;  // only the block's rows are loaded
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = Q_BYTES;
    static constexpr int OFF_V = Q_BYTES + KV_BYTES;
    static constexpr int TILE_BYTES = Q_BYTES + 2 * KV_BYTES;
    // row-max exchange between the two warps of a lane group: buffers 0/1 alternate
    // by tile, buffers 2/3 by item (row sums at the epilogue); each [2 halves][rows]
    static constexpr int XCHG_BYTES = 4 * 2 * kRowsM * 4;
    static constexpr int SMEM_BYTES = TILE_BYTES + 1024 /*align slack*/ + 256 /*barriers etc*/ + XCHG_BYTES;
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(kRowsM, BS, 0, 0);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(kRowsM, D, 0, 1);
};

struct Barriers {
    uint64_t q_full, q_empty, k_full, k_empty, v_full, v_empty, s_full, p_full, o_full, o_empty, pv_done;
    uint64_t sched_full[2], sched_empty[2];
    uint64_t drain;
    int4 sched_item[2];   // {row, col start, count, valid}
    uint32_t tmem_base;
    int abort_flag;
};

constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the row max grows by more than 2^8

// 2^x on the MUFU unit (flushes subnormal results to zero; exp2(-inf) = 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA pipe, for finite x: x = n + f with n = round(x) and f in [-1/2, 1/2];
// 2^f by a cubic fitted here for least maximum relative error on [-1/2, 1/2]
// (iteratively reweighted least squares on Chebyshev nodes; max relative error
// 7.5e-5, far below the 2^-9 rounding of the bf16 P it feeds); 2^n is added to
// the exponent field.  x is clamped at -126, so results below 2^-126 are not
// exact (they are then under 1.2e-38).  Adding 1.5*2^23 rounds x to an integer
// held in the low mantissa bits of t, whose bit pattern shifted left by 23 is
// n in the exponent field.
constexpr float kExp2C0 = 0.99992806f, kExp2C1 = 0.69326097f, kExp2C2 = 0.24261114f, kExp2C3 = 0.05517167f;

__device__ __forceinline__ float ex2_poly(float x) {
    x = fmaxf(x, -126.0f);
    const float t = __fadd_rn(x, 12582912.0f);
    const float f = __fsub_rn(x, __fsub_rn(t, 12582912.0f));
    const float p = fmaf(fmaf(fmaf(kExp2C3, f, kExp2C2), f, kExp2C1), f, kExp2C0);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Of every 8 exponentials of a full (unmasked) block, this many run as ex2_poly on
// the FMA pipe instead of the MUFU unit, whose throughput otherwise equals the MMA
// time per tile.
constexpr int kPolyOf8 = 0;

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Named barrier for the two warps that share a lane group (ids 1..4; 0 is __syncthreads).
__device__ __forceinline__ void pair_sync(int group) {
    asm volatile("bar.sync %0, 64;" ::"r"(group + 1) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <int D, int BS>
__global__ void __launch_bounds__(kThreads, 2)
    sparse_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                           const __grid_constant__ CUtensorMap tmap_v, const int32_t *__restrict__ row_ptr,
                           const int32_t *__restrict__ col_idx, const int32_t *__restrict__ order, int n_items,
                           int *__restrict__ work_counter, int N, int nb, int causal, float scale_log2,
                           __nv_bfloat16 *__restrict__ O, float *__restrict__ LSE, int32_t *dev_status,
                           int test_stall) {
    using C = Cfg<D, BS>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzled tiles
    const uint32_t base_addr = smem_addr(smem_raw);
    unsigned char *smem = smem_raw + ((1024 - (base_addr & 1023)) & 1023);
    unsigned char *sQ = smem + C::OFF_Q;
    unsigned char *sK = smem + C::OFF_K;
    unsigned char *sV = smem + C::OFF_V;
    Barriers *bar = reinterpret_cast<Barriers *>(smem + C::TILE_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abort_flag = &bar->abort_flag;

    if (threadIdx.x == 0) {
        mbar_init(&bar->q_full, 1);
        mbar_init(&bar->q_empty, 1);
        mbar_init(&bar->k_full, 1);
        mbar_init(&bar->k_empty, 1);
        mbar_init(&bar->v_full, 1);
        mbar_init(&bar->v_empty, 1);
        mbar_init(&bar->s_full, 1);
        mbar_init(&bar->p_full, kSoftmaxWarps);
        mbar_init(&bar->o_full, 1);
        mbar_init(&bar->o_empty, kSoftmaxWarps);
        mbar_init(&bar->pv_done, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar->sched_full[i], 1);
            mbar_init(&bar->sched_empty[i], 1 + kSoftmaxWarps);
        }
        mbar_init(&bar->drain, 1);
        bar->abort_flag = 0;
        fence_barrier_init();
    }
    // Q rows beyond the block (block size 64) are never loaded: keep them zero.
    if (BS < kRowsM) {
        for (int kb = 0; kb < C::KBLK; ++kb) {
            uint4 *z = reinterpret_cast<uint4 *>(sQ + kb * kRowsM * 128 + BS * 128);
            for (int i = threadIdx.x; i < (kRowsM - BS) * 128 / 16; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
            uint32_t it = 0, kc = 0, vc = 0;
            uint32_t q_armed = 0;
            bool ok = true;
            while (ok) {
                const int idx = atomicAdd(work_counter, 1);
                const int row = (idx < n_items) ? order[idx] : -1;
                int start = 0, count = 0;
                if (row >= 0) {
                    start = row_ptr[row];
                    count = row_ptr[row + 1] - start;
                    if (count < 0) {
                        record_error(dev_status, FVATTN_ERR_BAD_CSR);
                        count = 0;
                    }
                }
                const uint32_t slot = it & 1;
                if (!mbar_wait(&bar->sched_empty[slot], ((it >> 1) & 1) ^ 1, abort_flag, dev_status)) break;
                bar->sched_item[slot] = make_int4(row, start, count, row >= 0);
                mbar_arrive(&bar->sched_full[slot]);
                if (row < 0) break;
                const int bh = row / nb;
                const int qb = row % nb;
                if (!mbar_wait(&bar->q_empty, (it & 1) ^ 1, abort_flag, dev_status)) break;
                // Test hook: CTA 0 leaves the Q tile of its first item unloaded, so the
                // MMA warp's bounded wait for it runs out (exercises the timeout path).
                if (!(test_stall && blockIdx.x == 0 && it == 0)) {
                    mbar_arrive_expect_tx(&bar->q_full, C::Q_LOAD_BYTES);
                    for (int kb = 0; kb < C::KBLK; ++kb)
                        tma_load_3d(sQ + kb * kRowsM * 128, &tmap_q, &bar->q_full, kb * 64, qb * BS, bh);
                    q_armed = it + 1;
                }
                int prev = -1;
                for (int j = 0; j < count && ok; ++j) {
                    int kblk = col_idx[start + j];
                    if (kblk < 0 || kblk >= nb || kblk <= prev) {
                        record_error(dev_status, FVATTN_ERR_BAD_CSR);
                        kblk = 0;  // load a valid tile; the softmax masks it out
                    } else {
                        prev = kblk;
                    }
                    if (!mbar_wait(&bar->k_empty, (kc & 1) ^ 1, abort_flag, dev_status)) { ok = false; break; }
                    mbar_arrive_expect_tx(&bar->k_full, C::KV_BYTES);
                    for (int kb = 0; kb < C::KBLK; ++kb)
                        tma_load_3d(sK + kb * BS * 128, &tmap_k, &bar->k_full, kb * 64, kblk * BS, bh);
                    ++kc;
                    if (!mbar_wait(&bar->v_empty, (vc & 1) ^ 1, abort_flag, dev_status)) { ok = false; break; }
                    mbar_arrive_expect_tx(&bar->v_full, C::KV_BYTES);
                    for (int kb = 0; kb < C::KBLK; ++kb)
                        tma_load_3d(sV + kb * BS * 128, &tmap_v, &bar->v_full, kb * 64, kblk * BS, bh);
                    ++vc;
                }
                ++it;
            }
            // wait for every load this thread issued to land before the CTA exits
            if (q_armed > 0) mbar_wait_teardown(&bar->q_full, (q_armed - 1) & 1);
            if (kc > 0) mbar_wait_teardown(&bar->k_full, (kc - 1) & 1);
            if (vc > 0) mbar_wait_teardown(&bar->v_full, (vc - 1) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t tS = tmem + kTmemS;
            const uint32_t tO = tmem + kTmemO;
            const uint32_t q0 = smem_addr(sQ), k0 = smem_addr(sK), v0 = smem_addr(sV);
            uint32_t it = 0, kc = 0, vc = 0, pc = 0;
            uint32_t pv_issued = 0, pv_seen = 0;  // P lives in S's columns: S_{j+1} waits for PV_j
            bool ok = true;
            while (ok) {
                const uint32_t slot = it & 1;
                if (!mbar_wait(&bar->sched_full[slot], (it >> 1) & 1, abort_flag, dev_status)) break;
                const int4 item = bar->sched_item[slot];
                mbar_arrive(&bar->sched_empty[slot]);
                if (!item.w) break;
                const int count = item.z;
                if (!mbar_wait(&bar->q_full, it & 1, abort_flag, dev_status)) break;
                for (int j = 0; j < count; ++j) {
                    // S = Q K_j^T
                    if (!mbar_wait(&bar->k_full, kc & 1, abort_flag, dev_status)) { ok = false; break; }
                    if (kWaitPvBeforeS && pv_issued > pv_seen) {
                        if (!mbar_wait(&bar->pv_done, pv_seen & 1, abort_flag, dev_status)) { ok = false; break; }
                        pv_seen = pv_issued;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t kb = k >> 2, ko = (k & 3) * 32;
                        const uint64_t da = smem_desc_sw128(q0 + kb * kRowsM * 128 + ko, 16, 1024);
                        const uint64_t db = smem_desc_sw128(k0 + kb * BS * 128 + ko, 16, 1024);
                        mma_ss(tS, da, db, C::IDESC_S, k > 0 ? 1u : 0u);
                    }
                    mma_commit(&bar->k_empty);
                    if (j == count - 1) mma_commit(&bar->q_empty);
                    mma_commit(&bar->s_full);
                    ++kc;
                    // O += P_j V_j once the softmax has written P_j (and rescaled O)
                    if (!mbar_wait(&bar->p_full, pc & 1, abort_flag, dev_status)) { ok = false; break; }
                    ++pc;
                    if (j == 0 && !mbar_wait(&bar->o_empty, (it & 1) ^ 1, abort_flag, dev_status)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(&bar->v_full, vc & 1, abort_flag, dev_status)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < BS / 16; ++k) {
                        // keys [16k, 16k+16): P of column half h sits at h*BS/2, packed in pairs
                        const uint32_t pcol = 8 * k + (k / (BS / 32)) * (BS / 4);
                        const uint64_t dv = smem_desc_sw128(v0 + k * 16 * 128, BS * 128, 1024);
                        mma_ts(tO, tS + pcol, dv, C::IDESC_PV, (j > 0 || k > 0) ? 1u : 0u);
                    }
                    mma_commit(&bar->v_empty);
                    mma_commit(&bar->pv_done);
                    ++pv_issued;
                    ++vc;
                }
                if (!ok) break;
                if (count == 0) {
                    mma_commit(&bar->q_empty);
                    if (!mbar_wait(&bar->o_empty, (it & 1) ^ 1, abort_flag, dev_status)) break;
                }
                mma_commit(&bar->o_full);
                ++it;
            }
            // every MMA issued by this thread completes before TMEM is released
            mma_commit(&bar->drain);
            mbar_wait_teardown(&bar->drain, 0);
        }
    } else {
        // ------------------------------------------------ softmax / epilogue
        // warp w: rows 32*(w%4) .. +31 (its TMEM lane quarter), key columns of half
        // h = w/4; the two warps of a lane group exchange their row maxima.
        constexpr int HALF = BS / 2;               // S columns per warp
        constexpr int OHALF = D / 2;               // O columns per warp
        const int g = warp & 3, h = warp >> 2;
        const int r = g * 32 + lane;                               // tile row = TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(g * 32) << 16;
        const uint32_t tS = tmem + kTmemS + lane_base + h * HALF;  // this warp's S columns; P goes
                                                                   // to the first HALF/2 of them
        const uint32_t tO = tmem + kTmemO + lane_base + h * OHALF;
        float *xchg = reinterpret_cast<float *>(smem + C::TILE_BYTES + 256);  // [4][2][kRowsM]
        uint32_t it = 0, sc = 0;
        while (true) {
            const uint32_t slot = it & 1;
            if (!mbar_wait(&bar->sched_full[slot], (it >> 1) & 1, abort_flag, dev_status)) break;
            const int4 item = bar->sched_item[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->sched_empty[slot]);
            if (!item.w) break;
            const int row = item.x, start = item.y, count = item.z;
            const int64_t bh = row / nb;
            const int qb = row % nb;
            const int t_row = qb * BS + r;                         // token index of this thread's row
            float m = -CUDART_INF_F, l = 0.0f;                     // l: this half's share of the row sum
            int prev = -1;
            bool ok = true;
            for (int j = 0; j < count; ++j) {
                int kblk = col_idx[start + j];
                const bool valid = kblk >= 0 && kblk < nb && kblk > prev;
                if (valid) prev = kblk;
                const int key0 = kblk * BS;
                // keys of this block that exist and are allowed for this row, counted
                // from the start of this warp's column half
                int lim = valid ? min(BS, N - key0) : 0;
                if (causal) lim = min(lim, t_row - key0 + 1);
                lim -= h * HALF;
                if (!mbar_wait(&bar->s_full, sc & 1, abort_flag, dev_status)) { ok = false; break; }
                ++sc;
                tc_fence_after();
                uint32_t v[HALF];
#pragma unroll
                for (int c0 = 0; c0 < HALF; c0 += 32)
                    tmem_ld32(tS + c0, *reinterpret_cast<uint32_t(*)[32]>(&v[c0]));
                tmem_wait_ld();
                if (lim < HALF) {  // ragged last block, causal diagonal, or a skipped index
#pragma unroll
                    for (int c = 0; c < HALF; ++c)
                        if (c >= lim) v[c] = __float_as_uint(-CUDART_INF_F);
                }
                float mq[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
                for (int c = 0; c < HALF; c += 8) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        mq[q] = max3f(mq[q], __uint_as_float(v[c + 2 * q]), __uint_as_float(v[c + 2 * q + 1]));
                }
                const float mine = max3f(mq[0], mq[1], fmaxf(mq[2], mq[3]));
                float *xb = xchg + (j & 1) * 2 * kRowsM;
                xb[h * kRowsM + r] = mine;
                pair_sync(g);
                const float mxs = fmaxf(mine, xb[(1 - h) * kRowsM + r]) * scale_log2;
                // The reference maximum only moves when the row maximum exceeds it by
                // more than 2^8: P stays below 256 and the rescale of O is rare.  O and
                // l always share the same reference, so the final O / l is exact.  Both
                // warps of a row take the same decision from the same values.
                const bool need = mxs > m + kRescaleLog2;
                const float m_new = need ? mxs : m;
                const float alpha = need ? ex2_approx(m - m_new) : 1.0f;
                const float neg_m = (m_new == -CUDART_INF_F) ? 0.0f : -m_new;
                float rs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                // P packed as bf16 pairs in place: v[c/2] <- (p[c], p[c+1])
                if (lim >= HALF) {
#pragma unroll
                    for (int c = 0; c < HALF; c += 2) {
                        const float x0 = fmaf(__uint_as_float(v[c]), scale_log2, neg_m);
                        const float x1 = fmaf(__uint_as_float(v[c + 1]), scale_log2, neg_m);
                        const float p0 = ((c & 7) >= 8 - kPolyOf8) ? ex2_poly(x0) : ex2_approx(x0);
                        const float p1 = ((c & 7) + 1 >= 8 - kPolyOf8) ? ex2_poly(x1) : ex2_approx(x1);
                        rs[(c >> 1) & 3] += p0 + p1;
                        v[c >> 1] = pack_bf16(p0, p1);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < HALF; c += 2) {
                        const float p0 = ex2_approx(fmaf(__uint_as_float(v[c]), scale_log2, neg_m));
                        const float p1 = ex2_approx(fmaf(__uint_as_float(v[c + 1]), scale_log2, neg_m));
                        rs[(c >> 1) & 3] += p0 + p1;
                        v[c >> 1] = pack_bf16(p0, p1);
                    }
                }
                if constexpr (HALF / 2 >= 32) {
#pragma unroll
                    for (int c0 = 0; c0 < HALF / 2; c0 += 32)
                        tmem_st32(tS + c0, *reinterpret_cast<const uint32_t(*)[32]>(&v[c0]));
                } else {
                    tmem_st16(tS, *reinterpret_cast<const uint32_t(*)[16]>(&v[0]));
                }
                l = l * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
                // rescale this warp's half of the running output (PV_{j-1} has completed:
                // the S_j commit tracks every earlier MMA of this CTA)
                if (__any_sync(0xffffffffu, need && j > 0)) {
#pragma unroll
                    for (int c0 = 0; c0 < OHALF; c0 += 32) {
                        uint32_t o[32];
                        tmem_ld32(tO + c0, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                        tmem_st32(tO + c0, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar->p_full);
                m = m_new;
            }
            if (!ok) break;
            // epilogue: row sum = both halves' shares
            float *xl = xchg + (2 + (it & 1)) * 2 * kRowsM;
            xl[h * kRowsM + r] = l;
            pair_sync(g);
            const float lsum = l + xl[(1 - h) * kRowsM + r];
            if (!mbar_wait(&bar->o_full, it & 1, abort_flag, dev_status)) break;
            tc_fence_after();
            const bool row_ok = r < BS && t_row < N;
            const float inv_l = (lsum > 0.0f) ? 1.0f / lsum : 0.0f;
            __nv_bfloat16 *orow = O + (bh * N + t_row) * D + h * OHALF;
#pragma unroll
            for (int c0 = 0; c0 < OHALF; c0 += 32) {
                uint32_t v[32];
                if (count > 0) {
                    tmem_ld32(tO + c0, v);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) v[c] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2)
                    pk[c >> 1] = pack_bf16(__uint_as_float(v[c]) * inv_l, __uint_as_float(v[c + 1]) * inv_l);
                if (row_ok) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c0);
#pragma unroll
                    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
            }
            if (row_ok && h == 0)
                LSE[bh * N + t_row] = (lsum > 0.0f) ? (m + __log2f(lsum)) * 0.69314718055994531f : -CUDART_INF_F;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->o_empty);
            ++it;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

// ------------------------------------------------------------------ launcher

int attn_smem_bytes(int d, int bs) {
    if (d == 128 && bs == 128) return Cfg<128, 128>::SMEM_BYTES;
    if (d == 128 && bs == 64) return Cfg<128, 64>::SMEM_BYTES;
    if (d == 64 && bs == 128) return Cfg<64, 128>::SMEM_BYTES;
    return Cfg<64, 64>::SMEM_BYTES;
}

template <int D, int BS>
static cudaError_t launch_t(const AttnLaunch &a, cudaStream_t stream) {
    auto kern = sparse_attn_fwd_kernel<D, BS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D, BS>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<a.grid, kThreads, Cfg<D, BS>::SMEM_BYTES, stream>>>(
        *a.tmap_q, *a.tmap_k, *a.tmap_v, a.row_ptr, a.col_idx, a.order, a.n_items, a.work_counter, a.N, a.nb,
        a.causal, a.scale_log2, static_cast<__nv_bfloat16 *>(a.O), a.LSE, a.dev_status, a.test_stall);
    return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const AttnLaunch &a, int d, int bs, cudaStream_t stream) {
    if (d == 128 && bs == 128) return launch_t<128, 128>(a, stream);
    if (d == 128 && bs == 64) return launch_t<128, 64>(a, stream);
    if (d == 64 && bs == 128) return launch_t<64, 128>(a, stream);
    return launch_t<64, 64>(a, stream);
}

}  // namespace fvattn
namespace fvattn { int attn_ctas_per_sm() { return 2; } }
