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
//   * One work item = two neighbouring query blocks (2i, 2i+1) of one head:
//     slots A and B, each with its own CSR row.  Top-p routing gives
//     neighbouring query blocks mostly the same key blocks, so the item walks
//     the merge of the two sorted block lists and loads every key block of the
//     union once; a block selected by only one of the rows is computed for that
//     row only (no wasted tensor-core work).  A persistent grid of one CTA per
//     SM pops items longest-first (FVAttn §1 "RLB" balances per-head work at
//     run time; here the SMs are balanced instead).
//   * Warps 0-3 run the softmax, rescale and epilogue of slot A, warps 4-7 those
//     of slot B (thread = query row = TMEM lane); warp 8 issues TMA loads; warp
//     9 issues tcgen05 MMAs; warps 10-11 complete the third warpgroup.  That
//     warpgroup hands registers to the softmax warpgroups (setmaxnreg), which
//     keep a whole 128-column S row per thread without spilling.  Per union
//     block the MMA warp issues
//     S_A, PV_B(previous B block), S_B, PV_A: while one warpgroup runs the
//     softmax of its tile, the tensor cores run the other slot's two GEMMs.
//   * Q tiles (one per slot) and a ring of K/V stages arrive by TMA (3-D tensor
//     maps over [B*H, N, d], 128-byte swizzle, out-of-range rows zero-filled).
//     The producer walks the same merge as the MMA warp, so the ring is
//     consumed in the order it is filled; a K stage is released after its S
//     GEMMs, a V stage after its PV GEMMs.
//   * S = Q K^T accumulates in tensor memory (TMEM) in fp32 (SS MMA, M=128,
//     N=block, K=16 steps over d).  The softmax warps read S with tcgen05.ld,
//     write P as bf16 back into the same TMEM columns, and O += P V runs as a
//     TS MMA with P taken from TMEM and V from shared memory (MN-major).  The
//     next S of a slot is queued behind that slot's PV: tcgen05 MMAs of one
//     thread execute in issue order, so the PV has read P before S overwrites
//     those columns.
//   * TMEM (512 columns): slot X uses S/P at X*256 and O at X*256 + 128.
//   * O (fp32) stays in TMEM for the whole item; the epilogue divides by l,
//     converts to bf16 and stores; LSE = (m + log2 l) ln 2.
//   * Every mbarrier wait is bounded; a timeout raises the CTA abort flag and
//     records FVATTN_ERR_DEVICE_TIMEOUT; all roles then drain and exit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <atomic>
#include <cstdint>
#include <math_constants.h>

#include "attn_fwd.cuh"
#include "common.cuh"
#include "ptx_sm100.cuh"

namespace fvattn {

namespace {

using namespace ptx;

constexpr int kRowsM = 128;           // query rows per tile (tcgen05 M)
constexpr int kSlots = 2;             // query blocks per work item
constexpr int kThreads = 384;         // 2 softmax warpgroups + one warpgroup for TMA and MMA issue
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;           // warps 10 and 11 only take part in the register hand-over
// Register hand-over (setmaxnreg): the launch gives every thread kLaunchRegs; the
// TMA/MMA warpgroup drops to kIssueRegs and the two softmax warpgroups, which
// hold a whole 128-column S row per thread, rise to kSoftmaxRegs.  The split must
// not exceed the launch pool (checked on the host before every launch).
constexpr int kLaunchRegs = 168;      // 65536 / 384, rounded down to a multiple of 8
constexpr int kIssueRegs = 80;
constexpr int kSoftmaxRegs = 208;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kIssueRegs <= kThreads * kLaunchRegs, "register split exceeds the pool");
static_assert(kSoftmaxRegs % 8 == 0 && kIssueRegs % 8 == 0, "setmaxnreg takes multiples of 8");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemSlot = 256;   // TMEM columns per slot
constexpr uint32_t kTmemO = 128;      // O offset inside a slot (S/P at offset 0)
constexpr int kMinSmem = 120 * 1024;  // more than half an SM's shared memory: one CTA per SM

template <int D, int BS>
struct Cfg {
    static constexpr int KBLK = D / 64;                   // 128-byte (64 x bf16) column blocks along d
    static constexpr int Q_BYTES = KBLK * kRowsM * 128;   // one Q tile buffer
    static constexpr int Q_LOAD_BYTES = KBLK * BS * 128;  // only the block's rows are loaded
    static constexpr int STAGE_BYTES = KBLK * BS * 128;   // one K or V tile
    static constexpr int NST = STAGE_BYTES >= 32768 ? 4 : 8;
    static constexpr int OFF_RING = kSlots * Q_BYTES;
    static constexpr int TILE_BYTES = OFF_RING + NST * STAGE_BYTES;
    static constexpr int NEED = TILE_BYTES + 1024 /*alignment slack*/ + 512 /*barriers*/;
    static constexpr int SMEM_BYTES = NEED > kMinSmem ? NEED : kMinSmem;
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(kRowsM, BS, 0, 0);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(kRowsM, D, 0, 1);
};

struct Barriers {
    uint64_t ring_full[8], ring_empty[8];
    uint64_t q_full[kSlots], q_empty[kSlots], s_full[kSlots], p_full[kSlots], o_full[kSlots], o_empty[kSlots];
    uint64_t sched_full[2], sched_empty[2];
    uint64_t drain;
    int4 sched_item[2][kSlots];  // per slot: {row or -1, col start, count, valid item}
    int4 ring_step[8];           // per K stage: {key block, row A uses it, row B uses it, last step of item}
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Barriers) <= 512, "barrier block exceeds its shared-memory reservation");

// One step of the merge of the two rows' key-block lists.
struct Step {
    int kblk;   // key block to load (0 for a skipped index)
    bool pa, pb;
};

// Walks the union of two strictly ascending key-block lists in order.  An entry
// that is out of range or not ascending is processed alone (its tile is loaded
// from block 0 and masked out by that row's softmax), so the producer, the MMA
// warp and the softmax warps all see each row's tiles in CSR order.
struct Merge {
    const int32_t *a, *b;
    int na, nbl, ia, ib, prev_a, prev_b, nkb;
    bool bad;  // the last step was a skipped index
    __device__ void init(const int32_t *col_idx, int4 sa, int4 sb, int nkb_) {
        a = col_idx + sa.y;
        na = sa.x >= 0 ? sa.z : 0;
        b = col_idx + sb.y;
        nbl = sb.x >= 0 ? sb.z : 0;
        ia = ib = 0;
        prev_a = prev_b = -1;
        nkb = nkb_;
        bad = false;
    }
    __device__ bool done() const { return ia >= na && ib >= nbl; }
    __device__ Step next() {
        const bool ha = ia < na, hb = ib < nbl;
        const int xa = ha ? a[ia] : 0, xb = hb ? b[ib] : 0;
        const bool va = ha && xa >= 0 && xa < nkb && xa > prev_a;
        const bool vb = hb && xb >= 0 && xb < nkb && xb > prev_b;
        Step s;
        bad = false;
        if (ha && !va) {
            s = {0, true, false};
            bad = true;
            ++ia;
        } else if (hb && !vb) {
            s = {0, false, true};
            bad = true;
            ++ib;
        } else if (ha && hb && xa == xb) {
            s = {xa, true, true};
            prev_a = prev_b = xa;
            ++ia;
            ++ib;
        } else if (ha && (!hb || xa < xb)) {
            s = {xa, true, false};
            prev_a = xa;
            ++ia;
        } else {
            s = {xb, false, true};
            prev_b = xb;
            ++ib;
        }
        return s;
    }
};

constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the row max grows by more than 2^8

// 2^x on the MUFU unit (flushes subnormal results to zero; exp2(-inf) = 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <int D, int BS>
__global__ void __launch_bounds__(kThreads, 1)
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
    unsigned char *sQ = smem;                    // slot X at X * Q_BYTES
    unsigned char *ring = smem + C::OFF_RING;    // stage s at s * STAGE_BYTES
    Barriers *bar = reinterpret_cast<Barriers *>(smem + C::TILE_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abort_flag = &bar->abort_flag;
    const int npair = (nb + 1) / 2;              // items per head

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&bar->ring_full[s], 1);
            mbar_init(&bar->ring_empty[s], 1);
        }
        for (int x = 0; x < kSlots; ++x) {
            mbar_init(&bar->q_full[x], 1);
            mbar_init(&bar->q_empty[x], 1);
            mbar_init(&bar->s_full[x], 1);
            mbar_init(&bar->p_full[x], 4);
            mbar_init(&bar->o_full[x], 1);
            mbar_init(&bar->o_empty[x], 4);
        }
        for (int k = 0; k < 2; ++k) {
            mbar_init(&bar->sched_full[k], 1);
            mbar_init(&bar->sched_empty[k], 1 + 8);
        }
        mbar_init(&bar->drain, 1);
        bar->abort_flag = 0;
        fence_barrier_init();
    }
    // Q rows beyond the block (block size 64) are never loaded: keep them zero.
    if (BS < kRowsM) {
        for (int x = 0; x < kSlots; ++x)
            for (int kb = 0; kb < C::KBLK; ++kb) {
                uint4 *z = reinterpret_cast<uint4 *>(sQ + x * C::Q_BYTES + kb * kRowsM * 128 + BS * 128);
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

    if (warp >= kTmaWarp) {
    // The register hand-over and the code that uses the new count sit in the same
    // branch, so the compiler allocates each role's registers against its own limit.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kIssueRegs));
    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_q);
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
            uint32_t it = 0, rc = 0;                  // items published, ring loads issued
            uint32_t q_armed[kSlots] = {0, 0};        // Q loads issued per slot
            uint32_t q_items[kSlots] = {0, 0};        // items with a Q tile per slot
            bool ok = true;
            while (ok) {
                const int idx = atomicAdd(work_counter, 1);
                const int p = (idx < n_items) ? order[idx] : -1;
                int4 sx[kSlots] = {make_int4(-1, 0, 0, 0), make_int4(-1, 0, 0, 0)};
                if (p >= 0) {
                    const int bh = p / npair, i2 = p % npair;
                    for (int x = 0; x < kSlots; ++x) {
                        if (2 * i2 + x >= nb) continue;  // an odd last block has no partner
                        const int rw = bh * nb + 2 * i2 + x;
                        int c = row_ptr[rw + 1] - row_ptr[rw];
                        if (c < 0) {
                            record_error(dev_status, FVATTN_ERR_BAD_CSR);
                            c = 0;
                        }
                        sx[x] = make_int4(rw, row_ptr[rw], c, 1);
                    }
                }
                const uint32_t k = it & 1;
                if (!mbar_wait(&bar->sched_empty[k], ((it >> 1) & 1) ^ 1, abort_flag, dev_status)) break;
                bar->sched_item[k][0] = sx[0];
                bar->sched_item[k][1] = sx[1];
                mbar_arrive(&bar->sched_full[k]);
                if (p < 0) break;
                const int bh = sx[0].x / nb;
                // Q tiles of the rows that have key blocks
                for (int x = 0; x < kSlots && ok; ++x) {
                    if (sx[x].x < 0 || sx[x].z == 0) continue;
                    if (!mbar_wait(&bar->q_empty[x], (q_items[x] & 1) ^ 1, abort_flag, dev_status)) {
                        ok = false;
                        break;
                    }
                    ++q_items[x];
                    // Test hook: CTA 0 leaves its first Q tile unloaded, so the MMA warp's
                    // bounded wait for it runs out (exercises the timeout path).
                    if (test_stall && blockIdx.x == 0 && it == 0) continue;
                    const int qb = sx[x].x % nb;
                    mbar_arrive_expect_tx(&bar->q_full[x], C::Q_LOAD_BYTES);
                    for (int kb = 0; kb < C::KBLK; ++kb)
                        tma_load_3d(sQ + x * C::Q_BYTES + kb * kRowsM * 128, &tmap_q, &bar->q_full[x], kb * 64,
                                    qb * BS, bh);
                    q_armed[x] = q_items[x];
                }
                // K and V of every block of the union, in merge order
                Merge mg;
                mg.init(col_idx, sx[0], sx[1], nb);
                while (ok && !mg.done()) {
                    const Step s = mg.next();
                    if (mg.bad) record_error(dev_status, FVATTN_ERR_BAD_CSR);
                    const bool last = mg.done();
                    for (int kv = 0; kv < 2 && ok; ++kv) {
                        const uint32_t st = rc % C::NST;
                        if (!mbar_wait(&bar->ring_empty[st], ((rc / C::NST) & 1) ^ 1, abort_flag, dev_status)) {
                            ok = false;
                            break;
                        }
                        // the MMA warp reads the step from its K stage once the stage is full
                        if (kv == 0) bar->ring_step[st] = make_int4(s.kblk, s.pa ? 1 : 0, s.pb ? 1 : 0, last ? 1 : 0);
                        mbar_arrive_expect_tx(&bar->ring_full[st], C::STAGE_BYTES);
                        for (int kb = 0; kb < C::KBLK; ++kb)
                            tma_load_3d(ring + st * C::STAGE_BYTES + kb * BS * 128, kv == 0 ? &tmap_k : &tmap_v,
                                        &bar->ring_full[st], kb * 64, s.kblk * BS, bh);
                        ++rc;
                    }
                }
                ++it;
            }
            // every load this thread issued lands before the CTA exits
            for (uint32_t st = 0; st < static_cast<uint32_t>(C::NST); ++st) {
                if (rc > st) {
                    const uint32_t times = (rc - st + C::NST - 1) / C::NST;
                    mbar_wait_teardown(&bar->ring_full[st], (times - 1) & 1);
                }
            }
            for (int x = 0; x < kSlots; ++x)
                if (q_armed[x] > 0) mbar_wait_teardown(&bar->q_full[x], (q_armed[x] - 1) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t q0 = smem_addr(sQ), r0 = smem_addr(ring);
            uint32_t it = 0, rc = 0;
            uint32_t qn[kSlots] = {0, 0}, on[kSlots] = {0, 0}, pc[kSlots] = {0, 0};
            bool ok = true;
            auto wait = [&](uint64_t *b, uint32_t parity) {
                if (ok && !mbar_wait(b, parity, abort_flag, dev_status)) ok = false;
                return ok;
            };
            // S_X = Q_X K^T from ring stage st
            auto issue_s = [&](int x, uint32_t st) {
                const uint32_t qa = q0 + x * C::Q_BYTES, kbase = r0 + st * C::STAGE_BYTES;
                const uint32_t tS = tmem + x * kTmemSlot;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t kb = k >> 2, ko = (k & 3) * 32;
                    const uint64_t da = smem_desc_sw128(qa + kb * kRowsM * 128 + ko, 16, 1024);
                    const uint64_t db = smem_desc_sw128(kbase + kb * BS * 128 + ko, 16, 1024);
                    mma_ss(tS, da, db, C::IDESC_S, k > 0 ? 1u : 0u);
                }
                mma_commit(&bar->s_full[x]);
            };
            // O_X (+)= P_X V from ring stage st
            auto issue_pv = [&](int x, uint32_t st, bool first) {
                const uint32_t vbase = r0 + st * C::STAGE_BYTES;
                const uint32_t tS = tmem + x * kTmemSlot, tO = tS + kTmemO;
#pragma unroll
                for (int k = 0; k < BS / 16; ++k) {
                    const uint64_t dv = smem_desc_sw128(vbase + k * 16 * 128, BS * 128, 1024);
                    mma_ts(tO, tS + k * 8, dv, C::IDESC_PV, (!first || k > 0) ? 1u : 0u);
                }
            };
            while (ok) {
                const uint32_t k = it & 1;
                if (!wait(&bar->sched_full[k], (it >> 1) & 1)) break;
                const int4 sx[kSlots] = {bar->sched_item[k][0], bar->sched_item[k][1]};
                mbar_arrive(&bar->sched_empty[k]);
                if (!sx[0].w) break;
                bool q_wait[kSlots], first_pv[kSlots];
                for (int x = 0; x < kSlots; ++x) {
                    q_wait[x] = sx[x].x >= 0 && sx[x].z > 0;
                    first_pv[x] = true;
                    // a row without key blocks: only the O handshake with its warpgroup
                    if (sx[x].x >= 0 && sx[x].z == 0 && wait(&bar->o_empty[x], (on[x] & 1) ^ 1)) {
                        mma_commit(&bar->o_full[x]);
                        ++on[x];
                    }
                }
                // the producer walks the merge of the two rows' block lists and leaves
                // each step in its K stage, so this thread never reads col_idx
                bool more = (sx[0].x >= 0 && sx[0].z > 0) || (sx[1].x >= 0 && sx[1].z > 0);
                int b_pending = -1;  // ring stage of V for the B tile whose PV is still to issue
                while (ok && more) {
                    const uint32_t kst = rc % C::NST, vst = (rc + 1) % C::NST;
                    const uint32_t kph = (rc / C::NST) & 1, vph = ((rc + 1) / C::NST) & 1;
                    rc += 2;
                    if (!wait(&bar->ring_full[kst], kph)) break;
                    const int4 step = bar->ring_step[kst];
                    const Step s = {step.x, step.y != 0, step.z != 0};
                    more = step.w == 0;
                    if (s.pa) {
                        if (q_wait[0]) {
                            if (!wait(&bar->q_full[0], qn[0] & 1)) break;
                            ++qn[0];
                            q_wait[0] = false;
                        }
                        tc_fence_after();
                        issue_s(0, kst);
                    }
                    if (b_pending >= 0) {
                        if (!wait(&bar->p_full[1], pc[1] & 1)) break;
                        ++pc[1];
                        if (first_pv[1] && !wait(&bar->o_empty[1], (on[1] & 1) ^ 1)) break;
                        tc_fence_after();
                        issue_pv(1, b_pending, first_pv[1]);
                        first_pv[1] = false;
                        mma_commit(&bar->ring_empty[b_pending]);
                        b_pending = -1;
                    }
                    if (s.pb) {
                        if (q_wait[1]) {
                            if (!wait(&bar->q_full[1], qn[1] & 1)) break;
                            ++qn[1];
                            q_wait[1] = false;
                        }
                        tc_fence_after();
                        issue_s(1, kst);
                    }
                    mma_commit(&bar->ring_empty[kst]);  // K read by every S above
                    if (!wait(&bar->ring_full[vst], vph)) break;
                    if (s.pa) {
                        if (!wait(&bar->p_full[0], pc[0] & 1)) break;
                        ++pc[0];
                        if (first_pv[0] && !wait(&bar->o_empty[0], (on[0] & 1) ^ 1)) break;
                        tc_fence_after();
                        issue_pv(0, vst, first_pv[0]);
                        first_pv[0] = false;
                    }
                    if (s.pb) {
                        b_pending = static_cast<int>(vst);
                    } else {
                        mma_commit(&bar->ring_empty[vst]);
                    }
                }
                if (ok && b_pending >= 0 && wait(&bar->p_full[1], pc[1] & 1)) {
                    ++pc[1];
                    if (!first_pv[1] || wait(&bar->o_empty[1], (on[1] & 1) ^ 1)) {
                        tc_fence_after();
                        issue_pv(1, b_pending, first_pv[1]);
                        first_pv[1] = false;
                        mma_commit(&bar->ring_empty[b_pending]);
                    }
                }
                if (!ok) break;
                for (int x = 0; x < kSlots; ++x) {
                    if (sx[x].x >= 0 && sx[x].z > 0) {
                        mma_commit(&bar->q_empty[x]);
                        mma_commit(&bar->o_full[x]);
                        ++on[x];
                    }
                }
                ++it;
            }
            // every MMA issued by this thread completes before TMEM is released
            mma_commit(&bar->drain);
            mbar_wait_teardown(&bar->drain, 0);
        }
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        // ------------------------------------------------ softmax / epilogue
        const int X = warp >> 2;                                   // slot of this warpgroup
        const int r = threadIdx.x & (kRowsM - 1);                  // tile row = TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + X * kTmemSlot + lane_base;
        const uint32_t tO = tS + kTmemO;
        uint32_t it = 0, sc = 0, on = 0;
        while (true) {
            const uint32_t k = it & 1;
            if (!mbar_wait(&bar->sched_full[k], (it >> 1) & 1, abort_flag, dev_status)) break;
            const int4 item = bar->sched_item[k][X];
            const bool valid_item = bar->sched_item[k][0].w != 0;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->sched_empty[k]);
            ++it;
            if (!valid_item) break;
            if (item.x < 0) continue;                              // slot B of an odd last block
            const int row = item.x, start = item.y, count = item.z;
            const int64_t bh = row / nb;
            const int qb = row % nb;
            const int t_row = qb * BS + r;                         // token index of this thread's row
            float m = -CUDART_INF_F, l = 0.0f;
            int prev = -1;
            bool ok = true;
            for (int j = 0; j < count; ++j) {
                int kblk = col_idx[start + j];
                const bool valid = kblk >= 0 && kblk < nb && kblk > prev;
                if (valid) prev = kblk;
                const int key0 = kblk * BS;
                // keys of this block that exist and are allowed for this row
                int lim = valid ? min(BS, N - key0) : 0;
                if (causal) lim = min(lim, t_row - key0 + 1);
                if (!mbar_wait(&bar->s_full[X], sc & 1, abort_flag, dev_status)) { ok = false; break; }
                ++sc;
                tc_fence_after();
                // the whole S row of this thread: BS fp32 values
                uint32_t v[BS];
#pragma unroll
                for (int c0 = 0; c0 < BS; c0 += 32) tmem_ld32(tS + c0, *reinterpret_cast<uint32_t(*)[32]>(&v[c0]));
                tmem_wait_ld();
                if (lim < BS) {  // ragged last block, causal diagonal, or a skipped index
#pragma unroll
                    for (int c = 0; c < BS; ++c)
                        if (c >= lim) v[c] = __float_as_uint(-CUDART_INF_F);
                }
                float mq[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
                for (int c = 0; c < BS; c += 8) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        mq[q] = max3f(mq[q], __uint_as_float(v[c + 2 * q]), __uint_as_float(v[c + 2 * q + 1]));
                }
                const float mxs = max3f(mq[0], mq[1], fmaxf(mq[2], mq[3])) * scale_log2;
                // The reference maximum only moves when the row maximum exceeds it by
                // more than 2^8: P stays below 256 and the rescale of O is rare.  O and
                // l always share the same reference, so the final O / l is exact.
                const bool need = mxs > m + kRescaleLog2;
                const float m_new = need ? mxs : m;
                const float alpha = need ? ex2_approx(m - m_new) : 1.0f;
                const float neg_m = (m_new == -CUDART_INF_F) ? 0.0f : -m_new;
                float rs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                // P packed as bf16 pairs in place: v[c/2] <- (p[c], p[c+1])
                // one loop for full and masked tiles (masked scores are -inf, and 2^-inf = 0),
                // which keeps the kernel's code small enough for the instruction caches
#pragma unroll
                for (int c = 0; c < BS; c += 2) {
                    const float p0 = ex2_approx(fmaf(__uint_as_float(v[c]), scale_log2, neg_m));
                    const float p1 = ex2_approx(fmaf(__uint_as_float(v[c + 1]), scale_log2, neg_m));
                    rs[(c >> 1) & 3] += p0 + p1;
                    v[c >> 1] = pack_bf16(p0, p1);
                }
#pragma unroll
                for (int c0 = 0; c0 < BS / 2; c0 += 32)
                    tmem_st32(tS + c0, *reinterpret_cast<const uint32_t(*)[32]>(&v[c0]));
                l = l * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
                // rescale the running output (this slot's previous PV has completed: it
                // was issued before this S, and the S commit tracks every earlier MMA)
                if (__any_sync(0xffffffffu, need && j > 0)) {
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
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
                if (lane == 0) mbar_arrive(&bar->p_full[X]);
                m = m_new;
            }
            if (!ok) break;
            // epilogue
            if (!mbar_wait(&bar->o_full[X], on & 1, abort_flag, dev_status)) break;
            ++on;
            tc_fence_after();
            const bool row_ok = r < BS && t_row < N;
            const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
            __nv_bfloat16 *orow = O + (bh * N + t_row) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
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
            if (row_ok) LSE[bh * N + t_row] = (l > 0.0f) ? (m + __log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->o_empty[X]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------- work order
// Items are ordered head-major, longest first: heads by their total selected
// blocks (descending, equal totals by head index), and inside a head the items
// by their block count (descending, equal counts by item index).  All SMs then
// work on about one head at a time, whose K and V stay in L2, and the grid ends
// on the lightest head's shortest items.

constexpr int kOrderThreads = 1024;

// "x comes after y": key descending, index ascending.
__device__ __forceinline__ bool later(int kx, int ix, int ky, int iy) { return kx < ky || (kx == ky && ix > iy); }

// Sorts n <= 2 * kOrderThreads * reps (key, index) pairs in shared memory, padded to np2.
__device__ void bitonic_sort(int *key, int *idx, int np2) {
    for (int k = 2; k <= np2; k <<= 1) {
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
            for (int e = threadIdx.x; e < (np2 >> 1); e += blockDim.x) {
                const int a = (e / jj) * 2 * jj + (e % jj), b = a + jj;
                const bool up = (a & k) == 0;
                const bool swap = up ? later(key[a], idx[a], key[b], idx[b]) : later(key[b], idx[b], key[a], idx[a]);
                if (swap) {
                    const int tk = key[a], ti = idx[a];
                    key[a] = key[b];
                    idx[a] = idx[b];
                    key[b] = tk;
                    idx[b] = ti;
                }
            }
            __syncthreads();
        }
    }
}

// One CTA: head_rank[h] = position of head h in the order of head totals.
__global__ void __launch_bounds__(kOrderThreads) head_rank_kernel(const int32_t *__restrict__ row_ptr, int BH, int nb,
                                                                  int np2, int32_t *__restrict__ head_rank) {
    extern __shared__ int sm_order[];
    int *key = sm_order, *idx = sm_order + np2;
    for (int e = threadIdx.x; e < np2; e += blockDim.x) {
        key[e] = e < BH ? row_ptr[static_cast<int64_t>(e + 1) * nb] - row_ptr[static_cast<int64_t>(e) * nb] : -1;
        idx[e] = e < BH ? e : 0x7fffffff;
    }
    __syncthreads();
    bitonic_sort(key, idx, np2);
    for (int e = threadIdx.x; e < BH; e += blockDim.x) head_rank[idx[e]] = e;
}

// One CTA per head: its items sorted by block count, written at head_rank[h] * npair.
__global__ void __launch_bounds__(kOrderThreads) item_order_kernel(const int32_t *__restrict__ row_ptr, int nb,
                                                                   int np2, const int32_t *__restrict__ head_rank,
                                                                   int32_t *__restrict__ order) {
    extern __shared__ int sm_order[];
    int *key = sm_order, *idx = sm_order + np2;
    const int npair = (nb + 1) / 2;
    const int64_t bh = blockIdx.x;
    for (int e = threadIdx.x; e < np2; e += blockDim.x) {
        if (e < npair) {
            const int64_t r = bh * nb + 2 * e;
            const int64_t r_end = (2 * e + 2 <= nb) ? r + 2 : r + 1;
            key[e] = row_ptr[r_end] - row_ptr[r];
            idx[e] = e;
        } else {
            key[e] = -1;
            idx[e] = 0x7fffffff;
        }
    }
    __syncthreads();
    bitonic_sort(key, idx, np2);
    const int64_t base = static_cast<int64_t>(head_rank[bh]) * npair;
    for (int e = threadIdx.x; e < npair; e += blockDim.x)
        order[base + e] = static_cast<int32_t>(bh * npair + idx[e]);
}

}  // namespace

// ------------------------------------------------------------------ launcher

int attn_smem_bytes(int d, int bs) {
    if (d == 128 && bs == 128) return Cfg<128, 128>::SMEM_BYTES;
    if (d == 128 && bs == 64) return Cfg<128, 64>::SMEM_BYTES;
    if (d == 64 && bs == 128) return Cfg<64, 128>::SMEM_BYTES;
    return Cfg<64, 64>::SMEM_BYTES;
}

int attn_ctas_per_sm() { return 1; }

int64_t attn_num_items(int64_t BH, int nb) { return BH * ((nb + 1) / 2); }

static int pow2_at_least(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

cudaError_t launch_item_order(const int32_t *row_ptr, int64_t BH, int nb, int32_t *head_rank, int32_t *order,
                              cudaStream_t stream) {
    const int hp2 = pow2_at_least(static_cast<int>(BH));
    const int ip2 = pow2_at_least((nb + 1) / 2);
    head_rank_kernel<<<1, kOrderThreads, 2 * hp2 * sizeof(int), stream>>>(row_ptr, static_cast<int>(BH), nb, hp2,
                                                                           head_rank);
    item_order_kernel<<<static_cast<unsigned>(BH), kOrderThreads, 2 * ip2 * sizeof(int), stream>>>(
        row_ptr, nb, ip2, head_rank, order);
    return cudaGetLastError();
}

template <int D, int BS>
static cudaError_t launch_t(const AttnLaunch &a, cudaStream_t stream) {
    auto kern = sparse_attn_fwd_kernel<D, BS>;
    // The register hand-over waits until the pool holds the requested registers, so
    // it must fit in what the launch allocates: checked once per instantiation.
    static std::atomic<int> regs_ok{0};  // 0 unknown, 1 fits, -1 does not
    if (regs_ok.load() == 0) {
        cudaFuncAttributes fa{};
        cudaError_t e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        regs_ok.store(2 * 128 * kSoftmaxRegs + 128 * kIssueRegs <= fa.numRegs * kThreads ? 1 : -1);
    }
    if (regs_ok.load() < 0) return cudaErrorInvalidConfiguration;
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
