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
//   * One work item = 128 query rows of one head: at block 128 one query block
//     (a CSR row), at block 64 two neighbouring query blocks 2i and 2i+1 (a
//     pair).  A pair walks the union of its two rows' key-block lists; each
//     half of the tile masks the key blocks its own row did not select, which
//     leaves its m, l and O exactly as they were, so every row gets the result
//     of its own list and the M = 128 MMAs carry no zero rows.  The TMA warp
//     builds a pair's union in shared memory (per-row bitmaps, then a warp
//     scan) when it takes the item.  A tile is always 128 key columns: at
//     block 64, two consecutive entries of the union (two 64-row TMA boxes in
//     one ring stage; an odd union's last tile reads rows past N, zero-filled,
//     for its second half), so the MMAs and the softmax have the same shapes,
//     and the same per-tile overheads, at both block sizes.  A persistent grid of one CTA per SM pops
//     items from a queue ordered head-major and longest-first (FVAttn §1 "RLB"
//     balances per-head work at run time; here the SMs are balanced instead,
//     and the head order keeps one or two heads' K and V in L2 while all SMs
//     work on them).
//   * Warps 0-3 run the softmax and the epilogue (thread = query row = TMEM
//     lane); warp 4 issues TMA loads of K and V tiles into a ring of shared
//     memory stages; warp 5 issues the tcgen05 MMAs.
//   * Tensor memory (512 columns) holds Q twice (the current and the next
//     item), S twice and O once (fp32): S = Q K^T of tile j+2 is computed
//     while the softmax works on tile j+1 and the tensor cores run
//     O += P_j V_j, so the tensor cores never wait for the softmax of the tile
//     they need next.  Q comes from TMEM (TS MMA: only K is read from shared
//     memory for S), P is written into the columns of its S buffer and read
//     from there by the PV MMA (V from shared memory, MN-major).
//   * tcgen05 MMAs of one thread execute in issue order: S of tile j+2 is
//     issued after PV of tile j, which reads the P in the same columns.
//   * The softmax reads the whole S row of its thread (tcgen05.ld), takes the
//     row maximum, and writes P in place; the running reference maximum moves
//     only when a row's maximum exceeds it by more than 2^8, so the rescale of
//     O in tensor memory is rare.  The scale-and-shift of the scores and the
//     row sums run on packed fp32 pairs (one instruction per two columns): the
//     softmax warp, not a pipe, is the critical path, so instructions count.
//   * O stays in TMEM for the whole item; the epilogue divides by l, converts
//     to bf16 and stores; LSE = (m + log2 l) ln 2.  The softmax warps load the
//     next item's Q into TMEM before the epilogue, so the next item's first two
//     S tiles overlap it.
//   * Every mbarrier wait is bounded; a timeout raises the CTA abort flag and
//     records FVATTN_ERR_DEVICE_TIMEOUT; all roles then drain and exit.
//
// FP8 variant ("Accelerating HunyuanVideo inference with ParaAttention"
// (WaveSpeed), § "FP8 dynamic quantization": attention run on FP8 activations):
// Q, K and V arrive as e4m3 codes with one power-of-two scale 2^e per (head,
// block) (the block quantization of quant.cu), and both GEMMs run as tcgen05
// kind::f8f6f4 MMAs (e4m3 x e4m3, fp32 accumulation; twice the bf16 rate).
//   * S: the codes' dot products are exact products summed in fp32; the tile's
//     scale 2^(e_q + e_k) is folded into the softmax scale of that tile.
//   * PV: P is rounded to e4m3 (one scale for all rows of a key block: its
//     2^(e_v - E), E the largest e_v the row has taken so far, so that P <= 256
//     stays in range; the power of two rides in the exponent argument) and
//     written four codes per TMEM column; the row sum l uses the unrounded P
//     (the scaled values summed, then scaled back exactly by 2^(E - e_v)).
//     When a later block has a larger e_v, O is rescaled by the exact power of
//     two 2^(E_old - E_new) (together with the maximum rescale).  The epilogue
//     multiplies by 2^E / l.
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
constexpr int kKT = 128;              // key columns per tile (tcgen05 N of S, K of PV)
constexpr int kThreads = 192;         // softmax warpgroup + TMA warp + MMA warp
constexpr int kCtasPerSm = 1;         // kernels that hold tensor memory are resident one CTA per SM
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxStages = 12;
constexpr int kRingBytes = 192 * 1024;
constexpr int kUnionCap = kMaxCount;           // entries of one pair's key-block union
constexpr int kBitmapWords = kMaxCount / 32;   // one row's key-block bitmap

template <int D, int BS, bool F8>
struct Cfg {
    static constexpr int EB = F8 ? 1 : 2;                 // bytes per operand element (e4m3 or bf16)
    static_assert((D * EB) % 128 == 0, "rows of d operands must fill whole 128-byte swizzle spans");
    static constexpr int KBLK = D * EB / 128;             // 128-byte column blocks along d
    static constexpr int X_CHUNK = 128 / EB;              // elements per 128-byte column block
    static constexpr int KSTEP = 32 / EB;                 // K of one MMA (32 bytes of operand)
    // A tile is kKT = 128 key columns: one key block at block 128, two key blocks
    // (two entries of a pair's union, 64 rows each) at block 64.
    static constexpr int HALVES = kKT / BS;               // key blocks per tile
    static constexpr int STAGE_BYTES = KBLK * kKT * 128;  // one K or V tile
    static constexpr int NST = kRingBytes / STAGE_BYTES < kMaxStages ? kRingBytes / STAGE_BYTES : kMaxStages;
    static constexpr int TILE_BYTES = NST * STAGE_BYTES;
    // block 64: an item is a pair of query blocks; its key-block union lives in
    // shared memory, two slots of uint16 entries (block << 2 | row bits), plus the
    // two rows' bitmaps the union is built from
    static constexpr bool PAIR = BS == 64;
    static constexpr int UNION_BYTES = PAIR ? 2 * kUnionCap * 2 + 2 * kBitmapWords * 4 : 0;
    static constexpr int SMEM_BYTES = TILE_BYTES + 1024 /*alignment slack*/ + 512 /*barriers*/ + UNION_BYTES;
    static_assert(!PAIR || 2 * BS == kRowsM, "a pair fills the M = 128 tile");
    // TMEM columns: Q buffers (packed operands), S buffers (fp32; P as bf16 pairs or
    // e4m3 quads in their first columns), O (fp32)
    static constexpr uint32_t Q_COLS = D * EB / 4;
    static constexpr uint32_t T_Q0 = 0, T_Q1 = Q_COLS, T_S0 = 128, T_S1 = 128 + kKT, T_O = 128 + 2 * kKT;
    static_assert(2 * Q_COLS <= 128 && T_O + D <= kTmemCols, "TMEM layout exceeds 512 columns");
    static constexpr uint32_t IDESC_S = F8 ? idesc_e4m3_f32(kRowsM, kKT, 0, 0) : idesc_bf16_f32(kRowsM, kKT, 0, 0);
    static constexpr uint32_t IDESC_PV = F8 ? idesc_e4m3_f32(kRowsM, D, 0, 1) : idesc_bf16_f32(kRowsM, D, 0, 1);
};

struct Barriers {
    uint64_t ring_full[kMaxStages], ring_empty[kMaxStages];
    uint64_t q_full[2], s_full[2], p_full[2];
    uint64_t pv_done, o_full, o_empty;
    uint64_t sched_full[2], sched_empty[2];
    uint64_t drain;
    // {item (row, or pair of rows), CSR start (pairs: union entries), tiles, queue index + 1 (0: no more items)}
    int4 sched_item[2];
    long long t_start;   // diagnostic: global timer at the start of the CTA's work
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Barriers) <= 512, "barrier block exceeds its shared-memory reservation");

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

// Four fp32 values -> four e4m3 codes (a in the low byte): nearest, ties to even,
// saturating (the inputs here are at most 256, inside the e4m3 range).
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
    return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// x * 2^e for the block-scale exponents (exact; the clamp keeps absurd exponent
// sums of degenerate blocks finite).
__device__ __forceinline__ float pow2_scale(float x, int e) { return ldexpf(x, max(-200, min(e, 126))); }

// ------------------------------------------------------------- block-64 pairs
// Pair i of head bh: query blocks 2i (row A) and 2i+1 (row B, absent when nb is
// odd and i is the last pair).  The 32 lanes of a warp set one bit per selected
// key block in two bitmaps bm[0, nw) (A) and bm[nw, 2 nw) (B), nw = ceil(nb / 32);
// entries outside [0, nb) are left out.  With CHECK, also whether a row is
// malformed (a negative count, an entry outside [0, nb), or one not above the
// entry before it).
template <bool CHECK>
__device__ bool pair_bitmaps(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx, int64_t bh,
                             int pair, int nb, uint32_t *bm, int lane) {
    const int nw = (nb + 31) >> 5;
    for (int w = lane; w < 2 * nw; w += 32) bm[w] = 0u;
    __syncwarp();
    const int64_t ra = bh * nb + 2 * pair;
    const bool has_b = 2 * pair + 1 < nb;
    const int a0 = __ldg(row_ptr + ra), a1 = __ldg(row_ptr + ra + 1);
    const int b1 = has_b ? __ldg(row_ptr + ra + 2) : a1;
    bool bad = CHECK && (a1 < a0 || b1 < a1);
    for (int h = 0; h < 2; ++h) {
        const int s0 = h ? a1 : a0, s1 = h ? b1 : a1;
        for (int k = s0 + lane; k < s1; k += 32) {
            const int x = __ldg(col_idx + k);
            if (x >= 0 && x < nb) atomicOr(bm + h * nw + (x >> 5), 1u << (x & 31));
            else if (CHECK) bad = true;
            if (CHECK && k > s0 && __ldg(col_idx + k - 1) >= x) bad = true;
        }
    }
    __syncwarp();
    return __any_sync(0xffffffffu, bad);
}

// The pair's union from its bitmaps, ascending, as entries (block << 2) | (1 if row
// A selected it) | (2 if row B did), written to out[0, count) by the 32 lanes (each
// lane takes a run of words; a warp scan of their bit counts places the runs).
// Returns count (<= nb) on every lane.
__device__ int pair_union(const uint32_t *bm, int nb, uint16_t *out, int lane) {
    const int nw = (nb + 31) >> 5;
    const int wpl = (nw + 31) >> 5;  // words per lane (<= kBitmapWords / 32)
    const int w0 = lane * wpl;
    int cnt = 0;
    for (int q = 0; q < wpl; ++q)
        if (w0 + q < nw) cnt += __popc(bm[w0 + q] | bm[nw + w0 + q]);
    int inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
    }
    int pos = inc - cnt;
    for (int q = 0; q < wpl; ++q) {
        const int w = w0 + q;
        if (w >= nw) break;
        const uint32_t a = bm[w], b = bm[nw + w];
        uint32_t u = a | b;
        while (u) {
            const int bit = __ffs(u) - 1;
            u &= u - 1;
            out[pos++] = static_cast<uint16_t>(((w * 32 + bit) << 2) | ((a >> bit) & 1u) | (((b >> bit) & 1u) << 1));
        }
    }
    return __shfl_sync(0xffffffffu, inc, 31);
}

template <int D, int BS, bool F8>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    sparse_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                           const unsigned char *__restrict__ Qg, const int32_t *__restrict__ row_ptr,
                           const int32_t *__restrict__ col_idx, const int32_t *__restrict__ order, int n_items,
                           int *__restrict__ work_counter, int N, int nb, int causal, float scale_log2,
                           __nv_bfloat16 *__restrict__ O, float *__restrict__ LSE, int32_t *dev_status,
                           int test_stall, long long *__restrict__ cta_busy_ns, const int32_t *__restrict__ q_exp,
                           const int32_t *__restrict__ k_exp, const int32_t *__restrict__ v_exp) {
    using C = Cfg<D, BS, F8>;
    constexpr int NST = C::NST;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzled tiles
    const uint32_t base_addr = smem_addr(smem_raw);
    unsigned char *ring = smem_raw + ((1024 - (base_addr & 1023)) & 1023);  // stage s at s * STAGE_BYTES
    Barriers *bar = reinterpret_cast<Barriers *>(ring + C::TILE_BYTES);
    // pairs only: the two union slots and the bitmaps
    uint16_t *uni = reinterpret_cast<uint16_t *>(ring + C::TILE_BYTES + 512);
    uint32_t *bmap = reinterpret_cast<uint32_t *>(ring + C::TILE_BYTES + 512 + 2 * kUnionCap * 2);
    const int ipb = C::PAIR ? (nb + 1) >> 1 : nb;  // items per head

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abort_flag = &bar->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&bar->ring_full[s], 1);
            mbar_init(&bar->ring_empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bar->q_full[x], 4);
            mbar_init(&bar->s_full[x], 1);
            mbar_init(&bar->p_full[x], 4);
            mbar_init(&bar->sched_full[x], 1);
            mbar_init(&bar->sched_empty[x], 1 + 4);
        }
        mbar_init(&bar->pv_done, 1);
        mbar_init(&bar->o_full, 1);
        mbar_init(&bar->o_empty, 4);
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
    if (cta_busy_ns && threadIdx.x == 0) {
        long long t0;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
        bar->t_start = t0;
    }

    if (warp == kTmaWarp && C::PAIR) {
        // ------------------------------------------------- producer (pairs)
        // The whole warp builds each pair's union into the item's slot; lane 0
        // pops items, publishes them and issues the loads.
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
        uint32_t it = 0, rc = 0;  // items published, ring loads issued (lane 0)
        while (true) {
            int idx = 0, pr = -1;
            if (lane == 0) {
                idx = atomicAdd(work_counter, 1);
                pr = (idx < n_items) ? order[idx] : -1;
            }
            idx = __shfl_sync(0xffffffffu, idx, 0);
            pr = __shfl_sync(0xffffffffu, pr, 0);
            const uint32_t k = it & 1;
            // the slot is free once the previous item in it has been consumed
            int free_ok = 1;
            if (lane == 0) free_ok = mbar_wait(&bar->sched_empty[k], ((it >> 1) & 1) ^ 1, abort_flag, dev_status);
            if (!__shfl_sync(0xffffffffu, free_ok, 0)) break;
            uint16_t *ul = uni + k * kUnionCap;
            int count = 0;
            if (pr >= 0) {
                pair_bitmaps<false>(row_ptr, col_idx, pr / ipb, pr % ipb, nb, bmap, lane);
                count = pair_union(bmap, nb, ul, lane);
            }
            __threadfence_block();  // the union entries before lane 0 publishes the item
            __syncwarp();
            int ok = 1;
            if (lane == 0) {
                // item: {pair, union entries, tiles (two entries each), queue index + 1}
                const int tiles = (count + 1) >> 1;
                bar->sched_item[k] = make_int4(pr, count, tiles, pr >= 0 ? idx + 1 : 0);
                mbar_arrive(&bar->sched_full[k]);
                if (pr >= 0) {
                    const int bh = pr / ipb;
                    for (int j = 0; j < tiles && ok; ++j) {
                        // the two key blocks of the tile (the union is ascending and in
                        // range); an odd union's last tile loads rows past N for its
                        // second half, which the TMA unit fills with zeros
                        const int row0 = (ul[2 * j] >> 2) * BS;
                        const int row1 = (2 * j + 1 < count) ? (ul[2 * j + 1] >> 2) * BS : nb * BS;
                        for (int kv = 0; kv < 2; ++kv) {
                            const uint32_t st = rc % NST;
                            if (!mbar_wait(&bar->ring_empty[st], ((rc / NST) & 1) ^ 1, abort_flag, dev_status)) {
                                ok = 0;
                                break;
                            }
                            mbar_arrive_expect_tx(&bar->ring_full[st], C::STAGE_BYTES);
                            for (int kb = 0; kb < C::KBLK; ++kb) {
                                unsigned char *dst = ring + st * C::STAGE_BYTES + kb * kKT * 128;
                                const CUtensorMap *map = kv == 0 ? &tmap_k : &tmap_v;
                                tma_load_3d(dst, map, &bar->ring_full[st], kb * C::X_CHUNK, row0, bh);
                                tma_load_3d(dst + BS * 128, map, &bar->ring_full[st], kb * C::X_CHUNK, row1, bh);
                            }
                            ++rc;
                        }
                    }
                }
            }
            ++it;
            if (pr < 0 || !__shfl_sync(0xffffffffu, ok, 0)) break;
        }
        // every load lane 0 issued lands before the CTA exits
        if (lane == 0) {
            for (uint32_t st = 0; st < static_cast<uint32_t>(NST); ++st) {
                if (rc > st) {
                    const uint32_t times = (rc - st + NST - 1) / NST;
                    mbar_wait_teardown(&bar->ring_full[st], (times - 1) & 1);
                }
            }
        }
    } else if (warp == kTmaWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
            uint32_t it = 0, rc = 0;  // items published, ring loads issued
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
                    item = make_int4(rw, row_ptr[rw], c, idx + 1);
                }
                const uint32_t k = it & 1;
                if (!mbar_wait(&bar->sched_empty[k], ((it >> 1) & 1) ^ 1, abort_flag, dev_status)) break;
                bar->sched_item[k] = item;
                mbar_arrive(&bar->sched_full[k]);
                ++it;
                if (rw < 0) break;
                const int bh = rw / nb;
                int prev = -1;
                int kblk_next = item.z > 0 ? __ldg(col_idx + item.y) : 0;  // loaded one tile ahead
                for (int j = 0; j < item.z && ok; ++j) {
                    int kblk = kblk_next;
                    if (j + 1 < item.z) kblk_next = __ldg(col_idx + item.y + j + 1);
                    if (kblk >= 0 && kblk < nb && kblk > prev) {
                        prev = kblk;
                    } else {  // skipped by the softmax; any in-range tile will do
                        record_error(dev_status, FVATTN_ERR_BAD_CSR);
                        kblk = 0;
                    }
                    for (int kv = 0; kv < 2; ++kv) {
                        const uint32_t st = rc % NST;
                        if (!mbar_wait(&bar->ring_empty[st], ((rc / NST) & 1) ^ 1, abort_flag, dev_status)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bar->ring_full[st], C::STAGE_BYTES);
                        for (int kb = 0; kb < C::KBLK; ++kb)
                            tma_load_3d(ring + st * C::STAGE_BYTES + kb * kKT * 128, kv == 0 ? &tmap_k : &tmap_v,
                                        &bar->ring_full[st], kb * C::X_CHUNK, kblk * BS, bh);
                        ++rc;
                    }
                }
            }
            // every load this thread issued lands before the CTA exits
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
                if (ok && !mbar_wait(b, parity, abort_flag, dev_status)) ok = false;
                return ok;
            };
            // S[scol] = Q[qcol] K^T: Q from TMEM, K of ring stage st (K-major in shared
            // memory).  The descriptors of the k-steps are one base descriptor plus the
            // step's byte offset >> 4 (shared-memory addresses stay below 2^18, so the
            // 14-bit address field never carries).
            auto issue_s = [&](uint32_t qcol, uint32_t scol, uint32_t st) {
                const uint64_t kdesc = smem_desc_sw128(r0 + st * C::STAGE_BYTES, 16, 1024);
#pragma unroll
                for (int k = 0; k < D * C::EB / 32; ++k) {
                    const uint64_t db = kdesc + (((k >> 2) * kKT * 128 + (k & 3) * 32) >> 4);
                    if (F8)
                        mma_ts_f8_nc(tmem + scol, tmem + qcol + k * 8, db, C::IDESC_S, k > 0 ? 1u : 0u);
                    else
                        mma_ts_nc(tmem + scol, tmem + qcol + k * 8, db, C::IDESC_S, k > 0 ? 1u : 0u);
                }
            };
            // O (+)= P V, P from the S buffer at scol, V of ring stage st (MN-major)
            auto issue_pv = [&](uint32_t scol, uint32_t st, bool first) {
                const uint64_t vdesc = smem_desc_sw128(r0 + st * C::STAGE_BYTES, kKT * 128, 1024);
#pragma unroll
                for (int k = 0; k < kKT / C::KSTEP; ++k) {
                    const uint64_t dv = vdesc + ((k * C::KSTEP * 128) >> 4);
                    if (F8)
                        mma_ts_f8_nc(tmem + C::T_O, tmem + scol + k * 8, dv, C::IDESC_PV, (!first || k > 0) ? 1u : 0u);
                    else
                        mma_ts_nc(tmem + C::T_O, tmem + scol + k * 8, dv, C::IDESC_PV, (!first || k > 0) ? 1u : 0u);
                }
            };
            while (ok) {
                const uint32_t k = it & 1;
                if (!wait(&bar->sched_full[k], (it >> 1) & 1)) break;
                const int4 item = bar->sched_item[k];
                mbar_arrive(&bar->sched_empty[k]);
                ++it;
                if (!item.w) break;
                const int count = item.z;
                if (count == 0) {  // a row without key blocks: only the O handshake
                    if (!wait(&bar->o_empty, (on & 1) ^ 1)) break;
                    mma_commit(&bar->o_full);
                    ++on;
                    continue;
                }
                if (!wait(&bar->q_full[qn & 1], (qn >> 1) & 1)) break;
                tc_fence_after();
                const uint32_t qcol = (qn & 1) ? C::T_Q1 : C::T_Q0;
                // S of the first two key blocks, into both S buffers
                for (int j = 0; j < 2 && j < count; ++j) {
                    const uint32_t ki = rc + 2 * j;
                    if (!wait(&bar->ring_full[ki % NST], (ki / NST) & 1)) break;
                    const uint32_t sb = (tc + j) & 1;
                    issue_s(qcol, sb ? C::T_S1 : C::T_S0, ki % NST);
                    mma_commit(&bar->s_full[sb]);
                    mma_commit(&bar->ring_empty[ki % NST]);
                }
                for (int j = 0; j < count && ok; ++j) {
                    const uint32_t t = tc + j, sb = t & 1, scol = sb ? C::T_S1 : C::T_S0;
                    if (!wait(&bar->p_full[sb], (t >> 1) & 1)) break;
                    if (j == 0 && !wait(&bar->o_empty, (on & 1) ^ 1)) break;
                    const uint32_t vi = rc + 2 * j + 1;
                    if (!wait(&bar->ring_full[vi % NST], (vi / NST) & 1)) break;
                    tc_fence_after();
                    issue_pv(scol, vi % NST, j == 0);
                    mma_commit(&bar->ring_empty[vi % NST]);
                    mma_commit(&bar->pv_done);
                    if (j + 2 < count) {  // the S buffer just read by PV takes block j+2
                        const uint32_t ki = rc + 2 * (j + 2);
                        if (!wait(&bar->ring_full[ki % NST], (ki / NST) & 1)) break;
                        issue_s(qcol, scol, ki % NST);
                        mma_commit(&bar->s_full[sb]);
                        mma_commit(&bar->ring_empty[ki % NST]);
                    }
                }
                if (!ok) break;
                mma_commit(&bar->o_full);
                ++on;
                ++qn;
                rc += 2 * static_cast<uint32_t>(count);
                tc += static_cast<uint32_t>(count);
            }
            // every MMA issued by this thread completes before TMEM is released
            mma_commit(&bar->drain);
            mbar_wait_teardown(&bar->drain, 0);
        }
    } else {
        // ------------------------------------------------ softmax / epilogue (warps 0-3)
        const int r = threadIdx.x;                                  // tile row = TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        uint32_t it = 0, tc = 0, qn = 0, on = 0;  // items read, tiles, Q loads, outputs
        bool ok = true;
        // Items are read in queue order; item number n sits in slot n & 1.  A pair's
        // slot also holds its key-block union, so the slot is released only after the
        // item's last tile (release_item); a row's slot is released at once.
        auto next_item = [&](int4 &out) {
            const uint32_t k = it & 1;
            if (!mbar_wait(&bar->sched_full[k], (it >> 1) & 1, abort_flag, dev_status)) return false;
            out = bar->sched_item[k];
            __syncwarp();
            if (!C::PAIR && lane == 0) mbar_arrive(&bar->sched_empty[k]);
            ++it;
            return true;
        };
        auto release_item = [&](uint32_t n) {
            if (C::PAIR) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar->sched_empty[n & 1]);
            }
        };
        // This thread's query row of `itm` (zeros past the block or past N) into the
        // Q buffer of Q load number qn, as packed operands (bf16 pairs or e4m3 quads,
        // in order).
        auto load_q = [&](const int4 &itm) {
            const int64_t bhq = itm.x / ipb;
            const int tq = (itm.x % ipb) * kRowsM + r;
            const bool in = tq < N;
            const uint4 *src = reinterpret_cast<const uint4 *>(Qg + (bhq * N + (in ? tq : 0)) * (D * C::EB));
            const uint32_t tQ = tmem + lane_base + ((qn & 1) ? C::T_Q1 : C::T_Q0);
#pragma unroll
            for (int c0 = 0; c0 < static_cast<int>(C::Q_COLS); c0 += 32) {
                uint32_t q[32];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 x = in ? __ldg(src + c0 / 4 + i) : make_uint4(0, 0, 0, 0);
                    q[4 * i] = x.x;
                    q[4 * i + 1] = x.y;
                    q[4 * i + 2] = x.z;
                    q[4 * i + 3] = x.w;
                }
                tmem_st32(tQ + c0, q);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            // Test hook: the queue's first item never has its Q reported as loaded, so
            // the MMA warp's bounded wait for it runs out (exercises the timeout path).
            if (lane == 0 && !(test_stall && itm.w == 1)) mbar_arrive(&bar->q_full[qn & 1]);
        };
        int4 item;
        if (next_item(item)) {
            if (item.w && item.z > 0) load_q(item);
            while (item.w) {
                // rows: item.y = CSR start, item.z = key blocks (tiles); pairs: item.y =
                // union entries, item.z = tiles (two entries each)
                const int start = item.y, count = item.z;
                const uint32_t slot_n = it - 1;  // queue number of this item (its slot: & 1)
                const int64_t bh = item.x / ipb;
                const int t_row = (item.x % ipb) * kRowsM + r;  // token index of this thread's row
                const int qb = t_row / BS;                     // this row's query block
                const int half = C::PAIR ? (r >> 6) : 0;       // pairs: row A (0) or row B (1) of the item
                const uint16_t *ul = uni + (slot_n & 1) * kUnionCap;
                float m = -CUDART_INF_F, l = 0.0f;
                int prev = -1;
                // rows: the next tile's key block, loaded one tile ahead
                int kblk_next = (!C::PAIR && count > 0) ? __ldg(col_idx + start) : 0;
                // e4m3 operands: the row's Q exponent, the running V reference exponent E
                const int eq = (F8 && qb < nb) ? __ldg(q_exp + bh * nb + qb) : 0;
                int e_ref = 0;
                bool have_ref = false;
                for (int j = 0; j < count; ++j) {
                    // the tile's key blocks (-1: none) and whether this row takes each
                    int kb[C::HALVES];
                    bool mine[C::HALVES];
                    if constexpr (C::PAIR) {
#pragma unroll
                        for (int h = 0; h < C::HALVES; ++h) {
                            const int e = (C::HALVES * j + h < start) ? static_cast<int>(ul[C::HALVES * j + h]) : -1;
                            kb[h] = e >= 0 ? (e >> 2) : -1;
                            mine[h] = e >= 0 && ((e >> half) & 1);
                        }
                    } else {
                        kb[0] = kblk_next;
                        if (j + 1 < count) kblk_next = __ldg(col_idx + start + j + 1);
                        mine[0] = true;
                    }
                    // per key block: the keys that exist and are allowed for this row, the
                    // score scale (log2 units) and, for e4m3, the V exponent; E moves up to
                    // the largest V exponent this row has taken
                    int lim[C::HALVES], ev[C::HALVES];
                    float sc[C::HALVES];
                    int e_new = e_ref;
                    bool e_up = false;
#pragma unroll
                    for (int h = 0; h < C::HALVES; ++h) {
                        const bool valid = kb[h] >= 0 && kb[h] < nb && kb[h] > prev;
                        if (valid) prev = kb[h];
                        mine[h] = mine[h] && valid;
                        const int key0 = kb[h] * BS;
                        lim[h] = mine[h] ? min(BS, N - key0) : 0;
                        if (causal) lim[h] = min(lim[h], t_row - key0 + 1);
                        sc[h] = scale_log2;
                        ev[h] = 0;
                        if (F8 && mine[h]) {
                            sc[h] = pow2_scale(scale_log2, eq + __ldg(k_exp + bh * nb + kb[h]));
                            ev[h] = __ldg(v_exp + bh * nb + kb[h]);
                            if (!(have_ref || e_up) || ev[h] > e_new) {
                                e_new = ev[h];
                                e_up = true;
                            }
                        }
                    }
                    const uint32_t sb = tc & 1;
                    if (!mbar_wait(&bar->s_full[sb], (tc >> 1) & 1, abort_flag, dev_status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tS = tmem + lane_base + (sb ? C::T_S1 : C::T_S0);
                    // the whole S row of this thread: kKT fp32 values
                    uint32_t v[kKT];
#pragma unroll
                    for (int c0 = 0; c0 < kKT; c0 += 32)
                        tmem_ld32(tS + c0, *reinterpret_cast<uint32_t(*)[32]>(&v[c0]));
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < C::HALVES; ++h) {
                        if (lim[h] < BS) {  // ragged last block, causal diagonal, a skipped index or none
#pragma unroll
                            for (int c = 0; c < BS; ++c)
                                if (c >= lim[h]) v[h * BS + c] = __float_as_uint(-CUDART_INF_F);
                        }
                    }
                    float mxs = -CUDART_INF_F;
#pragma unroll
                    for (int h = 0; h < C::HALVES; ++h) {
                        float mq[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
                        for (int c = h * BS; c < (h + 1) * BS; c += 8) {
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                mq[q] = max3f(mq[q], __uint_as_float(v[c + 2 * q]), __uint_as_float(v[c + 2 * q + 1]));
                        }
                        mxs = fmaxf(mxs, max3f(mq[0], mq[1], fmaxf(mq[2], mq[3])) * sc[h]);
                    }
                    // The reference maximum only moves when the row maximum exceeds it by
                    // more than 2^8: P stays below 256 and the rescale of O is rare.  O and
                    // l always share the same reference, so the final O / l is exact.
                    const bool need = mxs > m + kRescaleLog2;
                    const float m_new = need ? mxs : m;
                    const float alpha_m = need ? ex2_approx(m - m_new) : 1.0f;  // rescale of l and O
                    const float neg_m = (m_new == -CUDART_INF_F) ? 0.0f : -m_new;
                    float rs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                    if constexpr (!F8) {
                        // P packed as bf16 pairs in place, v[c/2] <- (p[c], p[c+1]); one loop for
                        // full and masked tiles (masked scores are -inf, and 2^-inf = 0).  The
                        // scaling and the row sums run on fp32 pairs (one instruction per two
                        // columns).
                        uint64_t sc2[C::HALVES];
#pragma unroll
                        for (int h = 0; h < C::HALVES; ++h) sc2[h] = f32x2_pack(sc[h], sc[h]);
                        const uint64_t nm2 = f32x2_pack(neg_m, neg_m);
                        uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
                        for (int c = 0; c < kKT; c += 2) {
                            float x0, x1;
                            f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(v[c]), __uint_as_float(v[c + 1])),
                                                   sc2[c / BS], nm2),
                                         x0, x1);
                            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            acc2[(c >> 1) & 1] = f32x2_add(acc2[(c >> 1) & 1], f32x2_pack(p0, p1));
                            v[c >> 1] = pack_bf16(p0, p1);
                        }
                        f32x2_unpack(acc2[0], rs[0], rs[1]);
                        f32x2_unpack(acc2[1], rs[2], rs[3]);
#pragma unroll
                        for (int c0 = 0; c0 < kKT / 2; c0 += 32)
                            tmem_st32(tS + c0, *reinterpret_cast<const uint32_t(*)[32]>(&v[c0]));
                    } else {
                        // P * 2^(e_v - E) as e4m3 quads in place, v[c/4] <- (p[c] .. p[c+3]).  The
                        // power of two goes into the exponent, 2^(s sc - m + e_v - E), and the
                        // row sum takes the scaled values back by 2^(E - e_v) once per key block
                        // (exact: a power of two).
                        // (scaling and row sums on fp32 pairs, one instruction per two columns)
                        uint64_t sc2[C::HALVES], nm2[C::HALVES], rh2[C::HALVES];
#pragma unroll
                        for (int h = 0; h < C::HALVES; ++h) {
                            const float nmh = neg_m + static_cast<float>(ev[h] - e_new);
                            sc2[h] = f32x2_pack(sc[h], sc[h]);
                            nm2[h] = f32x2_pack(nmh, nmh);
                            rh2[h] = 0ull;
                        }
#pragma unroll
                        for (int c = 0; c < kKT; c += 4) {
                            float x0, x1, x2, x3;
                            f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(v[c]), __uint_as_float(v[c + 1])),
                                                   sc2[c / BS], nm2[c / BS]),
                                         x0, x1);
                            f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(v[c + 2]), __uint_as_float(v[c + 3])),
                                                   sc2[c / BS], nm2[c / BS]),
                                         x2, x3);
                            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            const float p2 = ex2_approx(x2), p3 = ex2_approx(x3);
                            rh2[c / BS] = f32x2_add(f32x2_add(rh2[c / BS], f32x2_pack(p0, p1)), f32x2_pack(p2, p3));
                            v[c >> 2] = pack_e4m3x4(p0, p1, p2, p3);
                        }
                        tmem_st32(tS, *reinterpret_cast<const uint32_t(*)[32]>(&v[0]));
#pragma unroll
                        for (int h = 0; h < C::HALVES; ++h) {
                            float a0, a1;
                            f32x2_unpack(rh2[h], a0, a1);
                            rs[h] = pow2_scale(a0 + a1, e_new - ev[h]);
                        }
                    }
                    float alpha = alpha_m;
                    if (F8 && e_up && have_ref) alpha = pow2_scale(alpha_m, e_ref - e_new);  // O in units of 2^E
                    l = l * alpha_m + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
                    // Rescale the running output.  The PV of the previous block may still be
                    // accumulating into O: wait for it first (its completion is phase tc-1
                    // of pv_done; the PV of this block cannot start before P is published).
                    // (a row without an earlier block, m = -inf, has O = 0: nothing to rescale)
                    if (__any_sync(0xffffffffu, (need && m != -CUDART_INF_F) || (e_up && have_ref))) {
                        if (!mbar_wait(&bar->pv_done, (tc - 1) & 1, abort_flag, dev_status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t tO = tmem + lane_base + C::T_O;
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
                    if (lane == 0) mbar_arrive(&bar->p_full[sb]);
                    m = m_new;
                    e_ref = e_new;
                    have_ref = have_ref || e_up;
                    ++tc;
                }
                if (!ok) break;
                release_item(slot_n);
                if (count > 0) ++qn;
                // the next item's Q goes into TMEM before this item's epilogue, so its first
                // S tiles overlap the epilogue
                int4 nxt;
                if (!next_item(nxt)) break;
                if (nxt.w && nxt.z > 0) load_q(nxt);
                // epilogue
                if (!mbar_wait(&bar->o_full, on & 1, abort_flag, dev_status)) break;
                ++on;
                tc_fence_after();
                const bool row_ok = t_row < N;
                const float inv_l = (l > 0.0f) ? (F8 ? pow2_scale(1.0f / l, e_ref) : 1.0f / l) : 0.0f;
                __nv_bfloat16 *orow = O + (bh * N + t_row) * D;
                const uint32_t tO = tmem + lane_base + C::T_O;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    if (count > 0) {
                        tmem_ld32(tO + c0, o);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = 0u;
                    }
                    uint32_t pkk[16];
#pragma unroll
                    for (int c = 0; c < 32; c += 2)
                        pkk[c >> 1] = pack_bf16(__uint_as_float(o[c]) * inv_l, __uint_as_float(o[c + 1]) * inv_l);
                    if (row_ok) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + c0);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(pkk[4 * q], pkk[4 * q + 1], pkk[4 * q + 2], pkk[4 * q + 3]);
                    }
                }
                if (row_ok)
                    LSE[bh * N + t_row] = (l > 0.0f) ? (m + __log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar->o_empty);
                item = nxt;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (cta_busy_ns && threadIdx.x == 0) {
        long long t_end;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_end));
        cta_busy_ns[blockIdx.x] = t_end - bar->t_start;
    }
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// Block 64: the key-block union size of every pair (one warp per pair), the work
// of its item; also checks the two rows and records FVATTN_ERR_BAD_CSR for a
// malformed one (the attention kernel then uses each row's in-range entries).
constexpr int kPairWarps = 8;
__global__ void __launch_bounds__(kPairWarps * 32)
    pair_count_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx, int64_t BH, int nb,
                      int32_t *__restrict__ counts, int32_t *dev_status) {
    __shared__ uint32_t bm_s[kPairWarps][2 * kBitmapWords];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int np = (nb + 1) >> 1;
    const int nw = (nb + 31) >> 5;
    uint32_t *bm = bm_s[warp];
    for (int64_t pr = static_cast<int64_t>(blockIdx.x) * kPairWarps + warp; pr < BH * np;
         pr += static_cast<int64_t>(gridDim.x) * kPairWarps) {
        const bool bad = pair_bitmaps<true>(row_ptr, col_idx, pr / np, static_cast<int>(pr % np), nb, bm, lane);
        if (bad && lane == 0) record_error(dev_status, FVATTN_ERR_BAD_CSR);
        int c = 0;
        for (int w = lane; w < nw; w += 32) c += __popc(bm[w] | bm[nw + w]);
        c = __reduce_add_sync(0xffffffffu, c);
        if (lane == 0) counts[pr] = c;
        __syncwarp();  // the bitmaps are reused by the next pair
    }
}

// Natural order (rows by index), the comparison point for the load-imbalance factor.
__global__ void natural_order_kernel(int64_t n, int32_t *__restrict__ order) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        order[i] = static_cast<int32_t>(i);
}

// ------------------------------------------------------------- work order
// Items (CSR rows) are ordered head-major, longest first: heads by their total
// selected blocks (descending, equal totals by head index), and inside a head
// the rows by their block count (descending, equal counts by row index).  All
// SMs then work on about one head at a time, whose K and V stay in L2, and the
// grid ends on the lightest head's shortest rows.

constexpr int kOrderThreads = 1024;

// "x comes after y": key descending, index ascending.
__device__ __forceinline__ bool later(int kx, int ix, int ky, int iy) { return kx < ky || (kx == ky && ix > iy); }

// Sorts np2 (a power of two) (key, index) pairs in shared memory into "later" order.
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

// One CTA per head: its rows sorted by block count, written at head_rank[h] * nb.
__global__ void __launch_bounds__(kOrderThreads) row_order_kernel(const int32_t *__restrict__ row_ptr, int nb,
                                                                  int np2, const int32_t *__restrict__ head_rank,
                                                                  int32_t *__restrict__ order) {
    extern __shared__ int sm_order[];
    int *key = sm_order, *idx = sm_order + np2;
    const int64_t bh = blockIdx.x;
    for (int e = threadIdx.x; e < np2; e += blockDim.x) {
        if (e < nb) {
            const int64_t rw = bh * nb + e;
            key[e] = row_ptr[rw + 1] - row_ptr[rw];
            idx[e] = e;
        } else {
            key[e] = -1;
            idx[e] = 0x7fffffff;
        }
    }
    __syncthreads();
    bitonic_sort(key, idx, np2);
    const int64_t base = static_cast<int64_t>(head_rank[bh]) * nb;
    for (int e = threadIdx.x; e < nb; e += blockDim.x) order[base + e] = static_cast<int32_t>(bh * nb + idx[e]);
}

}  // namespace

// ------------------------------------------------------------------ launcher

int attn_smem_bytes(int d, int bs) {
    if (d == 128 && bs == 128) return Cfg<128, 128, false>::SMEM_BYTES;
    if (d == 128 && bs == 64) return Cfg<128, 64, false>::SMEM_BYTES;
    if (d == 64 && bs == 128) return Cfg<64, 128, false>::SMEM_BYTES;
    return Cfg<64, 64, false>::SMEM_BYTES;
}

int attn_ctas_per_sm() { return kCtasPerSm; }

int64_t attn_num_items(int64_t BH, int nb, int bs) { return BH * (bs == 64 ? (nb + 1) / 2 : nb); }

cudaError_t launch_pair_counts(const int32_t *row_ptr, const int32_t *col_idx, int64_t BH, int nb, int32_t *counts,
                               int32_t *dev_status, cudaStream_t stream) {
    const int64_t pairs = BH * ((nb + 1) / 2);
    const int64_t need = (pairs + kPairWarps - 1) / kPairWarps;
    const int grid = static_cast<int>(need < 4096 ? (need > 0 ? need : 1) : 4096);
    pair_count_kernel<<<grid, kPairWarps * 32, 0, stream>>>(row_ptr, col_idx, BH, nb, counts, dev_status);
    return cudaGetLastError();
}

static int pow2_at_least(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

cudaError_t launch_item_order(const int32_t *row_ptr, int64_t BH, int nb, int32_t *head_rank, int32_t *order,
                              cudaStream_t stream) {
    const int hp2 = pow2_at_least(static_cast<int>(BH));
    const int ip2 = pow2_at_least(nb);
    head_rank_kernel<<<1, kOrderThreads, 2 * hp2 * sizeof(int), stream>>>(row_ptr, static_cast<int>(BH), nb, hp2,
                                                                           head_rank);
    row_order_kernel<<<static_cast<unsigned>(BH), kOrderThreads, 2 * ip2 * sizeof(int), stream>>>(row_ptr, nb, ip2,
                                                                                                  head_rank, order);
    return cudaGetLastError();
}

cudaError_t launch_natural_order(int64_t n, int32_t *order, cudaStream_t stream) {
    const int grid = static_cast<int>(n / 256 + 1 < 1024 ? n / 256 + 1 : 1024);
    natural_order_kernel<<<grid, 256, 0, stream>>>(n, order);
    return cudaGetLastError();
}

template <int D, int BS, bool F8>
static cudaError_t launch_t(const AttnLaunch &a, cudaStream_t stream) {
    auto kern = sparse_attn_fwd_kernel<D, BS, F8>;
    // Checked once per instantiation: the number of resident CTAs per SM sizes the
    // persistent grid.
    static int per_sm = 0;  // 0 unknown, > 0 resident CTAs per SM, < 0 not launchable
    if (per_sm == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D, BS, F8>::SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        int occ = 0;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, Cfg<D, BS, F8>::SMEM_BYTES)) !=
            cudaSuccess)
            return e;
        if (occ < 1) {
            set_last_error("attention kernel: no CTA fits on an SM");
            per_sm = -1;
        } else {
            per_sm = occ < kCtasPerSm ? occ : kCtasPerSm;
        }
    }
    if (per_sm < 0) return cudaErrorInvalidConfiguration;
    const int64_t cap = static_cast<int64_t>(per_sm) * a.sms;
    const int grid = static_cast<int>(a.n_items < cap ? a.n_items : cap);
    if (a.grid_out) *a.grid_out = grid;
    if (grid <= 0) return cudaSuccess;
    kern<<<grid, kThreads, Cfg<D, BS, F8>::SMEM_BYTES, stream>>>(
        *a.tmap_k, *a.tmap_v, static_cast<const unsigned char *>(a.Q), a.row_ptr, a.col_idx, a.order, a.n_items,
        a.work_counter, a.N, a.nb, a.causal, a.scale_log2, static_cast<__nv_bfloat16 *>(a.O), a.LSE, a.dev_status,
        a.test_stall, a.cta_busy_ns, a.q_exp, a.k_exp, a.v_exp);
    return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const AttnLaunch &a, int d, int bs, cudaStream_t stream) {
    if (d == 128 && bs == 128) return launch_t<128, 128, false>(a, stream);
    if (d == 128 && bs == 64) return launch_t<128, 64, false>(a, stream);
    if (d == 64 && bs == 128) return launch_t<64, 128, false>(a, stream);
    return launch_t<64, 64, false>(a, stream);
}

cudaError_t launch_sparse_attn_fp8(const AttnLaunch &a, int bs, cudaStream_t stream) {
    if (bs == 128) return launch_t<128, 128, true>(a, stream);
    return launch_t<128, 64, true>(a, stream);
}

}  // namespace fvattn
