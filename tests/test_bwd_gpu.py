"""Gradient parity on the GPU: fvattn_sparse_bwd against the fp64 oracle's
derivatives of sum(dO * O), applied to the GPU's routed mask (FVAttn review, §1
"Top-p routing"; FlashAttention review, §Background "Motivation" for the
forward it differentiates)."""
import numpy as np
import pytest
import torch

import workloads as W
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu


def rand_bits(rng, shape):
    return W.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


# Tolerance, from the arithmetic: P and dS are rounded to bf16 (relative 2^-9) before
# the tensor-core products, which accumulate in fp32, and the outputs are rounded to
# bf16 (2^-9).  dQ = sum_u dS_u k_u / sqrt(d) sums terms whose dS add up to zero in
# every row, so its relative error is 2^-9 times the cancellation ratio
# sum |dS k| / |sum dS k| (a few on peaked rows): 2e-2 in the Frobenius norm leaves
# a factor ~10; the largest single error is held to 3e-2 of the largest entry.
REL_FRO, REL_MAX = 2e-2, 3e-2


def grads_close(name, got, ref):
    """bf16 gradients against fp64: relative Frobenius error and largest error
    relative to the largest reference entry."""
    g = got.float().cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)
    mx = np.max(np.abs(g - ref)) / max(np.max(np.abs(ref)), 1e-30)
    print(f"{name}: rel fro {rel:.2e}, max/maxref {mx:.2e}")
    assert rel < REL_FRO, (name, rel)
    assert mx < REL_MAX, (name, mx)


def run_case(oracle_mod, B, H, N, d, p=None, causal=False, seed=0, csr=None):
    import top_routed_block_b200 as fv
    rng = np.random.default_rng(seed)
    if p is not None:
        w = W.Workload("bwd", B=B, H=H, N=N, d=d, bs=128, p=p, dist="structured", grid=(1, 1, N),
                       head_scale=("uniform", 0.5, 4.0), seed=seed)
        Q, K, V = W.generate(w)
    else:
        Q, K, V = (rand_bits(rng, (B, H, N, d)) for _ in range(3))
    dO = rand_bits(rng, (B, H, N, d))
    dQ_, dK_, dV_, dO_ = (to_dev(x) for x in (Q, K, V, dO))
    if csr is None:
        r = fv.fvattn_route(dQ_, dK_, p, 128)
        fv.check_status(r.dev_status, "route")
        rp_t, ci_t = r.row_ptr, r.col_idx
    else:
        rp_t = torch.from_numpy(csr[0]).cuda()
        ci_t = torch.from_numpy(csr[1] if csr[1].size else np.zeros(1, np.int32)).cuda()
    O, LSE, st = fv.fvattn_sparse_fwd(dQ_, dK_, dV_, rp_t, ci_t, 128, causal)
    fv.check_status(st, "fwd")
    gQ, gK, gV, st = fv.fvattn_sparse_bwd(dQ_, dK_, dV_, O, LSE, dO_, rp_t, ci_t, 128, causal)
    fv.check_status(st, "bwd")
    rp = rp_t.cpu().numpy()
    ci = ci_t[: int(rp[-1])].cpu().numpy()
    rQ, rK, rV = oracle_mod.attn_bwd(Q, K, V, dO, 128, causal, rp, ci)
    grads_close("dQ", gQ, rQ)
    grads_close("dK", gK, rK)
    grads_close("dV", gV, rV)
    # deterministic: no atomics anywhere
    gQ2, gK2, gV2, st = fv.fvattn_sparse_bwd(dQ_, dK_, dV_, O, LSE, dO_, rp_t, ci_t, 128, causal)
    fv.check_status(st, "bwd again")
    assert torch.equal(gQ, gQ2) and torch.equal(gK, gK2) and torch.equal(gV, gV2)


@pytest.mark.parametrize("d", [128, 64])
def test_bwd_routed_ragged(oracle_mod, d):
    run_case(oracle_mod, B=1, H=3, N=1000, d=d, p=0.8, seed=51)


def test_bwd_dense_causal(oracle_mod):
    csr = oracle_mod.dense_csr(1, 2, 640, 128, causal=True)
    run_case(oracle_mod, B=1, H=2, N=640, d=128, causal=True, seed=52, csr=csr)


def test_bwd_dense_non_causal_two_batches(oracle_mod):
    csr = oracle_mod.dense_csr(2, 2, 512, 128, causal=False)
    run_case(oracle_mod, B=2, H=2, N=512, d=128, seed=53, csr=csr)


def test_bwd_user_mask_with_empty_rows_and_unselected_keys(oracle_mod):
    # 5 blocks per head; row 1 selects nothing, block 3 is selected by no row
    rows = [[0, 2], [], [0, 1, 2, 4], [4], [1, 2]]
    rp, ci = [0], []
    for _h in range(2):
        for r in rows:
            ci.extend(r)
            rp.append(len(ci))
    csr = (np.asarray(rp, np.int32), np.asarray(ci, np.int32))
    run_case(oracle_mod, B=1, H=2, N=600, d=64, seed=54, csr=csr)


def test_bwd_routed_more_blocks_and_heads(oracle_mod):
    """32 key blocks per head and 8 heads, routed at p = 0.9: long CSR rows and
    columns, several items per CTA."""
    run_case(oracle_mod, B=1, H=8, N=4096, d=128, p=0.9, seed=55)


def _cheap_key_groups(rp, ci, w, rng, max_groups=10, max_select=2, per_block=4):
    """Sampled key tokens for dK/dV at full size: key blocks that at most
    ``max_select`` query blocks select (at least one), one per head in a seeded
    head order, up to ``max_groups`` heads; four tokens per block, the ragged tail
    included when it is the block.  The oracle rebuilds every selecting query
    row's softmax for each block, so this bounds its work."""
    BH, nb = w.B * w.H, w.nb
    toks, rows = [], 0
    for bh in rng.permutation(BH):
        if len(toks) == max_groups:
            break
        cols = ci[rp[bh * nb]:rp[(bh + 1) * nb]]
        counts = np.bincount(cols, minlength=nb)
        sel = np.flatnonzero((counts > 0) & (counts <= max_select))
        if sel.size == 0:
            continue
        kb = int(rng.choice(sel))
        rows += int(counts[kb]) * w.bs
        t0, t1 = kb * w.bs, min(w.N, (kb + 1) * w.bs)
        ts = rng.choice(np.arange(t0, t1), size=min(per_block, t1 - t0), replace=False)
        toks.append(bh * w.N + np.sort(ts))
    return (np.concatenate(toks).astype(np.int64) if toks else np.zeros(0, np.int64)), rows


FULL_BWD = [(W.VIDEO, False), (W.DENSE_CAUSAL, True), (W.LONG, False)]


@pytest.mark.parametrize("w,causal", FULL_BWD, ids=lambda x: x.name if hasattr(x, "name") else str(x))
def test_bwd_full_size_sampled(w, causal, oracle_mod):
    """Full-size gradients (video: the configuration the benchmark times; long video:
    118,800 tokens with a 16-token last block) on
    samples: dQ rows of query blocks 0, the ragged last one and two random ones in
    every head, and dK/dV rows of key blocks selected by one or two query blocks
    (which bounds the oracle's work) in up to ten heads.  The mask comes from the oracle's own
    routing (video, long video) or is the dense causal one, so no oracle input comes
    from the GPU; O and LSE for the backward come from the GPU forward on that mask."""
    import top_routed_block_b200 as fv
    rng = np.random.default_rng(61)
    Q, K, V = W.generate(w)
    if causal:
        rp, ci = oracle_mod.dense_csr(w.B, w.H, w.N, w.bs, True)
    else:
        r = oracle_mod.route(Q, K, w.p, w.bs)
        rp, ci = r.row_ptr, r.col_idx
    dO = W.f32_to_bf16_bits(rng.standard_normal(Q.shape).astype(np.float32))
    dQ_, dK_, dV_, dO_ = (to_dev(x) for x in (Q, K, V, dO))
    rp_t = torch.from_numpy(np.ascontiguousarray(rp, np.int32)).cuda()
    ci_t = torch.from_numpy(np.ascontiguousarray(ci, np.int32)).cuda()
    O, LSE, st = fv.fvattn_sparse_fwd(dQ_, dK_, dV_, rp_t, ci_t, w.bs, causal)
    fv.check_status(st, "fwd")
    gQ, gK, gV, st = fv.fvattn_sparse_bwd(dQ_, dK_, dV_, O, LSE, dO_, rp_t, ci_t, w.bs, causal)
    fv.check_status(st, "bwd")
    q_tok = W.sample_tokens(w, per_head_blocks=2, rows_per_block=2)
    k_tok, rows = _cheap_key_groups(rp, ci, w, rng)
    assert k_tok.size >= 8, "no affordable key blocks to sample"
    rq, rk, rv = oracle_mod.attn_bwd_sampled(Q, K, V, dO, w.bs, causal, rp, ci, q_tok, k_tok)
    d = w.d
    grads_close("dQ (sampled)", gQ.reshape(-1, d)[torch.from_numpy(q_tok).cuda()], rq)
    kt = torch.from_numpy(k_tok).cuda()
    grads_close("dK (sampled)", gK.reshape(-1, d)[kt], rk)
    grads_close("dV (sampled)", gV.reshape(-1, d)[kt], rv)
    print(w.name, "query rows", q_tok.size, "key rows", k_tok.size, "oracle query rows rebuilt", rows)
