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
