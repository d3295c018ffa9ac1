"""Slack-aware augmentation on the GPU (fvattn_route_sasa) against the oracle
(FVAttn review, §1 Key Terms "SASA" and §3; reading: the ranks are the SMs of the
persistent attention grid, the list schedule of the attention queue fixes each
machine's slack, which is filled round robin with its rows' next routing
candidates).

Small cases: the oracle routes, orders and augments on its own; the GPU's
augmented CSR and added counts are equal to its, bit for bit, and the added
probability mass within 1e-12 (the GPU's softmax uses CUDA's fp64 exp).  Each
small case is checked first to have no row whose kept mass lies within 1e-6 of
p, where the two routings may legitimately differ.

Full size (video): the routing candidates the GPU reports equal the oracle's on
every row that is not within 1e-6 of p; the plan is then checked, bit for bit,
against the oracle's augmentation applied to the GPU's own routed mask and
candidates (as attention parity checks O on the GPU's own mask)."""
import numpy as np
import pytest
import torch

import workloads as W
from tests.gpu_util import near_p_rows, to_dev

pytestmark = pytest.mark.gpu

SMALL = [
    W.Workload("sasa_routed", B=1, H=4, N=3000, d=128, bs=128, p=0.7, dist="structured", grid=(5, 20, 30),
               head_scale=("uniform", 0.5, 4.0), seed=81),
    W.Workload("sasa_bs64", B=2, H=3, N=2000, d=64, bs=64, p=0.8, dist="structured", grid=(5, 20, 20),
               head_scale=("uniform", 0.5, 4.0), seed=82),
    W.Workload("sasa_iid", B=1, H=2, N=1024, d=64, bs=64, p=0.6, seed=83),
    # more than 256 key blocks per row (the selection sorts 512 positions per row)
    W.Workload("sasa_wide", B=1, H=2, N=20000, d=64, bs=64, p=0.8, dist="structured", grid=(5, 40, 100),
               head_scale=("uniform", 0.5, 4.0), seed=84),
]


def gpu_sasa(w, Q, K, machines):
    import top_routed_block_b200 as fv
    r = fv.fvattn_route_sasa(to_dev(Q), to_dev(K), w.p, w.bs, machines, candidates=True)
    fv.check_status(r.dev_status, "fvattn_route_sasa")
    rp = r.row_ptr.cpu().numpy()
    return (rp, r.col_idx[: int(rp[-1])].cpu().numpy(), r.head_counts.cpu().numpy(), r.added.cpu().numpy(),
            r.added_mass.cpu().numpy(), r.cand.cpu().numpy(), r.cand_p.cpu().numpy())


def check_against(s_ref, got, BH, nb):
    rp, ci, hc, added, mass = got[:5]
    assert np.array_equal(added, s_ref.added)
    assert np.array_equal(rp, s_ref.row_ptr)
    assert np.array_equal(ci, s_ref.col_idx)
    assert np.array_equal(hc, np.diff(rp.astype(np.int64)).reshape(BH, nb).sum(1))
    assert np.allclose(mass, s_ref.added_mass, rtol=1e-12, atol=0)


@pytest.mark.parametrize("machines", [1, 3, 16, 148, 256])
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_sasa_small_independent(w, machines, oracle_mod):
    Q, K, _ = W.generate(w)
    r, cand, cand_p = oracle_mod.route_candidates(Q, K, w.p, w.bs, 8)
    assert not near_p_rows(r, w.p).any(), "choose a case without near-p rows"
    order = oracle_mod.head_order(r.row_ptr, w.B * w.H, w.nb)
    s_ref = oracle_mod.sasa(r.row_ptr, r.col_idx, cand, cand_p, order, machines)
    got = gpu_sasa(w, Q, K, machines)
    assert np.array_equal(got[5], cand)
    assert np.allclose(got[6], cand_p, rtol=1e-12, atol=0)
    check_against(s_ref, got, w.B * w.H, w.nb)
    if machines == 1:
        assert not s_ref.added.any()


@pytest.mark.slow
def test_sasa_video_full_size(oracle_mod):
    import top_routed_block_b200 as fv
    w = W.VIDEO
    Q, K, _ = W.generate(w)
    machines = torch.cuda.get_device_properties(0).multi_processor_count
    got = gpu_sasa(w, Q, K, machines)
    rp_g, ci_g, _, added, mass, cand_g, cand_pg = got
    # the routed mask underneath (same routing as fvattn_route) and the candidates
    base = fv.fvattn_route(to_dev(Q), to_dev(K), w.p, w.bs)
    fv.check_status(base.dev_status)
    brp = base.row_ptr.cpu().numpy()
    bci = base.col_idx[: int(brp[-1])].cpu().numpy()
    r, cand, cand_p = oracle_mod.route_candidates(Q, K, w.p, w.bs, 8)
    ok = ~near_p_rows(r, w.p)
    assert np.array_equal(cand_g[ok], cand[ok])
    assert np.allclose(cand_pg[ok], cand_p[ok], rtol=1e-12, atol=0)
    order = oracle_mod.head_order(brp, w.B * w.H, w.nb)
    s_ref = oracle_mod.sasa(brp, bci, cand_g, cand_pg, order, machines)
    check_against(s_ref, got, w.B * w.H, w.nb)
    # the augmented mask contains the routed one
    for row in range(0, w.rows, 97):
        assert set(bci[brp[row]:brp[row + 1]]) <= set(ci_g[rp_g[row]:rp_g[row + 1]])
    print(f"video: {int(added.sum())} blocks added over {machines} machines to {int((added > 0).sum())} rows, "
          f"mass {mass.sum():.4f}")


@pytest.mark.parametrize("w", [SMALL[0], SMALL[1]], ids=lambda w: w.name)
def test_attention_on_the_augmented_mask(w, oracle_mod):
    """The augmented mask drives the attention like any mask (at block 64 the paired
    query blocks walk the union of their augmented lists): every token against the
    oracle on that mask."""
    import top_routed_block_b200 as fv
    from tests.gpu_util import compare_attention
    Q, K, V = W.generate(w)
    dQ, dK, dV = to_dev(Q), to_dev(K), to_dev(V)
    r = fv.fvattn_route_sasa(dQ, dK, w.p, w.bs, 148)
    fv.check_status(r.dev_status, "fvattn_route_sasa")
    assert int(r.added.sum().item()) > 0, "choose a case where the plan adds blocks"
    O, LSE, st = fv.fvattn_sparse_fwd(dQ, dK, dV, r.row_ptr, r.col_idx, w.bs, False)
    fv.check_status(st, "forward on the augmented mask")
    rp = r.row_ptr.cpu().numpy()
    ci = r.col_idx[: int(rp[-1])].cpu().numpy()
    tokens = np.arange(w.B * w.H * w.N, dtype=np.int64)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, False, rp, ci, tokens)
    compare_attention(O, LSE, Oref, Lref, tokens, w.d, w.name)


def test_sasa_rejects_bad_machine_counts():
    # null pointers: were the machine check to regress, the null check would still stop the call
    import top_routed_block_b200 as fv
    lib = fv.load_library()
    for m in (0, 257):
        assert lib.fvattn_route_sasa(None, None, 1, 1, 256, 64, 64, 0.5, m, None, None, 0, None, None, None, None,
                                     None, None, 0, None, None) == fv.FVATTN_ERR_UNSUPPORTED
