"""Longest-first work order on the GPU against the oracle's sort, bit-exact
(FVAttn review, §1 "RLB" and §3: per-head work balanced once the mask is known;
here the rows are ordered by selected-block count, ties by row id)."""
import numpy as np
import pytest
import torch

import workloads as W
from tests.gpu_util import gpu_route, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,maxc,seed", [(1, 1, 0), (17, 8, 1), (1024, 256, 2), (1025, 256, 3),
                                            (10240, 256, 4), (22296, 929, 5), (70000, 4096, 6)])
def test_lpt_random_counts(rows, maxc, seed, oracle_mod):
    import top_routed_block_b200 as fv
    rng = np.random.default_rng(seed)
    counts = rng.integers(0, maxc + 1, size=rows)
    counts[rng.random(rows) < 0.3] = maxc // 2      # many ties
    rp = np.zeros(rows + 1, np.int32)
    rp[1:] = np.cumsum(counts)
    order, st = fv.fvattn_lpt_order(torch.from_numpy(rp).cuda(), maxc)
    fv.check_status(st)
    assert np.array_equal(order.cpu().numpy(), oracle_mod.lpt_order(rp))


def test_lpt_on_routed_mask(oracle_mod):
    import top_routed_block_b200 as fv
    w = W.VIDEO
    Q, K, _ = W.generate(w)
    rp, _, _ = gpu_route(to_dev(Q), to_dev(K), w.p, w.bs)
    order, st = fv.fvattn_lpt_order(torch.from_numpy(rp).cuda(), w.nb)
    fv.check_status(st)
    assert np.array_equal(order.cpu().numpy(), oracle_mod.lpt_order(rp))


def test_lpt_count_out_of_range_reported():
    import top_routed_block_b200 as fv
    rp = np.array([0, 3, 20, 22], np.int32)   # row 1 holds 17 > max_count
    order, st = fv.fvattn_lpt_order(torch.from_numpy(rp).cuda(), 8)
    torch.cuda.synchronize()
    assert int(st.item()) == fv.FVATTN_ERR_BAD_CSR


def _head_major_order(rp, BH, nb):
    """Brute force: heads by total selected blocks (descending, ties by lower head),
    then the rows of each head by block count (descending, ties by lower row)."""
    counts = np.diff(rp.astype(np.int64)).reshape(BH, nb)
    heads = sorted(range(BH), key=lambda h: (-int(counts[h].sum()), h))
    out = []
    for h in heads:
        out += [h * nb + i for i in sorted(range(nb), key=lambda i: (-int(counts[h, i]), i))]
    return np.array(out, np.int32)


def _expected_items(rp, ci, BH, nb, block, oracle_mod):
    """The items' CSR: the rows at block 128, the oracle's pairs at block 64."""
    if block == 128:
        return rp, nb
    pp, _, _ = oracle_mod.pair_items(rp, ci, BH, nb)
    return pp, (nb + 1) // 2


@pytest.mark.parametrize("B,H,N,block,maxc,seed", [(1, 1, 128, 128, 1, 0), (1, 3, 1000, 128, 8, 1),
                                                   (2, 5, 4000, 64, 63, 2), (1, 3, 900, 64, 15, 7),
                                                   (1, 40, 32760, 128, 256, 3), (4, 1024, 1280, 128, 10, 4),
                                                   (1, 8, 32768, 64, 512, 5)])
def test_attention_work_order_is_head_major_longest_first(B, H, N, block, maxc, seed, oracle_mod):
    """The queue fvattn_sparse_fwd pops its work items from, against a brute-force sort
    (many equal counts and equal head totals, so the tie-breaks are exercised).  At
    block 64 an item is a pair of rows (query blocks 2i, 2i+1) sized by the union of
    their key blocks, from the oracle."""
    import top_routed_block_b200 as fv
    rng = np.random.default_rng(seed)
    nb = -(-N // block)
    BH = B * H
    counts = rng.integers(0, min(maxc, nb) + 1, size=(BH, nb))
    counts[rng.random((BH, nb)) < 0.4] = min(maxc, nb) // 2
    if BH >= 4:
        counts[1] = counts[3]                     # two heads with equal totals
    rp = np.zeros(BH * nb + 1, np.int32)
    rp[1:] = np.cumsum(counts.reshape(-1))
    ci = np.concatenate([np.sort(rng.choice(nb, size=int(c), replace=False)) for c in counts.reshape(-1)]
                        + [np.zeros(0, np.int64)]).astype(np.int32)
    if BH >= 4:
        # equal head totals at block 64 too: head 1 repeats head 3's lists
        ci1 = ci[rp[3 * nb]:rp[4 * nb]]
        ci = np.concatenate([ci[:rp[nb]], ci1, ci[rp[2 * nb]:]]).astype(np.int32)
    dci = torch.from_numpy(ci if ci.size else np.zeros(1, np.int32)).cuda()
    order, st = fv.fvattn_attn_work_order(torch.from_numpy(rp).cuda(), B, H, N, block, dci)
    fv.check_status(st, "work order")
    assert order.numel() == fv.fvattn_attn_num_items(B, H, N, block)
    ip, per_head = _expected_items(rp, ci, BH, nb, block, oracle_mod)
    assert np.array_equal(order.cpu().numpy(), _head_major_order(ip, BH, per_head))


@pytest.mark.parametrize("w", [W.VIDEO, W.VIDEO_BS64], ids=lambda w: w.name)
def test_attention_work_order_on_routed_mask(w, oracle_mod):
    import top_routed_block_b200 as fv
    Q, K, _ = W.generate(w)
    rp, ci, _ = gpu_route(to_dev(Q), to_dev(K), w.p, w.bs)
    order, st = fv.fvattn_attn_work_order(torch.from_numpy(rp).cuda(), w.B, w.H, w.N, w.bs,
                                          torch.from_numpy(ci).cuda())
    fv.check_status(st, "work order")
    ip, per_head = _expected_items(rp, ci, w.B * w.H, w.nb, w.bs, oracle_mod)
    assert np.array_equal(order.cpu().numpy(), _head_major_order(ip, w.B * w.H, per_head))


def test_pair_work_order_reports_malformed_rows():
    """Block 64: a row with an index out of range or not ascending is reported as
    FVATTN_ERR_BAD_CSR by the pass that sizes the pairs."""
    import top_routed_block_b200 as fv
    rp = np.array([0, 2, 4, 6, 8], np.int32)                    # one head, nb = 4 (N = 256)
    for ci in ([0, 1, 1, 9, 2, 3, 0, 3], [0, 1, 1, 2, 3, 2, 0, 3], [0, 1, 1, 2, 2, 3, -1, 3]):
        order, st = fv.fvattn_attn_work_order(torch.from_numpy(rp).cuda(), 1, 1, 256, 64,
                                              torch.tensor(ci, dtype=torch.int32).cuda())
        torch.cuda.synchronize()
        assert int(st.item()) == fv.FVATTN_ERR_BAD_CSR, ci
    order, st = fv.fvattn_attn_work_order(torch.from_numpy(rp).cuda(), 1, 1, 256, 64,
                                          torch.tensor([0, 1, 1, 2, 2, 3, 0, 3], dtype=torch.int32).cuda())
    fv.check_status(st, "work order")
    assert order.cpu().tolist() == [0, 1]          # unions {0, 1, 2} and {0, 2, 3}: equal sizes
