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
