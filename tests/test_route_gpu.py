"""Routing parity on the GPU: the CSR block mask from fvattn_route against the
fp64 oracle, bit-exact up to the near-p exclusion (FVAttn review, §1 Key
Terms "Top-p routing"; score as fixed by this library)."""
import numpy as np
import pytest

import workloads as W
from tests.gpu_util import compare_routes, gpu_route, to_dev

pytestmark = pytest.mark.gpu

SMALL = [
    W.TINY,
    W.Workload("small_ragged_d128", B=1, H=3, N=1000, d=128, bs=128, p=0.7, dist="structured", grid=(5, 8, 25),
               head_scale=("uniform", 0.5, 4.0), seed=31),
    W.Workload("small_b2_d64_bs128", B=2, H=2, N=777, d=64, bs=128, p=0.5, dist="structured", grid=(7, 3, 37),
               head_scale=("uniform", 1.0, 6.0), seed=32),
    W.Workload("small_bs64_d128", B=1, H=3, N=2000, d=128, bs=64, p=0.9, dist="structured", grid=(5, 20, 20),
               head_scale=("uniform", 0.5, 4.0), seed=33),
    W.Workload("small_many_blocks", B=1, H=2, N=1024 * 64 - 5, d=64, bs=64, p=0.95, dist="structured",
               grid=(1, 1, 1024 * 64 - 5), head_scale=("uniform", 0.5, 4.0), seed=34),
    W.Workload("single_block", B=1, H=2, N=50, d=64, bs=64, p=0.9, seed=35),
    W.Workload("p_one_small", B=2, H=2, N=700, d=128, bs=128, p=1.0, seed=36),
    # key-block counts that land in each register-sort width of the selection kernel
    W.Workload("nb47_d64", B=1, H=3, N=3000, d=64, bs=64, p=0.8, dist="structured", grid=(3, 10, 100),
               head_scale=("uniform", 0.5, 4.0), seed=37),
    W.Workload("nb313_d64", B=1, H=2, N=20000, d=64, bs=64, p=0.9, dist="structured", grid=(5, 40, 100),
               head_scale=("uniform", 0.5, 4.0), seed=38),
    W.Workload("nb600_d128", B=1, H=2, N=600 * 64 - 17, d=128, bs=64, p=0.7, dist="structured",
               grid=(1, 1, 600 * 64 - 17), head_scale=("uniform", 0.5, 8.0), seed=39),
]


def run_case(w, oracle_mod):
    Q, K, _ = W.generate(w)
    ora = oracle_mod.route(Q, K, w.p, w.bs)
    gpu = gpu_route(to_dev(Q), to_dev(K), w.p, w.bs)
    excluded = compare_routes(gpu, ora, w.p, w.nb, w.B * w.H)
    print(f"{w.name}: rows {w.rows} nnz {gpu[0][-1]} excluded(near p) {excluded} "
          f"near-tie cuts (checked bit-exact) {compare_routes.last_near_ties}")
    return gpu, ora


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_route_small(w, oracle_mod):
    run_case(w, oracle_mod)


@pytest.mark.parametrize("w", [W.VIDEO, W.DENSE, W.LONG], ids=lambda w: w.name)
def test_route_full_size(w, oracle_mod):
    (rp, ci, hc), ora = run_case(w, oracle_mod)
    if w.p >= 1.0:
        assert np.all(np.diff(rp) == w.nb)


@pytest.mark.parametrize("w", W.sweep(), ids=lambda w: w.name)
def test_route_sweep(w, oracle_mod):
    run_case(w, oracle_mod)


def test_route_capacity_overflow_reported(oracle_mod):
    """A col_idx buffer smaller than the selection sets FVATTN_ERR_CAPACITY and
    leaves row_ptr complete."""
    import torch
    import top_routed_block_b200 as fv
    w = SMALL[1]
    Q, K, _ = W.generate(w)
    ora = oracle_mod.route(Q, K, w.p, w.bs)
    dQ, dK = to_dev(Q), to_dev(K)
    out = fv.RouteResult(torch.empty(w.rows + 1, dtype=torch.int32, device="cuda"),
                         torch.empty(4, dtype=torch.int32, device="cuda"),
                         torch.empty(w.B * w.H, dtype=torch.int32, device="cuda"),
                         torch.zeros(1, dtype=torch.int32, device="cuda"))
    fv.fvattn_route(dQ, dK, w.p, w.bs, out=out)
    torch.cuda.synchronize()
    assert int(out.dev_status.item()) == fv.FVATTN_ERR_CAPACITY
    assert int(out.row_ptr[-1].item()) == int(ora.row_ptr[-1])


@pytest.mark.parametrize("nb", [1, 8, 47, 128, 256, 313, 929])
def test_route_all_ties_keep_lowest_indices(nb):
    """K = 0 makes every score 0 and every probability exactly 1/nb, so the
    selection is decided by the tie-break alone: the first ceil(p*nb) blocks by
    index (FVAttn review, §1 "Top-p routing"; ties by lower index)."""
    p = 0.3
    bs, d = 64, 64
    N = nb * bs - (5 if nb > 1 else 0)
    rng = np.random.default_rng(nb)
    Q = rng.standard_normal((1, 2, N, d)).astype(np.float32)
    Qb = (Q.view(np.uint32) >> 16).astype(np.uint16)       # bf16 by truncation: any values will do
    Kb = np.zeros_like(Qb)
    rp, ci, hc = gpu_route(to_dev(Qb), to_dev(Kb), p, bs)
    k = int(np.ceil(p * nb))
    assert np.all(np.diff(rp) == k)
    for row in range(2 * nb):
        assert np.array_equal(ci[rp[row]:rp[row + 1]], np.arange(k))
    assert np.all(hc == k * nb)
