"""Helpers shared by the GPU parity tests: move bf16 bit patterns to the device,
run the library, and compare against the oracle with the stated tolerances.

Tolerances (bf16 inputs, fp32 accumulation):
  * routing CSR: bit-exact, except rows whose kept mass with or without the
    last kept block lies within 1e-6 of p (reported, then excluded);
  * O: max |err| <= 2e-2 and mean |err| <= 2e-3 against the oracle run on the
    GPU's own mask;
  * LSE: |err| <= 1e-3.
"""
from __future__ import annotations

import numpy as np
import torch

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3
NEAR_P = 1e-6
NEAR_TIE = 1e-12   # relative probability gap at the cut below which a row is reported as a near-tie


def to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def gpu_route(Q, K, p, bs):
    import top_routed_block_b200 as fv
    r = fv.fvattn_route(Q, K, p, bs)
    fv.check_status(r.dev_status, "fvattn_route")
    rp = r.row_ptr.cpu().numpy()
    ci = r.col_idx[: int(rp[-1])].cpu().numpy()
    return rp, ci, r.head_counts.cpu().numpy()


def near_p_rows(oracle_route, p):
    g = oracle_route.diag
    if p >= 1.0:
        return np.zeros(g.shape[0], bool)
    return (np.abs(g[:, 0] - p) < NEAR_P) | (np.abs(g[:, 1] - p) < NEAR_P)


def near_tie_rows(oracle_route, p):
    """Rows whose cut falls between two blocks of almost equal probability (relative
    gap below 1e-12): a swap there would change the set without moving the mass near
    p.  Reported, and still held to bit-exactness (the fp64 pipelines agree to ~1e-15)."""
    g = oracle_route.diag
    if p >= 1.0:
        return np.zeros(g.shape[0], bool)
    has_next = np.isfinite(g[:, 3])
    return has_next & ((g[:, 4] - g[:, 5]) <= NEAR_TIE * g[:, 4])


def compare_routes(gpu, ora, p, nb, BH):
    """Returns the number of excluded rows; asserts everything else is identical.
    Rows with a near-tie at the cut are counted in `compare_routes.last_near_ties`."""
    rp, ci, hc = gpu
    near = near_p_rows(ora, p)
    rows = rp.size - 1
    assert rows == ora.row_ptr.size - 1
    gc = np.diff(rp)
    oc = np.diff(ora.row_ptr)
    bad = []
    for r in range(rows):
        if near[r]:
            continue
        if gc[r] != oc[r] or not np.array_equal(ci[rp[r]:rp[r + 1]], ora.col_idx[ora.row_ptr[r]:ora.row_ptr[r + 1]]):
            bad.append(r)
    assert not bad, f"{len(bad)} routing rows differ, first {bad[:5]}"
    # the GPU CSR is well formed everywhere, excluded rows included
    assert rp[0] == 0 and np.all(gc >= 1) and np.all(gc <= nb)
    for r in range(rows):
        row = ci[rp[r]:rp[r + 1]]
        assert np.all(np.diff(row) > 0) and row[0] >= 0 and row[-1] < nb
    heads_ok = ~near.reshape(BH, nb).any(1)
    assert np.array_equal(hc[heads_ok], ora.head_counts[heads_ok])
    assert np.array_equal(hc, gc.reshape(BH, nb).sum(1))
    compare_routes.last_near_ties = int((near_tie_rows(ora, p) & ~near).sum())
    return int(near.sum())


def compare_attention(O_gpu: torch.Tensor, LSE_gpu: torch.Tensor, O_ref: np.ndarray, LSE_ref: np.ndarray,
                      tokens: np.ndarray, d: int, what: str = ""):
    o = O_gpu.reshape(-1, d).float()[torch.from_numpy(tokens).to(O_gpu.device)].cpu().numpy().astype(np.float64)
    l = LSE_gpu.reshape(-1)[torch.from_numpy(tokens).to(O_gpu.device)].cpu().numpy().astype(np.float64)
    err = np.abs(o - O_ref)
    fin = np.isfinite(LSE_ref)
    assert np.array_equal(fin, np.isfinite(l)), f"{what}: LSE finiteness differs"
    lerr = np.abs(l[fin] - LSE_ref[fin]) if fin.any() else np.zeros(1)
    msg = (f"{what}: O max {err.max():.3e} mean {err.mean():.3e}; LSE max {lerr.max():.3e}; "
           f"worst token {int(tokens[np.argmax(err.max(1))])}")
    assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS and lerr.max() <= LSE_ABS, msg
    return err.max(), err.mean(), lerr.max()
