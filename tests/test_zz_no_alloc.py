"""fvattn_sparse_fwd_noalloc: the sparse forward for callers that cannot
allocate device memory at call time (hosts that own every allocation and
only hand the library a stream and tensors, or steps that must not pay for
the device synchronisation of cudaMalloc/cudaFree).  It uses one fixed
library-owned device array as scratch instead of a caller workspace.

Checked through the C ABI:
  * against fvattn_sparse_fwd on the same inputs: bit for bit, since both run
    the same launches and every output row depends only on its own inputs;
  * for calls in a row on two shapes, interleaved (a, b, a, b), so every call
    after the first finds the scratch holding another call's contents;
  * against the fp64 oracle on sampled tokens (query block 0, the last ragged
    block and random blocks of every head);
  * for the size limit, with null pointers, so a regression in the host-side
    size check fails on the null-pointer check instead of launching anything.
This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import workloads as W
from tests.gpu_util import compare_attention

pytestmark = pytest.mark.gpu

CASES = [
    W.Workload("noalloc_a", B=1, H=4, N=4000, d=128, bs=128, p=0.8, dist="structured", grid=(10, 20, 20),
               head_scale=("uniform", 0.5, 4.0), seed=51),
    W.Workload("noalloc_b", B=2, H=2, N=1500, d=64, bs=64, p=0.9, dist="structured", grid=(6, 10, 25),
               head_scale=("uniform", 0.5, 4.0), seed=52),
]


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _sample_tokens(w, rng):
    toks = []
    for bh in range(w.B * w.H):
        for qb in sorted({0, w.nb - 1, *rng.integers(0, w.nb, 2).tolist()}):
            lo, hi = qb * w.bs, min(w.N, (qb + 1) * w.bs)
            toks.append(bh * w.N + np.arange(lo, hi))
    return np.concatenate(toks).astype(np.int64)


def test_noalloc_matches_workspace_entry_point_bitwise(oracle_mod):
    import top_routed_block_b200 as fv
    prep = []
    for w in CASES:
        Q, K, V = W.generate(w)
        dQ, dK, dV = _dev(Q), _dev(K), _dev(V)
        r = fv.fvattn_route(dQ, dK, w.p, w.bs)
        fv.check_status(r.dev_status)
        O_ref, LSE_ref, st = fv.fvattn_sparse_fwd(dQ, dK, dV, r.row_ptr, r.col_idx, w.bs, w.causal)
        fv.check_status(st)
        prep.append((w, (Q, K, V), (dQ, dK, dV), r, O_ref, LSE_ref))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = {}
    for w, _, (dQ, dK, dV), r, O_ref, LSE_ref in prep + prep:
        O = torch.full_like(dQ, float("nan"))
        LSE = torch.full((w.B, w.H, w.N), float("nan"), dtype=torch.float32, device="cuda")
        fv.fvattn_sparse_fwd_noalloc(dQ, dK, dV, r.row_ptr, r.col_idx, w.bs, w.causal, O=O, LSE=LSE,
                                     dev_status=status)
        fv.check_status(status, "fvattn_sparse_fwd_noalloc")
        assert torch.equal(O.view(torch.int16), O_ref.view(torch.int16)), w.name
        assert torch.equal(LSE.view(torch.int32), LSE_ref.view(torch.int32)), w.name
        outs[w.name] = (O, LSE)
    rng = np.random.default_rng(7)
    for w, (Q, K, V), _, r, _, _ in prep:
        O, LSE = outs[w.name]
        rp = r.row_ptr.cpu().numpy()
        ci = r.col_idx[: int(rp[-1])].cpu().numpy()
        tokens = _sample_tokens(w, rng)
        Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, w.causal, rp, ci, tokens)
        compare_attention(O, LSE, Oref, Lref, tokens, w.d, w.name)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import top_routed_block_b200 as fv
    lib = fv.load_library()
    B, H, N, block = 16, 256, 65536, 128    # 2097152 rows: more than the scratch holds
    assert fv.fvattn_fwd_workspace_bytes(B, H, N, block) > 4 << 20
    rc = lib.fvattn_sparse_fwd_noalloc(None, None, None, None, None, B, H, N, 128, block, 0, None, None, None, None)
    assert rc == fv.FVATTN_ERR_CAPACITY
