"""Sparse attention parity on the GPU: O and LSE from fvattn_sparse_fwd against
the fp64 oracle evaluated on the GPU's own block mask (FlashAttention review,
§Background "Motivation" and §Model; FVAttn review, §1 "Top-p routing").

Small cases compare every token (several tiles, ragged tails, both block
sizes and head dims, causal and not); the full-size workloads compare a seeded
sample of tokens: query block 0, the last (ragged) query block and random
query blocks of every head."""
import numpy as np
import pytest
import torch

import workloads as W
from tests.gpu_util import compare_attention, gpu_route, to_dev

pytestmark = pytest.mark.gpu

SMALL = [
    (W.TINY, False),
    (W.Workload("small_ragged_d128", B=1, H=3, N=1000, d=128, bs=128, p=0.7, dist="structured", grid=(5, 8, 25),
                head_scale=("uniform", 0.5, 4.0), seed=31), False),
    (W.Workload("small_b2_d64_bs128", B=2, H=2, N=777, d=64, bs=128, p=0.5, dist="structured", grid=(7, 3, 37),
                head_scale=("uniform", 1.0, 6.0), seed=32), False),
    (W.Workload("small_bs64_d128", B=1, H=3, N=2000, d=128, bs=64, p=0.9, dist="structured", grid=(5, 20, 20),
                head_scale=("uniform", 0.5, 4.0), seed=33), False),
    (W.Workload("small_bs64_d64_iid", B=1, H=2, N=300, d=64, bs=64, p=0.6, seed=37), False),
    (W.Workload("p_one_small", B=2, H=2, N=700, d=128, bs=128, p=1.0, seed=36), False),
    (W.Workload("p_one_small_causal", B=2, H=2, N=700, d=128, bs=128, p=1.0, seed=36), True),
    (W.Workload("p_one_bs64_d64_causal", B=1, H=2, N=500, d=64, bs=64, p=1.0, seed=38), True),
    # block 64, an odd number of query blocks (the last pair holds one row) and a
    # ragged last block of 4 tokens
    (W.Workload("bs64_odd_nb_causal", B=1, H=2, N=900, d=128, bs=64, p=1.0, seed=47), True),
    (W.Workload("bs64_odd_nb_routed", B=2, H=2, N=900, d=64, bs=64, p=0.7, dist="structured", grid=(4, 15, 15),
                head_scale=("uniform", 0.5, 4.0), seed=48), False),
    # d = 64 at block 128: many items, ragged tails, causal and routed
    (W.Workload("d64_bs128_routed", B=1, H=4, N=3000, d=64, bs=128, p=0.7, dist="structured",
                grid=(5, 20, 30), head_scale=("uniform", 0.5, 4.0), seed=51), False),
    (W.Workload("d64_bs128_causal", B=2, H=3, N=1500, d=64, bs=128, p=1.0, seed=52), True),
    (W.Workload("large_scores", B=1, H=2, N=600, d=128, bs=128, p=0.8, dist="structured", grid=(6, 10, 10),
                head_scale=("const", 6.0), seed=39), False),
]


def causal_csr(w, oracle_mod):
    return oracle_mod.dense_csr(w.B, w.H, w.N, w.bs, causal=True)


def run_fwd(dQ, dK, dV, rp, ci, bs, causal):
    import top_routed_block_b200 as fv
    drp = torch.from_numpy(np.ascontiguousarray(rp, np.int32)).cuda()
    dci = torch.from_numpy(np.ascontiguousarray(ci if ci.size else np.zeros(1), np.int32)).cuda()
    O, LSE, st = fv.fvattn_sparse_fwd(dQ, dK, dV, drp, dci, bs, causal)
    fv.check_status(st, "fvattn_sparse_fwd")
    return O, LSE


@pytest.mark.parametrize("w,causal", SMALL, ids=lambda x: x.name if hasattr(x, "name") else str(x))
def test_attention_small_every_token(w, causal, oracle_mod):
    Q, K, V = W.generate(w)
    dQ, dK, dV = to_dev(Q), to_dev(K), to_dev(V)
    if causal:
        rp, ci = causal_csr(w, oracle_mod)
    else:
        rp, ci, _ = gpu_route(dQ, dK, w.p, w.bs)
    O, LSE = run_fwd(dQ, dK, dV, rp, ci, w.bs, causal)
    tokens = np.arange(w.B * w.H * w.N, dtype=np.int64)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, causal, rp, ci, tokens)
    print(w.name, compare_attention(O, LSE, Oref, Lref, tokens, w.d, w.name))


@pytest.mark.parametrize("d", [128, 64])
def test_attention_custom_mask_with_empty_rows(d, oracle_mod):
    """Arbitrary ascending key-block sets, empty rows included (O = 0, LSE = -inf)."""
    rng = np.random.default_rng(40)
    w = W.Workload("custom", B=1, H=2, N=900, d=d, bs=128, p=1.0, seed=40)
    Q, K, V = W.generate(w)
    rows, nb = w.rows, w.nb
    sets = []
    for r in range(rows):
        if r % 5 == 0:
            sets.append([])
        else:
            sets.append(sorted(rng.choice(nb, size=int(rng.integers(1, nb + 1)), replace=False).tolist()))
    rp = np.zeros(rows + 1, np.int32)
    rp[1:] = np.cumsum([len(s) for s in sets])
    ci = np.asarray([j for s in sets for j in s], np.int32)
    O, LSE = run_fwd(to_dev(Q), to_dev(K), to_dev(V), rp, ci, w.bs, False)
    tokens = np.arange(w.B * w.H * w.N, dtype=np.int64)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, False, rp, ci, tokens)
    compare_attention(O, LSE, Oref, Lref, tokens, w.d, "custom")
    empty_tok = tokens[(tokens % w.N) < w.bs]  # query block 0 of head 0 is row 0: empty
    assert torch.all(O.reshape(-1, w.d)[: w.bs].float() == 0)
    assert torch.all(torch.isinf(LSE.reshape(-1)[: w.bs]))
    assert empty_tok.size > 0


@pytest.mark.parametrize("N,causal", [(900, False), (1024, False), (900, True)])
def test_block64_pairs_with_every_pattern(N, causal, oracle_mod):
    """Block 64 runs neighbouring query blocks 2i and 2i+1 as one tile over the union of
    their key blocks.  Pairs cycle through: both rows empty (O = 0, LSE = -inf), only
    the second row non-empty, equal lists, disjoint lists, and independent lists; an
    odd block count leaves the last row alone."""
    rng = np.random.default_rng(49 + N)
    w = W.Workload("pairs", B=1, H=3, N=N, d=128, bs=64, p=1.0, seed=49)
    Q, K, V = W.generate(w)
    nb = w.nb
    sets = []
    for h in range(w.H):
        for i in range(0, nb, 2):
            kind = (i // 2 + h) % 5
            rand = lambda: sorted(rng.choice(nb, size=int(rng.integers(1, nb + 1)), replace=False).tolist())
            if kind == 0:
                a, b = [], []
            elif kind == 1:
                a, b = [], rand()
            elif kind == 2:
                a = rand()
                b = list(a)
            elif kind == 3:
                perm = rng.permutation(nb)
                a, b = sorted(perm[: nb // 2].tolist()), sorted(perm[nb // 2:].tolist())
            else:
                a, b = rand(), rand()
            sets.append(a)
            if i + 1 < nb:
                sets.append(b)
    rp = np.zeros(len(sets) + 1, np.int32)
    rp[1:] = np.cumsum([len(x) for x in sets])
    ci = np.asarray([j for x in sets for j in x], np.int32)
    O, LSE = run_fwd(to_dev(Q), to_dev(K), to_dev(V), rp, ci, w.bs, causal)
    tokens = np.arange(w.B * w.H * w.N, dtype=np.int64)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, causal, rp, ci, tokens)
    compare_attention(O, LSE, Oref, Lref, tokens, w.d, "pairs")
    # head 0, pair 0: both rows empty
    assert torch.all(O.reshape(-1, w.d)[: 2 * w.bs].float() == 0)
    assert torch.all(torch.isinf(LSE.reshape(-1)[: 2 * w.bs]))


@pytest.mark.parametrize("N,causal", [(50, False), (50, True), (100, False), (128, True)])
def test_block64_one_pair(N, causal, oracle_mod):
    """Block 64 with one or two query blocks: a single pair, its second row absent
    (N <= 64) or present; every token."""
    w = W.Workload("one_pair", B=2, H=2, N=N, d=64, bs=64, p=1.0, seed=53)
    Q, K, V = W.generate(w)
    rp, ci = oracle_mod.dense_csr(w.B, w.H, w.N, w.bs, causal=causal)
    O, LSE = run_fwd(to_dev(Q), to_dev(K), to_dev(V), rp, ci, w.bs, causal)
    tokens = np.arange(w.B * w.H * w.N, dtype=np.int64)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, causal, rp, ci, tokens)
    compare_attention(O, LSE, Oref, Lref, tokens, w.d, "one_pair")


@pytest.mark.slow
def test_block64_largest_block_count(oracle_mod):
    """Block 64 at the largest supported block count (4096 query blocks, a ragged last
    block): the first pair's rows select every key block, so its union fills the
    whole union slot; the other rows hold a few blocks, the last one included.
    Sampled tokens: the first pair, the last pair and random pairs."""
    rng = np.random.default_rng(54)
    nb = 4096
    w = W.Workload("nb4096", B=1, H=1, N=nb * 64 - 5, d=64, bs=64, p=1.0, seed=54)
    Q, K, V = W.generate(w)
    sets = [list(range(nb)), list(range(nb))]
    for r in range(2, nb):
        k = int(rng.integers(1, 9))
        sets.append(sorted(set(rng.choice(nb, size=k, replace=False).tolist()) | {nb - 1}))
    rp = np.zeros(nb + 1, np.int32)
    rp[1:] = np.cumsum([len(x) for x in sets])
    ci = np.asarray([j for x in sets for j in x], np.int32)
    O, LSE = run_fwd(to_dev(Q), to_dev(K), to_dev(V), rp, ci, w.bs, False)
    pairs = [0, nb // 2 - 1] + rng.choice(np.arange(1, nb // 2 - 1), size=6, replace=False).tolist()
    tokens = np.concatenate([np.arange(p * 128, min(w.N, p * 128 + 128)) for p in sorted(pairs)]).astype(np.int64)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, False, rp, ci, tokens)
    compare_attention(O, LSE, Oref, Lref, tokens, w.d, "nb4096")


def test_block64_bad_csr_is_reported_and_in_range_entries_are_computed(oracle_mod):
    """Block 64: an out-of-range index and a repeated one are reported as
    FVATTN_ERR_BAD_CSR; every row is computed over its in-range entries."""
    import top_routed_block_b200 as fv
    w = W.Workload("badcsr64", B=1, H=1, N=256, d=64, bs=64, p=1.0, seed=50)
    Q, K, V = W.generate(w)
    rp = np.array([0, 2, 4, 6, 8], np.int32)
    ci = np.array([0, 1, 1, 9, 2, 2, 0, 3], np.int32)   # row 1: index 9 out of range; row 2: repeat
    good_rp = np.array([0, 2, 3, 4, 6], np.int32)
    good_ci = np.array([0, 1, 1, 2, 0, 3], np.int32)
    dQ, dK, dV = to_dev(Q), to_dev(K), to_dev(V)
    O, LSE, st = fv.fvattn_sparse_fwd(dQ, dK, dV, torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(),
                                      w.bs, False)
    torch.cuda.synchronize()
    assert int(st.item()) == fv.FVATTN_ERR_BAD_CSR
    tokens = np.arange(w.N, dtype=np.int64)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, False, good_rp, good_ci, tokens)
    compare_attention(O, LSE, Oref, Lref, tokens, w.d, "badcsr64")


def test_attention_uniform_probabilities_give_mean_of_values(oracle_mod):
    """K = 0 makes every probability equal: O is the mean of the selected V rows.
    This isolates the P.V product (P layout in tensor memory, V descriptor)."""
    w = W.Workload("uniform", B=1, H=1, N=512, d=128, bs=128, p=1.0, seed=41)
    Q, _, V = W.generate(w)
    K = np.zeros_like(Q)
    rp = np.array([0, 1, 2, 4, 8], np.int32)
    ci = np.array([0, 3, 1, 2, 0, 1, 2, 3], np.int32)
    O, LSE = run_fwd(to_dev(Q), to_dev(K), to_dev(V), rp, ci, w.bs, False)
    tokens = np.arange(w.N, dtype=np.int64)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, False, rp, ci, tokens)
    compare_attention(O, LSE, Oref, Lref, tokens, w.d, "uniform")


def test_attention_one_hot_values_expose_probabilities(oracle_mod):
    """V[u, c] = 1 if c == u mod d: O[t, c] is the probability mass of the keys
    u = c (mod d), so every P column is checked separately."""
    w = W.Workload("onehot", B=1, H=1, N=256, d=64, bs=128, p=1.0, seed=42)
    Q, K, _ = W.generate(w)
    Vf = np.zeros((1, 1, w.N, w.d), np.float32)
    for u in range(w.N):
        Vf[0, 0, u, u % w.d] = 1.0
    V = W.f32_to_bf16_bits(Vf)
    rp, ci = oracle_mod.dense_csr(1, 1, w.N, w.bs)
    O, LSE = run_fwd(to_dev(Q), to_dev(K), to_dev(V), rp, ci, w.bs, False)
    tokens = np.arange(w.N, dtype=np.int64)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, False, rp, ci, tokens)
    compare_attention(O, LSE, Oref, Lref, tokens, w.d, "onehot")


FULL = [(W.VIDEO, False), (W.DENSE, False), (W.DENSE_CAUSAL, True), (W.LONG, False), (W.VIDEO_BS64, False)]


@pytest.mark.parametrize("w,causal", FULL, ids=lambda x: x.name if hasattr(x, "name") else str(x))
def test_attention_full_size_sampled(w, causal, oracle_mod):
    Q, K, V = W.generate(w)
    dQ, dK, dV = to_dev(Q), to_dev(K), to_dev(V)
    if causal:
        rp, ci = causal_csr(w, oracle_mod)
    else:
        rp, ci, _ = gpu_route(dQ, dK, w.p, w.bs)
    O, LSE = run_fwd(dQ, dK, dV, rp, ci, w.bs, causal)
    tokens = W.sample_tokens(w, per_head_blocks=2, rows_per_block=24)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, causal, rp, ci, tokens)
    print(w.name, compare_attention(O, LSE, Oref, Lref, tokens, w.d, w.name))


@pytest.mark.parametrize("w", W.sweep(), ids=lambda w: w.name)
def test_attention_sweep_sampled(w, oracle_mod):
    Q, K, V = W.generate(w)
    dQ, dK, dV = to_dev(Q), to_dev(K), to_dev(V)
    rp, ci, _ = gpu_route(dQ, dK, w.p, w.bs)
    O, LSE = run_fwd(dQ, dK, dV, rp, ci, w.bs, False)
    tokens = W.sample_tokens(w, per_head_blocks=2, rows_per_block=12)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, False, rp, ci, tokens)
    compare_attention(O, LSE, Oref, Lref, tokens, w.d, w.name)


def test_bad_csr_is_reported_and_the_rest_is_computed(oracle_mod):
    """Out-of-range and non-ascending column indices are skipped and reported as
    FVATTN_ERR_BAD_CSR; the device stays usable and other rows are exact."""
    import top_routed_block_b200 as fv
    w = W.Workload("badcsr", B=1, H=1, N=512, d=128, bs=128, p=1.0, seed=43)
    Q, K, V = W.generate(w)
    rp = np.array([0, 2, 4, 6, 8], np.int32)
    ci = np.array([0, 1, 1, 9, 2, 2, 0, 3], np.int32)   # row 1: index 9 out of range; row 2: repeat
    good_rp = np.array([0, 2, 3, 4, 6], np.int32)
    good_ci = np.array([0, 1, 1, 2, 0, 3], np.int32)
    dQ, dK, dV = to_dev(Q), to_dev(K), to_dev(V)
    drp = torch.from_numpy(rp).cuda()
    dci = torch.from_numpy(ci).cuda()
    O, LSE, st = fv.fvattn_sparse_fwd(dQ, dK, dV, drp, dci, w.bs, False)
    torch.cuda.synchronize()
    assert int(st.item()) == fv.FVATTN_ERR_BAD_CSR
    tokens = np.arange(w.N, dtype=np.int64)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, False, good_rp, good_ci, tokens)
    compare_attention(O, LSE, Oref, Lref, tokens, w.d, "badcsr")
    # the context is still healthy
    O2, LSE2 = run_fwd(dQ, dK, dV, good_rp, good_ci, w.bs, False)
    compare_attention(O2, LSE2, Oref, Lref, tokens, w.d, "after-badcsr")


HOST_CASES = [
    # 24 heads of 0.5 MB: under two chunks of 64 MB, so the chunks halve at once (12, 6, 3, 2, 1)
    W.Workload("host_path", B=2, H=12, N=2000, d=128, bs=128, p=0.8, dist="structured", grid=(5, 20, 20),
               head_scale=("uniform", 0.5, 4.0), seed=44),
    # 20 heads of 8 MB: a full 8-head chunk first, then the halving tail (8, 6, 3, 2, 1)
    W.Workload("host_path_chunks", B=1, H=20, N=32768, d=128, bs=128, p=0.9, dist="structured",
               grid=(8, 64, 64), head_scale=("uniform", 0.5, 4.0), seed=46),
]


@pytest.mark.parametrize("w", HOST_CASES, ids=lambda w: w.name)
def test_host_buffer_path_matches_device_path(w):
    """fvattn_attention_host (chunked copies in, routing, attention, copies out)
    returns exactly what the device entry points return: heads are independent."""
    import top_routed_block_b200 as fv
    Q, K, V = W.generate(w)
    dQ, dK, dV = to_dev(Q), to_dev(K), to_dev(V)
    plan = fv.FvattnPlan(w.B, w.H, w.N, w.d, w.bs)
    O_dev, L_dev, _ = plan(dQ, dK, dV, w.p)
    plan.check()
    O_dev, L_dev = O_dev.clone(), L_dev.clone()
    pin = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    hQ, hK, hV = pin(Q), pin(K), pin(V)
    hO = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16).pin_memory()
    hL = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
    for _ in range(2):
        hO.fill_(float("nan"))
        fv.fvattn_attention_host(hQ, hK, hV, w.p, w.bs, False, plan=plan, dQ=torch.empty_like(dQ),
                                 dK=torch.empty_like(dK), dV=torch.empty_like(dV), hO=hO, hLSE=hL)
        assert torch.equal(hO, O_dev.cpu())
        assert torch.equal(hL, L_dev.cpu())


@pytest.mark.parametrize("d,bs", [(128, 128), (64, 128), (128, 64)])
def test_profiled_forward_reports_busy_time_and_matches(d, bs):
    """fvattn_sparse_fwd_profiled returns exactly what fvattn_sparse_fwd returns, in
    either work order (rows are independent), plus a positive busy time per CTA."""
    import top_routed_block_b200 as fv
    w = W.Workload("profiled", B=1, H=6, N=3000, d=d, bs=bs, p=0.8, dist="structured", grid=(5, 20, 30),
                   head_scale=("uniform", 0.5, 4.0), seed=45)
    Q, K, V = W.generate(w)
    dQ, dK, dV = to_dev(Q), to_dev(K), to_dev(V)
    r = fv.fvattn_route(dQ, dK, w.p, w.bs)
    fv.check_status(r.dev_status, "route")
    O_ref, L_ref, st = fv.fvattn_sparse_fwd(dQ, dK, dV, r.row_ptr, r.col_idx, w.bs, False)
    fv.check_status(st, "fwd")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for natural in (False, True):
        O, L, st, busy = fv.fvattn_sparse_fwd_profiled(dQ, dK, dV, r.row_ptr, r.col_idx, w.bs, False,
                                                       natural_order=natural)
        fv.check_status(st, "profiled")
        assert torch.equal(O, O_ref) and torch.equal(L, L_ref)
        b = busy.cpu().numpy()
        assert 1 <= b.size <= min(sms, w.rows)
        assert np.all(b > 0)
