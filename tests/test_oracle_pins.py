"""Pins for the fp64 CPU oracle (no GPU).

Each test checks the oracle against something other than itself: exact
rational or 50-digit Decimal brute force of the definitions, closed forms and
the invariants of the top-p rule.

Definitions followed (page title, section):
  * FVAttn review, §1 Key Terms "Top-p routing": key blocks are added in order
    of importance until the cumulative probability reaches p.
  * FlashAttention review, §Background "Motivation": S = QK^T, P = softmax(S),
    O = PV; §Model "Tiling Softmax": block-wise softmax combines exactly.
The routing score itself (mean-pooled blocks, qbar.kbar/sqrt(d), softmax over
key blocks, ties to the lower index) is this library's reading, since the
pages only name it.
"""
from __future__ import annotations

import itertools
import math
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

import workloads as W
from workloads import bf16_bits_to_f32, f32_to_bf16_bits

getcontext().prec = 60


def bf16(a) -> np.ndarray:
    return f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def rand_bf16(rng, shape, scale=1.0):
    return bf16(rng.standard_normal(shape).astype(np.float32) * scale)


def fvals(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(bits).astype(np.float64)


# ----------------------------------------------------------------- pooling

def test_pool_constant_blocks(oracle_mod):
    N, bs, d = 200, 64, 8
    X = np.zeros((1, 2, N, d), np.float32)
    for h in range(2):
        for i in range(4):
            X[0, h, i * bs:(i + 1) * bs] = (h * 4 + i) * 0.5 - 1.25
    out = oracle_mod.pool(bf16(X), bs)
    for h in range(2):
        for i in range(4):
            assert np.all(out[0, h, i] == (h * 4 + i) * 0.5 - 1.25)


def test_pool_ragged_block_divides_by_valid_tokens(oracle_mod):
    N, bs, d = 70, 64, 4
    X = np.zeros((1, 1, N, d), np.float32)
    for t in range(N):
        for c in range(d):
            X[0, 0, t, c] = (t % 7) - 3 + 0.25 * c
    out = oracle_mod.pool(bf16(X), bs)
    for i, (t0, t1) in enumerate([(0, 64), (64, 70)]):
        for c in range(d):
            exact = sum(Fraction(float(X[0, 0, t, c])) for t in range(t0, t1)) / (t1 - t0)
            assert abs(Fraction(out[0, 0, i, c]) - exact) <= abs(exact) * Fraction(1, 2**50) + Fraction(1, 2**60)
    # the last block holds 6 tokens; dividing by the block size would be 64/6 times smaller
    assert out[0, 0, 1, 0] != 0.0


# ------------------------------------------------------- attention (rows)

def decimal_attention(q, keys, vals):
    """50-digit brute force of softmax(q.k/sqrt(d)) v over the given keys."""
    d = len(q)
    if not keys:
        return [Decimal(0)] * d, None
    scale = Decimal(1) / Decimal(d).sqrt()
    s = [sum(Decimal(float(q[c])) * Decimal(float(k[c])) for c in range(d)) * scale for k in keys]
    m = max(s)
    w = [(x - m).exp() for x in s]
    z = sum(w)
    out = [sum(w[a] * Decimal(float(vals[a][c])) for a in range(len(vals))) / z for c in range(d)]
    return out, m + z.ln()


def random_csr(rng, rows, nb, p_keep=0.5, allow_empty=True):
    row_ptr = [0]
    cols = []
    for r in range(rows):
        sel = [j for j in range(nb) if rng.random() < p_keep]
        if not sel and not allow_empty:
            sel = [int(rng.integers(nb))]
        cols.extend(sel)
        row_ptr.append(len(cols))
    return np.asarray(row_ptr, np.int32), np.asarray(cols, np.int32)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,bs,d", [(11, 4, 4), (8, 4, 8), (1, 4, 4), (9, 3, 2)])
def test_attn_rows_matches_decimal_brute_force(oracle_mod, N, bs, d, causal):
    rng = np.random.default_rng(N * 100 + bs * 10 + d + causal)
    B, H = 1, 2
    Q, K, V = (rand_bf16(rng, (B, H, N, d)) for _ in range(3))
    nb = -(-N // bs)
    row_ptr, col_idx = random_csr(rng, B * H * nb, nb)
    # the first row empty and the second row full, whatever the draw
    counts = np.diff(row_ptr).tolist()
    rows_cols = [list(col_idx[row_ptr[r]:row_ptr[r + 1]]) for r in range(len(counts))]
    rows_cols[0] = []
    if len(rows_cols) > 1:
        rows_cols[1] = list(range(nb))
    row_ptr = np.zeros(len(rows_cols) + 1, np.int32)
    row_ptr[1:] = np.cumsum([len(c) for c in rows_cols])
    col_idx = np.asarray([j for c in rows_cols for j in c], np.int32)
    tokens = np.arange(B * H * N, dtype=np.int64)
    O, LSE = oracle_mod.attn_rows(Q, K, V, bs, causal, row_ptr, col_idx, tokens)
    Ot, LSEt = oracle_mod.attn_tiled(Q, K, V, bs, causal, row_ptr, col_idx, tokens)
    Qf, Kf, Vf = fvals(Q), fvals(K), fvals(V)
    for g in tokens:
        bh, t = divmod(int(g), N)
        b, h = divmod(bh, H)
        row = bh * nb + t // bs
        keys = []
        for e in range(row_ptr[row], row_ptr[row + 1]):
            kb = int(col_idx[e])
            for u in range(kb * bs, min(N, kb * bs + bs)):
                if causal and u > t:
                    continue
                keys.append(u)
        ref_o, ref_lse = decimal_attention(Qf[b, h, t], [Kf[b, h, u] for u in keys], [Vf[b, h, u] for u in keys])
        for impl_o, impl_lse in ((O, LSE), (Ot, LSEt)):
            assert np.allclose(impl_o[g], [float(x) for x in ref_o], rtol=0, atol=1e-12)
            if ref_lse is None:
                assert impl_lse[g] == -np.inf
            else:
                assert abs(impl_lse[g] - float(ref_lse)) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_attn_rows_equals_dense_attention_with_minus_inf_bias(oracle_mod, causal):
    """Masked-dense equivalence: the sparse attention on a block mask M equals dense
    softmax(Q K^T / sqrt(d) + bias) V over all N keys, with bias 0 on M (and u <= t if
    causal) and -inf elsewhere, written as fp64 matrix algebra; rows whose bias is all
    -inf give O = 0 and LSE = -inf.  Ragged last block, empty and full rows."""
    rng = np.random.default_rng(17 + causal)
    B, H, N, d, bs = 2, 2, 200, 16, 64
    nb = -(-N // bs)
    row_ptr, col_idx = random_csr(rng, B * H * nb, nb, p_keep=0.5, allow_empty=True)
    Q, K, V = (rand_bf16(rng, (B, H, N, d)) for _ in range(3))
    tokens = np.arange(B * H * N, dtype=np.int64)
    O, LSE = oracle_mod.attn_rows(Q, K, V, bs, causal, row_ptr, col_idx, tokens)
    Qf, Kf, Vf = fvals(Q), fvals(K), fvals(V)
    for bh in range(B * H):
        b, h = divmod(bh, H)
        allowed = np.zeros((N, N), bool)  # [query token, key token]
        for qb in range(nb):
            row = bh * nb + qb
            for kb in col_idx[row_ptr[row]:row_ptr[row + 1]]:
                allowed[qb * bs:(qb + 1) * bs, kb * bs:(kb + 1) * bs] = True
        if causal:
            allowed &= np.tril(np.ones((N, N), bool))
        S = Qf[b, h] @ Kf[b, h].T / math.sqrt(d) + np.where(allowed, 0.0, -np.inf)
        m = S.max(axis=1, keepdims=True)
        has = np.isfinite(m[:, 0])
        E = np.where(has[:, None], np.exp(S - np.where(has[:, None], m, 0.0)), 0.0)
        z = E.sum(axis=1)
        ref_o = np.where(has[:, None], (E @ Vf[b, h]) / np.where(has, z, 1.0)[:, None], 0.0)
        ref_lse = np.where(has, m[:, 0] + np.log(np.where(has, z, 1.0)), -np.inf)
        got_o = O[bh * N:(bh + 1) * N]
        got_lse = LSE[bh * N:(bh + 1) * N]
        assert np.max(np.abs(got_o - ref_o)) < 1e-12
        assert np.array_equal(np.isinf(got_lse), np.isinf(ref_lse))
        fin = np.isfinite(ref_lse)
        assert np.max(np.abs(got_lse[fin] - ref_lse[fin])) < 1e-12


def test_attn_closed_form_zero_keys_gives_mean_of_values(oracle_mod):
    rng = np.random.default_rng(7)
    B, H, N, d, bs = 1, 1, 40, 8, 16
    Q = rand_bf16(rng, (B, H, N, d))
    K = bf16(np.zeros((B, H, N, d)))
    V = rand_bf16(rng, (B, H, N, d))
    nb = 3
    row_ptr = np.array([0, 1, 3, 6], np.int32)
    col_idx = np.array([2, 0, 2, 0, 1, 2], np.int32)
    tokens = np.arange(N, dtype=np.int64)
    O, LSE = oracle_mod.attn_rows(Q, K, V, bs, False, row_ptr, col_idx, tokens)
    Vf = fvals(V)[0, 0]
    for t in range(N):
        row = t // bs
        keys = [u for e in range(row_ptr[row], row_ptr[row + 1])
                for u in range(col_idx[e] * bs, min(N, col_idx[e] * bs + bs))]
        for c in range(d):
            exact = sum(Fraction(Vf[u, c]) for u in keys) / len(keys)
            assert abs(O[t, c] - float(exact)) <= 1e-14
        assert abs(LSE[t] - math.log(len(keys))) <= 1e-14
    assert nb == 3


def test_attn_closed_form_single_key_and_constant_values(oracle_mod):
    Q = bf16([[[[0.5, -1.0, 2.0, 0.25]]]])
    K = bf16([[[[1.0, 1.0, -0.5, 4.0]]]])
    V = bf16([[[[3.0, -2.0, 0.125, 7.0]]]])
    O, LSE = oracle_mod.attn_rows(Q, K, V, 64, False, np.array([0, 1], np.int32), np.array([0], np.int32),
                                  np.array([0], np.int64))
    assert np.array_equal(O[0], [3.0, -2.0, 0.125, 7.0])
    assert LSE[0] == (0.5 - 1.0 - 1.0 + 1.0) / 2.0
    rng = np.random.default_rng(3)
    Q, K = rand_bf16(rng, (1, 1, 100, 16)), rand_bf16(rng, (1, 1, 100, 16), 3.0)
    V = bf16(np.full((1, 1, 100, 16), 1.5))
    row_ptr, col_idx = oracle_mod.dense_csr(1, 1, 100, 32)
    O, _ = oracle_mod.attn_rows(Q, K, V, 32, False, row_ptr, col_idx, np.arange(100, dtype=np.int64))
    assert np.max(np.abs(O - 1.5)) <= 1e-14


@pytest.mark.parametrize("causal", [False, True])
def test_tiled_online_softmax_equals_row_softmax(oracle_mod, causal):
    rng = np.random.default_rng(11)
    B, H, N, d, bs = 1, 2, 300, 32, 64
    Q, K, V = rand_bf16(rng, (B, H, N, d), 2.0), rand_bf16(rng, (B, H, N, d), 2.0), rand_bf16(rng, (B, H, N, d))
    row_ptr, col_idx = random_csr(rng, B * H * 5, 5, p_keep=0.6)
    tokens = np.arange(B * H * N, dtype=np.int64)
    O, L = oracle_mod.attn_rows(Q, K, V, bs, causal, row_ptr, col_idx, tokens)
    Ot, Lt = oracle_mod.attn_tiled(Q, K, V, bs, causal, row_ptr, col_idx, tokens)
    assert np.max(np.abs(O - Ot)) <= 1e-12
    fin = np.isfinite(L)
    assert np.array_equal(fin, np.isfinite(Lt))
    assert np.max(np.abs(L[fin] - Lt[fin])) <= 1e-12


# ------------------------------------------------------------------ routing

def check_csr(route, rows, nb):
    rp, ci = route.row_ptr, route.col_idx
    assert rp[0] == 0 and rp.size == rows + 1 and np.all(np.diff(rp) >= 1)
    for r in range(rows):
        cols = ci[rp[r]:rp[r + 1]]
        assert np.all(np.diff(cols) > 0) and cols[0] >= 0 and cols[-1] < nb


def test_route_uniform_scores_select_lowest_indices(oracle_mod):
    """K = 0 makes every score 0 and every probability 1/nb: the kept set is the
    first ceil(p*nb) blocks by index -- this pins the tie-break."""
    rng = np.random.default_rng(5)
    B, H, N, d, bs = 1, 2, 640, 16, 64
    Q = rand_bf16(rng, (B, H, N, d))
    K = bf16(np.zeros((B, H, N, d)))
    for p, expect in ((0.35, 4), (0.55, 6), (0.73, 8), (0.05, 1)):
        r = oracle_mod.route(Q, K, p, bs)
        check_csr(r, B * H * 10, 10)
        assert np.all(r.counts == expect)
        for row in range(B * H * 10):
            assert list(r.col_idx[r.row_ptr[row]:r.row_ptr[row + 1]]) == list(range(expect))
        assert np.all(r.head_counts == 10 * expect)


def test_route_reaching_p_exactly_counts(oracle_mod):
    """Eight uniform blocks (probability 1/8, exact in binary): with p = 1/2 the
    mass of four blocks equals p exactly, and "reaches p" keeps four, not five."""
    rng = np.random.default_rng(6)
    Q = rand_bf16(rng, (1, 1, 512, 16))
    K = bf16(np.zeros((1, 1, 512, 16)))
    r = oracle_mod.route(Q, K, 0.5, 64)
    assert np.all(r.counts == 4)
    assert np.all(r.diag[:, 0] == 0.5)


def test_route_worked_example_by_hand(oracle_mod):
    """Hand-derived instance.  Q tokens all (1,0,0,0); K block means in channel 0
    are (0, 2, 1, 2) for blocks 0..3 (d=4, so scale 1/2): scores (0, 1, .5, 1).
    Probabilities e^s/Z with Z = 1 + 2e + e^.5 are (.1237, .3362, .2039, .3362).
    Order by score, equal scores by index: 1, 3, 2, 0; cumulative mass
    .3362, .6724, .8763, 1.  Hence p=.3 -> {1}; p=.5 -> {1,3}; p=.7 -> {1,2,3};
    p=.9 -> {0,1,2,3}."""
    N, bs, d = 8, 2, 4
    Q = np.zeros((1, 1, N, d), np.float32)
    Q[..., 0] = 1.0
    K = np.zeros((1, 1, N, d), np.float32)
    K[0, 0, 2:4, 0] = [1.0, 3.0]   # mean 2
    K[0, 0, 4:6, 0] = [0.5, 1.5]   # mean 1
    K[0, 0, 6:8, 0] = [2.0, 2.0]   # mean 2
    K[0, 0, 0:2, 1] = [5.0, -5.0]  # block 0 mean 0 in every channel
    z = 1 + 2 * math.e + math.exp(0.5)
    probs = [1 / z, math.e / z, math.exp(0.5) / z, math.e / z]
    assert abs(probs[1] + probs[3] - 0.6724) < 1e-4
    for p, want in ((0.3, [1]), (0.5, [1, 3]), (0.7, [1, 2, 3]), (0.9, [0, 1, 2, 3])):
        r = oracle_mod.route(bf16(Q), bf16(K), p, bs)
        for row in range(4):
            assert list(r.col_idx[r.row_ptr[row]:r.row_ptr[row + 1]]) == want
        assert r.head_counts[0] == 4 * len(want)


def test_route_one_hot_block(oracle_mod):
    B, H, N, d, bs = 1, 1, 640, 16, 64
    Q = bf16(np.ones((B, H, N, d)))
    Kf = np.zeros((B, H, N, d), np.float32)
    Kf[0, 0, 5 * bs:6 * bs] = 4.0   # score 4*16/4 = 16 against 0 elsewhere
    r = oracle_mod.route(Q, bf16(Kf), 0.99, bs)
    assert np.all(r.counts == 1) and np.all(r.col_idx == 5)


def test_route_p_to_zero_is_argmax_with_lowest_index(oracle_mod):
    B, H, N, d, bs = 1, 1, 640, 16, 64
    Q = bf16(np.ones((B, H, N, d)))
    Kf = np.zeros((B, H, N, d), np.float32)
    Kf[0, 0, 2 * bs:3 * bs] = 1.0
    Kf[0, 0, 7 * bs:8 * bs] = 1.0
    r = oracle_mod.route(Q, bf16(Kf), 1e-300, bs)
    assert np.all(r.counts == 1) and np.all(r.col_idx == 2)


def test_route_p_one_keeps_every_block(oracle_mod):
    rng = np.random.default_rng(9)
    Q, K = rand_bf16(rng, (2, 3, 500, 32), 3.0), rand_bf16(rng, (2, 3, 500, 32), 3.0)
    r = oracle_mod.route(Q, K, 1.0, 64)
    nb = 8
    assert np.all(r.counts == nb)
    rp, ci = oracle_mod.dense_csr(2, 3, 500, 64)
    assert np.array_equal(r.row_ptr, rp) and np.array_equal(r.col_idx, ci)


def test_route_invariants_and_monotone_in_p(oracle_mod):
    from workloads import Workload, generate
    w = Workload("t", B=1, H=4, N=24 * 32, d=32, bs=32, p=0.9, dist="structured", grid=(3, 16, 16),
                 head_scale=("uniform", 0.5, 4.0), seed=21)
    Q, K, _ = generate(w)
    prev = None
    for p in (0.1, 0.3, 0.5, 0.7, 0.9, 0.95, 0.99):
        r = oracle_mod.route(Q, K, p, w.bs)
        check_csr(r, w.rows, w.nb)
        g = r.diag
        assert np.all(g[:, 0] >= p)                       # kept mass reaches p
        assert np.all(g[:, 1] < p)                        # one block fewer does not
        assert np.all(g[:, 2] >= g[:, 3])                 # kept scores >= dropped scores
        assert np.all(g[:, 4] >= g[:, 5])                 # kept probability >= dropped
        hc = r.counts.reshape(w.B * w.H, w.nb).sum(1)
        assert np.array_equal(hc, r.head_counts)
        if prev is not None:
            assert np.all(r.counts >= prev)
        prev = r.counts


def exact_route_row(qbar, kbars, p):
    """Exact scores (d a perfect square) and 60-digit probabilities; the shortest
    set reaching p found by exhaustive search over subsets."""
    d = len(qbar)
    root = math.isqrt(d)
    assert root * root == d
    s = [sum(qbar[c] * k[c] for c in range(d)) / root for k in kbars]
    m = max(s)
    e = [(Decimal(x.numerator) / Decimal(x.denominator) - Decimal(m.numerator) / Decimal(m.denominator)).exp()
         for x in s]
    z = sum(e)
    prob = [x / z for x in e]
    nb = len(kbars)
    P = Decimal(repr(p))
    for size in range(1, nb + 1):
        best = None
        for sub in itertools.combinations(range(nb), size):
            mass = sum(prob[j] for j in sub)
            if mass >= P and (best is None or mass > best[0]):
                best = (mass, sub)
        if best is not None:
            order = sorted(range(nb), key=lambda j: (-s[j], j))
            chosen = sorted(order[:size])
            top_mass = sum(prob[j] for j in chosen)
            near = min(abs(top_mass - P), abs(top_mass - prob[order[size - 1]] - P))
            return chosen, near
    return list(range(nb)), Decimal(0)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_route_matches_exhaustive_exact_search(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    B, H, N, d, bs = 1, 2, 6 * 4 - 1, 16, 4      # 6 blocks, the last ragged
    Q, K = rand_bf16(rng, (B, H, N, d), 2.0), rand_bf16(rng, (B, H, N, d), 2.0)
    Qf, Kf = fvals(Q), fvals(K)
    nb = 6

    def pooled(X, bh, i):
        t0, t1 = i * bs, min(N, i * bs + bs)
        return [sum(Fraction(X[0, bh, t, c]) for t in range(t0, t1)) / (t1 - t0) for c in range(d)]

    for p in (0.2, 0.5, 0.8, 0.95):
        r = oracle_mod.route(Q, K, p, bs)
        for bh in range(H):
            kb = [pooled(Kf, bh, j) for j in range(nb)]
            for i in range(nb):
                want, near = exact_route_row(pooled(Qf, bh, i), kb, p)
                if near < Decimal("1e-9"):
                    continue
                row = bh * nb + i
                assert list(r.col_idx[r.row_ptr[row]:r.row_ptr[row + 1]]) == want


# -------------------------------------------------------------- LPT order

def test_lpt_order_brute_force(oracle_mod):
    rng = np.random.default_rng(4)
    for rows in (0, 1, 7, 300):
        counts = rng.integers(0, 12, size=rows)
        rp = np.zeros(rows + 1, np.int32)
        rp[1:] = np.cumsum(counts)
        got = oracle_mod.lpt_order(rp)
        want = sorted(range(rows), key=lambda r: (-int(counts[r]), r))
        assert list(got) == want


# ------------------------------------------------------ stored fixtures

def test_golden_tiny_route_unchanged(oracle_mod):
    """tests/golden/tiny_route.json was written by tests/golden/make_golden.py
    (oracle only); the oracle must keep reproducing it."""
    import json
    import os
    from workloads import TINY, generate
    with open(os.path.join(os.path.dirname(__file__), "golden", "tiny_route.json")) as f:
        g = json.load(f)
    Q, K, _ = generate(TINY)
    r = oracle_mod.route(Q, K, TINY.p, TINY.bs)
    assert r.row_ptr.tolist() == g["row_ptr"]
    assert r.col_idx.tolist() == g["col_idx"]
    assert r.head_counts.tolist() == g["head_counts"]


def test_workload_generators_are_seeded_and_shaped():
    from workloads import ALL, TINY, Workload, generate
    a = generate(TINY)
    b = generate(TINY)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    assert a[0].shape == (1, 2, 512, 64) and a[0].dtype == np.uint16
    w = Workload("s", B=1, H=3, N=4 * 6 * 8, d=16, bs=32, p=0.9, dist="structured", grid=(4, 6, 8),
                 head_scale=("uniform", 0.5, 4.0), seed=5)
    Q, K, V = generate(w)
    assert Q.shape == (1, 3, 192, 16)
    qf, kf, vf = (bf16_bits_to_f32(x).astype(np.float64) for x in (Q, K, V))
    assert qf.std() > 1.0                                  # noise plus the per-head field
    assert np.corrcoef(qf.ravel(), kf.ravel())[0, 1] > 0.2  # Q and K share the field
    assert abs(np.corrcoef(qf.ravel(), vf.ravel())[0, 1]) < 0.1
    assert ALL["video_dit"].N == 32760 and ALL["video_dit"].nb == 256
    assert ALL["long_video"].N == 118800 and ALL["long_video"].nb == 929
    assert len([k for k in ALL if k.startswith("sweep")]) == 20


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.5, 0.0, 1e-30], np.float32)
    b = f32_to_bf16_bits(x)
    back = bf16_bits_to_f32(b)
    assert back[0] == 1.0 and back[1] == 1.0          # tie rounds to even
    assert back[2] == 1.0 + 2**-6                       # tie rounds up to even
    assert back[3] == -2.5 and back[4] == 0.0


# ------------------------------------------------------- attention gradients

def numpy_forward(Qf, Kf, Vf, bs, causal, row_ptr, col_idx):
    """Plain fp64 numpy statement of the masked attention forward (brute force)."""
    B, H, N, d = Qf.shape
    nb = -(-N // bs)
    O = np.zeros_like(Qf)
    for b in range(B):
        for h in range(H):
            for t in range(N):
                row = (b * H + h) * nb + t // bs
                keys = [u for kb in col_idx[row_ptr[row]:row_ptr[row + 1]]
                        for u in range(kb * bs, min((kb + 1) * bs, N)) if not (causal and u > t)]
                if not keys:
                    continue
                s = Kf[b, h, keys] @ Qf[b, h, t] / math.sqrt(d)
                w = np.exp(s - s.max())
                O[b, h, t] = (w / w.sum()) @ Vf[b, h, keys]
    return O


@pytest.mark.parametrize("causal", [False, True])
def test_attn_bwd_matches_finite_differences(oracle_mod, causal):
    """Directional derivatives of L = sum(dO * O) by central differences of an
    independent fp64 forward equal the oracle's gradients."""
    rng = np.random.default_rng(7 + causal)
    B, H, N, d, bs = 1, 2, 70, 16, 32
    nb = -(-N // bs)
    row_ptr, col_idx = random_csr(rng, B * H * nb, nb, p_keep=0.6, allow_empty=True)
    Q, K, V, dO = (rand_bf16(rng, (B, H, N, d)) for _ in range(4))
    dQ, dK, dV = oracle_mod.attn_bwd(Q, K, V, dO, bs, causal, row_ptr, col_idx)
    Qf, Kf, Vf, dOf = fvals(Q), fvals(K), fvals(V), fvals(dO)

    def loss(Qx, Kx, Vx):
        return float(np.sum(dOf * numpy_forward(Qx, Kx, Vx, bs, causal, row_ptr, col_idx)))

    h = 1e-5
    for which, grad in (("Q", dQ), ("K", dK), ("V", dV)):
        for _ in range(3):
            r = rng.standard_normal((B, H, N, d))
            args_p = [Qf, Kf, Vf]
            args_m = [Qf, Kf, Vf]
            i = "QKV".index(which)
            args_p[i] = args_p[i] + h * r
            args_m[i] = args_m[i] - h * r
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            an = float(np.sum(grad * r))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (which, fd, an)


@pytest.mark.parametrize("causal", [False, True])
def test_attn_bwd_dense_matches_torch_autograd(oracle_mod, causal):
    """With every block selected the oracle's gradients equal fp64 autograd of
    softmax(QK^T/sqrt(d))V (lower-triangular mask if causal)."""
    import torch
    rng = np.random.default_rng(11 + causal)
    B, H, N, d, bs = 1, 2, 96, 16, 32
    nb = N // bs
    row_ptr, col_idx = oracle_mod.dense_csr(B, H, N, bs, causal)
    Q, K, V, dO = (rand_bf16(rng, (B, H, N, d)) for _ in range(4))
    dQ, dK, dV = oracle_mod.attn_bwd(Q, K, V, dO, bs, causal, row_ptr, col_idx)
    q, k, v = (torch.tensor(fvals(x), dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    s = q @ k.transpose(-1, -2) / math.sqrt(d)
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    o = torch.softmax(s, dim=-1) @ v
    (o * torch.tensor(fvals(dO), dtype=torch.float64)).sum().backward()
    for mine, ref in ((dQ, q.grad), (dK, k.grad), (dV, v.grad)):
        assert np.max(np.abs(mine - ref.numpy())) < 1e-11


def test_attn_bwd_dense_identities(oracle_mod):
    """Dense, non-causal: every softmax row sums to one and is invariant to a common
    shift of the keys, so sum_u dV_u = sum_t dO_t and sum_u dK_u = 0 per head."""
    rng = np.random.default_rng(13)
    B, H, N, d, bs = 2, 2, 100, 8, 32
    row_ptr, col_idx = oracle_mod.dense_csr(B, H, N, bs, False)
    Q, K, V, dO = (rand_bf16(rng, (B, H, N, d)) for _ in range(4))
    dQ, dK, dV = oracle_mod.attn_bwd(Q, K, V, dO, bs, False, row_ptr, col_idx)
    assert np.max(np.abs(dV.sum(axis=2) - fvals(dO).sum(axis=2))) < 1e-10
    assert np.max(np.abs(dK.sum(axis=2))) < 1e-10


@pytest.mark.parametrize("causal", [False, True])
def test_attn_bwd_sampled_equals_full_gradients(oracle_mod, causal):
    """The sampled-token gradients are the full oracle's rows, value for value: query
    tokens anywhere (ragged last block, empty CSR rows), key tokens grouped and
    ungrouped, a key block no row selects (zero gradients), a repeated token."""
    rng = np.random.default_rng(21 + causal)
    B, H, N, d, bs = 2, 2, 100, 16, 32
    nb = -(-N // bs)
    row_ptr, col_idx = random_csr(rng, B * H * nb, nb, p_keep=0.5, allow_empty=True)
    Q, K, V, dO = (rand_bf16(rng, (B, H, N, d)) for _ in range(4))
    dQ, dK, dV = oracle_mod.attn_bwd(Q, K, V, dO, bs, causal, row_ptr, col_idx)
    total = B * H * N
    q_tok = np.r_[rng.choice(total, 20, replace=False), total - 1, 0]
    k_tok = np.r_[rng.choice(total, 24, replace=False), 3, 3, N - 1, total - 1]
    sq, sk, sv = oracle_mod.attn_bwd_sampled(Q, K, V, dO, bs, causal, row_ptr, col_idx, q_tok, k_tok)
    flat = lambda a: a.reshape(total, d)
    assert np.array_equal(sq, flat(dQ)[q_tok])
    assert np.array_equal(sk, flat(dK)[k_tok])
    assert np.array_equal(sv, flat(dV)[k_tok])


def test_attn_bwd_sampled_dense_matches_torch_autograd(oracle_mod):
    """Dense non-causal: the sampled rows equal fp64 autograd of softmax(QK^T/sqrt(d))V."""
    import torch
    rng = np.random.default_rng(23)
    B, H, N, d, bs = 1, 2, 80, 16, 32
    row_ptr, col_idx = oracle_mod.dense_csr(B, H, N, bs, False)
    Q, K, V, dO = (rand_bf16(rng, (B, H, N, d)) for _ in range(4))
    q, k, v = (torch.tensor(fvals(x), dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    o = torch.softmax(q @ k.transpose(-1, -2) / math.sqrt(d), dim=-1) @ v
    (o * torch.tensor(fvals(dO), dtype=torch.float64)).sum().backward()
    toks = np.array([0, 31, 32, 79, N + 5, 2 * N - 1])
    sq, sk, sv = oracle_mod.attn_bwd_sampled(Q, K, V, dO, bs, False, row_ptr, col_idx, toks, toks)
    for mine, ref in ((sq, q.grad), (sk, k.grad), (sv, v.grad)):
        assert np.max(np.abs(mine - ref.numpy().reshape(-1, d)[toks])) < 1e-11


# ---------------------------------------------------------------- e4m3 quantization

def test_e4m3_known_codes_ties_saturation_and_nan(oracle_mod):
    """Values of the E4M3FN format itself: exponent bias 7, 3 mantissa bits,
    subnormals m * 2^-9, largest finite 448, NaN at 0x7F; nearest rounding with
    ties to the even code; saturation at 448."""
    enc = oracle_mod.e4m3_encode
    table = oracle_mod.e4m3_decode_table()
    assert table[0x38] == 1.0 and table[0xB8] == -1.0 and table[0x7E] == 448.0 and table[0xFE] == -448.0
    assert table[0x08] == 2.0 ** -6 and table[0x01] == 2.0 ** -9 and table[0x07] == 7 * 2.0 ** -9
    assert table[0x39] == 1.125 and table[0x3F] == 1.875 and table[0x40] == 2.0
    assert np.isnan(table[0x7F]) and np.isnan(table[0xFF])
    assert enc(0.0) == 0x00 and enc(1.0) == 0x38 and enc(-2.0) == 0xC0 and enc(448.0) == 0x7E
    assert enc(1.0625) == 0x38          # halfway 1 | 1.125: to the even code 0x38
    assert enc(1.1875) == 0x3A          # halfway 1.125 | 1.25: to the even code 0x3A
    assert enc(1.07) == 0x39 and enc(1.05) == 0x38
    assert enc(2.0 ** -10) == 0x00      # halfway 0 | 2^-9: to the even code 0
    assert enc(3 * 2.0 ** -10) == 0x02  # halfway 2^-9 | 2^-8: to the even code 2
    assert enc(500.0) == 0x7E and enc(1e30) == 0x7E and enc(-1e30) == 0xFE and enc(464.0) == 0x7E
    assert enc(float("nan")) == 0x7F


def test_e4m3_round_trip_and_monotone(oracle_mod):
    enc = oracle_mod.e4m3_encode
    table = oracle_mod.e4m3_decode_table()
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert enc(table[c]) == c or (c == 0x80 and enc(table[c]) in (0x00, 0x80)), hex(c)
    xs = np.linspace(-460.0, 460.0, 20001)
    vals = table[[enc(x) for x in xs]]
    assert np.all(np.diff(vals) >= 0)


def test_quant_e4m3_block_scales_and_error_bound(oracle_mod):
    """Every block's scaled maximum lands in (224, 448]; an all-zero block gets the
    scale 2^0 and zero codes; each value is within half an e4m3 step of the input
    (relative 2^-4 in the normal range, 2^-10 * scale below it); the dequantized
    values are exact bf16 values."""
    rng = np.random.default_rng(31)
    B, H, N, d, bs = 2, 2, 300, 16, 64
    x = rng.standard_normal((B, H, N, d)).astype(np.float32)
    x[0, 1, 64:128] = 0.0                               # an all-zero block
    x[1, 0, 128:192] *= 1e-30                            # a tiny-magnitude block
    x[1, 1, 256:] *= 1e20                                # a huge-magnitude ragged last block
    X = f32_to_bf16_bits(x)
    codes, exps = oracle_mod.quant_e4m3(X, bs)
    xv = fvals(X)
    nb = -(-N // bs)
    for b in range(B):
        for h in range(H):
            for k in range(nb):
                blk = xv[b, h, k * bs:(k + 1) * bs]
                amax = np.max(np.abs(blk))
                e = int(exps[b, h, k])
                if amax == 0.0:
                    assert e == 0 and np.all(codes[b, h, k * bs:(k + 1) * bs] == 0)
                else:
                    assert 224.0 < amax * 2.0 ** -e <= 448.0
    deq = oracle_mod.dequant_e4m3(codes, exps, bs)
    scale = np.ldexp(1.0, np.repeat(exps, bs, axis=2)[:, :, :N])[..., None]
    err = np.abs(deq - xv)
    normal = np.abs(xv) >= 2.0 ** -6 * scale
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(xv[normal]))
    assert np.all(err[~normal] <= 2.0 ** -10 * np.broadcast_to(scale, xv.shape)[~normal])
    assert np.array_equal(fvals(f32_to_bf16_bits(deq.astype(np.float32))), deq)


def test_e4m3_input_rounding_against_the_attention_tolerances(oracle_mod):
    """Why the FP8 attention kernel is not built: exact fp64 attention on the
    e4m3-dequantized Q, K, V, against the same on the bf16 inputs, with the same mask.
    On structured inputs (peaked heads, scales up to 4, the video recipe at 4096
    tokens) input rounding alone moves O and LSE by whole units, far outside the
    path's tolerances (O max 2e-2, mean 2e-3, LSE 1e-3).  On i.i.d. inputs O stays
    inside, LSE does not."""
    import workloads as Wl
    deq = lambda X, bs: f32_to_bf16_bits(oracle_mod.dequant_e4m3(*oracle_mod.quant_e4m3(X, bs), bs).astype(np.float32))
    w = Wl.Workload("fp8probe", B=1, H=4, N=4096, d=128, bs=128, p=0.9, dist="structured", grid=(4, 32, 32),
                    head_scale=("uniform", 0.5, 4.0), seed=9)
    Q, K, V = Wl.generate(w)
    r = oracle_mod.route(Q, K, w.p, w.bs)
    toks = Wl.sample_tokens(w, per_head_blocks=2, rows_per_block=8)
    O0, L0 = oracle_mod.attn_rows(Q, K, V, w.bs, False, r.row_ptr, r.col_idx, toks)
    O1, L1 = oracle_mod.attn_rows(deq(Q, w.bs), deq(K, w.bs), deq(V, w.bs), w.bs, False, r.row_ptr, r.col_idx, toks)
    assert np.abs(O1 - O0).max() > 0.5 and np.abs(L1 - L0).max() > 0.5
    w2 = Wl.Workload("fp8iid", B=1, H=2, N=4096, d=128, bs=128, p=1.0, seed=10)
    Q, K, V = Wl.generate(w2)
    rp, ci = oracle_mod.dense_csr(1, 2, 4096, 128, False)
    toks = Wl.sample_tokens(w2, per_head_blocks=2, rows_per_block=8)
    O0, L0 = oracle_mod.attn_rows(Q, K, V, 128, False, rp, ci, toks)
    O1, L1 = oracle_mod.attn_rows(deq(Q, 128), deq(K, 128), deq(V, 128), 128, False, rp, ci, toks)
    err = np.abs(O1 - O0)
    assert err.max() < 2e-2 and err.mean() < 2e-3
    assert np.abs(L1 - L0).max() > 1e-3


# ------------------------------------------------------------------ SASA (NEXT-1)
# FVAttn review §1 Key Terms "SASA" and §3: after balancing, ranks with slack compute
# extra high-value blocks.  One GPU: ranks = SMs of the persistent grid (reading in
# oracle_sasa).  Pinned to closed forms, a hand-worked schedule and Graham's bound.

def test_route_candidates_uniform_scores_closed_form(oracle_mod):
    # K = 0: every score is 0, every probability 1/nb; the cut takes the first
    # ceil(p * nb) blocks by index and the candidates are the next ones by index.
    B, H, N, d, bs, p, kc = 1, 2, 640, 64, 64, 0.35, 8
    nb = N // bs
    rng = np.random.default_rng(3)
    Q = W.f32_to_bf16_bits(rng.standard_normal((B, H, N, d)).astype(np.float32))
    K = np.zeros_like(Q)
    r, cand, cand_p = oracle_mod.route_candidates(Q, K, p, bs, kc)
    keep = int(np.ceil(p * nb))
    for row in range(B * H * nb):
        assert list(r.col_idx[r.row_ptr[row]:r.row_ptr[row + 1]]) == list(range(keep))
        want = list(range(keep, min(nb, keep + kc))) + [-1] * max(0, keep + kc - nb)
        assert list(cand[row]) == want
        assert np.allclose(cand_p[row][: nb - keep], 1.0 / nb, rtol=0, atol=1e-15)


def test_route_candidates_are_the_best_unselected_blocks(oracle_mod):
    w = W.Workload("cand", B=1, H=3, N=1500, d=64, bs=64, p=0.6, dist="structured", grid=(6, 10, 25),
                   head_scale=("uniform", 0.5, 4.0), seed=7)
    Q, K, _ = W.generate(w)
    r, cand, cand_p = oracle_mod.route_candidates(Q, K, w.p, w.bs, 8)
    r0 = oracle_mod.route(Q, K, w.p, w.bs)
    assert np.array_equal(r.row_ptr, r0.row_ptr) and np.array_equal(r.col_idx, r0.col_idx)
    for row in range(w.rows):
        sel = set(r.col_idx[r.row_ptr[row]:r.row_ptr[row + 1]].tolist())
        c = [x for x in cand[row].tolist() if x >= 0]
        assert not sel.intersection(c) and len(set(c)) == len(c)
        assert len(c) == min(8, w.nb - len(sel))
        pr = cand_p[row][: len(c)]
        # non-increasing, below the last kept probability, the first equals the first dropped one
        assert np.all(np.diff(pr) <= 0) and (len(c) == 0 or pr[0] <= r.diag[row, 4])
        assert len(c) == 0 or pr[0] == r.diag[row, 5]


@pytest.mark.parametrize("BH,nb,seed", [(1, 5, 0), (3, 7, 1), (8, 16, 2)])
def test_head_order_brute_force(oracle_mod, BH, nb, seed):
    rng = np.random.default_rng(seed)
    counts = rng.integers(0, 5, size=(BH, nb))
    if BH > 2:
        counts[2] = counts[0]
    rp = np.zeros(BH * nb + 1, np.int32)
    rp[1:] = np.cumsum(counts.reshape(-1))
    heads = sorted(range(BH), key=lambda h: (-int(counts[h].sum()), h))
    want = [h * nb + i for h in heads for i in sorted(range(nb), key=lambda i: (-int(counts[h, i]), i))]
    assert list(oracle_mod.head_order(rp, BH, nb)) == want


def test_pair_items_hand_worked(oracle_mod):
    # one head, nb = 5 (three pairs, the last holding row 4 alone):
    # rows 0: {0, 2}, 1: {1, 2, 4}, 2: {3}, 3: {}, 4: {0, 4}
    rp = np.array([0, 2, 5, 6, 6, 8], np.int32)
    ci = np.array([0, 2, 1, 2, 4, 3, 0, 4], np.int32)
    pp, pc, pb = oracle_mod.pair_items(rp, ci, 1, 5)
    assert list(pp) == [0, 4, 5, 7]
    assert list(pc) == [0, 1, 2, 4, 3, 0, 4]
    assert list(pb) == [1, 2, 3, 2, 1, 1, 1]


@pytest.mark.parametrize("BH,nb,seed", [(1, 1, 0), (2, 7, 1), (3, 16, 2), (2, 33, 3)])
def test_pair_items_are_set_unions(oracle_mod, BH, nb, seed):
    rng = np.random.default_rng(seed)
    sets = []
    for r in range(BH * nb):
        kind = r % 4
        if kind == 0:
            sets.append([])
        elif kind == 1 and sets[-1]:
            sets.append(list(sets[-1]))         # the same list as the row before
        else:
            sets.append(sorted(rng.choice(nb, size=int(rng.integers(1, nb + 1)), replace=False).tolist()))
    rp = np.zeros(BH * nb + 1, np.int32)
    rp[1:] = np.cumsum([len(x) for x in sets])
    ci = np.asarray([j for x in sets for j in x], np.int32)
    pp, pc, pb = oracle_mod.pair_items(rp, ci, BH, nb)
    np_ = (nb + 1) // 2
    assert pp.size == BH * np_ + 1
    for b in range(BH):
        for i in range(np_):
            e0, e1 = pp[b * np_ + i], pp[b * np_ + i + 1]
            a = set(sets[b * nb + 2 * i])
            bb = set(sets[b * nb + 2 * i + 1]) if 2 * i + 1 < nb else set()
            cols = list(pc[e0:e1])
            assert cols == sorted(a | bb)
            assert [c for c, x in zip(cols, pb[e0:e1]) if x & 1] == sorted(a)
            assert [c for c, x in zip(cols, pb[e0:e1]) if x & 2] == sorted(bb)
            assert all(x in (1, 2, 3) for x in pb[e0:e1])


def _csr(counts):
    rp = np.zeros(len(counts) + 1, np.int32)
    rp[1:] = np.cumsum(counts)
    ci = np.concatenate([np.arange(c, dtype=np.int32) * 2 for c in counts]) if sum(counts) else np.zeros(0, np.int32)
    return rp, ci


def test_sasa_hand_worked_schedule(oracle_mod):
    # rows 0, 1, 2 with 3, 2, 2 blocks, queue order 0, 1, 2, two machines:
    # row 0 -> m0 (load 3), row 1 -> m1 (2), row 2 -> m1 (4); makespan 4, slack m0 = 1, m1 = 0,
    # so row 0 (the only row of m0) gets its first candidate.
    rp, ci = _csr([3, 2, 2])
    cand = np.array([[1, 3, -1], [1, 3, 5], [1, -1, -1]], np.int32)
    cand_p = np.array([[0.2, 0.1, 0.0], [0.3, 0.2, 0.1], [0.4, 0.0, 0.0]])
    s = oracle_mod.sasa(rp, ci, cand, cand_p, np.array([0, 1, 2], np.int32), 2)
    assert list(s.added) == [1, 0, 0]
    assert list(s.row_ptr) == [0, 4, 6, 8]
    assert list(s.col_idx[:4]) == [0, 1, 2, 4]
    assert s.added_mass[0] == 0.2 and s.added_mass[1] == 0.0
    # round robin: rows of 6, 1 and 2 blocks in that order on two machines: row 0 -> m0 (6),
    # row 1 -> m1 (1), row 2 -> m1 (3); m1's slack of 3 goes row 1, row 2, row 1
    rp, ci = _csr([6, 1, 2])
    cand = np.array([[-1] * 4, [1, 3, 5, 7], [1, 5, 7, 9]], np.int32)
    s = oracle_mod.sasa(rp, ci, cand, np.zeros((3, 4)), np.array([0, 1, 2], np.int32), 2)
    assert list(s.added) == [0, 2, 1]
    # one machine: no slack, nothing added
    s = oracle_mod.sasa(rp, ci, cand, np.zeros((3, 4)), np.array([0, 1, 2], np.int32), 1)
    assert not s.added.any() and np.array_equal(s.row_ptr, rp) and np.array_equal(s.col_idx, ci)


@pytest.mark.parametrize("rows,machines,kc,seed", [(40, 3, 4, 0), (200, 16, 8, 1), (1000, 148, 8, 2), (10, 30, 2, 3)])
def test_sasa_schedule_and_augmentation_invariants(oracle_mod, rows, machines, kc, seed):
    rng = np.random.default_rng(seed)
    counts = rng.integers(1, 60, size=rows)
    rp, ci = _csr(counts.tolist())
    cand = np.full((rows, kc), -1, np.int32)
    avail = rng.integers(0, kc + 1, size=rows)
    for r in range(rows):
        cand[r, : avail[r]] = 2 * counts[r] + 1 + 2 * np.arange(avail[r])   # odd: never among the selected
    cand_p = rng.random((rows, kc))
    order = np.argsort(-counts, kind="stable").astype(np.int32)
    s = oracle_mod.sasa(rp, ci, cand, cand_p, order, machines)
    # replay the schedule (least-loaded machine, lowest index on ties) to get per-machine loads
    load = np.zeros(machines, np.int64)
    mach = np.zeros(rows, np.int64)
    for r in order:
        m = int(np.argmin(load))
        mach[r] = m
        load[m] += counts[r]
    T = load.max()
    # Graham's list-scheduling bound
    assert T <= counts.sum() / machines + counts.max()
    for m in range(machines):
        rs = np.nonzero(mach == m)[0]
        extra = int(s.added[rs].sum())
        assert load[m] + extra <= T
        # the slack is used up unless every row of the machine ran out of candidates
        assert load[m] + extra == T or all(s.added[r] == avail[r] for r in rs)
    assert np.all(s.added <= avail)
    for r in range(rows):
        row = s.col_idx[s.row_ptr[r]:s.row_ptr[r + 1]]
        want = sorted(list(ci[rp[r]:rp[r + 1]]) + list(cand[r, : s.added[r]]))
        assert list(row) == want
        assert s.added_mass[r] == pytest.approx(cand_p[r, : s.added[r]].sum(), abs=1e-15)


# ------------------------------------------------------------------ RLB (NEXT-2)
# FVAttn review §1 Key Terms "RLB" and §3: heads move between GPUs once their work is
# known.  Pinned to hand-worked plans, the sum-of-squares descent every move makes, the
# absence of an improving move at the end, and an exhaustive optimum on tiny instances.

def _rlb_apply(work, moves):
    ranks, units = work.shape
    owner = np.repeat(np.arange(ranks), units)
    loads = work.sum(1).astype(np.int64)
    flat = work.reshape(-1)
    ss = [int((loads ** 2).sum())]
    for u, s, d in moves:
        assert owner[u] == s and s != d
        owner[u] = d
        loads[s] -= flat[u]
        loads[d] += flat[u]
        ss.append(int((loads ** 2).sum()))
    return owner, loads, ss


def test_rlb_hand_worked(oracle_mod):
    assert oracle_mod.rlb_plan(np.array([[10, 1], [1, 1]])).tolist() == [[1, 0, 1]]
    # loads 10 / 0: both 5s are below the gap; the lower home index moves, then the loads are equal
    assert oracle_mod.rlb_plan(np.array([[5, 5], [0, 0]])).tolist() == [[0, 0, 1]]
    assert oracle_mod.rlb_plan(np.array([[3, 4], [4, 3]])).size == 0          # already balanced
    assert oracle_mod.rlb_plan(np.array([[7, 9, 1]])).size == 0               # one rank
    # three ranks: 12 / 2 / 1 -> rank 0 gives 4 to rank 2 (gap 11) and 4 to rank 1 (gap 6): 4 / 6 / 5;
    # then rank 1 gives its home unit 0 (work 1, below the gap 2) to rank 0: 5 / 5 / 5
    moves = oracle_mod.rlb_plan(np.array([[4, 4, 4], [1, 1, 0], [1, 0, 0]]))
    _, loads, _ = _rlb_apply(np.array([[4, 4, 4], [1, 1, 0], [1, 0, 0]]), moves)
    assert moves.tolist() == [[0, 0, 2], [1, 0, 1], [3, 1, 0]] and loads.tolist() == [5, 5, 5]


@pytest.mark.parametrize("ranks,units,seed", [(2, 4, 0), (3, 8, 1), (8, 5, 2), (8, 40, 3), (4, 1, 4)])
def test_rlb_invariants(oracle_mod, ranks, units, seed):
    rng = np.random.default_rng(seed)
    work = rng.integers(0, 200, size=(ranks, units)) * (rng.random((ranks, 1)) * 3 + 0.2)
    work = work.astype(np.int64)
    moves = oracle_mod.rlb_plan(work)
    owner, loads, ss = _rlb_apply(work, moves)
    assert all(b < a for a, b in zip(ss, ss[1:]))               # every move lowers the sum of squares
    assert loads.max() <= work.sum(1).max()
    src, dst = int(np.argmax(loads)), int(np.argmin(loads))
    gap = loads[src] - loads[dst]
    flat = work.reshape(-1)
    assert not any(owner[u] == src and 0 < flat[u] < gap for u in range(flat.size))


def test_rlb_close_to_exhaustive_optimum_on_tiny_instances(oracle_mod):
    import itertools as it
    rng = np.random.default_rng(9)
    for _ in range(40):
        ranks, units = int(rng.integers(2, 4)), int(rng.integers(1, 4))
        work = rng.integers(0, 30, size=(ranks, units)).astype(np.int64)
        flat = work.reshape(-1)
        best = min(max(sum(int(flat[u]) for u in range(flat.size) if a[u] == r) for r in range(ranks))
                   for a in it.product(range(ranks), repeat=flat.size))
        _, loads, _ = _rlb_apply(work, oracle_mod.rlb_plan(work))
        assert best <= loads.max() <= best + flat.max()


def test_near_tie_report_flags_exact_ties_at_the_cut(oracle_mod):
    """The GPU routing tests report rows whose cut separates two blocks of (almost)
    equal probability.  With K = 0 every score ties, so every row cut short of all
    blocks is such a row; on structured inputs none is expected."""
    from tests.gpu_util import near_tie_rows
    w = W.Workload("ties", B=1, H=2, N=1000, d=64, bs=64, p=0.5, seed=5)
    Q, K, _ = W.generate(w)
    r = oracle_mod.route(Q, np.zeros_like(K), w.p, w.bs)
    cut = np.diff(r.row_ptr) < w.nb
    assert cut.all() and np.array_equal(near_tie_rows(r, w.p), cut)
    w2 = W.Workload("no_ties", B=1, H=2, N=1000, d=64, bs=64, p=0.7, dist="structured", grid=(4, 10, 25),
                    head_scale=("uniform", 0.5, 4.0), seed=6)
    Q2, K2, _ = W.generate(w2)
    assert not near_tie_rows(oracle_mod.route(Q2, K2, w2.p, w2.bs), w2.p).any()
