"""Test infrastructure: the fp64 CPU oracle for top-p routed block-sparse attention.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The product (``top_routed_block_b200``)
never does, and the oracle shares no code with it.

The arithmetic lives in ``fvattn_oracle.c`` (plain C loops, fp64, index-order
sums, compiled with ``-ffp-contract=off``).  This module only builds that file
and marshals numpy arrays into it.  Sources, per function, are cited in the C
file: the FVAttn review, §1 Key Terms (top-p routing) and §1 RLB / §3 (per-head
work after the mask), and the FlashAttention review, §Background "Motivation"
(S = QK^T, P = softmax(S), O = PV) and §Model "Tiling Softmax".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fvattn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library in-tree (gcc, -O2, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               "-pthread", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_pool.argtypes = [P, i64, i32, i32, i32, P, i32]
        lib.oracle_route.argtypes = [P, P, i32, i32, i32, i32, i32, dbl, P, P, i64, P, P, i32]
        lib.oracle_attn_rows.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, P, P, P, i64, P, P, i32]
        lib.oracle_attn_tiled.argtypes = lib.oracle_attn_rows.argtypes
        lib.oracle_lpt_order.argtypes = [P, i64, P]
        lib.oracle_route_cand.argtypes = [P, P, i32, i32, i32, i32, i32, dbl, P, P, i64, P, P, P, P, i32, i32]
        lib.oracle_head_order.argtypes = [P, i64, i64, P]
        lib.oracle_pair_items.argtypes = [P, P, i64, i64, P, P, P]
        lib.oracle_sasa.argtypes = [P, P, i64, P, P, i32, P, i32, P, P, P, P, i64]
        lib.oracle_rlb_plan.argtypes = [P, i32, i32, i32, P, P, P, P]
        lib.oracle_attn_bwd.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i32, P, P, P, P, P, i32]
        lib.oracle_attn_bwd_sampled.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i32, P, P, P, i64, P, P, P,
                                                i64, P, P, i32]
        lib.oracle_quant_e4m3.argtypes = [P, i64, i32, i32, i32, P, P]
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_double.restype = dbl
        lib.oracle_e4m3_from_double.argtypes = [dbl]
        lib.oracle_e4m3_from_double.restype = ctypes.c_uint8
        for f in ("oracle_pool", "oracle_route", "oracle_attn_rows", "oracle_attn_tiled", "oracle_lpt_order",
                  "oracle_attn_bwd", "oracle_attn_bwd_sampled", "oracle_quant_e4m3", "oracle_route_cand",
                  "oracle_head_order", "oracle_sasa", "oracle_rlb_plan"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _bits(x: np.ndarray) -> np.ndarray:
    """bf16 tensors travel as their uint16 bit patterns."""
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return x


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def pool(X: np.ndarray, bs: int, nthreads: int | None = None) -> np.ndarray:
    """Mean of each block of ``bs`` tokens over the tokens that exist: X [B,H,N,d] -> [B,H,nb,d] fp64."""
    X = _bits(X)
    B, H, N, d = X.shape
    nb = -(-N // bs)
    out = np.empty((B, H, nb, d), dtype=np.float64)
    rc = _load().oracle_pool(_ptr(X), B * H, N, d, bs, _ptr(out), nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_pool failed ({rc})")
    return out


class Route:
    """CSR block mask from the oracle, with per-row diagnostics.

    ``diag[r]`` = (mass kept, mass without the last kept block, last kept score,
    first dropped score, last kept probability, first dropped probability).
    """

    def __init__(self, row_ptr, col_idx, head_counts, diag):
        self.row_ptr, self.col_idx, self.head_counts, self.diag = row_ptr, col_idx, head_counts, diag

    @property
    def counts(self) -> np.ndarray:
        return np.diff(self.row_ptr)


def route(Q: np.ndarray, K: np.ndarray, p: float, bs: int, nthreads: int | None = None) -> Route:
    Q, K = _bits(Q), _bits(K)
    B, H, N, d = Q.shape
    if K.shape != Q.shape:
        raise ValueError("Q and K shapes differ")
    nb = -(-N // bs)
    rows = B * H * nb
    row_ptr = np.empty(rows + 1, dtype=np.int32)
    cap = rows * nb
    col_idx = np.empty(max(cap, 1), dtype=np.int32)
    head_counts = np.empty(B * H, dtype=np.int32)
    diag = np.empty((rows, 6), dtype=np.float64)
    rc = _load().oracle_route(_ptr(Q), _ptr(K), B, H, N, d, bs, float(p), _ptr(row_ptr), _ptr(col_idx), cap,
                              _ptr(head_counts), _ptr(diag), nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_route failed ({rc})")
    return Route(row_ptr, col_idx[: row_ptr[-1]].copy(), head_counts, diag)


def _attn(fn, Q, K, V, bs, causal, row_ptr, col_idx, tokens, nthreads):
    Q, K, V = _bits(Q), _bits(K), _bits(V)
    B, H, N, d = Q.shape
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
    col_idx = np.ascontiguousarray(col_idx, dtype=np.int32)
    if col_idx.size == 0:
        col_idx = np.zeros(1, dtype=np.int32)
    O = np.empty((tokens.size, d), dtype=np.float64)
    LSE = np.empty(tokens.size, dtype=np.float64)
    rc = fn(_ptr(Q), _ptr(K), _ptr(V), B, H, N, d, bs, 1 if causal else 0, _ptr(row_ptr), _ptr(col_idx),
            _ptr(tokens), tokens.size, _ptr(O), _ptr(LSE), nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle attention failed ({rc})")
    return O, LSE


def attn_rows(Q, K, V, bs, causal, row_ptr, col_idx, tokens, nthreads=None):
    """Row-wise definition. ``tokens`` are flat indices (b*H + h)*N + t. Returns O [n,d], LSE [n] (fp64)."""
    return _attn(_load().oracle_attn_rows, Q, K, V, bs, causal, row_ptr, col_idx, tokens, nthreads)


def attn_tiled(Q, K, V, bs, causal, row_ptr, col_idx, tokens, nthreads=None):
    """Block-by-block online softmax; equal to :func:`attn_rows` up to rounding."""
    return _attn(_load().oracle_attn_tiled, Q, K, V, bs, causal, row_ptr, col_idx, tokens, nthreads)


def attn_bwd(Q, K, V, dO, bs, causal, row_ptr, col_idx, nthreads=None):
    """Gradients of sum(dO * O) for the attention of :func:`attn_rows` (all bf16 bit
    patterns [B,H,N,d]). Returns dQ, dK, dV as fp64 [B,H,N,d]."""
    Q, K, V, dO = _bits(Q), _bits(K), _bits(V), _bits(dO)
    B, H, N, d = Q.shape
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
    col_idx = np.ascontiguousarray(col_idx, dtype=np.int32)
    if col_idx.size == 0:
        col_idx = np.zeros(1, dtype=np.int32)
    dQ = np.empty((B, H, N, d), dtype=np.float64)
    dK = np.empty_like(dQ)
    dV = np.empty_like(dQ)
    rc = _load().oracle_attn_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(dO), B, H, N, d, bs, 1 if causal else 0,
                                 _ptr(row_ptr), _ptr(col_idx), _ptr(dQ), _ptr(dK), _ptr(dV),
                                 nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_attn_bwd failed")
    return dQ, dK, dV


def attn_bwd_sampled(Q, K, V, dO, bs, causal, row_ptr, col_idx, q_tokens, k_tokens, nthreads=None):
    """The gradients of :func:`attn_bwd` at sampled tokens only (global indices
    b*H*N + h*N + t): dQ rows of ``q_tokens`` and dK, dV rows of ``k_tokens``, fp64
    [n, d] each.  Key tokens are grouped by (head, key block) internally so that one
    query row's softmax serves every sampled key of its block."""
    Q, K, V, dO = _bits(Q), _bits(K), _bits(V), _bits(dO)
    B, H, N, d = Q.shape
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
    col_idx = np.ascontiguousarray(col_idx, dtype=np.int32)
    if col_idx.size == 0:
        col_idx = np.zeros(1, dtype=np.int32)
    q_tokens = np.ascontiguousarray(q_tokens, dtype=np.int64)
    k_tokens = np.ascontiguousarray(k_tokens, dtype=np.int64)
    key = (k_tokens // N) * (N // bs + 1) + (k_tokens % N) // bs  # (head, key block)
    perm = np.argsort(key, kind="stable")
    ks = np.ascontiguousarray(k_tokens[perm])
    starts = np.flatnonzero(np.r_[True, np.diff(key[perm]) != 0]) if ks.size else np.zeros(0, np.int64)
    group_ptr = np.ascontiguousarray(np.r_[starts, ks.size], dtype=np.int64)
    dQ = np.empty((max(q_tokens.size, 1), d), dtype=np.float64)
    dKs = np.empty((max(ks.size, 1), d), dtype=np.float64)
    dVs = np.empty_like(dKs)
    rc = _load().oracle_attn_bwd_sampled(_ptr(Q), _ptr(K), _ptr(V), _ptr(dO), B, H, N, d, bs, 1 if causal else 0,
                                         _ptr(row_ptr), _ptr(col_idx), _ptr(q_tokens), q_tokens.size, _ptr(dQ),
                                         _ptr(ks), _ptr(group_ptr), group_ptr.size - 1, _ptr(dKs), _ptr(dVs),
                                         nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_attn_bwd_sampled failed")
    dK = np.empty((k_tokens.size, d), dtype=np.float64)
    dV = np.empty_like(dK)
    dK[perm] = dKs[: ks.size]
    dV[perm] = dVs[: ks.size]
    return dQ[: q_tokens.size], dK, dV


def e4m3_encode(x: float) -> int:
    """The e4m3 code of one value: nearest, ties to the even code, saturating at 448."""
    return int(_load().oracle_e4m3_from_double(float(x)))


def e4m3_decode_table() -> np.ndarray:
    """fp64 value of each of the 256 e4m3 codes (NaN for 0x7F and 0xFF)."""
    lib = _load()
    return np.array([lib.oracle_e4m3_to_double(c) for c in range(256)], dtype=np.float64)


def quant_e4m3(X, bs):
    """Block quantization of bf16 bit patterns [B,H,N,d] to e4m3: codes uint8
    [B,H,N,d] and the power-of-two scale exponent of every (batch*head, block),
    int32 [B,H,nb]; value = e4m3 value of the code * 2^exponent."""
    X = _bits(X)
    B, H, N, d = X.shape
    nb = -(-N // bs)
    codes = np.empty((B, H, N, d), dtype=np.uint8)
    exps = np.empty((B, H, nb), dtype=np.int32)
    rc = _load().oracle_quant_e4m3(_ptr(X), B * H, N, d, bs, _ptr(codes), _ptr(exps))
    if rc != 0:
        raise ValueError("oracle_quant_e4m3 failed")
    return codes, exps


def dequant_e4m3(codes, exps, bs):
    """fp64 values of block-quantized e4m3 data (see :func:`quant_e4m3`)."""
    B, H, N, d = codes.shape
    table = e4m3_decode_table()
    scale = np.ldexp(1.0, np.repeat(exps, bs, axis=2)[:, :, :N])
    return table[codes] * scale[..., None]


def route_candidates(Q: np.ndarray, K: np.ndarray, p: float, bs: int, kc: int, nthreads: int | None = None):
    """:func:`route` plus, per row, the kc key blocks that follow the cut in the
    routing order (-1 past the last block) and their probabilities."""
    Q, K = _bits(Q), _bits(K)
    B, H, N, d = Q.shape
    nb = -(-N // bs)
    rows = B * H * nb
    row_ptr = np.empty(rows + 1, dtype=np.int32)
    cap = rows * nb
    col_idx = np.empty(max(cap, 1), dtype=np.int32)
    head_counts = np.empty(B * H, dtype=np.int32)
    diag = np.empty((rows, 6), dtype=np.float64)
    cand = np.empty((rows, max(kc, 1)), dtype=np.int32)
    cand_p = np.empty((rows, max(kc, 1)), dtype=np.float64)
    rc = _load().oracle_route_cand(_ptr(Q), _ptr(K), B, H, N, d, bs, float(p), _ptr(row_ptr), _ptr(col_idx), cap,
                                   _ptr(head_counts), _ptr(diag), _ptr(cand), _ptr(cand_p), kc,
                                   nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_route_cand failed ({rc})")
    return Route(row_ptr, col_idx[: row_ptr[-1]].copy(), head_counts, diag), cand[:, :kc], cand_p[:, :kc]


def head_order(row_ptr: np.ndarray, BH: int, nb: int) -> np.ndarray:
    """The attention queue: heads by total selected blocks (desc, ties lower head),
    rows of a head by block count (desc, ties lower row)."""
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
    order = np.empty(BH * nb, dtype=np.int32)
    if _load().oracle_head_order(_ptr(row_ptr), BH, nb, _ptr(order)) != 0:
        raise ValueError("oracle_head_order failed")
    return order


def pair_items(row_ptr: np.ndarray, col_idx: np.ndarray, BH: int, nb: int):
    """Work items at block 64: pairs of query blocks (2i, 2i+1) of a head, each the
    union of the two rows' key blocks.  Returns (pair_ptr, pair_col, pair_bits), a CSR
    over the BH * ceil(nb/2) pairs; bits 1: row 2i selected the block, 2: row 2i+1."""
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
    col_idx = np.ascontiguousarray(col_idx if len(col_idx) else np.zeros(1), dtype=np.int32)
    np_ = (nb + 1) // 2
    pair_ptr = np.empty(BH * np_ + 1, dtype=np.int32)
    cap = max(int(row_ptr[-1]), 1)
    pair_col = np.empty(cap, dtype=np.int32)
    pair_bits = np.empty(cap, dtype=np.int32)
    if _load().oracle_pair_items(_ptr(row_ptr), _ptr(col_idx), BH, nb, _ptr(pair_ptr), _ptr(pair_col),
                                 _ptr(pair_bits)) != 0:
        raise ValueError("oracle_pair_items failed")
    n = int(pair_ptr[-1])
    return pair_ptr, pair_col[:n].copy(), pair_bits[:n].copy()


class Sasa:
    """Augmented CSR and, per row, the number and probability mass of the added blocks."""

    def __init__(self, row_ptr, col_idx, added, added_mass):
        self.row_ptr, self.col_idx, self.added, self.added_mass = row_ptr, col_idx, added, added_mass


def sasa(row_ptr, col_idx, cand, cand_p, order, machines: int) -> Sasa:
    """Slack-aware augmentation of a routed mask over `machines` SMs (see
    oracle_sasa in fvattn_oracle.c)."""
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
    col_idx = np.ascontiguousarray(col_idx if len(col_idx) else np.zeros(1), dtype=np.int32)
    cand = np.ascontiguousarray(cand, dtype=np.int32)
    cand_p = np.ascontiguousarray(cand_p, dtype=np.float64)
    order = np.ascontiguousarray(order, dtype=np.int32)
    rows = row_ptr.size - 1
    kc = cand.shape[1] if cand.ndim == 2 else 0
    added = np.empty(max(rows, 1), dtype=np.int32)
    mass = np.empty(max(rows, 1), dtype=np.float64)
    rp = np.empty(rows + 1, dtype=np.int32)
    cap = int(row_ptr[-1]) + rows * kc
    ci = np.empty(max(cap, 1), dtype=np.int32)
    rc = _load().oracle_sasa(_ptr(row_ptr), _ptr(col_idx), rows, _ptr(cand), _ptr(cand_p), kc, _ptr(order),
                             int(machines), _ptr(added), _ptr(mass), _ptr(rp), _ptr(ci), cap)
    if rc != 0:
        raise ValueError(f"oracle_sasa failed ({rc})")
    return Sasa(rp, ci[: rp[-1]].copy(), added[:rows], mass[:rows])


def rlb_plan(work: np.ndarray, max_moves: int | None = None):
    """Head moves balancing per-rank work (work: int [ranks, units]); returns the
    moves as an int32 array [n, 3] of (home unit r*units+i, source rank, destination)."""
    work = np.ascontiguousarray(work, dtype=np.int64)
    ranks, units = work.shape
    cap = ranks * units * 4 if max_moves is None else max_moves
    mu = np.empty(max(cap, 1), np.int32)
    ms = np.empty(max(cap, 1), np.int32)
    md = np.empty(max(cap, 1), np.int32)
    n = ctypes.c_int32(0)
    if _load().oracle_rlb_plan(_ptr(work), ranks, units, cap, _ptr(mu), _ptr(ms), _ptr(md), ctypes.byref(n)) != 0:
        raise ValueError("oracle_rlb_plan failed")
    return np.stack([mu[: n.value], ms[: n.value], md[: n.value]], axis=1)


def lpt_order(row_ptr: np.ndarray) -> np.ndarray:
    """Rows sorted by selected-block count descending, ties by row id ascending."""
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
    rows = row_ptr.size - 1
    order = np.empty(max(rows, 1), dtype=np.int32)
    rc = _load().oracle_lpt_order(_ptr(row_ptr), rows, _ptr(order))
    if rc != 0:
        raise ValueError("oracle_lpt_order failed")
    return order[:rows]


def dense_csr(B: int, H: int, N: int, bs: int, causal: bool = False):
    """Every key block for every query block (lower triangle of blocks if causal)."""
    nb = -(-N // bs)
    counts = []
    cols = []
    for _bh in range(B * H):
        for i in range(nb):
            js = list(range(i + 1)) if causal else list(range(nb))
            counts.append(len(js))
            cols.extend(js)
    row_ptr = np.zeros(len(counts) + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum(counts)
    return row_ptr, np.asarray(cols, dtype=np.int32)
