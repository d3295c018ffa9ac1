"""FP8 (e4m3) block-sparse attention forward (fvattn_sparse_fwd_fp8) against the
fp64 oracle applied to the dequantized inputs ("Accelerating HunyuanVideo
inference with ParaAttention" (WaveSpeed), § "FP8 dynamic quantization": attention
on FP8 activations; reading: OCP E4M3FN codes with one power-of-two scale per
(head, block)).

The oracle's inputs come from the oracle's own quantizer; the GPU quantizer's
codes are asserted byte-equal to them first, so both sides see the same values.
The dequantized values are exact bf16 values, so the reference is the plain
attention oracle on them.

Tolerance (derived; the mode is approximate by construction):
  * S: e4m3 x e4m3 products are exact and summed in fp32, so a score's error is
    at most d * 2^-24 * sum_c |q_c k_c| / sqrt(d) (fp32 summation bound), e_s.
  * P: the PV MMA takes P as e4m3 (3 mantissa bits): a value in the normal range
    is off by at most 2^-4 of itself; a value scaled below the normal range
    (the tile's V scale is 2^(e_v - E) <= 1, so up to 2^(max e_v - min e_v) of the
    head below) is off by at most 2^-10 2^(E - e_v) absolute, or flushed to zero
    (off by at most itself).  With P normalised to its row maximum:
      |dO_c| <= [sum_u (2^-4 P_u + min(P_u, 2^(-10 + D_h))) |v_uc|] / sum_u P_u
                + 2 max_u e_s,u * [sum_u P_u |v_uc|] / sum_u P_u     (score errors)
                + 2^-8 |O_c|                                          (bf16 output)
    with D_h = max - min block exponent of V over the head.
  * LSE uses the unrounded P: |dLSE| <= max_u e_s,u + 1e-5 (fp32 log and sum).
Checked element by element on every token of small cases and on sampled tokens
(query block 0, the last ragged block, random blocks of every head) at full size."""
import numpy as np
import pytest
import torch

import workloads as W
from tests.gpu_util import gpu_route, to_dev

pytestmark = pytest.mark.gpu

SMALL = [
    (W.Workload("fp8_small_routed", B=1, H=3, N=1000, d=128, bs=128, p=0.7, dist="structured", grid=(5, 8, 25),
                head_scale=("uniform", 0.5, 4.0), seed=61), False),
    (W.Workload("fp8_small_dense", B=2, H=2, N=700, d=128, bs=128, p=1.0, seed=62), False),
    (W.Workload("fp8_small_causal", B=1, H=2, N=900, d=128, bs=128, p=1.0, seed=63), True),
    (W.Workload("fp8_small_bs64", B=1, H=2, N=1500, d=128, bs=64, p=0.9, dist="structured", grid=(6, 10, 25),
                head_scale=("uniform", 0.5, 4.0), seed=64), False),
    (W.Workload("fp8_large_scores", B=1, H=2, N=600, d=128, bs=128, p=0.8, dist="structured", grid=(6, 10, 10),
                head_scale=("const", 6.0), seed=65), False),
    # block 64, causal, an odd block count (the last pair holds one row) and a ragged last block
    (W.Workload("fp8_bs64_causal_odd", B=1, H=2, N=900, d=128, bs=64, p=1.0, seed=66), True),
]


def quantize_both(oracle_mod, X, bs):
    """Oracle codes and exponents (the reference's inputs) and the GPU quantizer's,
    asserted equal byte for byte."""
    import top_routed_block_b200 as fv
    codes_o, exps_o = oracle_mod.quant_e4m3(X, bs)
    codes_g, exps_g = fv.fvattn_quant_e4m3(to_dev(X), bs)
    torch.cuda.synchronize()
    assert np.array_equal(exps_g.cpu().numpy(), exps_o)
    assert np.array_equal(codes_g.cpu().numpy(), codes_o)
    return codes_o, exps_o, codes_g, exps_g


def dequant_bits(oracle_mod, codes, exps, bs):
    """Dequantized values as bf16 bit patterns (exact: e4m3 values times powers of two
    are bf16 values) and as fp64."""
    x = oracle_mod.dequant_e4m3(codes, exps, bs)
    bits = W.f32_to_bf16_bits(x.astype(np.float32))
    assert np.array_equal(W.bf16_bits_to_f32(bits).astype(np.float64), x)
    return bits, x


def allowed_keys(rp, ci, w, causal, bh, t):
    r = bh * w.nb + t // w.bs
    ks = [np.arange(kb * w.bs, min(w.N, (kb + 1) * w.bs)) for kb in ci[rp[r]:rp[r + 1]]]
    keys = np.concatenate(ks) if ks else np.zeros(0, np.int64)
    return keys[keys <= t] if causal else keys


def bounds(Qd, Kd, Vd, vexp, rp, ci, w, causal, tokens, O_ref):
    """Per-element bound on |O_gpu - O_ref| and per-token bound on |LSE_gpu - LSE_ref|
    (see the module docstring), from the dequantized fp64 inputs."""
    d = w.d
    Qf, Kf, Vf = (x.reshape(w.B * w.H, w.N, d) for x in (Qd, Kd, Vd))
    ob = np.zeros((tokens.size, d))
    lb = np.zeros(tokens.size)
    for i, tok in enumerate(tokens):
        bh, t = divmod(int(tok), w.N)
        keys = allowed_keys(rp, ci, w, causal, bh, t)
        if keys.size == 0:
            continue
        ev = vexp.reshape(w.B * w.H, w.nb)[bh]
        Dh = float(ev.max() - ev.min())
        q = Qf[bh, t]
        k = Kf[bh, keys]
        s = k @ q / np.sqrt(d)
        es = d * 2.0 ** -24 * (np.abs(k) @ np.abs(q)) / np.sqrt(d)
        P = np.exp(s - s.max())
        l = P.sum()
        av = np.abs(Vf[bh, keys])
        pv = P @ av
        ob[i] = ((2.0 ** -4) * pv + np.minimum(P, 2.0 ** (-10 + Dh)) @ av) / l + 2.0 * es.max() * pv / l \
            + 2.0 ** -8 * np.abs(O_ref[i]) + 1e-6
        lb[i] = es.max() + 1e-5
    return ob, lb


def check(O, LSE, O_ref, L_ref, ob, lb, tokens, d, what):
    o = O.reshape(-1, d).float()[torch.from_numpy(tokens).to(O.device)].cpu().numpy().astype(np.float64)
    l = LSE.reshape(-1)[torch.from_numpy(tokens).to(O.device)].cpu().numpy().astype(np.float64)
    err = np.abs(o - O_ref)
    fin = np.isfinite(L_ref)
    assert np.array_equal(fin, np.isfinite(l)), f"{what}: LSE finiteness differs"
    lerr = np.abs(l[fin] - L_ref[fin])
    over = err > ob
    msg = (f"{what}: O max {err.max():.3e} mean {err.mean():.3e} (bound mean {ob.mean():.3e}), "
           f"{int(over.sum())} elements over the bound; LSE max {lerr.max() if lerr.size else 0:.3e}")
    assert not over.any(), msg
    assert (lerr <= lb[fin]).all(), msg
    return msg


def run_case(w, causal, oracle_mod, tokens):
    import top_routed_block_b200 as fv
    Q, K, V = W.generate(w)
    qc, qe, dqc, dqe = quantize_both(oracle_mod, Q, w.bs)
    kc, ke, dkc, dke = quantize_both(oracle_mod, K, w.bs)
    vc, ve, dvc, dve = quantize_both(oracle_mod, V, w.bs)
    if causal:
        rp, ci = oracle_mod.dense_csr(w.B, w.H, w.N, w.bs, causal=True)
    else:
        rp, ci, _ = gpu_route(to_dev(Q), to_dev(K), w.p, w.bs)
    drp = torch.from_numpy(np.ascontiguousarray(rp, np.int32)).cuda()
    dci = torch.from_numpy(np.ascontiguousarray(ci, np.int32)).cuda()
    O, LSE, st = fv.fvattn_sparse_fwd_fp8(dqc, dkc, dvc, dqe, dke, dve, drp, dci, w.bs, causal)
    fv.check_status(st, "fvattn_sparse_fwd_fp8")
    Qb, Qd = dequant_bits(oracle_mod, qc, qe, w.bs)
    Kb, Kd = dequant_bits(oracle_mod, kc, ke, w.bs)
    Vb, Vd = dequant_bits(oracle_mod, vc, ve, w.bs)
    O_ref, L_ref = oracle_mod.attn_rows(Qb, Kb, Vb, w.bs, causal, rp, ci, tokens)
    ob, lb = bounds(Qd, Kd, Vd, ve, rp, ci, w, causal, tokens, O_ref)
    return check(O, LSE, O_ref, L_ref, ob, lb, tokens, w.d, w.name)


@pytest.mark.parametrize("w,causal", SMALL, ids=lambda x: x.name if hasattr(x, "name") else str(x))
def test_fp8_small_every_token(w, causal, oracle_mod):
    print(run_case(w, causal, oracle_mod, np.arange(w.B * w.H * w.N, dtype=np.int64)))


def sampled_tokens(w, seed):
    rng = np.random.default_rng(seed)
    toks = []
    for bh in range(w.B * w.H):
        for qb in sorted({0, w.nb - 1, *rng.integers(0, w.nb, 2).tolist()}):
            lo, hi = qb * w.bs, min(w.N, (qb + 1) * w.bs)
            toks.append(bh * w.N + np.arange(lo, hi, 16))
    return np.concatenate(toks).astype(np.int64)


@pytest.mark.slow
@pytest.mark.parametrize("w,causal", [(W.VIDEO, False), (W.DENSE, False), (W.DENSE, True)],
                         ids=["video_dit", "dense", "dense_causal"])
def test_fp8_full_size_sampled(w, causal, oracle_mod):
    print(run_case(w, causal, oracle_mod, sampled_tokens(w, 17)))


def test_fp8_rejects_unsupported_shapes():
    import top_routed_block_b200 as fv
    lib = fv.load_library()
    # d = 64 (e4m3 rows of 64 bytes) is not supported; null pointers are checked after the shape
    assert lib.fvattn_sparse_fwd_fp8(None, None, None, None, None, None, None, None, 1, 1, 256, 64, 128, 0, None,
                                     None, None, 0, None, None) == fv.FVATTN_ERR_UNSUPPORTED
