"""e4m3 block quantization on the GPU (fvattn_quant_e4m3) against the oracle's
quant_e4m3, byte for byte: codes and per-block scale exponents (the FP8 input step;
reading: OCP E4M3FN values, power-of-two block scales, nearest rounding with ties to
the even code, saturation at 448)."""
import numpy as np
import pytest
import torch

import workloads as W
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu


def run_and_compare(oracle_mod, X, bs):
    import top_routed_block_b200 as fv
    codes, exps = fv.fvattn_quant_e4m3(to_dev(X), bs)
    torch.cuda.synchronize()
    rc, re = oracle_mod.quant_e4m3(X, bs)
    got_c, got_e = codes.cpu().numpy(), exps.cpu().numpy()
    assert np.array_equal(got_e, re), np.argwhere(got_e != re)[:5]
    bad = np.argwhere(got_c != rc)
    assert bad.size == 0, (bad[:5], got_c[tuple(bad[0])], rc[tuple(bad[0])])
    return got_c, got_e


def edge_values(rng, shape):
    """Normal values with every kind of block: all zero, tiny, huge, and values sitting
    exactly halfway between e4m3 neighbours after scaling (ties)."""
    x = rng.standard_normal(shape).astype(np.float32)
    B, H, N, d = shape
    x[0, 0, 0:64] = 0.0
    x[0, 1, 64:128] *= 1e-30
    x[-1, -1, 128:192] *= 1e25
    # block max 256 (scale 2^0); 1.0625, 1.1875, 2^-10 and 3*2^-10 are exact ties
    x[0, 0, 192:256] = 1.0
    x[0, 0, 192, 0] = 256.0
    x[0, 0, 193, :8] = [1.0625, 1.1875, -1.0625, 2.0 ** -10, 3 * 2.0 ** -10, 17.0, 18.0, 19.0]
    return x


@pytest.mark.parametrize("d,bs,N", [(64, 64, 300), (128, 128, 1000), (128, 64, 777), (64, 128, 257)])
def test_quant_e4m3_matches_oracle(oracle_mod, d, bs, N):
    rng = np.random.default_rng(71 + d + bs)
    x = edge_values(rng, (2, 3, N, d))
    run_and_compare(oracle_mod, W.f32_to_bf16_bits(x), bs)


def test_quant_e4m3_infinities_saturate_and_nan_stays_nan(oracle_mod):
    rng = np.random.default_rng(73)
    x = rng.standard_normal((1, 2, 256, 64)).astype(np.float32)
    x[0, 0, 3, 5] = np.inf              # block 0 of head 0 keeps the scale 2^0
    x[0, 0, 4, 6] = -np.inf
    X = W.f32_to_bf16_bits(x)
    codes, exps = run_and_compare(oracle_mod, X, 64)
    assert exps[0, 0, 0] == 0 and codes[0, 0, 3, 5] == 0x7E and codes[0, 0, 4, 6] == 0xFE
    import top_routed_block_b200 as fv
    x[0, 1, 70, 1] = np.nan             # NaN does not count toward its block's maximum
    X = W.f32_to_bf16_bits(x)
    codes, exps = fv.fvattn_quant_e4m3(to_dev(X), 64)
    rc, re = oracle_mod.quant_e4m3(X, 64)
    c = codes.cpu().numpy()
    assert np.array_equal(exps.cpu().numpy(), re)
    assert c[0, 1, 70, 1] in (0x7F, 0xFF)
    mask = np.ones(c.shape, bool)
    mask[0, 1, 70, 1] = False
    assert np.array_equal(c[mask], rc[mask])


def test_quant_e4m3_full_size_video_q(oracle_mod):
    """Q of the video-DiT configuration (B1 H40 N32760 d128, block 128), every byte."""
    Q, _, _ = W.generate(W.VIDEO)
    codes, exps = run_and_compare(oracle_mod, Q, W.VIDEO.bs)
    assert exps.shape == (1, 40, W.VIDEO.nb)
