"""GPU parity of the row scorer (few tokens per call: decode steps and short prefills).

Shapes the tensor-core scorer does not take (fewer than 64 tokens, fp32) go through the row
scorer when n <= 512 and through the generic warp scorer otherwise; both are checked against the oracle's product-key selection, including ragged
row counts, top above k_half, non-multiple-of-32 n, fp32 and bf16, and exact ties.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import sdm_synth as S
from tests.parity import compare_selection, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sdm():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_state_linear_score_b200 as m
    m.device_error(clear=True)
    return m


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def _dims(sdm, wl):
    return sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R,
                    wl.x_dtype, wl.v_dtype)


def _check(sdm, orc, wl, x, sk, top, exact_only=False):
    d = _dims(sdm, wl)
    idx, w = sdm.score_topk(d, x, sk, top)
    torch.cuda.synchronize()
    assert sdm.device_error() == 0
    idx_o, sc_o, w_o = orc.score(f64(x), f64(sk), wl.k_half, top, mode=oracle.MODE_PK)
    gi = idx.cpu().numpy()
    if exact_only:
        np.testing.assert_array_equal(gi, idx_o)
    exact, near, bad = compare_selection(orc, f64(x), f64(sk), gi, idx_o, sc_o, wl.n_sub)
    assert not bad, f"selections differ beyond near ties at {bad[:5]}"
    assert near <= max(2, 0.01 * gi[..., 0].size), (exact, near)
    same = np.all(gi == idx_o, axis=-1)
    assert same.any()
    assert np.abs(f64(w)[same] - w_o[same]).max() < 1e-5
    return idx, w


CASES = {
    # name: (x dtype, B, H, T, d_k, n, k_half, top)
    "decode_mid": ("bf16", 7, 3, 1, 128, 256, 32, 32),
    "top_above_k": ("bf16", 3, 2, 5, 64, 40, 8, 20),
    "f32_k64": ("f32", 2, 2, 9, 32, 100, 64, 64),
    "n512": ("bf16", 2, 1, 3, 128, 512, 64, 48),
    "top_k_squared": ("f32", 5, 1, 3, 16, 16, 4, 16),
    "n_one_lane": ("bf16", 1, 2, 6, 32, 20, 5, 7),
    "fallback_large_n": ("bf16", 1, 2, 2, 128, 600, 16, 16),
    "fallback_f32_large_n": ("f32", 2, 1, 4, 32, 700, 8, 8),
}


@pytest.mark.parametrize("name", list(CASES))
def test_row_scorer_vs_oracle(sdm, orc, name):
    xd, B, H, T, d_k, n, kh, top = CASES[name]
    wl = S.MID.scaled(B=B, H=H, T=T, d_k=d_k, n_sub=n, d_v=16, k_half=kh, W=min(top, 64),
                      R=min(top, 64), x_dtype=xd, v_dtype="f32", subkey_var=2.0 / d_k,
                      seed=2000 + len(name))
    inp = {k: v.cuda() for k, v in S.generate(wl, with_m0=False).items()}
    for x, sk in ((inp["k"], inp["skw"]), (inp["q"], inp["skr"])):
        _check(sdm, orc, wl, x, sk, top)


def test_row_scorer_exact_ties(sdm, orc):
    """Zero queries (every score 0) and repeated sub-key rows: ties go to the lower index."""
    wl = S.MID.scaled(B=5, H=2, T=1, n_sub=64, k_half=16, W=24, R=24, d_v=16, v_dtype="f32")
    inp = {k: v.cuda() for k, v in S.generate(wl, with_m0=False).items()}
    x = inp["k"].clone()
    x[0].zero_()                      # every score of batch 0 is exactly 0
    sk = inp["skw"].clone()
    sk[:, :, 8:16] = sk[:, :, 0:8]    # sub-keys 8..15 repeat 0..7 in every table
    sk[:, :, 40:48] = sk[:, :, 0:8]
    _check(sdm, orc, wl, x, sk, wl.W, exact_only=True)


def test_decode_step_reads_both_roles(sdm, orc):
    """The decode step scores both roles in one launch; each matches the oracle."""
    wl = S.DECODE.scaled(B=6, H=3, T=1, decode_steps=1, n_sub=128, k_half=32, W=32, R=24)
    inp = {k: v.cuda() for k, v in S.generate(wl).items()}
    d = _dims(sdm, wl)
    st = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st)
    o, (wi, wv, ri, rv) = sdm.decode_step(d, inp["q"][:, :, 0].contiguous(),
                                          inp["k"][:, :, 0].contiguous(),
                                          inp["v"][:, :, 0].contiguous(),
                                          inp["alpha"][:, :, 0].contiguous(),
                                          inp["beta"][:, :, 0].contiguous(), inp["skw"],
                                          inp["skr"], st)
    torch.cuda.synchronize()
    assert sdm.device_error() == 0
    for x, sk, top, gi, gw in ((inp["k"][:, :, :1], inp["skw"], wl.W, wi, wv),
                               (inp["q"][:, :, :1], inp["skr"], wl.R, ri, rv)):
        idx_o, sc_o, w_o = orc.score(f64(x), f64(sk), wl.k_half, top, mode=oracle.MODE_PK)
        g = gi.view(wl.B, wl.H, 1, top).cpu().numpy()
        exact, near, bad = compare_selection(orc, f64(x), f64(sk), g, idx_o, sc_o, wl.n_sub)
        assert not bad and near <= 2, (exact, near, bad[:3])
