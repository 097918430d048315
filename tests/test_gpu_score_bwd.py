"""GPU parity of sdm_score_backward (the gradient through the scoring, selections held
fixed) against the oracle's score_backward, on the GPU scorer's own selections."""
from __future__ import annotations

import pytest
import torch

import oracle
import sdm_synth as S
from tests.parity import check_err, f64, normwise_rel_err

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


CASES = {
    # name: (x dtype, B, H, T, d_k, n, k_half, top)
    "tiny_f32": ("f32", 1, 2, 40, 32, 16, 4, 4),
    "mid_bf16": ("bf16", 2, 2, 70, 128, 256, 32, 32),
    "top_above_32": ("bf16", 1, 2, 30, 64, 64, 48, 48),
    "wide_half": ("f32", 2, 1, 12, 256, 32, 8, 16),
}


@pytest.mark.parametrize("name", list(CASES))
def test_score_backward_vs_oracle(sdm, orc, name):
    xd, B, H, T, d_k, n, kh, top = CASES[name]
    wl = S.MID.scaled(B=B, H=H, T=T, d_k=d_k, n_sub=n, d_v=16, k_half=kh, W=min(top, 64),
                      R=min(top, 64), x_dtype=xd, v_dtype="f32", subkey_var=2.0 / d_k,
                      seed=3000 + len(name))
    inp = {k: v.cuda() for k, v in S.generate(wl, with_m0=False).items()}
    d = sdm.Dims(B, H, T, d_k, n, 16, kh, wl.W, wl.R, xd, "f32")
    g = torch.Generator(device="cuda").manual_seed(7)
    for x, sk in ((inp["k"], inp["skw"]), (inp["q"], inp["skr"])):
        idx, w = sdm.score_topk(d, x, sk, top)
        idx, w = idx.view(B, H, T, top), w.view(B, H, T, top)
        dw = torch.randn(B, H, T, top, device="cuda", generator=g)
        dx, dsk = sdm.score_backward(d, x, sk, top, idx, w, dw)
        torch.cuda.synchronize()
        assert sdm.device_error() == 0
        dx_o, dsk_o = orc.score_backward(f64(x), f64(sk), idx.cpu().numpy(), f64(dw))
        check_err(normwise_rel_err(f64(dx), dx_o), 1e-4, "dx")
        check_err(normwise_rel_err(f64(dsk), dsk_o), 1e-4, "dsubkeys")
        # a second call adds to the table gradient
        _, dsk2 = sdm.score_backward(d, x, sk, top, idx, w, dw, dsubkeys=dsk.clone())
        torch.cuda.synchronize()
        check_err(normwise_rel_err(f64(dsk2), 2 * dsk_o), 1e-4, "dsubkeys accumulated")
