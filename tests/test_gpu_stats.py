"""GPU parity of the memory-utilisation diagnostics (sdm_weight_stats) against the oracle.

Appendix D.1 "Memory Utilization and Access": cumulative top-k mass and the entropy-based
effective-key measure of post-softmax selected-slot weights, with means and token-level
quantiles.  Per-row values and means are compared within fp32 rounding; the GPU quantiles
must be exactly the order statistics of the GPU's own per-row values, and within the largest
per-row difference of the oracle's (order statistics are 1-Lipschitz in the max norm).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import sdm_synth as S

pytestmark = pytest.mark.gpu

PROBS = (0.0, 0.1, 0.5, 0.9, 1.0)


@pytest.fixture(scope="module")
def sdm():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_state_linear_score_b200 as m
    return m


def check(sdm, w: torch.Tensor, probs=PROBS):
    orc = oracle.default()
    g = sdm.weight_stats(w, probs)
    torch.cuda.synchronize()
    r = orc.weight_stats(w.double().cpu().numpy(), probs)
    K = w.shape[-1]
    cum = g["cum"].double().cpu().numpy()
    eff = g["eff"].double().cpu().numpy().reshape(-1)
    assert np.abs(cum - r["cum"]).max() <= 1e-5 * K
    d_eff = np.abs(eff - r["eff"].reshape(-1)).max()
    assert d_eff <= 2e-6
    assert np.abs(g["mean_cum"].double().cpu().numpy() - r["mean_cum"]).max() <= 1e-5 * K
    assert abs(float(g["mean_eff"]) - r["mean_eff"]) <= 2e-6
    srt = np.sort(g["eff"].cpu().numpy().reshape(-1))
    rows = srt.size
    for q, p, qo in zip(g["quant"].cpu().numpy(), probs, r["quant"]):
        assert q == srt[int(np.floor(p * (rows - 1)))]  # exact order statistic
        assert abs(float(q) - qo) <= d_eff + 1e-7
    return g


def test_stats_of_scoring_weights(sdm):
    # the write and read weights the scoring produces on the mid-size workload (several
    # blocks of rows plus a ragged tail)
    wl = S.MID.scaled(T=300)
    inp = S.generate(wl, device="cuda")
    d = sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R,
                 wl.x_dtype, wl.v_dtype)
    widx, ww, ridx, rw = sdm.selection_buffers(d)
    sdm.score_topk(d, inp["k"], inp["skw"], wl.W, widx, ww)
    sdm.score_topk(d, inp["q"], inp["skr"], wl.R, ridx, rw)
    for w in (ww, rw):
        g = check(sdm, w)
        assert abs(float(g["mean_cum"][-1]) - 1.0) < 1e-5  # softmax rows sum to 1


def test_stats_closed_forms(sdm):
    K = 16
    g = check(sdm, torch.full((1000, K), 1.0 / K, device="cuda"))
    assert torch.allclose(g["eff"], torch.ones_like(g["eff"]), atol=1e-6)
    w = torch.zeros(513, K, device="cuda")
    w[:, 0] = 1.0
    g = check(sdm, w)
    assert torch.allclose(g["eff"], torch.full_like(g["eff"], 1.0 / K), atol=1e-7)


@pytest.mark.parametrize("rows,K", [(1, 1), (1, 64), (255, 7), (257, 64), (70001, 32)])
def test_stats_shapes(sdm, rows, K):
    gen = torch.Generator(device="cuda").manual_seed(rows * 131 + K)
    x = torch.rand(rows, K, device="cuda", generator=gen) + 0.01
    w = torch.sort(x / x.sum(1, keepdim=True), dim=1, descending=True).values
    check(sdm, w.contiguous())


def test_stats_full_size_long_context_rows(sdm):
    # as many rows as the long-context workload's read weights (B*H*T = 4,194,304), K = 64;
    # sampled per-row checks, exact quantiles of the GPU values
    wl = S.LONG
    rows, K = wl.B * wl.H * wl.T, wl.R
    gen = torch.Generator(device="cuda").manual_seed(5)
    x = torch.randn(rows, K, device="cuda", generator=gen)
    w = torch.softmax(x, dim=1)
    w = torch.sort(w, dim=1, descending=True).values.contiguous()
    g = sdm.weight_stats(w, PROBS)
    torch.cuda.synchronize()
    idx = torch.randint(0, rows, (2000,), generator=torch.Generator().manual_seed(1))
    r = oracle.default().weight_stats(w[idx.cuda()].double().cpu().numpy(), PROBS)
    assert np.abs(g["eff"][idx.cuda()].double().cpu().numpy() - r["eff"]).max() <= 2e-6
    assert np.abs(g["cum"][idx.cuda()].double().cpu().numpy() - r["cum"]).max() <= 1e-5 * K
    srt = np.sort(g["eff"].cpu().numpy())
    for q, p in zip(g["quant"].cpu().numpy(), PROBS):
        assert q == srt[int(np.floor(p * (rows - 1)))]
    mean_eff = float(np.mean(g["eff"].double().cpu().numpy()))
    assert abs(float(g["mean_eff"]) - mean_eff) <= 1e-6


def test_stats_validation(sdm):
    w = torch.full((4, 8), 0.125, device="cuda")
    with pytest.raises(sdm.SdmError):
        sdm.weight_stats(w, probs=(1.5,))
    with pytest.raises(sdm.SdmError):
        sdm.weight_stats(torch.full((4, 65), 1 / 65, device="cuda"))
