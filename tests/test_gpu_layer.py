"""GPU parity of the tensor-core GEMM and of the SDM layer's output side.

GEMM: bf16 operands, fp32 accumulation (tcgen05) against numpy fp64 on the same bf16
values: products of bf16 are exact in fp32, so the only error is fp32 accumulation,
bounded by about K * 2^-24 relative to sum |a||b|.  Layer output: RMS-norm, swish gate
and the output projection against the oracle; the GPU rounds the gated, normalised
operand to bf16 before the projection, so the bound is the bf16 tolerance of the
recurrence tests (normwise 2e-2).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import sdm_synth as S
from tests.parity import TOL, f64, normwise_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sdm():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_state_linear_score_b200 as m
    m.device_error(clear=True)
    return m


def gemm_check(sdm, M, N, K, seed):
    gen = torch.Generator(device="cuda").manual_seed(seed)
    A = torch.randn(M, K, device="cuda", generator=gen).to(torch.bfloat16)
    Bt = torch.randn(N, K, device="cuda", generator=gen).to(torch.bfloat16)
    C = sdm.gemm_bf16(A, Bt)
    torch.cuda.synchronize()
    a, b = f64(A), f64(Bt)
    ref = a @ b.T
    bound = (np.abs(a) @ np.abs(b).T) * (K * 2.0 ** -24) + 1e-30
    err = np.abs(f64(C) - ref)
    assert (err <= 4 * bound).all(), float((err / bound).max())
    return C


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (256, 512, 512), (200, 300, 72), (1, 16, 8),
                                   (129, 257, 136), (1000, 48, 520)])
def test_gemm_vs_fp64(sdm, M, N, K):
    gemm_check(sdm, M, N, K, seed=M * 7 + N * 3 + K)


def test_gemm_full_size_projection(sdm):
    # the mid workload's output projection: M = B*T = 8192, K = H*d_v = 512, N = d_model =
    # 4*H*n = 4096; sampled rows against fp64
    M, N, K = 8192, 4096, 512
    gen = torch.Generator(device="cuda").manual_seed(3)
    A = torch.randn(M, K, device="cuda", generator=gen).to(torch.bfloat16)
    Bt = torch.randn(N, K, device="cuda", generator=gen).to(torch.bfloat16)
    C = sdm.gemm_bf16(A, Bt)
    torch.cuda.synchronize()
    rows = torch.randint(0, M, (64,), generator=torch.Generator().manual_seed(4)).cuda()
    a, b = f64(A[rows]), f64(Bt)
    ref = a @ b.T
    bound = (np.abs(a) @ np.abs(b).T) * (K * 2.0 ** -24)
    assert (np.abs(f64(C[rows]) - ref) <= 4 * bound).all()
    assert sdm.device_error() == 0


def test_layer_out_vs_oracle(sdm):
    orc = oracle.default()
    for (B, H, T, dv, dm) in [(2, 2, 40, 16, 64), (1, 4, 130, 128, 300), (2, 3, 7, 64, 8)]:
        gen = torch.Generator(device="cuda").manual_seed(B * 100 + T)
        o = torch.randn(B, H, T, dv, device="cuda", generator=gen)
        g = torch.randn(B, T, H * dv, device="cuda", generator=gen).to(torch.bfloat16)
        wn = torch.rand(dv, device="cuda", generator=gen) + 0.5
        Wo_t = (torch.randn(dm, H * dv, device="cuda", generator=gen) / np.sqrt(H * dv)).to(torch.bfloat16)
        d = sdm.Dims(B, H, T, 128, 16, dv, 4, 4, 4, "bf16", "bf16")
        y = sdm.layer_out(d, o, g, wn, Wo_t, eps=1e-6)
        torch.cuda.synchronize()
        ref = orc.layer_out(f64(o), f64(g), f64(wn), f64(Wo_t), eps=1e-6)
        assert normwise_rel_err(f64(y), ref) <= TOL["bf16"]


def test_layer_out_after_prefill(sdm):
    # the read output of a real prefill through the output side, mid shapes (d_model =
    # 4*H*n); rows sampled against the oracle
    orc = oracle.default()
    wl = S.MID.scaled(T=256)
    inp = S.generate(wl, device="cuda")
    d = sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R,
                 wl.x_dtype, wl.v_dtype)
    st = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st)
    out, _ = sdm.prefill(d, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                         inp["skw"], inp["skr"], st)
    dm = 4 * wl.H * wl.n_sub
    gen = torch.Generator(device="cuda").manual_seed(11)
    g = torch.randn(wl.B, wl.T, wl.H * wl.d_v, device="cuda", generator=gen).to(torch.bfloat16)
    wn = torch.ones(wl.d_v, device="cuda")
    Wo_t = (torch.randn(dm, wl.H * wl.d_v, device="cuda", generator=gen) /
            np.sqrt(wl.H * wl.d_v)).to(torch.bfloat16)
    y = sdm.layer_out(d, out, g, wn, Wo_t)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 77, 255, 256, 300, 511])
    ref = orc.layer_out(f64(out), f64(g), f64(wn), f64(Wo_t), rows=rows)
    got = f64(y).reshape(wl.B * wl.T, dm)[rows]
    assert normwise_rel_err(got, ref) <= TOL["bf16"]
    assert sdm.device_error() == 0


def test_gemm_validation(sdm):
    A = torch.zeros(4, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sdm.SdmError):
        sdm.gemm_bf16(A, torch.zeros(4, 12, dtype=torch.bfloat16, device="cuda"))  # K % 8
