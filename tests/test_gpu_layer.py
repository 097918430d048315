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
from tests.parity import TOL, check_err, f64, normwise_rel_err

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
                                   (129, 257, 136), (1000, 48, 520),
                                   # more tiles than SMs: several tiles per persistent CTA,
                                   # both TMEM accumulators, the stage ring across tiles
                                   (2560, 3072, 64), (2048, 2560, 328),
                                   # K > 1024: the deep-ring configuration
                                   (300, 520, 1544), (1280, 4096, 2048)])
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
        check_err(normwise_rel_err(f64(y), ref), TOL["bf16"], "y")


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
    check_err(normwise_rel_err(got, ref), TOL["bf16"])
    assert sdm.device_error() == 0


def test_layer_out_fused_into_the_read(sdm):
    """The row pass with the output side's RMS-norm and swish gate fused into it: its fp32
    read output equals the plain row pass's bit for bit, its bf16 operand a matches the
    oracle's normalised and gated read, and y = a @ Wo matches the oracle's layer output."""
    orc = oracle.default()
    for wl in (S.MID.scaled(T=256), S.HEADLINE.scaled(B=2, H=2, T=200, n_sub=128)):
        inp = S.generate(wl, device="cuda")
        d = sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R,
                     wl.x_dtype, wl.v_dtype)
        sel = sdm.score_qk(d, inp["q"], inp["k"], inp["skw"], inp["skr"])
        ws = sdm.workspace(d)
        st = sdm.State(d, inp["M0"])
        sdm.state_reset(d, st)
        sdm.forward_plan(d, inp["alpha"], inp["beta"], *sel, st, ws)
        out0 = torch.empty((wl.B, wl.H, wl.T, wl.d_v), device="cuda")
        sdm.forward_run(d, inp["v"], inp["beta"], *sel, st, out0, ws)
        gen = torch.Generator(device="cuda").manual_seed(5)
        g = torch.randn(wl.B, wl.T, wl.H * wl.d_v, device="cuda", generator=gen).to(torch.bfloat16)
        wn = 0.5 + torch.rand(wl.d_v, device="cuda", generator=gen)
        st2 = sdm.State(d, inp["M0"])
        sdm.state_reset(d, st2)
        sdm.forward_plan(d, inp["alpha"], inp["beta"], *sel, st2, ws)
        out1, a = sdm.forward_run_gated(d, inp["v"], inp["beta"], *sel, st2, g, wn, 1e-6, ws=ws)
        dm = 4 * wl.H * wl.n_sub
        Wo_t = (torch.randn(dm, wl.H * wl.d_v, device="cuda", generator=gen) /
                np.sqrt(wl.H * wl.d_v)).to(torch.bfloat16)
        y = sdm.gemm_bf16(a.reshape(wl.B * wl.T, wl.H * wl.d_v), Wo_t)
        torch.cuda.synchronize()
        assert torch.equal(out0, out1)
        # a against the normalised, gated read computed from the same fp32 read in fp64
        o64 = f64(out1).transpose(0, 2, 1, 3)  # [B,T,H,d_v]
        rms = np.sqrt((o64 ** 2).mean(-1, keepdims=True) + 1e-6)
        z = f64(g).reshape(wl.B, wl.T, wl.H, wl.d_v)
        a_ref = (o64 / rms * f64(wn) * (z / (1 + np.exp(-z)))).reshape(wl.B, wl.T, -1)
        check_err(normwise_rel_err(f64(a), a_ref), TOL["bf16"], "a")
        rows = np.array([0, 1, 77, wl.B * wl.T - 1])
        ref = orc.layer_out(f64(out1), f64(g), f64(wn), f64(Wo_t), rows=rows)
        check_err(normwise_rel_err(f64(y).reshape(wl.B * wl.T, dm)[rows], ref), TOL["bf16"], "y")
        assert sdm.device_error() == 0


def test_gemm_validation(sdm):
    A = torch.zeros(4, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sdm.SdmError):
        sdm.gemm_bf16(A, torch.zeros(4, 12, dtype=torch.bfloat16, device="cuda"))  # K % 8


def _layer_in_case(sdm, B, H, T, dk, dv, dm, n_sub, vdt, seed):
    gen = torch.Generator(device="cuda").manual_seed(seed)
    hs = 2 * dk + 2 * dv + 2
    x = torch.randn(B, T, dm, device="cuda", generator=gen).to(torch.bfloat16)
    Win_t = (torch.randn(H * hs, dm, device="cuda", generator=gen) / np.sqrt(dm)).to(torch.bfloat16)
    A_log = torch.randn(H, device="cuda", generator=gen) * 0.5
    dt = torch.randn(H, device="cuda", generator=gen) * 0.5
    d = sdm.Dims(B, H, T, dk, n_sub, dv, 8, 8, 8, "bf16", vdt)
    return d, x, Win_t, A_log, dt


@pytest.mark.parametrize("B,H,T,dk,dv,dm,vdt", [(2, 2, 50, 32, 16, 64, "bf16"),
                                                (1, 4, 130, 128, 128, 512, "bf16"),
                                                (2, 3, 9, 16, 8, 40, "f32")])
def test_layer_in_vs_oracle(sdm, B, H, T, dk, dv, dm, vdt):
    d, x, Win_t, A_log, dt = _layer_in_case(sdm, B, H, T, dk, dv, dm, 16, vdt, seed=T + dm)
    r = sdm.layer_in(d, x, Win_t, A_log, dt)
    torch.cuda.synchronize()
    ref = oracle.default().layer_in(f64(x), f64(Win_t), f64(A_log), f64(dt), H, dk, dv)
    for name in ("q", "k", "v", "g"):
        assert normwise_rel_err(f64(r[name]), ref[name]) <= 1e-2, name  # bf16 outputs
    # gates: fp32 from fp32 accumulation of exact bf16 products
    assert np.abs(f64(r["alpha"]) - ref["alpha"]).max() <= 1e-4
    assert np.abs(f64(r["beta"]) - ref["beta"]).max() <= 1e-4
    assert sdm.device_error() == 0


def test_layer_forward_chain(sdm):
    """x -> layer_in -> prefill (scoring + recurrence) -> layer_out, mid-like shapes, each
    stage against the oracle fed the GPU's previous stage (bf16 rounding at the stage
    boundaries is the GPU's own)."""
    orc = oracle.default()
    B, H, T, dk, dv, n, k, W = 1, 2, 96, 128, 128, 64, 16, 16
    dm = 4 * H * n
    d, x, Win_t, A_log, dt = _layer_in_case(sdm, B, H, T, dk, dv, dm, n, "bf16", seed=5)
    d = sdm.Dims(B, H, T, dk, n, dv, k, W, W, "bf16", "bf16")
    gen = torch.Generator(device="cuda").manual_seed(6)
    skw = (torch.randn(H, 2, n, dk // 2, device="cuda", generator=gen) / 8).to(torch.bfloat16)
    skr = (torch.randn(H, 2, n, dk // 2, device="cuda", generator=gen) / 8).to(torch.bfloat16)
    M0 = torch.randn(H, n * n, dv, device="cuda", generator=gen) * 0.02
    wn = torch.rand(dv, device="cuda", generator=gen) + 0.5
    Wo_t = (torch.randn(dm, H * dv, device="cuda", generator=gen) / np.sqrt(H * dv)).to(torch.bfloat16)
    r = sdm.layer_in(d, x, Win_t, A_log, dt)
    st = sdm.State(d, M0)
    sdm.state_reset(d, st)
    o, (widx, ww, ridx, rw) = sdm.prefill(d, r["q"], r["k"], r["v"], r["alpha"], r["beta"],
                                          skw, skr, st)
    y = sdm.layer_out(d, o, r["g"], wn, Wo_t)
    torch.cuda.synchronize()
    ref_in = orc.layer_in(f64(x), f64(Win_t), f64(A_log), f64(dt), H, dk, dv)
    assert normwise_rel_err(f64(r["q"]), ref_in["q"]) <= 1e-2
    outs = []
    for h in range(H):
        s = orc.fresh_lazy_state(f64(M0[h]))
        outs.append(orc.recur_lazy(f64(r["v"][0, h]), f64(r["alpha"][0, h]), f64(r["beta"][0, h]),
                                   widx[0, h].cpu().numpy(), f64(ww[0, h]), ridx[0, h].cpu().numpy(),
                                   f64(rw[0, h]), s))
    ref_o = np.stack(outs).reshape(B, H, T, dv)
    check_err(normwise_rel_err(f64(o), ref_o), TOL["bf16"], "o")
    ref_y = orc.layer_out(f64(o), f64(r["g"]), f64(wn), f64(Wo_t))
    check_err(normwise_rel_err(f64(y), ref_y), TOL["bf16"], "y")
    assert sdm.device_error() == 0
