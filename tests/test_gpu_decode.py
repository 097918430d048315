"""GPU parity of the one-launch decode step (decode_fused_kernel: a cluster of two CTAs scores
four sequences' keys and queries and runs their recurrence steps) against the oracle: every step's
selections of both roles, the outputs and the final memory of every (b,h), under both decay
rules, for the three sub-key counts it takes (n = 128, 256, 512: 4, 8, 16 scores per lane),
d_v = 64, 128, 192 (one or two float4 columns per lane), bf16 and fp32 values, and numbers of
sequences that leave the last cluster partly empty (B = 3, 5)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import sdm_synth as S
from tests.parity import TOL, check_err, f64, normwise_rel_err
from tests.test_gpu_parity import check_selection

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


def _dims(sdm, wl, T=None, decay="all"):
    return sdm.Dims(wl.B, wl.H, wl.T if T is None else T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half,
                    wl.W, wl.R, wl.x_dtype, wl.v_dtype, decay=decay)


@pytest.mark.parametrize("n_sub,d_v,vdt,W,R,decay", [
    (128, 64, "bf16", 32, 32, "all"),
    (256, 128, "bf16", 32, 32, "all"),
    (256, 128, "bf16", 32, 32, "touched"),
    (512, 192, "f32", 32, 32, "all"),
    (256, 128, "f32", 16, 24, "all"),
])
def test_decode_fused_vs_oracle(sdm, orc, n_sub, d_v, vdt, W, R, decay):
    wl = S.DECODE.scaled(B=3 if n_sub != 256 else 5, H=2, T=24, decode_steps=5, n_sub=n_sub, d_v=d_v, v_dtype=vdt,
                         k_half=32, W=W, R=R)
    inp = {k: v.cuda() for k, v in S.generate(wl).items()}
    d = _dims(sdm, wl, decay=decay)
    dd = _dims(sdm, wl, T=1, decay=decay)
    assert sdm.decode_path(dd) == sdm.DECODE_FUSED
    st = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st)
    T0 = wl.T
    sl = lambda x: x[:, :, :T0].contiguous()
    out0, sel0 = sdm.prefill(d, sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["alpha"]),
                             sl(inp["beta"]), inp["skw"], inp["skr"], st)
    outs, sels = [], []
    for s in range(wl.decode_steps):
        t = T0 + s
        o, sel = sdm.decode_step(dd, inp["q"][:, :, t].contiguous(), inp["k"][:, :, t].contiguous(),
                                 inp["v"][:, :, t].contiguous(), inp["alpha"][:, :, t].contiguous(),
                                 inp["beta"][:, :, t].contiguous(), inp["skw"], inp["skr"], st)
        outs.append(o.clone())
        sels.append([x.clone().view(wl.B, wl.H, 1, -1) for x in sel])
    M = sdm.state_materialize(d, st)
    torch.cuda.synchronize()
    assert sdm.device_error() == 0
    for s, (wi, wv, ri, rv) in enumerate(sels):
        t = T0 + s
        check_selection(orc, inp["k"][:, :, t:t + 1], inp["skw"], wi, wv, wl.k_half, W, n_sub)
        check_selection(orc, inp["q"][:, :, t:t + 1], inp["skr"], ri, rv, wl.k_half, R, n_sub)
    cat = lambda i: torch.cat([sel0[i]] + [x[i] for x in sels], dim=2).cpu()
    widx, ww, ridx, rw = cat(0), cat(1), cat(2), cat(3)
    got = torch.cat([out0] + [o[:, :, None] for o in outs], dim=2)
    for b in range(wl.B):
        for h in range(wl.H):
            args = (f64(inp["v"][b, h]), f64(inp["alpha"][b, h]), f64(inp["beta"][b, h]),
                    np.asarray(widx[b, h]), f64(ww[b, h]), np.asarray(ridx[b, h]), f64(rw[b, h]))
            if decay == "touched":
                o_ref, M_ref = orc.recur_touched(*args, f64(inp["M0"][h]))
            else:
                stt = orc.fresh_lazy_state(f64(inp["M0"][h]))
                o_ref = orc.recur_lazy(*args, stt)
                M_ref = orc.materialize(stt)
            check_err(normwise_rel_err(f64(got[b, h]), o_ref), TOL[vdt], f"out (b,h)={(b, h)}")
            check_err(normwise_rel_err(f64(M[b, h]), M_ref), TOL[vdt], f"memory (b,h)={(b, h)}")
