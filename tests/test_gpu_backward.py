"""GPU parity of sdm_backward (the recurrence's gradients, A.3-style in-place replay and
undo) against the oracle's reverse-mode backward (recur_backward), element by element per
(b,h): dv, dalpha, dbeta, dww, drw and the gradient of the starting memory; and the state
given to the call comes back bit for bit.
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


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def _state_bits(st):
    # bit patterns: pristine rows of M are never initialised and may hold NaNs
    return (st.M.view(torch.int32).clone(), st.stamp.view(torch.int64).clone(),
            st.Lambda.view(torch.int64).clone())


def _case(sdm, orc, wl, decay, pool, seed, start_tokens=0, end_grad=False):
    inp = {k: v.cuda() for k, v in S.generate(wl).items()}
    T0, T = start_tokens, wl.T - start_tokens
    g = torch.Generator().manual_seed(seed)
    widx = S.random_indices(wl.B, wl.H, wl.T, wl.N, wl.W, g, pool=pool).cuda()
    ridx = S.random_indices(wl.B, wl.H, wl.T, wl.N, wl.R, g, pool=pool).cuda()
    ww = S.random_weights(wl.B, wl.H, wl.T, wl.W, g).cuda()
    rw = S.random_weights(wl.B, wl.H, wl.T, wl.R, g).cuda()
    dout = torch.randn(wl.B, wl.H, T, wl.d_v, generator=g).cuda()
    dM_end = torch.randn(wl.B, wl.H, wl.N, wl.d_v, generator=g).cuda() if end_grad else None
    mk = lambda t: sdm.Dims(wl.B, wl.H, t, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R,
                            wl.x_dtype, wl.v_dtype, decay=decay)
    st = sdm.State(mk(wl.T), inp["M0"])
    sdm.state_reset(mk(wl.T), st)
    sl = lambda x, a, b: x[:, :, a:b].contiguous()
    if T0 > 0:  # a first call leaves a non-fresh state
        sdm.forward(mk(T0), sl(inp["v"], 0, T0), sl(inp["alpha"], 0, T0), sl(inp["beta"], 0, T0),
                    sl(widx, 0, T0), sl(ww, 0, T0), sl(ridx, 0, T0), sl(rw, 0, T0), st)
    d = mk(T)
    args = [sl(x, T0, wl.T) for x in (inp["v"], inp["alpha"], inp["beta"], widx, ww, ridx, rw)]
    M_start = sdm.state_materialize(d, st)
    before = _state_bits(st)
    grads = sdm.backward(d, *args, st, dout, dM_end=dM_end)
    torch.cuda.synchronize()
    assert sdm.device_error() == 0
    after = _state_bits(st)
    assert all(torch.equal(x, y) for x, y in zip(before, after)), "state not restored"
    tol = TOL[wl.v_dtype]
    c = [x.cpu() for x in args]
    for b in range(wl.B):
        for h in range(wl.H):
            ref = orc.recur_backward(f64(c[0][b, h]), f64(c[1][b, h]), f64(c[2][b, h]),
                                     np.asarray(c[3][b, h]), f64(c[4][b, h]), np.asarray(c[5][b, h]),
                                     f64(c[6][b, h]), f64(M_start[b, h]), f64(dout[b, h]),
                                     touched=decay == "touched",
                                     dM_end=None if dM_end is None else f64(dM_end[b, h]))
            for key, gk in (("dv", "dv"), ("dalpha", "dalpha"), ("dbeta", "dbeta"),
                            ("dww", "dww"), ("drw", "drw"), ("dM0", "dM_in")):
                err = normwise_rel_err(f64(grads[gk][b, h]), ref[key])
                check_err(err, tol, f"{key} (b,h)={(b, h)}")


@pytest.mark.parametrize("decay", ["all", "touched"])
@pytest.mark.parametrize("T,pool,W,R,dv,vdt", [
    (60, 20, 4, 4, 16, "f32"),      # slots repeat across tokens, reads meet writes
    (33, 40, 8, 6, 32, "f32"),
    (80, 300, 16, 16, 128, "bf16"),
    (24, 64, 40, 24, 64, "f32"),    # eight rows per warp
    (20, 50, 6, 6, 256, "f32"),     # two float4 columns per lane
    (1, 10, 4, 4, 16, "f32"),
])
def test_backward_vs_oracle(sdm, orc, decay, T, pool, W, R, dv, vdt):
    wl = S.TINY.scaled(B=2, H=2, T=T, n_sub=20, d_v=dv, k_half=8, W=W, R=R, v_dtype=vdt,
                       alpha=("uniform", 0.6, 1.0))
    _case(sdm, orc, wl, decay, pool, seed=T * 7 + W)


@pytest.mark.parametrize("decay", ["all", "touched"])
def test_backward_from_a_non_fresh_state(sdm, orc, decay):
    """The call starts where a previous forward call left the state (stamps, Lambda, rows)."""
    wl = S.TINY.scaled(B=1, H=2, T=90, n_sub=16, d_v=16, k_half=8, W=5, R=5,
                       alpha=("uniform", 0.7, 1.0))
    _case(sdm, orc, wl, decay, pool=30, seed=5, start_tokens=50)


@pytest.mark.parametrize("decay", ["all", "touched"])
@pytest.mark.parametrize("T,pool,W,R,dv,vdt,start", [
    (40, 20, 4, 4, 16, "f32", 0),      # heavy slot reuse
    (60, 300, 16, 16, 128, "bf16", 0),
    (70, 30, 5, 5, 16, "f32", 30),     # from a non-fresh state
])
def test_backward_end_gradient(sdm, orc, decay, T, pool, W, R, dv, vdt, start):
    """A gradient for the memory after the last token (dM_end), as a sequence split into
    calls needs: every gradient against the oracle given the same dM_end."""
    wl = S.TINY.scaled(B=2, H=2, T=T, n_sub=20, d_v=dv, k_half=8, W=W, R=R, v_dtype=vdt,
                       alpha=("uniform", 0.6, 1.0))
    _case(sdm, orc, wl, decay, pool, seed=T * 3 + W + start, start_tokens=start, end_grad=True)
