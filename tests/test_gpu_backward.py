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


def _calls_setup(sdm, wl, decay, pool, seed):
    inp = {k: v.cuda() for k, v in S.generate(wl).items()}
    g = torch.Generator().manual_seed(seed)
    widx = S.random_indices(wl.B, wl.H, wl.T, wl.N, wl.W, g, pool=pool).cuda()
    ridx = S.random_indices(wl.B, wl.H, wl.T, wl.N, wl.R, g, pool=pool).cuda()
    ww = S.random_weights(wl.B, wl.H, wl.T, wl.W, g).cuda()
    rw = S.random_weights(wl.B, wl.H, wl.T, wl.R, g).cuda()
    dout = torch.randn(wl.B, wl.H, wl.T, wl.d_v, generator=g).cuda()
    mk = lambda t: sdm.Dims(wl.B, wl.H, t, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R,
                            wl.x_dtype, wl.v_dtype, decay=decay)
    seq = [inp["v"], inp["alpha"], inp["beta"], widx, ww, ridx, rw]
    return inp, seq, dout, mk


@pytest.mark.parametrize("decay", ["all", "touched"])
def test_call_log_restores_state(sdm, decay):
    """sdm_call_log_save before a call and sdm_call_log_restore after it give back the state
    the call started from, bit for bit (rows, stamps, Lambda), also when the call writes the
    same slot several times and when it starts from a non-fresh state."""
    wl = S.TINY.scaled(B=2, H=3, T=70, n_sub=12, d_v=32, k_half=6, W=6, R=5,
                       alpha=("uniform", 0.7, 1.0))
    inp, seq, _, mk = _calls_setup(sdm, wl, decay, pool=25, seed=11)
    st = sdm.State(mk(wl.T), inp["M0"])
    sdm.state_reset(mk(wl.T), st)
    sl = lambda x, a, b: x[:, :, a:b].contiguous()
    for a, b in ((0, 30), (30, 70)):
        d = mk(b - a)
        part = [sl(x, a, b) for x in seq]
        before = _state_bits(st)
        log = sdm.call_log_save(d, part[3], st)
        sdm.forward(d, *part, st)
        changed = _state_bits(st)
        assert not all(torch.equal(x, y) for x, y in zip(before, changed))
        sdm.call_log_restore(d, part[3], log, st)
        after = _state_bits(st)
        assert all(torch.equal(x, y) for x, y in zip(before, after)), "state not restored"
        sdm.forward(d, *part, st)  # then really advance to the next call
    torch.cuda.synchronize()
    assert sdm.device_error() == 0


@pytest.mark.parametrize("decay", ["all", "touched"])
@pytest.mark.parametrize("T,cuts,pool,W,R,dv,vdt", [
    (60, (25,), 20, 4, 4, 16, "f32"),          # slots shared across the two calls
    (90, (20, 55), 40, 8, 6, 32, "f32"),       # three calls
    (64, (32,), 300, 16, 16, 128, "bf16"),
])
def test_backward_across_calls(sdm, orc, decay, T, cuts, pool, W, R, dv, vdt):
    """A sequence run as several forward calls, each with its call log, differentiated call by
    call from the last: restore the call's log, sdm_backward over it from the restored state
    with the next call's dM_in as its dM_end.  Every gradient of every call, and the gradient
    of the memory at the start, against the oracle's backward over the whole sequence as one
    call; the state ends where the sequence started."""
    wl = S.TINY.scaled(B=2, H=2, T=T, n_sub=20, d_v=dv, k_half=8, W=W, R=R, v_dtype=vdt,
                       alpha=("uniform", 0.6, 1.0))
    inp, seq, dout, mk = _calls_setup(sdm, wl, decay, pool, seed=T + W)
    st = sdm.State(mk(T), inp["M0"])
    sdm.state_reset(mk(T), st)
    M_start = sdm.state_materialize(mk(T), st)
    start_bits = _state_bits(st)
    bounds = [0, *cuts, T]
    sl = lambda x, a, b: x[:, :, a:b].contiguous()
    calls = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        d = mk(b - a)
        part = [sl(x, a, b) for x in seq]
        log = sdm.call_log_save(d, part[3], st)
        sdm.forward(d, *part, st)
        calls.append((a, b, d, part, log))
    grads = [None] * len(calls)
    dM_end = None
    for c in range(len(calls) - 1, -1, -1):
        a, b, d, part, log = calls[c]
        sdm.call_log_restore(d, part[3], log, st)
        grads[c] = sdm.backward(d, *part, st, sl(dout, a, b), dM_end=dM_end)
        dM_end = grads[c]["dM_in"]
    torch.cuda.synchronize()
    assert sdm.device_error() == 0
    assert all(torch.equal(x, y) for x, y in zip(start_bits, _state_bits(st)))
    tol = TOL[vdt]
    cat = lambda key: torch.cat([g[key] for g in grads], dim=2)
    c = [x.cpu() for x in seq]
    for b in range(wl.B):
        for h in range(wl.H):
            ref = orc.recur_backward(f64(c[0][b, h]), f64(c[1][b, h]), f64(c[2][b, h]),
                                     np.asarray(c[3][b, h]), f64(c[4][b, h]), np.asarray(c[5][b, h]),
                                     f64(c[6][b, h]), f64(M_start[b, h]), f64(dout[b, h]),
                                     touched=decay == "touched")
            for key in ("dv", "dalpha", "dbeta", "dww", "drw"):
                check_err(normwise_rel_err(f64(cat(key)[b, h]), ref[key]), tol,
                          f"{key} (b,h)={(b, h)}")
            check_err(normwise_rel_err(f64(grads[0]["dM_in"][b, h]), ref["dM0"]), tol,
                      f"dM0 (b,h)={(b, h)}")
