"""GPU parity of the touched-slots decay variant (sdm_dims.decay = "touched": alpha scales
only each token's write slots) against the oracle's plain definition (recur_touched).

Cases: heavy slot sharing inside chunks (every in-chunk link and chain product), a call of
more than 512 chunks (the plan's walk instead of the per-slot masks), scoring + recurrence
through sdm_prefill, decode steps continuing a prefill, and the two decay readings
agreeing at alpha = 1 and differing below it.
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


def _dims(sdm, wl, T=None, decay="touched"):
    return sdm.Dims(wl.B, wl.H, wl.T if T is None else T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half,
                    wl.W, wl.R, wl.x_dtype, wl.v_dtype, decay=decay)


def _oracle_bh(orc, inp, b, h, widx, ww, ridx, rw, T0=0, T1=None):
    sl = slice(T0, T1)
    return orc.recur_touched(f64(inp["v"][b, h, sl]), f64(inp["alpha"][b, h, sl]),
                             f64(inp["beta"][b, h, sl]), np.asarray(widx[b, h]), f64(ww[b, h]),
                             np.asarray(ridx[b, h]), f64(rw[b, h]), f64(inp["M0"][h]))


def _forward_touched(sdm, orc, wl, inp, widx, ww, ridx, rw, tol):
    d = _dims(sdm, wl)
    st = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st)
    out = sdm.forward(d, inp["v"], inp["alpha"], inp["beta"], widx, ww, ridx, rw, st)
    M = sdm.state_materialize(d, st)
    torch.cuda.synchronize()
    assert sdm.device_error() == 0
    wc, wwc, rc, rwc = widx.cpu(), ww.cpu(), ridx.cpu(), rw.cpu()
    for b in range(wl.B):
        for h in range(wl.H):
            o_ref, M_ref = _oracle_bh(orc, inp, b, h, wc, wwc, rc, rwc)
            e_out = normwise_rel_err(f64(out[b, h]), o_ref)
            e_mem = normwise_rel_err(f64(M[b, h]), M_ref)
            check_err(e_out, tol, f"out (b,h)={(b, h)}")
            check_err(e_mem, tol, f"memory (b,h)={(b, h)}")
    return out, M


@pytest.mark.parametrize("T,pool,W,R", [(300, 40, 8, 8), (97, 12, 4, 6), (64, 64, 16, 16),
                                        (1, 20, 4, 4), (33, 9, 9, 3)])
def test_touched_shared_slots(sdm, orc, T, pool, W, R):
    """Heavy slot sharing inside chunks (small pool): every chain product of the plan."""
    wl = S.TINY.scaled(B=2, H=2, T=T, n_sub=16, d_v=16, k_half=8, W=W, R=R,
                       alpha=("uniform", 0.5, 1.0))
    inp = {k: v.cuda() for k, v in S.generate(wl).items()}
    g = torch.Generator().manual_seed(T * 37 + pool)
    widx = S.random_indices(2, 2, T, wl.N, W, g, pool=pool).cuda()
    ridx = S.random_indices(2, 2, T, wl.N, R, g, pool=pool).cuda()
    ww = S.random_weights(2, 2, T, W, g).cuda()
    rw = S.random_weights(2, 2, T, R, g).cuda()
    _forward_touched(sdm, orc, wl, inp, widx, ww, ridx, rw, TOL["f32"])


def test_touched_walk_path(sdm, orc):
    """More than 512 chunks in one call: the plan's walk supplies the pristine signs."""
    wl = S.TINY.scaled(B=1, H=1, T=17000, n_sub=16, d_v=16, k_half=4, W=4, R=4,
                       alpha=("uniform", 0.97, 1.0))
    inp = {k: v.cuda() for k, v in S.generate(wl).items()}
    g = torch.Generator().manual_seed(19)
    widx = S.random_indices(1, 1, wl.T, wl.N, 4, g, pool=64).cuda()
    ridx = S.random_indices(1, 1, wl.T, wl.N, 4, g, pool=64).cuda()
    ww = S.random_weights(1, 1, wl.T, 4, g).cuda()
    rw = S.random_weights(1, 1, wl.T, 4, g).cuda()
    _forward_touched(sdm, orc, wl, inp, widx, ww, ridx, rw, TOL["f32"])


def test_touched_prefill_and_decode(sdm, orc):
    """Scoring + recurrence (sdm_prefill), then single-token steps, against the oracle run
    over all tokens on the GPU's selections; and the prefill split in two calls."""
    wl = S.MID.scaled(B=2, H=2, T=150, decode_steps=6, n_sub=64, k_half=16, W=16, R=16)
    inp = {k: v.cuda() for k, v in S.generate(wl).items()}
    T0, steps = wl.T, wl.decode_steps
    d = _dims(sdm, wl)
    st = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st)
    sl = lambda x, a, b: x[:, :, a:b].contiguous()
    out0, sel0 = sdm.prefill(d, sl(inp["q"], 0, T0), sl(inp["k"], 0, T0), sl(inp["v"], 0, T0),
                             sl(inp["alpha"], 0, T0), sl(inp["beta"], 0, T0), inp["skw"],
                             inp["skr"], st)
    dd = _dims(sdm, wl, T=1)
    outs, sels = [], []
    for s in range(steps):
        t = T0 + s
        o, sel = sdm.decode_step(dd, inp["q"][:, :, t].contiguous(), inp["k"][:, :, t].contiguous(),
                                 inp["v"][:, :, t].contiguous(), inp["alpha"][:, :, t].contiguous(),
                                 inp["beta"][:, :, t].contiguous(), inp["skw"], inp["skr"], st)
        outs.append(o.clone())
        sels.append([x.clone().view(wl.B, wl.H, 1, -1) for x in sel])
    M = sdm.state_materialize(d, st)
    torch.cuda.synchronize()
    assert sdm.device_error() == 0
    cat = lambda i: torch.cat([sel0[i]] + [x[i] for x in sels], dim=2).cpu()
    widx, ww, ridx, rw = cat(0), cat(1), cat(2), cat(3)
    got = torch.cat([out0] + [o[:, :, None] for o in outs], dim=2)
    for b in range(wl.B):
        for h in range(wl.H):
            o_ref, M_ref = _oracle_bh(orc, inp, b, h, widx, ww, ridx, rw)
            check_err(normwise_rel_err(f64(got[b, h]), o_ref), TOL[wl.v_dtype], "out")
            check_err(normwise_rel_err(f64(M[b, h]), M_ref), TOL[wl.v_dtype], "memory")
    # the same tokens as two prefill calls from a fresh state
    st2 = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st2)
    T1 = 70
    d1, d2 = _dims(sdm, wl, T=T1), _dims(sdm, wl, T=T0 - T1)
    o1, _ = sdm.prefill(d1, sl(inp["q"], 0, T1), sl(inp["k"], 0, T1), sl(inp["v"], 0, T1),
                        sl(inp["alpha"], 0, T1), sl(inp["beta"], 0, T1), inp["skw"], inp["skr"], st2)
    o2, _ = sdm.prefill(d2, sl(inp["q"], T1, T0), sl(inp["k"], T1, T0), sl(inp["v"], T1, T0),
                        sl(inp["alpha"], T1, T0), sl(inp["beta"], T1, T0), inp["skw"], inp["skr"],
                        st2)
    torch.cuda.synchronize()
    two = torch.cat([o1, o2], dim=2)
    assert normwise_rel_err(f64(two), f64(out0)) <= 1e-5


def test_touched_against_every_slot_decay(sdm, orc):
    """alpha = 1: the two readings give the same result; alpha < 1: they differ."""
    wl = S.TINY.scaled(B=2, H=2, T=120, n_sub=16, d_v=16, k_half=8, W=6, R=6,
                       alpha=("uniform", 0.6, 0.9))
    inp = {k: v.cuda() for k, v in S.generate(wl).items()}
    g = torch.Generator().manual_seed(23)
    widx = S.random_indices(2, 2, wl.T, wl.N, 6, g, pool=30).cuda()
    ridx = S.random_indices(2, 2, wl.T, wl.N, 6, g, pool=30).cuda()
    ww = S.random_weights(2, 2, wl.T, 6, g).cuda()
    rw = S.random_weights(2, 2, wl.T, 6, g).cuda()

    def run(decay, alpha):
        d = _dims(sdm, wl, decay=decay)
        st = sdm.State(d, inp["M0"])
        sdm.state_reset(d, st)
        out = sdm.forward(d, inp["v"], alpha, inp["beta"], widx, ww, ridx, rw, st)
        return f64(out), f64(sdm.state_materialize(d, st))

    ones = torch.ones_like(inp["alpha"])
    (oa, Ma), (ot, Mt) = run("all", ones), run("touched", ones)
    assert normwise_rel_err(ot, oa) <= 1e-6 and normwise_rel_err(Mt, Ma) <= 1e-6
    (oa, Ma), (ot, Mt) = run("all", inp["alpha"]), run("touched", inp["alpha"])
    assert normwise_rel_err(ot, oa) > 1e-2
    assert sdm.device_error() == 0
