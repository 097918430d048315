"""GPU parity: the CUDA path through the C ABI against the CPU oracle, element by element.

Inputs are the seeded synthetic workloads (sdm_synth) at sizes the oracle finishes in
seconds (several chunks and a ragged tail), plus the five workloads at full size with
sampled checks.  Tolerances: tests/parity.py.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import sdm_synth as S
from tests.parity import TOL, check_err, compare_selection, f64, normwise_rel_err, per_bh_rel_err

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


def dims_of(sdm, wl, T=None):
    return sdm.Dims(wl.B, wl.H, wl.T if T is None else T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half,
                    wl.W, wl.R, wl.x_dtype, wl.v_dtype)


def to_dev(d):
    return {k: v.cuda() for k, v in d.items()}


def oracle_select(orc, x, sk, k_half, top):
    return orc.score(f64(x), f64(sk), k_half, top, mode=oracle.MODE_PK)


def oracle_recurrence(orc, inp, widx, ww, ridx, rw, pairs, T0=0, T1=None):
    """Lazy oracle recurrence for the listed (b,h) from a fresh state; returns outs, states."""
    outs, states = [], []
    v, a, bta, M0 = inp["v"], inp["alpha"], inp["beta"], inp["M0"]
    for (b, h) in pairs:
        sl = slice(T0, T1)
        st = orc.fresh_lazy_state(f64(M0[h]))
        out = orc.recur_lazy(f64(v[b, h, sl]), f64(a[b, h, sl]), f64(bta[b, h, sl]),
                             np.asarray(widx[b, h]), f64(ww[b, h]), np.asarray(ridx[b, h]),
                             f64(rw[b, h]), st)
        outs.append(out)
        states.append(st)
    return outs, states


def check_selection(orc, x, sk, gpu_idx, gpu_w, k_half, top, n, max_near_frac=0.01):
    idx_o, sc_o, w_o = oracle_select(orc, x, sk, k_half, top)
    gi = gpu_idx.cpu().numpy()
    exact, near, bad = compare_selection(orc, f64(x), f64(sk), gi, idx_o, sc_o, n)
    assert not bad, f"selections differ beyond near ties at {bad[:5]}"
    assert near <= max(2, max_near_frac * gi[..., 0].size), (exact, near)
    same = np.all(gi == idx_o, axis=-1)
    if same.any():
        dw = np.abs(f64(gpu_w)[same] - w_o[same]).max()
        assert dw < 1e-5, dw
    return exact, near


# ------------------------------------------------------------------ scoring ---

@pytest.mark.parametrize("wl", [
    S.TINY,
    S.MID.scaled(B=1, H=2, T=333),
    S.HEADLINE.scaled(B=1, H=2, T=150),
    S.LONG.scaled(B=1, H=2, T=120),
    S.MID.scaled(B=3, H=2, T=70),   # one tensor-core tile per sequence, rows past T zero-filled
    S.MID.scaled(B=3, H=1, T=64),   # two sequences per tile, the last tile's second one absent
], ids=["tiny", "mid", "headline", "long", "mid_t70", "mid_t64_odd_b"])
def test_score_vs_oracle(sdm, orc, wl):
    inp = to_dev(S.generate(wl, with_m0=False))
    d = dims_of(sdm, wl)
    for x, sk, top in ((inp["k"], inp["skw"], wl.W), (inp["q"], inp["skr"], wl.R)):
        idx, w = sdm.score_topk(d, x, sk, top)
        torch.cuda.synchronize()
        check_selection(orc, x, sk, idx, w, wl.k_half, top, wl.n_sub)
    assert sdm.device_error() == 0


@pytest.mark.parametrize("wl", [S.MID.scaled(B=2, H=2, T=300), S.TINY.scaled(B=2, H=2, T=100),
                                S.HEADLINE.scaled(B=1, H=2, T=130)], ids=["mid", "tiny", "headline"])
def test_score_qk_matches_score_topk(sdm, wl):
    """Both roles in one call give exactly what two single-role calls give."""
    inp = to_dev(S.generate(wl, with_m0=False))
    d = dims_of(sdm, wl)
    widx, ww, ridx, rw = sdm.score_qk(d, inp["q"], inp["k"], inp["skw"], inp["skr"])
    wi2, ww2 = sdm.score_topk(d, inp["k"], inp["skw"], wl.W)
    ri2, rw2 = sdm.score_topk(d, inp["q"], inp["skr"], wl.R)
    torch.cuda.synchronize()
    assert torch.equal(widx, wi2) and torch.equal(ridx, ri2)
    assert torch.equal(ww, ww2) and torch.equal(rw, rw2)
    assert sdm.device_error() == 0


@pytest.mark.parametrize("wl", [S.MID.scaled(B=1, H=2, T=300), S.LONG.scaled(B=1, H=1, T=100)],
                         ids=["mid", "long"])
def test_score_exact_ties(sdm, orc, wl):
    """Sub-key tables whose rows come in identical pairs: every half-score has an exactly equal
    twin and pair sums tie in groups of four, so the selections' boundaries fall on exact ties
    again and again.  The oracle ranks exact ties by the lower index, as the kernel must: the
    indices are compared bit for bit (no near-tie allowance)."""
    inp = to_dev(S.generate(wl, with_m0=False))
    for key in ("skw", "skr"):
        sk = inp[key].clone()
        sk[:, :, 1::2] = sk[:, :, 0::2]
        inp[key] = sk.contiguous()
    d = dims_of(sdm, wl)
    for x, sk, top in ((inp["k"], inp["skw"], wl.W), (inp["q"], inp["skr"], wl.R)):
        idx, w = sdm.score_topk(d, x, sk, top)
        torch.cuda.synchronize()
        idx_o, _, w_o = oracle_select(orc, x, sk, wl.k_half, top)
        gi = idx.cpu().numpy()
        same = np.all(gi == idx_o, axis=-1)
        assert same.all(), f"{(~same).sum()} rows differ, first at {np.argwhere(~same)[:3].tolist()}"
        check_err(float(np.abs(f64(w) - w_o).max()), 1e-5, "weights")
    assert sdm.device_error() == 0


def test_score_brute_force_equivalence(sdm, orc):
    """k_half == top: GPU product-key selection equals the oracle's brute-force ranking."""
    wl = S.MID.scaled(B=1, H=1, T=64, n_sub=64, k_half=16, W=16, R=16)
    inp = to_dev(S.generate(wl, with_m0=False))
    d = dims_of(sdm, wl)
    idx, w = sdm.score_topk(d, inp["k"], inp["skw"], wl.W)
    idx_b, sc_b, w_b = orc.score(f64(inp["k"]), f64(inp["skw"]), wl.k_half, wl.W,
                                 mode=oracle.MODE_BRUTE)
    exact, near, bad = compare_selection(orc, f64(inp["k"]), f64(inp["skw"]), idx.cpu().numpy(),
                                         idx_b, sc_b, wl.n_sub)
    assert not bad and near <= 2


# --------------------------------------------------------------- recurrence ---

def _forward_case(sdm, orc, wl, inp, widx, ww, ridx, rw, tol):
    d = dims_of(sdm, wl)
    st = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st)
    out = sdm.forward(d, inp["v"], inp["alpha"], inp["beta"], widx, ww, ridx, rw, st)
    M = sdm.state_materialize(d, st)
    torch.cuda.synchronize()
    assert sdm.device_error() == 0
    pairs = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    outs, states = oracle_recurrence(orc, inp, widx.cpu(), ww.cpu(), ridx.cpu(), rw.cpu(), pairs)
    for (b, h), o_ref, st_ref in zip(pairs, outs, states):
        e_out = normwise_rel_err(f64(out[b, h]), o_ref)
        e_mem = normwise_rel_err(f64(M[b, h]), orc.materialize(st_ref))
        check_err(e_out, tol, f"out (b,h)={(b, h)}")
        check_err(e_mem, tol, f"memory (b,h)={(b, h)}")
    lam_ref = np.array([s["Lambda"] for s in states])
    np.testing.assert_allclose(f64(st.Lambda).reshape(-1), lam_ref, rtol=1e-12, atol=1e-12)
    return out, st


@pytest.mark.parametrize("wl", [
    S.TINY,
    S.MID.scaled(B=1, H=2, T=333),
    S.HEADLINE.scaled(B=2, H=1, T=257, n_sub=128),
    S.LONG.scaled(B=1, H=1, T=100, n_sub=128),
], ids=["tiny", "mid", "headline", "long"])
def test_forward_oracle_selection(sdm, orc, wl):
    """Recurrence parity with the oracle's own slot selections fed to both sides."""
    inp = to_dev(S.generate(wl))
    ro, _, rwo = oracle_select(orc, inp["q"], inp["skr"], wl.k_half, wl.R)
    wo, _, wwo = oracle_select(orc, inp["k"], inp["skw"], wl.k_half, wl.W)
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()
    _forward_case(sdm, orc, wl, inp, t(wo, torch.int32), t(wwo, torch.float32),
                  t(ro, torch.int32), t(rwo, torch.float32), TOL[wl.v_dtype])


@pytest.mark.parametrize("T,pool,W,R", [(300, 40, 8, 8), (97, 12, 4, 6), (64, 64, 16, 16),
                                        (1, 20, 4, 4), (33, 9, 9, 3)])
def test_forward_shared_slots(sdm, orc, T, pool, W, R):
    """Heavy slot sharing inside chunks (small pool): exercises every in-chunk link path."""
    wl = S.TINY.scaled(B=2, H=2, T=T, n_sub=16, d_v=16, k_half=8, W=W, R=R,
                       alpha=("uniform", 0.5, 1.0))
    inp = to_dev(S.generate(wl))
    g = torch.Generator().manual_seed(T * 31 + pool)
    widx = S.random_indices(2, 2, T, wl.N, W, g, pool=pool).cuda()
    ridx = S.random_indices(2, 2, T, wl.N, R, g, pool=pool).cuda()
    ww = S.random_weights(2, 2, T, W, g).cuda()
    rw = S.random_weights(2, 2, T, R, g).cuda()
    _forward_case(sdm, orc, wl, inp, widx, ww, ridx, rw, TOL["f32"])


@pytest.mark.parametrize("vdt,dv", [("f32", 32), ("bf16", 64)])
def test_forward_sixteen_column_slices(sdm, orc, vdt, dv):
    """Enough sequences that the row pass takes 16-column slices (B*H*d_v/16 CTAs fill the
    SMs: 320 and 640 here), ragged last chunk, slots shared within and across chunks."""
    B, H, T, W, R = 4, 40, 70, 6, 5
    wl = S.TINY.scaled(B=B, H=H, T=T, n_sub=16, d_v=dv, k_half=8, W=W, R=R, v_dtype=vdt,
                       alpha=("uniform", 0.6, 1.0))
    inp = to_dev(S.generate(wl))
    g = torch.Generator().manual_seed(dv)
    widx = S.random_indices(B, H, T, wl.N, W, g, pool=60).cuda()
    ridx = S.random_indices(B, H, T, wl.N, R, g, pool=60).cuda()
    ww = S.random_weights(B, H, T, W, g).cuda()
    rw = S.random_weights(B, H, T, R, g).cuda()
    _forward_case(sdm, orc, wl, inp, widx, ww, ridx, rw, TOL[vdt])


def test_forward_long_call_walk_path(sdm, orc):
    """More than 512 chunks in one call: the plan takes its sequential walk instead of the
    per-slot chunk masks; results must not depend on which is used."""
    wl = S.TINY.scaled(B=1, H=1, T=17000, n_sub=16, d_v=16, k_half=4, W=4, R=4,
                       alpha=("uniform", 0.97, 1.0))
    inp = to_dev(S.generate(wl))
    g = torch.Generator().manual_seed(17)
    widx = S.random_indices(1, 1, wl.T, wl.N, 4, g, pool=64).cuda()
    ridx = S.random_indices(1, 1, wl.T, wl.N, 4, g, pool=64).cuda()
    ww = S.random_weights(1, 1, wl.T, 4, g).cuda()
    rw = S.random_weights(1, 1, wl.T, 4, g).cuda()
    _forward_case(sdm, orc, wl, inp, widx, ww, ridx, rw, TOL["f32"])


def test_prefill_end_to_end(sdm, orc):
    """Scoring + recurrence: selections against the oracle, outputs against the oracle's
    recurrence run on the GPU's selections (so a near tie cannot fail the output check)."""
    for wl in (S.TINY, S.MID.scaled(B=2, H=2, T=200)):
        inp = to_dev(S.generate(wl))
        d = dims_of(sdm, wl)
        st = sdm.State(d, inp["M0"])
        sdm.state_reset(d, st)
        out, (widx, ww, ridx, rw) = sdm.prefill(d, inp["q"], inp["k"], inp["v"], inp["alpha"],
                                                inp["beta"], inp["skw"], inp["skr"], st)
        torch.cuda.synchronize()
        check_selection(orc, inp["k"], inp["skw"], widx, ww, wl.k_half, wl.W, wl.n_sub)
        check_selection(orc, inp["q"], inp["skr"], ridx, rw, wl.k_half, wl.R, wl.n_sub)
        pairs = [(b, h) for b in range(wl.B) for h in range(wl.H)]
        outs, _ = oracle_recurrence(orc, inp, widx.cpu(), ww.cpu(), ridx.cpu(), rw.cpu(), pairs)
        ref = np.stack(outs).reshape(wl.B, wl.H, wl.T, wl.d_v)
        check_err(per_bh_rel_err(f64(out), ref), TOL[wl.v_dtype])


def test_shared_subkey_tables(sdm, orc):
    """One sub-key table for both roles (the same array passed as skw and skr): reads and
    writes then address the same slots for q = k, and everything still matches the oracle."""
    wl = S.MID.scaled(B=1, H=2, T=160)
    inp = to_dev(S.generate(wl))
    inp["q"] = inp["k"].clone()  # same key for reading and writing: same slots
    d = dims_of(sdm, wl)
    st = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st)
    out, (widx, ww, ridx, rw) = sdm.prefill(d, inp["q"], inp["k"], inp["v"], inp["alpha"],
                                            inp["beta"], inp["skw"], inp["skw"], st)
    torch.cuda.synchronize()
    check_selection(orc, inp["k"], inp["skw"], widx, ww, wl.k_half, wl.W, wl.n_sub)
    check_selection(orc, inp["q"], inp["skw"], ridx, rw, wl.k_half, wl.R, wl.n_sub)
    assert torch.equal(widx, ridx) and torch.equal(ww, rw)
    pairs = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    outs, _ = oracle_recurrence(orc, inp, widx.cpu(), ww.cpu(), ridx.cpu(), rw.cpu(), pairs)
    ref = np.stack(outs).reshape(wl.B, wl.H, wl.T, wl.d_v)
    check_err(per_bh_rel_err(f64(out), ref), TOL[wl.v_dtype])


def test_split_invariance(sdm, orc):
    """prefill(T) == prefill(T1) + prefill(T-T1) == prefill(T1) + (T-T1) decode steps."""
    wl = S.MID.scaled(B=2, H=2, T=90, n_sub=32, k_half=8, W=8, R=8, d_v=32)
    inp = to_dev(S.generate(wl))
    d = dims_of(sdm, wl)
    tol = TOL[wl.v_dtype]

    def sl(x, a, b):
        return x[:, :, a:b].contiguous()

    st = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st)
    full, _ = sdm.prefill(d, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["skw"],
                          inp["skr"], st)
    M_full = sdm.state_materialize(d, st)
    for T1 in (1, 37, 64):
        st2 = sdm.State(d, inp["M0"])
        sdm.state_reset(d, st2)
        outs = []
        for a, b in ((0, T1), (T1, wl.T)):
            dd = dims_of(sdm, wl, T=b - a)
            o, _ = sdm.prefill(dd, sl(inp["q"], a, b), sl(inp["k"], a, b), sl(inp["v"], a, b),
                               sl(inp["alpha"], a, b), sl(inp["beta"], a, b), inp["skw"],
                               inp["skr"], st2)
            outs.append(o)
        check_err(per_bh_rel_err(f64(torch.cat(outs, 2)), f64(full)), tol)
        check_err(per_bh_rel_err(f64(sdm.state_materialize(d, st2)), f64(M_full)), tol)
        st3 = sdm.State(d, inp["M0"])
        sdm.state_reset(d, st3)
        d1 = dims_of(sdm, wl, T=T1)
        o1, _ = sdm.prefill(d1, sl(inp["q"], 0, T1), sl(inp["k"], 0, T1), sl(inp["v"], 0, T1),
                            sl(inp["alpha"], 0, T1), sl(inp["beta"], 0, T1), inp["skw"],
                            inp["skr"], st3)
        outs = [o1]
        dd = dims_of(sdm, wl, T=1)
        for t in range(T1, wl.T):
            o, _ = sdm.decode_step(dd, inp["q"][:, :, t].contiguous(), inp["k"][:, :, t].contiguous(),
                                   inp["v"][:, :, t].contiguous(), inp["alpha"][:, :, t].contiguous(),
                                   inp["beta"][:, :, t].contiguous(), inp["skw"], inp["skr"], st3)
            outs.append(o.unsqueeze(2))
        check_err(per_bh_rel_err(f64(torch.cat(outs, 2)), f64(full)), tol)
        check_err(per_bh_rel_err(f64(sdm.state_materialize(d, st3)), f64(M_full)), tol)
    assert sdm.device_error() == 0


def test_decode_vs_oracle(sdm, orc):
    wl = S.DECODE.scaled(B=3, H=2, T=40, decode_steps=12, n_sub=64, k_half=16, W=16, R=16)
    inp = to_dev(S.generate(wl))
    d = dims_of(sdm, wl)
    st = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st)
    T0 = wl.T
    sl = lambda x: x[:, :, :T0].contiguous()
    out0, (w0, ww0, r0, rw0) = sdm.prefill(d, sl(inp["q"]), sl(inp["k"]), sl(inp["v"]),
                                           sl(inp["alpha"]), sl(inp["beta"]), inp["skw"],
                                           inp["skr"], st)
    dd = dims_of(sdm, wl, T=1)
    outs, sels = [], []
    for s in range(wl.decode_steps):
        t = T0 + s
        o, sel = sdm.decode_step(dd, inp["q"][:, :, t].contiguous(), inp["k"][:, :, t].contiguous(),
                                 inp["v"][:, :, t].contiguous(), inp["alpha"][:, :, t].contiguous(),
                                 inp["beta"][:, :, t].contiguous(), inp["skw"], inp["skr"], st)
        outs.append(o.clone())
        sels.append([x.clone() for x in sel])
    torch.cuda.synchronize()
    # selections of each step against the oracle
    for s, (wi, wv, ri, rv) in enumerate(sels):
        t = T0 + s
        check_selection(orc, inp["k"][:, :, t:t + 1], inp["skw"], wi, wv, wl.k_half, wl.W, wl.n_sub)
        check_selection(orc, inp["q"][:, :, t:t + 1], inp["skr"], ri, rv, wl.k_half, wl.R, wl.n_sub)
    for b in range(wl.B):
        for h in range(wl.H):
            widx = np.concatenate([w0[b, h].cpu().numpy()] + [x[0][b, h].cpu().numpy() for x in sels])
            ww = np.concatenate([f64(ww0[b, h])] + [f64(x[1][b, h]) for x in sels])
            ridx = np.concatenate([r0[b, h].cpu().numpy()] + [x[2][b, h].cpu().numpy() for x in sels])
            rw = np.concatenate([f64(rw0[b, h])] + [f64(x[3][b, h]) for x in sels])
            stt = orc.fresh_lazy_state(f64(inp["M0"][h]))
            ref = orc.recur_lazy(f64(inp["v"][b, h]), f64(inp["alpha"][b, h]), f64(inp["beta"][b, h]),
                                 widx, ww, ridx, rw, stt)
            got = np.concatenate([f64(out0[b, h])] + [f64(o[b, h])[None] for o in outs])
            check_err(normwise_rel_err(got, ref), TOL[wl.v_dtype])
            check_err(normwise_rel_err(f64(sdm.state_materialize(d, st)[b, h]),
                                       orc.materialize(stt)), TOL[wl.v_dtype], "memory")
    assert sdm.device_error() == 0


def test_empty_and_single_token(sdm, orc):
    wl = S.TINY.scaled(B=2, H=3, T=1)
    inp = to_dev(S.generate(wl))
    d0 = dims_of(sdm, wl, T=0)
    st = sdm.State(d0, inp["M0"])
    sdm.state_reset(d0, st)
    e = torch.empty((2, 3, 0, wl.d_k), device="cuda")
    out, _ = sdm.prefill(d0, e, e, torch.empty((2, 3, 0, wl.d_v), device="cuda"),
                         torch.empty((2, 3, 0), device="cuda"), torch.empty((2, 3, 0), device="cuda"),
                         inp["skw"], inp["skr"], st)
    assert out.numel() == 0 and torch.all(st.Lambda == 0)
    assert torch.equal(sdm.state_materialize(d0, st), inp["M0"].unsqueeze(0).expand(2, 3, -1, -1))
    test_forward_oracle_selection(sdm, orc, wl)


def test_device_error_bits(sdm):
    wl = S.TINY.scaled(B=1, H=1, T=40)
    inp = to_dev(S.generate(wl))
    d = dims_of(sdm, wl)
    g = torch.Generator().manual_seed(5)
    widx = S.random_indices(1, 1, 40, wl.N, wl.W, g).cuda()
    ridx = S.random_indices(1, 1, 40, wl.N, wl.R, g).cuda()
    ww = S.random_weights(1, 1, 40, wl.W, g).cuda()
    rw = S.random_weights(1, 1, 40, wl.R, g).cuda()
    st = sdm.State(d, inp["M0"])
    for what, bit in (("range", sdm.DEVERR_SLOT_RANGE), ("dup", sdm.DEVERR_DUP_WRITE),
                      ("alpha", sdm.DEVERR_ALPHA)):
        w2, r2, a2 = widx.clone(), ridx.clone(), inp["alpha"].clone()
        if what == "range":
            w2[0, 0, 7, 1] = wl.N + 5
            r2[0, 0, 3, 0] = -2
        elif what == "dup":
            w2[0, 0, 9, 2] = w2[0, 0, 9, 0]
        else:
            a2[0, 0, 11] = 0.0
        sdm.state_reset(d, st)
        out = sdm.forward(d, inp["v"], a2, inp["beta"], w2, ww, r2, rw, st)
        bits = sdm.device_error(clear=True)
        assert bits & bit, (what, bits)
        assert torch.isfinite(out).all()
    assert sdm.device_error() == 0


def test_host_validation_errors(sdm):
    wl = S.TINY
    inp = to_dev(S.generate(wl))
    bad = sdm.Dims(1, 1, 4, 30, 16, 16, 4, 4, 4)  # d_k/2 = 15 is not a multiple of 8
    with pytest.raises(sdm.SdmError):
        sdm.score_topk(bad, inp["k"], inp["skw"], 4)
    d = dims_of(sdm, wl)
    with pytest.raises(sdm.SdmError):
        sdm.score_topk(d, inp["k"], inp["skw"], 65)
    st = sdm.State(d, inp["M0"])
    tiny_ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    sel = sdm.selection_buffers(d)
    with pytest.raises(sdm.SdmError):
        sdm.forward(d, inp["v"], inp["alpha"], inp["beta"], *sel, st, ws=tiny_ws)


# ---------------------------------------------------------- full-size cases ---

def _full_case(sdm, orc, wl, n_rows=192, n_pairs=2, seed=0):
    """The workload at full size, in the launch configuration the bench times; checks
    sampled score rows against the oracle and whole (b,h) recurrences on the GPU's
    selections."""
    inp = S.generate(wl, device="cuda")
    d = dims_of(sdm, wl)
    T0 = wl.T
    cut = (lambda x: x[:, :, :T0].contiguous()) if wl.decode_steps else (lambda x: x)
    st = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st)
    out, (widx, ww, ridx, rw) = sdm.prefill(d, cut(inp["q"]), cut(inp["k"]), cut(inp["v"]),
                                            cut(inp["alpha"]), cut(inp["beta"]), inp["skw"],
                                            inp["skr"], st)
    torch.cuda.synchronize()
    assert sdm.device_error() == 0
    rng = np.random.default_rng(seed)
    rows = [(int(rng.integers(wl.B)), int(rng.integers(wl.H)), int(rng.integers(T0)))
            for _ in range(n_rows)]
    for x, sk, gi, gw, top in ((inp["k"], inp["skw"], widx, ww, wl.W),
                               (inp["q"], inp["skr"], ridx, rw, wl.R)):
        xs = torch.stack([x[b, h, t] for b, h, t in rows])[None, None]  # [1,1,n,d_k]
        hs = sorted({h for _, h, _ in rows})
        # score each sampled row against its own head's table
        for hh in hs:
            sel = [i for i, r in enumerate(rows) if r[1] == hh]
            gsel = torch.stack([gi[rows[i][0], hh, rows[i][2]] for i in sel])[None, None]
            wsel = torch.stack([gw[rows[i][0], hh, rows[i][2]] for i in sel])[None, None]
            check_selection(orc, xs[:, :, sel], sk[hh:hh + 1], gsel, wsel, wl.k_half, top,
                            wl.n_sub, max_near_frac=0.02)
    pairs = [(int(rng.integers(wl.B)), int(rng.integers(wl.H))) for _ in range(n_pairs)]
    Mfull = None
    for (b, h) in pairs:
        stt = orc.fresh_lazy_state(f64(inp["M0"][h]))
        ref = orc.recur_lazy(f64(inp["v"][b, h, :T0]), f64(inp["alpha"][b, h, :T0]),
                             f64(inp["beta"][b, h, :T0]), widx[b, h].cpu().numpy(), f64(ww[b, h]),
                             ridx[b, h].cpu().numpy(), f64(rw[b, h]), stt)
        check_err(normwise_rel_err(f64(out[b, h]), ref), TOL[wl.v_dtype])
        d1 = sdm.Dims(1, 1, T0, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R, wl.x_dtype,
                      wl.v_dtype)
        # materialise just this sequence through a one-sequence view of the state
        one = sdm.State.__new__(sdm.State)
        one.M = st.M[b, h:h + 1].unsqueeze(0).contiguous()
        one.stamp = st.stamp[b, h:h + 1].unsqueeze(0).contiguous()
        one.Lambda = st.Lambda[b, h:h + 1].unsqueeze(0).contiguous()
        one.M0 = inp["M0"][h:h + 1].contiguous()
        one._c = sdm._CState(one.M.data_ptr(), one.stamp.data_ptr(), one.Lambda.data_ptr(),
                             one.M0.data_ptr())
        Mone = sdm.state_materialize(d1, one)
        check_err(normwise_rel_err(f64(Mone[0, 0]), orc.materialize(stt)), TOL[wl.v_dtype])
        del one, Mone
    return inp, st, (widx, ww, ridx, rw)


@pytest.mark.slow
def test_full_mid_prefill(sdm, orc):
    _full_case(sdm, orc, S.MID)
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_full_headline_prefill(sdm, orc):
    _full_case(sdm, orc, S.HEADLINE, n_pairs=1)
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_full_decode(sdm, orc):
    wl = S.DECODE
    inp, st, sel0 = _full_case(sdm, orc, wl, n_rows=64, n_pairs=1)
    d = dims_of(sdm, wl, T=1)
    qd, kd, vd = (S.decode_layout(inp[k], wl.T) for k in ("q", "k", "v"))
    ad, bd = (S.decode_layout(inp[k], wl.T) for k in ("alpha", "beta"))
    sel = sdm.selection_buffers(d)
    steps = wl.decode_steps
    outs = torch.empty((steps, wl.B, wl.H, wl.d_v), device="cuda")
    wsel = torch.empty((steps, wl.B, wl.H, wl.W), dtype=torch.int32, device="cuda")
    rsel = torch.empty((steps, wl.B, wl.H, wl.R), dtype=torch.int32, device="cuda")
    wws = torch.empty((steps, wl.B, wl.H, wl.W), device="cuda")
    rws = torch.empty((steps, wl.B, wl.H, wl.R), device="cuda")
    for s in range(steps):
        sdm.decode_step(d, qd[s], kd[s], vd[s], ad[s], bd[s], inp["skw"], inp["skr"], st, sel=sel,
                        out=outs[s])
        wsel[s].copy_(sel[0].view(wl.B, wl.H, wl.W))
        wws[s].copy_(sel[1].view(wl.B, wl.H, wl.W))
        rsel[s].copy_(sel[2].view(wl.B, wl.H, wl.R))
        rws[s].copy_(sel[3].view(wl.B, wl.H, wl.R))
    torch.cuda.synchronize()
    assert sdm.device_error() == 0
    # every row's selection of both roles at the first and the last step
    for s in (0, steps - 1):
        for x, sk, top, gi, gw in ((kd[s], inp["skw"], wl.W, wsel[s], wws[s]),
                                   (qd[s], inp["skr"], wl.R, rsel[s], rws[s])):
            check_selection(orc, x.unsqueeze(2), sk, gi.unsqueeze(2), gw.unsqueeze(2), wl.k_half,
                            top, wl.n_sub)
    b, h = 5, 7
    widx = np.concatenate([sel0[0][b, h].cpu().numpy(), wsel[:, b, h].cpu().numpy()])
    ww = np.concatenate([f64(sel0[1][b, h]), f64(wws[:, b, h])])
    ridx = np.concatenate([sel0[2][b, h].cpu().numpy(), rsel[:, b, h].cpu().numpy()])
    rw = np.concatenate([f64(sel0[3][b, h]), f64(rws[:, b, h])])
    stt = orc.fresh_lazy_state(f64(inp["M0"][h]))
    ref = orc.recur_lazy(f64(inp["v"][b, h]), f64(inp["alpha"][b, h]), f64(inp["beta"][b, h]), widx,
                         ww, ridx, rw, stt)
    check_err(normwise_rel_err(f64(outs[:, b, h]), ref[wl.T:]), TOL[wl.v_dtype])
    del inp, st
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_full_long_context(sdm, orc):
    _full_case(sdm, orc, S.LONG, n_rows=96, n_pairs=1)
    torch.cuda.empty_cache()
