"""Checks that pin the CPU oracle to facts that do not come from the oracle itself.

Each function takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with what the definition or the mathematics fixes.  They are
run against the real oracle (tests/test_oracle_pins.py) and against planted
mutants of its C source (tests/test_oracle_mutants.py), where at least one of
them must fail for every mutant.

Sources: "Sparse Delta Memory: Scaling the State of Linear RNNs through
Sparsity" summary pages — §2 Background (Gated DeltaNet; Product Key Memory),
§3 Method (sparse updates, sparse addressing, sparse retrieval, connection to
GDN, learned initial state), §4 SDM Configuration (softmax-normalised
activations).
"""
from __future__ import annotations

import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _random_case(rng, T, N, dv, W, R, a_lo=0.8, a_hi=1.0):
    v = rng.standard_normal((T, dv))
    alpha = rng.uniform(a_lo, a_hi, T)
    beta = rng.uniform(0.0, 1.0, T)
    widx = np.stack([rng.choice(N, W, replace=False) for _ in range(T)]).astype(np.int32)
    ridx = np.stack([rng.choice(N, R, replace=False) for _ in range(T)]).astype(np.int32)
    ww = rng.uniform(0.05, 1.0, (T, W))
    ww /= ww.sum(1, keepdims=True)
    rw = rng.uniform(0.05, 1.0, (T, R))
    rw /= rw.sum(1, keepdims=True)
    M0 = rng.standard_normal((N, dv)) * 0.5
    return v, alpha, beta, widx, ww, ridx, rw, M0


# ---------------------------------------------------------------- scoring ---

def pin_pk_equals_brute(o):
    """Product-key top-W equals brute-force top-W over all N slots when k >= W
    (a pair with per-half ranks (a, b) is beaten by at least (a+1)(b+1)-1 pairs)."""
    rng = _rng(1)
    for (n, hd, k, top) in [(8, 4, 4, 4), (16, 8, 6, 5), (16, 16, 16, 16), (32, 8, 8, 8)]:
        sk = rng.standard_normal((2, n, hd))
        for _ in range(20):
            x = rng.standard_normal(2 * hd)
            ib, sb, wb = o.topk(x, sk, k, top, mode=0)
            ip, sp, wp = o.topk(x, sk, k, top, mode=1)
            assert np.array_equal(ib, ip), (n, hd, k, top, ib, ip)
            assert np.array_equal(sb, sp)


def pin_brute_matches_numpy(o):
    """Brute-force ranking equals a numpy matmul + lexsort of all N = n^2 slot scores."""
    rng = _rng(2)
    n, hd, top = 12, 6, 7
    sk = rng.standard_normal((2, n, hd))
    for _ in range(30):
        x = rng.standard_normal(2 * hd)
        s1 = sk[0] @ x[:hd]
        s2 = sk[1] @ x[hd:]
        full = (s1[:, None] + s2[None, :]).reshape(-1)  # slot s = i*n + j
        order = np.lexsort((np.arange(n * n), -full))[:top]
        idx, sc, w = o.topk(x, sk, n, top, mode=0)
        assert np.array_equal(idx, order), (idx, order)
        np.testing.assert_allclose(sc, full[order], rtol=0, atol=1e-12)
        e = np.exp(full[order] - full[order].max())
        np.testing.assert_allclose(w, e / e.sum(), rtol=1e-13, atol=0)


def pin_pk_depends_on_k(o):
    """With k < W the product-key shortlist must miss some brute-force winners."""
    rng = _rng(3)
    n, hd, k, top = 16, 4, 2, 4
    sk = rng.standard_normal((2, n, hd))
    differs = 0
    for _ in range(50):
        x = rng.standard_normal(2 * hd)
        ib, _, _ = o.topk(x, sk, k, top, mode=0)
        ip, _, _ = o.topk(x, sk, k, top, mode=1)
        differs += int(not np.array_equal(ib, ip))
        # every product-key pick lies in the k x k shortlist
        s1, s2 = o.half_scores(x, sk)
        top1 = set(np.lexsort((np.arange(n), -s1))[:k].tolist())
        top2 = set(np.lexsort((np.arange(n), -s2))[:k].tolist())
        for s in ip.tolist():
            assert s // n in top1 and s % n in top2
    assert differs > 0


def pin_tie_order(o):
    """Equal scores rank the lower slot first (reading: the pages fix no tie rule)."""
    hd, n = 2, 4
    sk = np.zeros((2, n, hd))
    sk[0] = [[1, 0], [2, 0], [1, 0], [0, 0]]   # s1 = [1, 2, 1, 0] for x[:2] = [1, 0]
    sk[1] = [[0, 1], [0, 1], [0, 0], [0, 3]]   # s2 = [1, 1, 0, 3] for x[2:] = [0, 1]
    x = np.array([1.0, 0.0, 0.0, 1.0])
    # slot scores: s(i,j) = s1[i] + s2[j]; best is (1,3)=5, then (0,3)=(2,3)=4 tie, ...
    idx, sc, _ = o.topk(x, sk, 4, 5, mode=0)
    s1 = np.array([1, 2, 1, 0.0])
    s2 = np.array([1, 1, 0, 3.0])
    full = (s1[:, None] + s2[None, :]).reshape(-1)
    expect = sorted(range(16), key=lambda s: (-full[s], s))[:5]
    assert idx.tolist() == expect, (idx, expect)
    assert idx.tolist()[:3] == [7, 3, 11]
    idx2, _, _ = o.topk(x, sk, 4, 5, mode=1)
    assert idx2.tolist() == expect


def pin_hand_scoring(o):
    """The hand-worked scoring example in tests/golden/hand_scoring.json."""
    with open(os.path.join(GOLDEN, "hand_scoring.json")) as f:
        g = json.load(f)
    for mode in (0, 1):
        idx, sc, w = o.topk(g["x"], g["subkeys"], g["k_half"], g["top"], mode=mode)
        assert idx.tolist() == g["idx"]
        assert sc.tolist() == g["score"]
        np.testing.assert_allclose(w, g["w"], rtol=1e-15, atol=0)


def pin_softmax(o):
    """Weights are softmax of the selected scores: positive, sum 1, best-first,
    and w_a / w_b = exp(s_a - s_b)."""
    rng = _rng(4)
    n, hd = 8, 4
    sk = rng.standard_normal((2, n, hd))
    for top in (1, 2, 5):
        for _ in range(10):
            x = rng.standard_normal(2 * hd)
            idx, sc, w = o.topk(x, sk, n, top, mode=1)
            assert np.all(w > 0)
            assert abs(w.sum() - 1.0) < 1e-14
            assert np.all(np.diff(sc) <= 0) and np.all(np.diff(w) <= 1e-16)
            if top >= 2:
                np.testing.assert_allclose(w[0] / w[1], np.exp(sc[0] - sc[1]), rtol=1e-12)
            if top == 1:
                assert w[0] == 1.0


def pin_batched_score(o):
    """Batched scoring equals per-vector scoring, with per-head tables."""
    rng = _rng(5)
    B, H, T, hd, n, k, top = 2, 3, 5, 4, 6, 3, 3
    x = rng.standard_normal((B, H, T, 2 * hd))
    sk = rng.standard_normal((H, 2, n, hd))
    idx, sc, w = o.score(x, sk, k, top, mode=1)
    for b in range(B):
        for h in range(H):
            for t in range(T):
                i1, s1, w1 = o.topk(x[b, h, t], sk[h], k, top, mode=1)
                assert np.array_equal(idx[b, h, t], i1)
                assert np.array_equal(w[b, h, t], w1)


# ------------------------------------------------------------- recurrence ---

def pin_beta_zero(o):
    """beta = 0: memory only decays, M_T = M0 * prod(alpha) and
    o_t = sum_j u_j M0[r_j] * prod_{s<=t} alpha_s."""
    rng = _rng(6)
    T, N, dv, W, R = 17, 20, 3, 4, 5
    v, alpha, beta, widx, ww, ridx, rw, M0 = _random_case(rng, T, N, dv, W, R)
    beta = np.zeros(T)
    cum = np.cumprod(alpha)
    expect_out = np.stack([(rw[t][:, None] * M0[ridx[t]]).sum(0) * cum[t] for t in range(T)])
    out_d, M_d = o.recur_dense(v, alpha, beta, widx, ww, ridx, rw, M0)
    np.testing.assert_allclose(out_d, expect_out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(M_d, M0 * cum[-1], rtol=1e-12, atol=1e-14)
    st = o.fresh_lazy_state(M0)
    out_l = o.recur_lazy(v, alpha, beta, widx, ww, ridx, rw, st)
    np.testing.assert_allclose(out_l, expect_out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(o.materialize(st), M0 * cum[-1], rtol=1e-12, atol=1e-14)


def pin_one_hot_exact(o):
    """alpha = 1, beta = 1, a single write slot with weight 1 and a read of that
    slot right after: the read returns v exactly (delta rule overwrite)."""
    rng = _rng(7)
    T, N, dv = 9, 12, 4
    v = rng.standard_normal((T, dv))
    s = rng.permutation(N)[:T].astype(np.int32)[:, None]  # each token writes a fresh slot
    ones = np.ones((T, 1))
    for M0 in (np.zeros((N, dv)), ):
        out_d, _ = o.recur_dense(v, np.ones(T), np.ones(T), s, ones, s, ones, M0)
        assert np.array_equal(out_d, v)
        st = o.fresh_lazy_state(M0)
        out_l = o.recur_lazy(v, np.ones(T), np.ones(T), s, ones, s, ones, st)
        assert np.array_equal(out_l, v)
    # non-zero M0: exact up to the one rounding of M + (v - M)
    M0 = rng.standard_normal((N, dv))
    out_d, _ = o.recur_dense(v, np.ones(T), np.ones(T), s, ones, s, ones, M0)
    np.testing.assert_allclose(out_d, v, rtol=0, atol=4 * np.finfo(float).eps * 8)


def pin_convex_update(o):
    """W = R = 1 at one slot: M <- alpha*M + beta*(v - alpha*M), a textbook
    exponential-moving-average step, and the read returns it."""
    rng = _rng(8)
    T, N, dv = 12, 5, 3
    v = rng.standard_normal((T, dv))
    alpha = rng.uniform(0.5, 1.0, T)
    beta = rng.uniform(0.0, 1.0, T)
    s = np.full((T, 1), 2, np.int32)
    ones = np.ones((T, 1))
    M0 = rng.standard_normal((N, dv))
    m = M0[2].copy()
    expect = []
    for t in range(T):
        m = (1 - beta[t]) * alpha[t] * m + beta[t] * v[t]
        expect.append(m.copy())
    out_d, M_d = o.recur_dense(v, alpha, beta, s, ones, s, ones, M0)
    np.testing.assert_allclose(out_d, np.stack(expect), rtol=1e-12, atol=1e-14)
    others = [i for i in range(N) if i != 2]
    np.testing.assert_allclose(M_d[others], M0[others] * np.prod(alpha), rtol=1e-12)


def pin_dense_limit_gdn(o):
    """All N slots selected (W = R = N, k = n): the sparse recurrence is exactly
    Gated DeltaNet with the dense key k_t = softmax weights over all slots,
    S_t = alpha_t (I - beta_t k k^T) S_{t-1} + beta_t k v^T, o_t = S_t^T q_t."""
    rng = _rng(9)
    n, hd, T, dv = 4, 3, 11, 5
    N = n * n
    skw = rng.standard_normal((2, n, hd))
    skr = rng.standard_normal((2, n, hd))
    kx = rng.standard_normal((T, 2 * hd))
    qx = rng.standard_normal((T, 2 * hd))
    v = rng.standard_normal((T, dv))
    alpha = rng.uniform(0.7, 1.0, T)
    beta = rng.uniform(0.0, 1.0, T)
    M0 = rng.standard_normal((N, dv)) * 0.3

    def dense_weights(x, sk):
        s = (sk[0] @ x[:hd])[:, None] + (sk[1] @ x[hd:])[None, :]
        e = np.exp(s.reshape(-1) - s.max())
        return e / e.sum()

    S = M0.copy()
    expect = []
    for t in range(T):
        kv = dense_weights(kx[t], skw)
        qv = dense_weights(qx[t], skr)
        S = alpha[t] * (np.eye(N) - beta[t] * np.outer(kv, kv)) @ S + beta[t] * np.outer(kv, v[t])
        expect.append(S.T @ qv)
    widx, ww, ridx, rw = [], [], [], []
    for t in range(T):
        i, _, w = o.topk(kx[t], skw, n, N, mode=1)
        widx.append(i); ww.append(w)
        i, _, w = o.topk(qx[t], skr, n, N, mode=1)
        ridx.append(i); rw.append(w)
    out_d, M_d = o.recur_dense(v, alpha, beta, np.array(widx), np.array(ww), np.array(ridx),
                               np.array(rw), M0)
    np.testing.assert_allclose(out_d, np.stack(expect), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(M_d, S, rtol=1e-11, atol=1e-12)


def pin_lazy_equals_dense(o):
    """Lazy decay (per-slot stamps) equals literal dense decay to 1e-12."""
    rng = _rng(10)
    for (T, N, dv, W, R) in [(40, 12, 3, 3, 4), (64, 50, 4, 6, 6), (30, 9, 2, 9, 9)]:
        v, alpha, beta, widx, ww, ridx, rw, M0 = _random_case(rng, T, N, dv, W, R, 0.5, 1.0)
        out_d, M_d = o.recur_dense(v, alpha, beta, widx, ww, ridx, rw, M0)
        st = o.fresh_lazy_state(M0)
        out_l = o.recur_lazy(v, alpha, beta, widx, ww, ridx, rw, st)
        scale = max(1.0, np.abs(out_d).max())
        assert np.abs(out_l - out_d).max() <= 1e-12 * scale
        assert np.abs(o.materialize(st) - M_d).max() <= 1e-12 * max(1.0, np.abs(M_d).max())


def pin_split_invariance(o):
    """One call over T tokens equals T1 tokens then T-T1 tokens, and equals T1
    tokens then T-T1 single-token calls (the lazy state carries everything)."""
    rng = _rng(11)
    T, N, dv, W, R = 30, 15, 3, 3, 4
    v, alpha, beta, widx, ww, ridx, rw, M0 = _random_case(rng, T, N, dv, W, R)
    st = o.fresh_lazy_state(M0)
    full = o.recur_lazy(v, alpha, beta, widx, ww, ridx, rw, st)
    for T1 in (0, 1, 13, 29):
        st2 = o.fresh_lazy_state(M0)
        a = o.recur_lazy(v[:T1], alpha[:T1], beta[:T1], widx[:T1], ww[:T1], ridx[:T1], rw[:T1], st2)
        b = o.recur_lazy(v[T1:], alpha[T1:], beta[T1:], widx[T1:], ww[T1:], ridx[T1:], rw[T1:], st2)
        assert np.array_equal(np.concatenate([a, b]), full)
        st3 = o.fresh_lazy_state(M0)
        parts = [o.recur_lazy(v[:T1], alpha[:T1], beta[:T1], widx[:T1], ww[:T1], ridx[:T1],
                              rw[:T1], st3)]
        for t in range(T1, T):
            sl = slice(t, t + 1)
            parts.append(o.recur_lazy(v[sl], alpha[sl], beta[sl], widx[sl], ww[sl], ridx[sl],
                                      rw[sl], st3))
        assert np.array_equal(np.concatenate(parts), full)
        assert np.array_equal(o.materialize(st3), o.materialize(st))
    _, M_d = o.recur_dense(v, alpha, beta, widx, ww, ridx, rw, M0)
    _, M_a = o.recur_dense(v[:7], alpha[:7], beta[:7], widx[:7], ww[:7], ridx[:7], rw[:7], M0)
    _, M_b = o.recur_dense(v[7:], alpha[7:], beta[7:], widx[7:], ww[7:], ridx[7:], rw[7:], M_a)
    assert np.array_equal(M_b, M_d)


def pin_hand_recurrence(o):
    """The hand-worked two-token example in tests/golden/hand_two_tokens.json."""
    with open(os.path.join(GOLDEN, "hand_two_tokens.json")) as f:
        g = json.load(f)
    args = [np.array(g[k], dtype=float) for k in ("v", "alpha", "beta")]
    widx, ridx = np.array(g["widx"]), np.array(g["ridx"])
    ww, rw = np.array(g["ww"], float), np.array(g["rw"], float)
    M0 = np.array(g["M0"], float)
    out_d, M_d = o.recur_dense(*args, widx, ww, ridx, rw, M0)
    assert out_d.tolist() == g["out"]
    assert M_d.tolist() == g["M_final"]
    st = o.fresh_lazy_state(M0)
    out_l = o.recur_lazy(*args, widx, ww, ridx, rw, st)
    assert out_l.tolist() == g["out"]
    assert o.materialize(st).tolist() == g["M_final"]


# ------------------------------------------- touched-slots decay variant ---

def pin_touched_hand(o):
    """The hand-worked three-token example in tests/golden/hand_touched_three_tokens.json."""
    with open(os.path.join(GOLDEN, "hand_touched_three_tokens.json")) as f:
        g = json.load(f)
    args = [np.array(g[k], dtype=float) for k in ("v", "alpha", "beta")]
    widx, ridx = np.array(g["widx"]), np.array(g["ridx"])
    ww, rw = np.array(g["ww"], float), np.array(g["rw"], float)
    out, M = o.recur_touched(*args, widx, ww, ridx, rw, np.array(g["M0"], float))
    assert out.tolist() == g["out"]
    assert M.tolist() == g["M_final"]


def pin_touched_alpha_one(o):
    """alpha = 1: no slot decays under either reading, so the touched-slots recurrence
    performs the dense one's arithmetic exactly."""
    rng = _rng(13)
    T, N, dv, W, R = 25, 14, 3, 4, 5
    v, alpha, beta, widx, ww, ridx, rw, M0 = _random_case(rng, T, N, dv, W, R)
    ones = np.ones(T)
    out_t, M_t = o.recur_touched(v, ones, beta, widx, ww, ridx, rw, M0)
    out_d, M_d = o.recur_dense(v, ones, beta, widx, ww, ridx, rw, M0)
    assert np.array_equal(out_t, out_d) and np.array_equal(M_t, M_d)


def pin_touched_all_slots_gdn(o):
    """Every slot written at every token (W = N, a fresh permutation per token): every
    slot decays once per token, which is the dense form (Gated DeltaNet)."""
    rng = _rng(14)
    T, N, dv, R = 12, 7, 3, 4
    v = rng.standard_normal((T, dv))
    alpha = rng.uniform(0.5, 1.0, T)
    beta = rng.uniform(0.0, 1.0, T)
    widx = np.stack([rng.permutation(N) for _ in range(T)]).astype(np.int32)
    ww = rng.dirichlet(np.ones(N), T)
    ridx = np.stack([rng.permutation(N)[:R] for _ in range(T)]).astype(np.int32)
    rw = rng.dirichlet(np.ones(R), T)
    M0 = rng.standard_normal((N, dv))
    out_t, M_t = o.recur_touched(v, alpha, beta, widx, ww, ridx, rw, M0)
    out_d, M_d = o.recur_dense(v, alpha, beta, widx, ww, ridx, rw, M0)
    np.testing.assert_allclose(out_t, out_d, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(M_t, M_d, rtol=1e-13, atol=1e-14)


def pin_touched_beta_zero(o):
    """beta = 0: a slot is multiplied by alpha_t exactly at the tokens that write it, so
    M_T[s] = M0[s] * prod_{t: s written at t} alpha_t, and o_t reads that product up to
    token t (slots never written keep M0)."""
    rng = _rng(15)
    T, N, dv, W, R = 19, 16, 3, 3, 4
    v, alpha, beta, widx, ww, ridx, rw, M0 = _random_case(rng, T, N, dv, W, R, 0.5, 1.0)
    widx = np.stack([rng.permutation(10)[:W] for _ in range(T)]).astype(np.int32)  # 10..15 unwritten
    fac = np.ones((T + 1, N))
    for t in range(T):
        fac[t + 1] = fac[t]
        fac[t + 1, widx[t]] *= alpha[t]
    expect = np.stack([(rw[t][:, None] * (M0[ridx[t]] * fac[t + 1, ridx[t]][:, None])).sum(0)
                       for t in range(T)])
    out_t, M_t = o.recur_touched(v, alpha, np.zeros(T), widx, ww, ridx, rw, M0)
    np.testing.assert_allclose(out_t, expect, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(M_t, M0 * fac[T][:, None], rtol=1e-12, atol=1e-14)
    untouched = np.setdiff1d(np.arange(N), widx.reshape(-1))
    assert untouched.size > 0 and np.array_equal(M_t[untouched], M0[untouched])


# ----------------------------------------------------------------- backward ---

def _fd_case(rng, T, N, dv, W, R):
    v, alpha, beta, widx, ww, ridx, rw, M0 = _random_case(rng, T, N, dv, W, R, 0.5, 1.0)
    # small N: slots repeat across tokens and reads meet this token's writes
    widx = np.stack([rng.permutation(N)[:W] for _ in range(T)]).astype(np.int32)
    ridx = np.stack([rng.permutation(N)[:R] for _ in range(T)]).astype(np.int32)
    dout = rng.standard_normal((T, dv))
    return v, alpha, beta, widx, ww, ridx, rw, M0, dout


def _check_fd(o, touched, case, G_end=None):
    """Central differences of L = sum(dout * out) (+ sum(G_end * M_T), the final memory)
    through the forward oracle, every input."""
    v, alpha, beta, widx, ww, ridx, rw, M0, dout = case
    fwd = o.recur_touched if touched else o.recur_dense
    g = o.recur_backward(v, alpha, beta, widx, ww, ridx, rw, M0, dout, touched=touched,
                         dM_end=G_end)

    def loss(**kw):
        a = dict(v=v, alpha=alpha, beta=beta, ww=ww, rw=rw, M0=M0)
        a.update(kw)
        out, MT = fwd(a["v"], a["alpha"], a["beta"], widx, a["ww"], ridx, a["rw"], a["M0"])
        return float((dout * out).sum()) + (0.0 if G_end is None else float((G_end * MT).sum()))

    h = 1e-6
    for name, arr, key in (("v", v, "dv"), ("alpha", alpha, "dalpha"), ("beta", beta, "dbeta"),
                           ("ww", ww, "dww"), ("rw", rw, "drw"), ("M0", M0, "dM0")):
        num = np.empty_like(arr)
        for idx in np.ndindex(arr.shape):
            ap, am = arr.copy(), arr.copy()
            ap[idx] += h
            am[idx] -= h
            num[idx] = (loss(**{name: ap}) - loss(**{name: am})) / (2 * h)
        np.testing.assert_allclose(g[key], num, rtol=1e-6, atol=1e-7, err_msg=name)


def pin_backward_finite_differences(o):
    """The backward equals central differences of the forward (every slot decays)."""
    rng = _rng(16)
    _check_fd(o, False, _fd_case(rng, 7, 6, 3, 2, 3))
    _check_fd(o, False, _fd_case(rng, 5, 4, 2, 4, 4))  # every slot written at every token


def pin_backward_touched_finite_differences(o):
    """The backward equals central differences of the forward (only the write slots decay)."""
    rng = _rng(17)
    _check_fd(o, True, _fd_case(rng, 7, 6, 3, 2, 3))
    _check_fd(o, True, _fd_case(rng, 6, 9, 2, 3, 2))


def pin_backward_end_gradient(o):
    """A gradient for the memory after the last token (a loss that also reads the final
    state): central differences of L = sum(dout * out) + sum(G * M_T) for both decay rules;
    with no token it passes through unchanged; with beta = 0 and no output gradient, every
    slot decays, so M_T = M0 prod(alpha): dM0 = prod(alpha) G and
    dalpha_t = <G, M0> prod over the other tokens of alpha."""
    rng = _rng(20)
    for touched in (False, True):
        case = _fd_case(rng, 6, 5, 3, 2, 2)
        _check_fd(o, touched, case, G_end=rng.standard_normal((5, 3)))
    T, N, dv, W, R = 5, 6, 2, 2, 2
    v, alpha, beta, widx, ww, ridx, rw, M0, dout = _fd_case(rng, T, N, dv, W, R)
    G = rng.standard_normal((N, dv))
    g0 = o.recur_backward(v[:0], alpha[:0], beta[:0], widx[:0], ww[:0], ridx[:0], rw[:0], M0,
                          dout[:0], dM_end=G)
    assert np.array_equal(g0["dM0"], G)
    g = o.recur_backward(v, alpha, np.zeros(T), widx, ww, ridx, rw, M0, np.zeros((T, dv)),
                         dM_end=G)
    P = float(np.prod(alpha))
    np.testing.assert_allclose(g["dM0"], P * G, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(g["dalpha"], float((G * M0).sum()) * P / alpha, rtol=1e-12)
    assert np.array_equal(g["drw"], np.zeros((T, R)))


def pin_backward_split_calls(o):
    """A sequence taken back in two calls (the second call's start-state gradient passed to
    the first as the gradient of its final memory) gives the single call's gradients."""
    rng = _rng(21)
    T, T1, N, dv, W, R = 10, 4, 6, 3, 2, 3
    v, alpha, beta, widx, ww, ridx, rw, M0, dout = _fd_case(rng, T, N, dv, W, R)
    for touched in (False, True):
        fwd = o.recur_touched if touched else o.recur_dense
        whole = o.recur_backward(v, alpha, beta, widx, ww, ridx, rw, M0, dout, touched=touched)
        a, b = slice(0, T1), slice(T1, T)
        _, M_mid = fwd(v[a], alpha[a], beta[a], widx[a], ww[a], ridx[a], rw[a], M0)
        g2 = o.recur_backward(v[b], alpha[b], beta[b], widx[b], ww[b], ridx[b], rw[b], M_mid,
                              dout[b], touched=touched)
        g1 = o.recur_backward(v[a], alpha[a], beta[a], widx[a], ww[a], ridx[a], rw[a], M0,
                              dout[a], touched=touched, dM_end=g2["dM0"])
        for key in ("dv", "dalpha", "dbeta", "dww", "drw"):
            np.testing.assert_allclose(np.concatenate([g1[key], g2[key]]), whole[key],
                                       rtol=1e-12, atol=1e-13, err_msg=key)
        np.testing.assert_allclose(g1["dM0"], whole["dM0"], rtol=1e-12, atol=1e-13)


def pin_backward_frozen_memory(o):
    """beta = 0, alpha = 1: the memory stays M0, so o_t = sum_j u_j M0[r_j] and
    dM0[s] = sum over (t, j) with r_j = s of u_j dout_t, du_j = <dout_t, M0[r_j]>,
    dv = dw = 0 (no write moves the memory)."""
    rng = _rng(18)
    T, N, dv, W, R = 9, 8, 3, 2, 3
    v, alpha, beta, widx, ww, ridx, rw, M0, dout = _fd_case(rng, T, N, dv, W, R)
    for touched in (False, True):
        g = o.recur_backward(v, np.ones(T), np.zeros(T), widx, ww, ridx, rw, M0, dout,
                             touched=touched)
        expect = np.zeros_like(M0)
        for t in range(T):
            for j in range(R):
                expect[ridx[t, j]] += rw[t, j] * dout[t]
        np.testing.assert_allclose(g["dM0"], expect, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(g["drw"], np.einsum("tc,tjc->tj", dout, M0[ridx]),
                                   rtol=1e-13, atol=1e-14)
        assert np.array_equal(g["dv"], np.zeros((T, dv))) and np.array_equal(g["dww"], np.zeros((T, W)))


def pin_score_backward_finite_differences(o):
    """The scoring backward equals central differences of L = sum dw * softmax(scores of the
    fixed selected slots), the scores written out here from the definition, for x and both
    sub-key tables."""
    rng = _rng(19)
    B, H, T, n, hd, top = 2, 2, 3, 5, 3, 6
    x = rng.standard_normal((B, H, T, 2 * hd))
    sk = rng.standard_normal((H, 2, n, hd))
    idx = np.stack([rng.permutation(n * n)[:top] for _ in range(B * H * T)]).reshape(B, H, T, top)
    dw = rng.standard_normal((B, H, T, top))

    def loss(x, sk):
        tot = 0.0
        for b in range(B):
            for h in range(H):
                for t in range(T):
                    i, j = idx[b, h, t] // n, idx[b, h, t] % n
                    sc = sk[h, 0, i] @ x[b, h, t, :hd] + sk[h, 1, j] @ x[b, h, t, hd:]
                    e = np.exp(sc - sc.max())
                    tot += float(dw[b, h, t] @ (e / e.sum()))
        return tot

    dx, dsk = o.score_backward(x, sk, idx, dw)
    eps = 1e-6
    for arr, g, isx in ((x, dx, True), (sk, dsk, False)):
        num = np.empty_like(arr)
        for ix in np.ndindex(arr.shape):
            ap, am = arr.copy(), arr.copy()
            ap[ix] += eps
            am[ix] -= eps
            num[ix] = ((loss(ap, sk) - loss(am, sk)) if isx else (loss(x, ap) - loss(x, am))) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8)


def pin_prefill_pairs(o):
    """The batched prefill equals product-key scoring followed by the lazy recurrence."""
    rng = _rng(12)
    B, H, T, hd, n, dv, k, W, R = 2, 2, 9, 3, 5, 4, 3, 3, 2
    q = rng.standard_normal((B, H, T, 2 * hd))
    kk = rng.standard_normal((B, H, T, 2 * hd))
    v = rng.standard_normal((B, H, T, dv))
    alpha = rng.uniform(0.8, 1.0, (B, H, T))
    beta = rng.uniform(0, 1, (B, H, T))
    skw = rng.standard_normal((H, 2, n, hd))
    skr = rng.standard_normal((H, 2, n, hd))
    M0 = rng.standard_normal((H, n * n, dv))
    pairs = [(1, 0), (0, 1)]
    out = o.prefill_pairs(q, kk, v, alpha, beta, skw, skr, M0, k, W, R, pairs)
    for pi, (b, h) in enumerate(pairs):
        wi, _, wwt = o.score(kk[b:b + 1, h:h + 1], skw[h:h + 1], k, W)
        ri, _, rwt = o.score(q[b:b + 1, h:h + 1], skr[h:h + 1], k, R)
        st = o.fresh_lazy_state(M0[h])
        ref = o.recur_lazy(v[b, h], alpha[b, h], beta[b, h], wi[0, 0], wwt[0, 0], ri[0, 0],
                           rwt[0, 0], st)
        assert np.array_equal(out[pi], ref)


# ------------------------------------------------------ utilisation diagnostics ---
# Appendix D.1 "Memory Utilization and Access": cumulative top-k mass and an entropy-based
# effective-key measure of the post-softmax selected-slot weights, with the mean and
# token-level quantiles over batch, head and time.

def pin_weight_stats_closed_forms(o):
    K = 8
    # uniform weights: mass k/K, exp(H)/K = 1
    r = o.weight_stats(np.full((5, K), 1.0 / K))
    assert np.allclose(r["cum"][0], np.arange(1, K + 1) / K, rtol=0, atol=1e-15)
    assert np.allclose(r["eff"], 1.0, rtol=0, atol=1e-14)
    # one-hot: mass 1 everywhere, exp(0)/K
    w = np.zeros((3, K))
    w[:, 0] = 1.0
    r = o.weight_stats(w)
    assert np.array_equal(r["cum"], np.ones((3, K)))
    assert np.allclose(r["eff"], 1.0 / K, rtol=0, atol=1e-15)
    # two-point weights (p, 1-p): H = -p ln p - (1-p) ln(1-p), natural log
    p = 0.8
    w = np.zeros((1, K))
    w[0, :2] = [p, 1 - p]
    r = o.weight_stats(w)
    H = -p * np.log(p) - (1 - p) * np.log(1 - p)
    assert abs(r["eff"][0] - np.exp(H) / K) < 1e-14
    assert abs(r["cum"][0, 0] - p) < 1e-15 and abs(r["cum"][0, 1] - 1.0) < 1e-15


def pin_weight_stats_summaries(o):
    rng = _rng(77)
    K, rows = 16, 1000  # p * (rows - 1) is not an integer for p = 0.1, 0.5, 0.9
    w = rng.dirichlet(np.full(K, 0.7), rows)
    w = -np.sort(-w, axis=1)  # best first
    probs = (0.0, 0.1, 0.5, 0.9, 1.0)
    r = o.weight_stats(w, probs)
    # per row: cumulative sums and exp(entropy)/K written out with numpy
    assert np.allclose(r["cum"], np.cumsum(w, axis=1), rtol=0, atol=1e-14)
    H = -(w * np.log(w)).sum(1)
    assert np.allclose(r["eff"], np.exp(H) / K, rtol=1e-13, atol=0)
    assert np.allclose(r["mean_cum"], np.cumsum(w, axis=1).mean(0), rtol=0, atol=1e-14)
    assert abs(r["mean_eff"] - (np.exp(H) / K).mean()) < 1e-13
    # order statistics at floor(p (rows-1)) of the ascending sort
    srt = np.sort(np.exp(H) / K)
    for q, pq in zip(r["quant"], probs):
        assert abs(q - srt[int(np.floor(pq * (rows - 1)))]) < 1e-13
    assert abs(r["mean_cum"][-1] - 1.0) < 1e-12


# ------------------------------------------------------------- layer output ---
# §3 Method "Sparse retrieval": RMS-normalised, elementwise gated, mixed across heads.

def _sig(z):
    return 1.0 / (1.0 + np.exp(-z))


def pin_layer_out_hand_example(o):
    # one head, d_v = 2, x = (3, 4): mean square 12.5, so the normalised row is
    # (3, 4) / sqrt(12.5); gate pre-activation z = 1 on both channels: swish(1) = sigma(1);
    # wn = (1, 2); Wo = identity
    x = np.array([3.0, 4.0]).reshape(1, 1, 1, 2)
    g = np.ones((1, 1, 2))
    wn = np.array([1.0, 2.0])
    y = o.layer_out(x, g, wn, np.eye(2), eps=0.0)
    s1 = 1.0 / (1.0 + np.exp(-1.0))
    exp = np.array([3.0, 8.0]) / np.sqrt(12.5) * s1
    assert np.allclose(y.reshape(2), exp, rtol=1e-14, atol=0)


def pin_layer_out_properties(o):
    rng = _rng(91)
    B, H, T, dv, dm = 2, 3, 5, 8, 7
    x = rng.standard_normal((B, H, T, dv))
    g = rng.standard_normal((B, T, H * dv))
    wn = rng.uniform(0.5, 1.5, dv)
    Wo = rng.standard_normal((dm, H * dv))
    y = o.layer_out(x, g, wn, Wo, eps=0.0)
    # RMS-norm makes each head's read scale-free
    assert np.allclose(o.layer_out(x * 7.5, g, wn, Wo, eps=0.0), y, rtol=1e-12, atol=1e-12)
    # a zero gate closes the output; swish(z) ~ z for large z, ~ 0 for very negative z
    assert np.array_equal(o.layer_out(x, np.zeros_like(g), wn, Wo, eps=0.0), np.zeros((B, T, dm)))
    big = o.layer_out(x, np.full_like(g, 40.0), wn, Wo, eps=0.0)
    assert np.allclose(big, 40.0 * o.layer_out(x, np.full_like(g, 1e6), wn, Wo, eps=0.0) / 1e6,
                       rtol=1e-12, atol=1e-12)
    # Wo selecting one head and channel returns that head's gated normalised channel
    h, c = 2, 5
    sel = np.zeros((1, H * dv))
    sel[0, h * dv + c] = 1.0
    ys = o.layer_out(x, g, wn, sel, eps=0.0)[..., 0]
    xn = x[:, h] / np.sqrt((x[:, h] ** 2).mean(-1, keepdims=True))
    z = g[:, :, h * dv + c]
    assert np.allclose(ys, xn[..., c] * wn[c] * z * _sig(z), rtol=1e-12, atol=1e-14)
    # mixing across heads is a linear map of the gated reads (numpy matmul, row subset)
    a = np.concatenate([x[:, hh] / np.sqrt((x[:, hh] ** 2).mean(-1, keepdims=True)) * wn
                        for hh in range(H)], axis=-1) * g * _sig(g)
    assert np.allclose(y, a @ Wo.T, rtol=1e-12, atol=1e-12)
    rows = np.array([7, 0, 3])
    assert np.allclose(o.layer_out(x, g, wn, Wo, eps=0.0, rows=rows), y.reshape(B * T, dm)[rows],
                       rtol=0, atol=0)
    # eps enters as mean square + eps
    e = 0.3
    ye = o.layer_out(x, g, wn, sel, eps=e)[..., 0]
    xe = x[:, h] / np.sqrt((x[:, h] ** 2).mean(-1, keepdims=True) + e)
    assert np.allclose(ye, xe[..., c] * wn[c] * z * _sig(z), rtol=1e-12, atol=1e-14)


# -------------------------------------------------------------- layer input ---

def pin_layer_in_routing_and_gates(o):
    H, dk, dv, dm = 2, 3, 2, 5
    hs = 2 * dk + 2 * dv + 2
    rng = _rng(93)
    B, T = 2, 3
    x = rng.standard_normal((B, T, dm))
    A_log = np.array([0.2, -0.7])
    dt = np.array([0.5, -1.0])
    # Win routes input dim (n mod dm) to output column n: every output is a known input value
    Win = np.zeros((H * hs, dm))
    for n in range(H * hs):
        Win[n, n % dm] = 1.0
    r = o.layer_in(x, Win, A_log, dt, H, dk, dv)
    col = lambda n: x[..., n % dm]  # [B, T]
    for h in range(H):
        base = h * hs
        for c in range(dk):
            assert np.array_equal(r["q"][:, h, :, c], col(base + c))
            assert np.array_equal(r["k"][:, h, :, c], col(base + dk + c))
        for c in range(dv):
            assert np.array_equal(r["v"][:, h, :, c], col(base + 2 * dk + c))
            assert np.array_equal(r["g"][:, :, h * dv + c], col(base + 2 * dk + dv + c))
        a = col(base + 2 * dk + 2 * dv)
        b = col(base + 2 * dk + 2 * dv + 1)
        sp = np.log1p(np.exp(a + dt[h]))
        assert np.allclose(r["alpha"][:, h], np.exp(-np.exp(A_log[h]) * sp), rtol=1e-14, atol=0)
        assert np.allclose(r["beta"][:, h], 1 / (1 + np.exp(-b)), rtol=1e-14, atol=0)
    # gate ranges: alpha in (0, 1), beta in (0, 1); a very negative a gives alpha -> 1
    assert ((r["alpha"] > 0) & (r["alpha"] < 1)).all() and ((r["beta"] > 0) & (r["beta"] < 1)).all()
    Wa = np.zeros((H * hs, dm))
    xs = np.full((1, 1, dm), -60.0)
    Wa[2 * dk + 2 * dv, 0] = 1.0
    assert abs(o.layer_in(xs, Wa, A_log, np.zeros(H), H, dk, dv)["alpha"][0, 0, 0] - 1.0) < 1e-20 + 1e-12


def pin_layer_in_linear(o):
    rng = _rng(94)
    H, dk, dv, dm, B, T = 3, 4, 2, 6, 2, 4
    hs = 2 * dk + 2 * dv + 2
    x = rng.standard_normal((B, T, dm))
    Win = rng.standard_normal((H * hs, dm))
    A_log, dt = rng.standard_normal(H), rng.standard_normal(H)
    r = o.layer_in(x, Win, A_log, dt, H, dk, dv)
    P = x @ Win.T  # numpy matmul: the projection
    for h in range(H):
        base = h * hs
        assert np.allclose(r["q"][:, h], P[..., base:base + dk], rtol=1e-12, atol=1e-12)
        assert np.allclose(r["v"][:, h], P[..., base + 2 * dk:base + 2 * dk + dv], rtol=1e-12, atol=1e-12)
    # projections are linear in x; the listed-rows form agrees with the full form
    r2 = o.layer_in(2 * x, Win, A_log, dt, H, dk, dv)
    assert np.allclose(r2["k"], 2 * r["k"], rtol=1e-12, atol=1e-12)
    rows = np.array([5, 0])
    rs = o.layer_in(x, Win, A_log, dt, H, dk, dv, rows=rows)
    assert np.array_equal(rs["g"], r["g"].reshape(B * T, -1)[rows])


ALL_PINS = [pin_pk_equals_brute, pin_brute_matches_numpy, pin_pk_depends_on_k, pin_tie_order,
            pin_hand_scoring, pin_softmax, pin_batched_score, pin_beta_zero, pin_one_hot_exact,
            pin_convex_update, pin_dense_limit_gdn, pin_lazy_equals_dense, pin_split_invariance,
            pin_hand_recurrence, pin_prefill_pairs, pin_weight_stats_closed_forms,
            pin_weight_stats_summaries, pin_layer_out_hand_example, pin_layer_out_properties,
            pin_layer_in_routing_and_gates, pin_layer_in_linear, pin_touched_hand,
            pin_touched_alpha_one, pin_touched_all_slots_gdn, pin_touched_beta_zero,
            pin_backward_finite_differences, pin_backward_touched_finite_differences,
            pin_backward_frozen_memory, pin_backward_end_gradient, pin_backward_split_calls, pin_score_backward_finite_differences]
