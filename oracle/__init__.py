"""CPU oracle for Sparse Delta Memory (SDM).  TEST INFRASTRUCTURE ONLY.

A plain, slow fp64 implementation (``sdm_oracle.c``) of what the SDM hot path
computes: product-key scoring with top-W / top-R selection and softmax weights,
and the sparse gated-delta recurrence over an N-slot memory that starts from M0.
Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path and
never imports it.

Readings of the method (the pages give prose, not equations) are written out in
``sdm_oracle.c``'s header; each C function names the passage it follows.

Parity status per function:
  half_scores / topk / score ... pinned (brute force vs product key, numpy matmul
                                 + argsort, exact-recall proof when k >= top)
  softmax weights ............. pinned (sum to 1, order, closed form on 2 slots)
  recur_dense ................. pinned (beta=0 closed form, one-hot write/read,
                                 dense Gated DeltaNet matrix form, hand example)
  recur_lazy .................. pinned (agrees with recur_dense to 1e-12)
  recur_backward .............. pinned (central finite differences of recur_dense and
                                 recur_touched for every input, with and without a gradient
                                 of the final memory; beta = 0 and alpha = 1 closed form;
                                 beta = 0 decay closed form of that gradient; two calls
                                 chained through it = one call)
  score_backward .............. pinned (central finite differences of the softmax of the
                                 selected slots' half-score sums, for x and the tables)
  recur_touched ............... pinned (hand example, alpha = 1 equals recur_dense,
                                 all slots written = recur_dense (Gated DeltaNet),
                                 beta = 0 closed form with unwritten slots at M0)
  materialize ................. pinned (beta=0 closed form)
  prefill_pairs ............... pinned through score + recur_lazy
  weight_stats ................ pinned (uniform and one-hot closed forms, two-point
                                 entropy, numpy sort for the order statistics)
  layer_in .................... pinned (one-hot routing of inputs to each output, gate
                                 closed forms, linearity, matmul)
  layer_out ................... pinned (hand RMS-norm example, scale invariance, swish
                                 closed forms, gate zero, head selection by Wo, matmul)
The softmax temperature and the tie order are readings the pages do not fix
(parity of those two choices is unpinned by the pages themselves).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "sdm_oracle.c")
LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_default = None

MODE_BRUTE = 0
MODE_PK = 1


def build(force: bool = False, src: str = SRC, out: str = LIB_PATH) -> str:
    """Compile the oracle C source into a shared library with gcc (-O2, OpenMP)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


class Oracle:
    """numpy front end over one build of the oracle library."""

    def __init__(self, lib_path: str = LIB_PATH):
        lib = ctypes.CDLL(lib_path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        lib.sdm_oracle_half_scores.argtypes = [P, P, I, I, P, P]
        lib.sdm_oracle_half_scores.restype = None
        lib.sdm_oracle_topk_vec.argtypes = [P, P, I, I, I, I, I, P, P, P]
        lib.sdm_oracle_topk_vec.restype = I
        lib.sdm_oracle_score.argtypes = [P, P, I, I, I, I, I, I, I, I, P, P, P, I]
        lib.sdm_oracle_score.restype = I
        lib.sdm_oracle_recur_dense.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P, P]
        lib.sdm_oracle_recur_dense.restype = I
        lib.sdm_oracle_recur_touched.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P, P]
        lib.sdm_oracle_recur_touched.restype = I
        lib.sdm_oracle_recur_backward.argtypes = [I, I, I, I, I, I] + [P] * 16
        lib.sdm_oracle_recur_backward.restype = I
        lib.sdm_oracle_score_backward.argtypes = [P, P, I, I, I, I, P, P, P, P]
        lib.sdm_oracle_score_backward.restype = I
        lib.sdm_oracle_recur_lazy.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P]
        lib.sdm_oracle_recur_lazy.restype = I
        lib.sdm_oracle_materialize.argtypes = [I, I, P, P, D, P]
        lib.sdm_oracle_materialize.restype = None
        lib.sdm_oracle_prefill_pairs.argtypes = [I, I, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P,
                                                 I, P, P, I]
        lib.sdm_oracle_prefill_pairs.restype = I
        lib.sdm_oracle_weight_stats.argtypes = [I, I, P, P, P, P, P, I, P, P]
        lib.sdm_oracle_weight_stats.restype = I
        lib.sdm_oracle_layer_out.argtypes = [I, I, I, I, I, P, P, P, D, P, I, P, P]
        lib.sdm_oracle_layer_out.restype = I
        lib.sdm_oracle_layer_in.argtypes = [I, I, I, I, I, I, P, P, P, P, I, P, P, P, P, P, P, P]
        lib.sdm_oracle_layer_in.restype = I
        lib.sdm_oracle_max_threads.argtypes = []
        lib.sdm_oracle_max_threads.restype = I
        self.lib = lib

    def max_threads(self) -> int:
        return int(self.lib.sdm_oracle_max_threads())

    def layer_out(self, o, g, wn, Wo_t, eps: float = 1e-6, rows=None):
        """Output side of an SDM layer: o [B,H,T,dv], g [B,T,H*dv], wn [dv], Wo_t [dm, H*dv]
        -> y [B,T,dm], or [len(rows), dm] for the listed rows (b*T + t)."""
        o = _f64(o)
        B, H, T, dv = o.shape
        Wo_t = _f64(Wo_t)
        dm = int(Wo_t.shape[0])
        full = rows is None
        r = np.arange(B * T, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
        y = np.empty((len(r), dm), dtype=np.float64)
        _check(self.lib.sdm_oracle_layer_out(B, H, T, dv, dm, _p(o), _p(_f64(g)), _p(_f64(wn)),
                                             float(eps), _p(Wo_t), len(r), _p(r), _p(y)),
               "layer_out")
        return y.reshape(B, T, dm) if full else y

    def layer_in(self, x, Win_t, A_log, dt_bias, H: int, dk: int, dv: int, rows=None):
        """Input side of an SDM layer: x [B,T,dm], Win_t [H*(2dk+2dv+2), dm] -> dict of q, k
        [B,H,T,dk], v [B,H,T,dv], g [B,T,H*dv], alpha, beta [B,H,T]; with rows (b*T + t) the
        outputs are per listed row: q [n,H,dk], v [n,H,dv], g [n,H*dv], alpha/beta [n,H]."""
        x = _f64(x)
        B, T, dm = x.shape
        full = rows is None
        r = np.arange(B * T, dtype=np.int64) if full else np.ascontiguousarray(rows, dtype=np.int64)
        n = len(r)
        q = np.empty((n, H, dk)); k = np.empty((n, H, dk)); v = np.empty((n, H, dv))
        g = np.empty((n, H * dv)); a = np.empty((n, H)); b = np.empty((n, H))
        _check(self.lib.sdm_oracle_layer_in(B, H, T, dk, dv, dm, _p(x), _p(_f64(Win_t)),
                                            _p(_f64(A_log)), _p(_f64(dt_bias)), n, _p(r), _p(q),
                                            _p(k), _p(v), _p(g), _p(a), _p(b)), "layer_in")
        if not full:
            return {"q": q, "k": k, "v": v, "g": g, "alpha": a, "beta": b}
        bht = lambda z: z.reshape(B, T, H, -1).transpose(0, 2, 1, 3)
        return {"q": bht(q), "k": bht(k), "v": bht(v), "g": g.reshape(B, T, H * dv),
                "alpha": a.reshape(B, T, H).transpose(0, 2, 1),
                "beta": b.reshape(B, T, H).transpose(0, 2, 1)}

    def weight_stats(self, w, probs=(0.1, 0.5, 0.9)):
        """Memory-utilisation diagnostics (Appendix D.1) of weight rows w [..., K] given best
        first: per-row cumulative mass and normalised effective keys exp(H)/K, their means,
        and order statistics of exp(H)/K at floor(p*(rows-1)).  Returns a dict."""
        w = _f64(w)
        K = int(w.shape[-1])
        rows = int(w.size // K)
        cum = np.empty(w.shape, dtype=np.float64)
        eff = np.empty(w.shape[:-1], dtype=np.float64)
        mean_cum = np.empty(K, dtype=np.float64)
        mean_eff = np.empty(1, dtype=np.float64)
        pr = _f64(probs)
        quant = np.empty(len(pr), dtype=np.float64)
        _check(self.lib.sdm_oracle_weight_stats(rows, K, _p(w), _p(cum), _p(eff), _p(mean_cum),
                                                _p(mean_eff), len(pr), _p(pr), _p(quant)),
               "weight_stats")
        return {"cum": cum, "eff": eff, "mean_cum": mean_cum, "mean_eff": float(mean_eff[0]),
                "quant": quant}

    def half_scores(self, x, sk):
        """s1[i] = <x[:h], C1[i]>, s2[j] = <x[h:], C2[j]> for one vector x [2h], sk [2,n,h]."""
        x, sk = _f64(x), _f64(sk)
        n, hd = sk.shape[1], sk.shape[2]
        assert x.shape == (2 * hd,)
        s1 = np.empty(n, np.float64)
        s2 = np.empty(n, np.float64)
        self.lib.sdm_oracle_half_scores(_p(x), _p(sk), n, hd, _p(s1), _p(s2))
        return s1, s2

    def topk(self, x, sk, k_half: int, top: int, mode: int = MODE_PK):
        """Best-first (idx, score, w) for one vector x [2h] against one role's tables sk [2,n,h]."""
        x, sk = _f64(x), _f64(sk)
        n, hd = sk.shape[1], sk.shape[2]
        idx = np.empty(top, np.int32)
        sc = np.empty(top, np.float64)
        w = np.empty(top, np.float64)
        _check(self.lib.sdm_oracle_topk_vec(_p(x), _p(sk), n, hd, k_half, top, mode, _p(idx), _p(sc),
                                            _p(w)), "topk")
        return idx, sc, w

    def score(self, x, sk, k_half: int, top: int, mode: int = MODE_PK, nthreads: int = 0):
        """Batched scoring: x [B,H,T,2h], sk [H,2,n,h] -> idx/score/w [B,H,T,top]."""
        x, sk = _f64(x), _f64(sk)
        B, H, T, dk = x.shape
        n, hd = sk.shape[2], sk.shape[3]
        assert dk == 2 * hd and sk.shape[0] == H and sk.shape[1] == 2
        idx = np.empty((B, H, T, top), np.int32)
        sc = np.empty((B, H, T, top), np.float64)
        w = np.empty((B, H, T, top), np.float64)
        _check(self.lib.sdm_oracle_score(_p(x), _p(sk), B, H, T, hd, n, k_half, top, mode, _p(idx),
                                         _p(sc), _p(w), nthreads), "score")
        return idx, sc, w

    def recur_dense(self, v, alpha, beta, widx, ww, ridx, rw, M):
        """Dense-decay recurrence for one (b,h).  Returns (out [T,dv], M_final [N,dv])."""
        v, alpha, beta = _f64(v), _f64(alpha), _f64(beta)
        widx, ridx, ww, rw = _i32(widx), _i32(ridx), _f64(ww), _f64(rw)
        M = _f64(M).copy()
        T, dv = v.shape
        N = M.shape[0]
        W, R = widx.shape[1], ridx.shape[1]
        out = np.empty((T, dv), np.float64)
        _check(self.lib.sdm_oracle_recur_dense(T, N, dv, W, R, _p(v), _p(alpha), _p(beta), _p(widx),
                                               _p(ww), _p(ridx), _p(rw), _p(M), _p(out)),
               "recur_dense")
        return out, M

    def recur_touched(self, v, alpha, beta, widx, ww, ridx, rw, M):
        """Touched-slots decay (alpha scales only the write slots) for one (b,h).

        Returns (out [T,dv], M_final [N,dv])."""
        v, alpha, beta = _f64(v), _f64(alpha), _f64(beta)
        widx, ridx, ww, rw = _i32(widx), _i32(ridx), _f64(ww), _f64(rw)
        M = _f64(M).copy()
        T, dv = v.shape
        N = M.shape[0]
        W, R = widx.shape[1], ridx.shape[1]
        out = np.empty((T, dv), np.float64)
        _check(self.lib.sdm_oracle_recur_touched(T, N, dv, W, R, _p(v), _p(alpha), _p(beta),
                                                 _p(widx), _p(ww), _p(ridx), _p(rw), _p(M),
                                                 _p(out)), "recur_touched")
        return out, M

    def score_backward(self, x, sk, idx, dw):
        """Gradient through the scoring with the selections idx [B,H,T,top] fixed.
        x [B,H,T,2h], sk [H,2,n,h], dw [B,H,T,top].  Returns (dx like x, dsk like sk)."""
        x, sk, dw = _f64(x), _f64(sk), _f64(dw)
        idx = _i32(idx)
        B, H, T, dk = x.shape
        n, hd = sk.shape[2], sk.shape[3]
        top = idx.shape[-1]
        dx = np.empty_like(x)
        dsk = np.zeros_like(sk)
        for h in range(H):
            xh = np.ascontiguousarray(x[:, h].reshape(B * T, dk))
            ih = np.ascontiguousarray(idx[:, h].reshape(B * T, top))
            dwh = np.ascontiguousarray(dw[:, h].reshape(B * T, top))
            dxh = np.empty_like(xh)
            dskh = np.zeros_like(sk[h])
            _check(self.lib.sdm_oracle_score_backward(_p(xh), _p(np.ascontiguousarray(sk[h])),
                                                      B * T, n, hd, top, _p(ih), _p(dwh),
                                                      _p(dxh), _p(dskh)), "score_backward")
            dx[:, h] = dxh.reshape(B, T, dk)
            dsk[h] = dskh
        return dx, dsk

    def recur_backward(self, v, alpha, beta, widx, ww, ridx, rw, M0, dout, touched=False,
                       dM_end=None):
        """Gradients of one (b,h)'s recurrence for output gradient dout [T,dv] (selections
        fixed) and, optionally, gradient dM_end [N,dv] with respect to the memory after the
        last token.  Returns dict dv [T,dv], dalpha [T], dbeta [T], dww [T,W], drw [T,R],
        dM0 [N,dv] (with respect to the state at the start)."""
        v, alpha, beta = _f64(v), _f64(alpha), _f64(beta)
        widx, ridx, ww, rw = _i32(widx), _i32(ridx), _f64(ww), _f64(rw)
        M0, dout = _f64(M0), _f64(dout)
        T, dv = v.shape
        N = M0.shape[0]
        W, R = widx.shape[1], ridx.shape[1]
        g = {"dv": np.empty((T, dv)), "dalpha": np.empty(T), "dbeta": np.empty(T),
             "dww": np.empty((T, W)), "drw": np.empty((T, R)), "dM0": np.empty((N, dv))}
        _check(self.lib.sdm_oracle_recur_backward(
            T, N, dv, W, R, 1 if touched else 0, _p(v), _p(alpha), _p(beta), _p(widx), _p(ww),
            _p(ridx), _p(rw), _p(M0), _p(dout), None if dM_end is None else _p(_f64(dM_end)),
            _p(g["dv"]), _p(g["dalpha"]), _p(g["dbeta"]),
            _p(g["dww"]), _p(g["drw"]), _p(g["dM0"])), "recur_backward")
        return g

    @staticmethod
    def fresh_lazy_state(M0h):
        """Lazy state of a fresh sequence: Mraw = M0 (copy), stamp = 0, Lambda = 0."""
        M0h = _f64(M0h)
        return {"Mraw": M0h.copy(), "stamp": np.zeros(M0h.shape[0], np.float64), "Lambda": 0.0}

    def recur_lazy(self, v, alpha, beta, widx, ww, ridx, rw, state):
        """Lazy-decay recurrence for one (b,h); `state` is updated in place.  Returns out [T,dv]."""
        v, alpha, beta = _f64(v), _f64(alpha), _f64(beta)
        widx, ridx, ww, rw = _i32(widx), _i32(ridx), _f64(ww), _f64(rw)
        T, dv = v.shape
        Mraw, stamp = state["Mraw"], state["stamp"]
        assert Mraw.dtype == np.float64 and Mraw.flags.c_contiguous and stamp.flags.c_contiguous
        N = Mraw.shape[0]
        W, R = widx.shape[1], ridx.shape[1]
        lam = ctypes.c_double(state["Lambda"])
        out = np.empty((T, dv), np.float64)
        _check(self.lib.sdm_oracle_recur_lazy(T, N, dv, W, R, _p(v), _p(alpha), _p(beta), _p(widx),
                                              _p(ww), _p(ridx), _p(rw), _p(Mraw), _p(stamp),
                                              ctypes.byref(lam), _p(out)), "recur_lazy")
        state["Lambda"] = lam.value
        return out

    def materialize(self, state):
        """Dense [N,dv] memory of a lazy state."""
        Mraw, stamp = state["Mraw"], state["stamp"]
        N, dv = Mraw.shape
        M = np.empty_like(Mraw)
        self.lib.sdm_oracle_materialize(N, dv, _p(Mraw), _p(stamp), float(state["Lambda"]), _p(M))
        return M

    def prefill_pairs(self, q, k, v, alpha, beta, skw, skr, M0, k_half: int, W: int, R: int, pairs,
                      nthreads: int = 0):
        """Score both roles and run the lazy recurrence from M0 for each (b,h) in `pairs`.

        Returns out [len(pairs), T, dv].  Used for the timed CPU baseline.
        """
        q, k, v, alpha, beta = _f64(q), _f64(k), _f64(v), _f64(alpha), _f64(beta)
        skw, skr, M0 = _f64(skw), _f64(skr), _f64(M0)
        B, H, T, dk = q.shape
        n, hd = skw.shape[2], skw.shape[3]
        dv = v.shape[3]
        pairs = _i32(np.asarray(pairs).reshape(-1, 2))
        out = np.empty((pairs.shape[0], T, dv), np.float64)
        _check(self.lib.sdm_oracle_prefill_pairs(B, H, T, hd, n, dv, k_half, W, R, _p(q), _p(k),
                                                 _p(v), _p(alpha), _p(beta), _p(skw), _p(skr),
                                                 _p(M0), pairs.shape[0], _p(pairs), _p(out),
                                                 nthreads), "prefill_pairs")
        return out


def default() -> Oracle:
    """The oracle built from sdm_oracle.c (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            build()
            _default = Oracle(LIB_PATH)
        return _default


def __getattr__(name):
    # module-level shortcuts: oracle.score(...), oracle.recur_lazy(...), ...
    if name in {"max_threads", "half_scores", "topk", "score", "recur_dense", "recur_lazy",
                "materialize", "prefill_pairs"}:
        return getattr(default(), name)
    if name == "fresh_lazy_state":
        return Oracle.fresh_lazy_state
    raise AttributeError(name)
