"""Seeded synthetic inputs for the Sparse Delta Memory hot path.

This module only draws random tensors with the shapes and distributions of the
five workloads; it holds none of the method's arithmetic.  Both the CUDA path
and the CPU oracle consume exactly the bytes it produces (the oracle receives
them upcast to fp64).

Notation follows the pages: B sequences, H heads, T tokens, key width d_k (two
halves of d_k/2), n sub-keys per half (N = n^2 slots), value width d_v, per-half
top-k, W write slots and R read slots per token, decay gate alpha, input gate
beta, initial memory M0.  A distribution written N(mu, s) takes s as the
VARIANCE (so N(0, 0.02^2) has std 0.02 and N(0, 0.1) has std sqrt(0.1)).
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d_k: int
    n_sub: int
    d_v: int
    k_half: int
    W: int
    R: int
    x_dtype: str  # "f32" or "bf16": q, k and the sub-key tables
    v_dtype: str  # "f32" or "bf16"
    alpha: tuple  # ("uniform", lo, hi) or ("sigmoid_normal", mean, var)
    beta: tuple
    subkey_var: float
    m0_std: float = 0.02
    clusters: int = 0  # >0: q and k are cluster centre + noise
    cluster_noise_var: float = 0.1
    decode_steps: int = 0  # >0: T tokens of prefill, then this many single-token steps
    seed: int = 1000

    @property
    def N(self) -> int:
        return self.n_sub * self.n_sub

    @property
    def hd(self) -> int:
        return self.d_k // 2

    def scaled(self, **kw) -> "Workload":
        """Same structure with some sizes replaced (e.g. fewer tokens for a parity test)."""
        return dataclasses.replace(self, **kw)


# The five workloads, in the order they are specified.
TINY = Workload("tiny", B=1, H=1, T=256, d_k=32, n_sub=16, d_v=16, k_half=4, W=4, R=4,
                x_dtype="f32", v_dtype="f32", alpha=("uniform", 0.9, 1.0), beta=("uniform", 0.0, 1.0),
                subkey_var=1.0 / 16, seed=1001)
MID = Workload("mid_prefill", B=2, H=4, T=4096, d_k=128, n_sub=256, d_v=128, k_half=32, W=32, R=32,
               x_dtype="bf16", v_dtype="bf16", alpha=("uniform", 0.95, 1.0),
               beta=("uniform", 0.0, 1.0), subkey_var=1.0 / 64, seed=1002)
HEADLINE = Workload("headline_prefill", B=8, H=16, T=8192, d_k=128, n_sub=512, d_v=64, k_half=16,
                    W=16, R=16, x_dtype="bf16", v_dtype="bf16", alpha=("sigmoid_normal", 3.0, 0.5),
                    beta=("sigmoid_normal", 0.0, 1.0), subkey_var=1.0 / 64, seed=1003)
DECODE = Workload("decode", B=64, H=16, T=512, d_k=128, n_sub=256, d_v=128, k_half=32, W=32, R=32,
                  x_dtype="bf16", v_dtype="bf16", alpha=("uniform", 0.95, 1.0),
                  beta=("uniform", 0.0, 1.0), subkey_var=1.0 / 64, decode_steps=1024, seed=1004)
LONG = Workload("long_context", B=1, H=32, T=131072, d_k=128, n_sub=1024, d_v=128, k_half=64, W=64,
                R=64, x_dtype="bf16", v_dtype="bf16", alpha=("uniform", 0.99, 1.0),
                beta=("uniform", 0.0, 1.0), subkey_var=1.0 / 64, clusters=4096, seed=1005)

WORKLOADS = {w.name: w for w in (TINY, MID, HEADLINE, DECODE, LONG)}
ORDER = [TINY, MID, HEADLINE, DECODE, LONG]


def torch_dtype(tag: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[tag]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _gate(spec, shape, g, device) -> torch.Tensor:
    kind = spec[0]
    if kind == "uniform":
        lo, hi = spec[1], spec[2]
        x = torch.empty(shape, dtype=torch.float32, device=device)
        x.uniform_(lo, hi, generator=g)
        if hi <= 1.0:  # keep the half-open interval [lo, hi) strictly below hi
            x.clamp_(max=math.nextafter(hi, 0.0))
        return x
    if kind == "sigmoid_normal":
        mean, var = spec[1], spec[2]
        x = torch.empty(shape, dtype=torch.float32, device=device)
        x.normal_(mean, math.sqrt(var), generator=g)
        return torch.sigmoid(x)
    raise ValueError(spec)


def _normal(shape, std, dtype, g, device) -> torch.Tensor:
    x = torch.empty(shape, dtype=torch.float32, device=device)
    x.normal_(0.0, std, generator=g)
    return x.to(dtype)


def _clustered(wl: Workload, T: int, g, device, centres) -> torch.Tensor:
    B, H = wl.B, wl.H
    which = torch.randint(0, wl.clusters, (B, H, T), generator=g, device=device)
    x = torch.empty((B, H, T, wl.d_k), dtype=torch.float32, device=device)
    x.normal_(0.0, math.sqrt(wl.cluster_noise_var), generator=g)
    x += centres[which]
    return x.to(torch_dtype(wl.x_dtype))


def generate(wl: Workload, device="cpu", seed: int | None = None, with_m0: bool = True) -> dict:
    """Draw every input of one workload.

    Returns a dict of tensors on `device`:
      q, k   [B,H,T_all,d_k]  (x_dtype)   T_all = T + decode_steps
      v      [B,H,T_all,d_v]  (v_dtype)
      alpha, beta [B,H,T_all] (f32)
      skw, skr [H,2,n,d_k/2]  (x_dtype)   write / read sub-key tables
      M0     [H,N,d_v]        (f32)       only when with_m0
    """
    seed = wl.seed if seed is None else seed
    g = _gen(device, seed)
    B, H, d_k, d_v = wl.B, wl.H, wl.d_k, wl.d_v
    T_all = wl.T + wl.decode_steps
    xd, vd = torch_dtype(wl.x_dtype), torch_dtype(wl.v_dtype)
    out = {}
    if wl.clusters > 0:
        centres = torch.empty((wl.clusters, d_k), dtype=torch.float32, device=device)
        centres.normal_(0.0, 1.0, generator=g)
        out["k"] = _clustered(wl, T_all, g, device, centres)
        out["q"] = _clustered(wl, T_all, g, device, centres)
        del centres
    else:
        out["q"] = _normal((B, H, T_all, d_k), 1.0, xd, g, device)
        out["k"] = _normal((B, H, T_all, d_k), 1.0, xd, g, device)
    out["v"] = _normal((B, H, T_all, d_v), 1.0, vd, g, device)
    out["alpha"] = _gate(wl.alpha, (B, H, T_all), g, device)
    out["beta"] = _gate(wl.beta, (B, H, T_all), g, device)
    sk_std = math.sqrt(wl.subkey_var)
    out["skw"] = _normal((H, 2, wl.n_sub, wl.hd), sk_std, xd, g, device)
    out["skr"] = _normal((H, 2, wl.n_sub, wl.hd), sk_std, xd, g, device)
    if with_m0:
        M0 = torch.empty((H, wl.N, d_v), dtype=torch.float32, device=device)
        for h in range(H):  # per head, so no full-size temporary is needed
            M0[h].normal_(0.0, wl.m0_std, generator=g)
        out["M0"] = M0
    return out


def decode_layout(x: torch.Tensor, T0: int) -> torch.Tensor:
    """Tokens T0.. of a [B,H,T_all,...] tensor rearranged step-major: [steps,B,H,...]."""
    return x[:, :, T0:].movedim(2, 0).contiguous()


def random_indices(B, H, T, N, top, g: torch.Generator, device="cpu", pool: int | None = None
                   ) -> torch.Tensor:
    """Distinct random slots per token, [B,H,T,top] int32 (for recurrence-only tests).

    Slots are drawn from `pool` (default N) randomly chosen slots, so a small pool
    makes nearby tokens share slots often.
    """
    pool = N if pool is None else pool
    assert top <= pool <= N
    r = torch.randint(0, pool - top + 1, (B, H, T, top), generator=g, device=device)
    r = r.sort(dim=-1).values + torch.arange(top, device=device)  # distinct, sorted
    order = torch.rand((B, H, T, top), generator=g, device=device).argsort(dim=-1)
    r = r.gather(-1, order)  # random order within the token
    perm = torch.randperm(N, generator=g, device=device)[:pool]
    return perm[r].to(torch.int32)


def random_weights(B, H, T, top, g: torch.Generator, device="cpu") -> torch.Tensor:
    """Positive weights summing to one per token, [B,H,T,top] f32 (for recurrence-only tests)."""
    w = torch.rand((B, H, T, top), generator=g, device=device) + 0.05
    return (w / w.sum(-1, keepdim=True)).to(torch.float32)
