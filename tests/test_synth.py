"""The seeded workload generator: shapes, dtypes, determinism and the stated distributions."""
import math

import torch

import sdm_synth as S


def test_shapes_and_dtypes_tiny():
    d = S.generate(S.TINY)
    wl = S.TINY
    assert d["q"].shape == (1, 1, 256, 32) and d["q"].dtype == torch.float32
    assert d["v"].shape == (1, 1, 256, 16)
    assert d["skw"].shape == (1, 2, 16, 16) and d["skr"].shape == (1, 2, 16, 16)
    assert d["M0"].shape == (1, wl.N, 16)
    assert d["alpha"].shape == (1, 1, 256)


def test_deterministic_and_seed_sensitive():
    a = S.generate(S.TINY)
    b = S.generate(S.TINY)
    c = S.generate(S.TINY, seed=7)
    for k in a:
        assert torch.equal(a[k], b[k])
    assert not torch.equal(a["q"], c["q"])


def test_distributions_mid_scaled():
    wl = S.MID.scaled(T=512, B=1, H=2)
    d = S.generate(wl)
    assert d["q"].dtype == torch.bfloat16 and d["skw"].dtype == torch.bfloat16
    a = d["alpha"]
    assert a.min() >= 0.95 and a.max() < 1.0
    assert d["beta"].min() >= 0.0 and d["beta"].max() <= 1.0
    assert abs(d["skw"].float().std().item() - math.sqrt(1 / 64)) < 0.01
    assert abs(d["M0"].std().item() - 0.02) < 0.001
    assert not torch.equal(d["skw"], d["skr"])


def test_headline_gates_are_sigmoid_normal():
    wl = S.HEADLINE.scaled(T=256, B=1, H=2, n_sub=32)
    d = S.generate(wl, with_m0=False)
    logit = torch.logit(d["alpha"].double())
    assert abs(logit.mean().item() - 3.0) < 0.1
    assert abs(logit.var().item() - 0.5) < 0.1


def test_clustered_keys():
    wl = S.LONG.scaled(T=2048, H=2, n_sub=16, clusters=8)
    d = S.generate(wl, with_m0=False)
    k = d["k"].float().reshape(-1, wl.d_k)
    # with 8 centres and noise variance 0.1, nearest-other-row distances are small
    dists = torch.cdist(k[:64], k[64:1024]).min(dim=1).values
    assert dists.max() < 0.5 * math.sqrt(2 * wl.d_k)


def test_random_indices_distinct():
    g = torch.Generator()
    g.manual_seed(3)
    idx = S.random_indices(2, 3, 50, 100, 7, g, pool=12)
    assert idx.shape == (2, 3, 50, 7)
    s = idx.sort(dim=-1).values
    assert (s[..., 1:] != s[..., :-1]).all()
    assert idx.min() >= 0 and idx.max() < 100
    assert len(torch.unique(idx)) <= 12


def test_decode_layout():
    x = torch.arange(2 * 3 * 5 * 4).reshape(2, 3, 5, 4)
    y = S.decode_layout(x, 2)
    assert y.shape == (3, 2, 3, 4)
    assert torch.equal(y[1, 1, 2], x[1, 2, 3])
