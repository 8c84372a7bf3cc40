"""Pins of the DCT-mix oracle to facts outside itself (Chiaroscuro Attention
summary, paper.rainbus.top/paper/2606.08327: "Prerequisites: DCT",
"Prerequisites: spectral entropy", "Method step details").

The transform is pinned to scipy's orthonormal DCT, Parseval and single-basis
inputs; the entropy to its closed forms (one coefficient: 0, flat spectrum: 1,
two equal coefficients: ln 2 / ln d) and to scale invariance; the mix to the
identity filter, the zero filter, a single-coefficient filter (a scaled cosine)
and a low-pass filter through scipy; y to torch's layer_norm.
"""
import math

import numpy as np
import pytest
import scipy.fft as sfft
import torch

import oracle

RNG = np.random.default_rng(20260601)


@pytest.mark.parametrize("d", [2, 7, 64, 256, 1024])
def test_dct2_is_scipys_orthonormal_type_ii(d):
    x = RNG.standard_normal((3, d))
    X = oracle.dct2(x)
    assert np.abs(X - sfft.dct(x, type=2, norm="ortho", axis=-1)).max() < 1e-11
    assert np.abs(oracle.idct2(X) - x).max() < 1e-11
    assert np.abs(oracle.idct2(x) - sfft.idct(x, type=2, norm="ortho", axis=-1)).max() < 1e-11


def test_parseval_and_single_basis_vector():
    d = 128
    x = RNG.standard_normal((4, d))
    X = oracle.dct2(x)
    assert np.allclose((X ** 2).sum(-1), (x ** 2).sum(-1), rtol=1e-12)
    n = np.arange(d)
    for k in (0, 1, 5, 127):
        basis = np.cos(np.pi * (2 * n + 1) * k / (2 * d))
        Xb = oracle.dct2(basis)
        others = np.delete(Xb, k)
        assert np.abs(others).max() < 1e-11 and abs(Xb[k]) > 1.0


def _mix(x, w=None, gamma=None, beta=None, eps=1e-5, tau=0.8954):
    x = torch.as_tensor(x, dtype=torch.float32)
    d = x.shape[-1]
    w = torch.ones(d) if w is None else torch.as_tensor(w, dtype=torch.float32)
    gamma = torch.ones(d) if gamma is None else torch.as_tensor(gamma, dtype=torch.float32)
    beta = torch.zeros(d) if beta is None else torch.as_tensor(beta, dtype=torch.float32)
    return oracle.dct_mix(x, w, gamma, beta, eps=eps, tau=tau)


def test_entropy_closed_forms():
    d = 256
    n = np.arange(d)
    rows = [
        np.full(d, 0.75),                                       # DC only: H = 0
        np.cos(np.pi * (2 * n + 1) * 9 / (2 * d)),              # one cosine: H = 0
        sfft.idct(np.ones(d), type=2, norm="ortho"),            # flat spectrum: H = 1
        sfft.idct(np.eye(d)[3] + np.eye(d)[40], type=2, norm="ortho"),   # two equal: ln2/ln d
        np.zeros(d),                                            # no energy: H = 0 (reading)
    ]
    r = _mix(np.stack(rows).astype(np.float32))
    # the rows pass through fp32, so the single-coefficient cases leak ~1e-7 of energy
    expect = [0.0, 0.0, 1.0, math.log(2) / math.log(d), 0.0]
    assert np.allclose(r["H"], expect, atol=5e-5), (r["H"], expect)
    assert r["H"][4] == 0.0


def test_entropy_brute_force_and_scale_invariance():
    d = 64
    x = RNG.standard_normal((6, d)).astype(np.float32)
    r = _mix(x)
    X = sfft.dct(x.astype(np.float64), type=2, norm="ortho", axis=-1)
    p = X ** 2 / (X ** 2).sum(-1, keepdims=True)
    h = -(p * np.log(p)).sum(-1) / math.log(d)
    assert np.abs(r["H"] - h).max() < 1e-12
    r2 = _mix(x * 8.0)      # a power-of-two scale is exact in fp32
    assert np.abs(r2["H"] - r["H"]).max() < 1e-12
    assert ((r["H"] >= 0) & (r["H"] <= 1)).all()


def test_route_is_h_at_most_tau_inclusive():
    d = 64
    x = np.stack([np.zeros(d), RNG.standard_normal(d)]).astype(np.float32)
    h = _mix(x)["H"]
    assert h[0] == 0.0
    assert list(_mix(x, tau=0.0)["route"]) == [1, 0]                 # H = 0 <= 0
    assert list(_mix(x, tau=-1e-3)["route"]) == [0, 0]
    assert list(_mix(x, tau=1.0)["route"]) == [1, 1]
    mid = float(np.float32(h[1]))
    assert _mix(x, tau=float(h[1]) + 1e-6)["route"][1] == 1
    assert _mix(x, tau=mid - 1e-4)["route"][1] == 0


def test_mix_identity_zero_and_single_coefficient_filters():
    d = 128
    x = RNG.standard_normal((5, d)).astype(np.float32)
    r = _mix(x)                                   # w = 1: iDCT(DCT(x)) = x
    assert np.abs(r["mix"] - x).max() < 1e-12
    r0 = _mix(x, w=np.zeros(d))
    assert np.abs(r0["mix"]).max() == 0.0
    j = 11
    wj = np.zeros(d, dtype=np.float32)
    wj[j] = 2.0
    rj = _mix(x, w=wj)
    n = np.arange(d)
    Xj = sfft.dct(x.astype(np.float64), type=2, norm="ortho", axis=-1)[:, j]
    expect = 2.0 * Xj[:, None] * math.sqrt(2.0 / d) * np.cos(np.pi * (2 * n + 1) * j / (2 * d))
    assert np.abs(rj["mix"] - expect).max() < 1e-12


def test_mix_low_pass_matches_scipy_and_y_matches_layer_norm():
    d = 256
    x = RNG.standard_normal((7, d)).astype(np.float32)
    w = np.where(np.arange(d) < 40, RNG.uniform(0, 1, d), 0.0).astype(np.float32)
    g = (1 + 0.1 * RNG.standard_normal(d)).astype(np.float32)
    b = (0.1 * RNG.standard_normal(d)).astype(np.float32)
    r = _mix(x, w=w, gamma=g, beta=b, eps=1e-5)
    X = sfft.dct(x.astype(np.float64), type=2, norm="ortho", axis=-1)
    m = sfft.idct(X * w.astype(np.float64), type=2, norm="ortho", axis=-1)
    assert np.abs(r["mix"] - m).max() < 1e-12
    z = torch.from_numpy(x.astype(np.float64) + m)
    y = torch.nn.functional.layer_norm(z, (d,), torch.from_numpy(g.astype(np.float64)),
                                       torch.from_numpy(b.astype(np.float64)),
                                       eps=float(np.float32(1e-5)))
    assert np.abs(r["y"] - y.numpy()).max() < 1e-10


def test_bf16_rows_are_widened_exactly():
    d = 64
    xb = torch.randn(3, d, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    rb = _mix(xb.float())
    w = torch.ones(d)
    r16 = oracle.dct_mix(xb, w, torch.ones(d), torch.zeros(d))
    for k in ("mix", "y", "H"):
        assert np.array_equal(r16[k], rb[k])
