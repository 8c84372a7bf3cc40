"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something other than its own formula:
a brute-force DFT, an independent FFT library (numpy), Parseval's theorem,
the O(L^2) time-domain form given by the convolution theorem, closed forms
(constant and single-tone inputs) and invariants of the method.  Sources:
SPECTRE walk-through (hotelren.com/news/5925787) §2.1 (convolution theorem),
§2.2 (pseudocode; "global circular-convolution-type attention"), §2.3
(frequency truncation).
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _brute_dft(x, sign=-1):
    n = x.shape[0]
    idx = np.arange(n)
    e = (np.outer(idx, idx) % n).astype(np.float64)
    W = np.exp(sign * 2j * np.pi * e / n)
    return W @ x


# ----------------------------------------------------------------------------
# the FFT itself
# ----------------------------------------------------------------------------
BRUTE_N = [1, 2, 3, 4, 5, 6, 7, 8, 12, 16, 24, 32, 48, 64, 96, 128, 192, 256, 384,
           512, 768, 1024, 1536, 2048, 3072, 4096]


@pytest.mark.parametrize("n", BRUTE_N)
@pytest.mark.parametrize("sign", [-1, 1])
def test_fft_matches_brute_force_dft(n, sign):
    r = _rng(n)
    x = r.standard_normal(n) + 1j * r.standard_normal(n)
    got = oracle.fft(x, sign)
    ref = _brute_dft(x, sign)
    err = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    assert err < 1e-12, err


@pytest.mark.parametrize("n", [256, 4096, 12288, 65536, 3 * 2 ** 15, 1048576])
def test_fft_matches_numpy(n):
    r = _rng(7 + n)
    x = r.standard_normal(n) + 1j * r.standard_normal(n)
    got = oracle.fft(x, -1)
    ref = np.fft.fft(x)
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err < 1e-12, err


@pytest.mark.parametrize("n", [8, 12, 256, 4096, 12288])
def test_parseval_on_real_input(n):
    r = _rng(100 + n)
    x = r.standard_normal(n)
    X = oracle.fft(x, -1)[: n // 2 + 1]
    e_time = np.sum(x * x)
    e_freq = (abs(X[0]) ** 2 + 2 * np.sum(abs(X[1:n // 2]) ** 2) + abs(X[n // 2]) ** 2) / n
    assert abs(e_time - e_freq) / e_time < 1e-12


# ----------------------------------------------------------------------------
# the mixer against its time-domain form
# ----------------------------------------------------------------------------
def _time_domain_out(q, k, v, gprime):
    """out = r (*) g' (*) v with r[tau] = sum_u q[u+tau] k[u]; all circular.

    q, k, v: [L] float64; gprime: [L] time-domain gate kernel (or None for
    the identity).  Direct O(L^2) sums."""
    L = q.shape[0]
    r = np.array([np.dot(np.roll(q, -tau), k) for tau in range(L)])
    if gprime is not None:
        r = np.array([np.dot(r, np.roll(gprime[::-1], t + 1)) for t in range(L)])
    return np.array([np.dot(r, np.roll(v[::-1], t + 1)) for t in range(L)])


def _gate_kernel(Grow, F, L):
    """g'[n] = (1/L) sum_f G'_f e^{2 pi i f n / L} for the Hermitian,
    truncated gate, written as a direct cosine sum."""
    n = np.arange(L)
    g = np.zeros(L)
    for f in range(L // 2 + 1):
        if f >= F:
            continue
        w = 1.0 if (f == 0 or (L % 2 == 0 and f == L // 2)) else 2.0
        g += w * Grow[f] * np.cos(2 * np.pi * f * n / L)
    return g / L


def _mk(B, L, C, seed, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    t = [torch.randn(B, L, C, generator=g).to(dtype) for _ in range(4)]
    return t


@pytest.mark.parametrize("L", [8, 12, 16, 24, 48, 64, 96, 128, 192, 256, 384, 512, 768, 1024])
def test_mixer_matches_time_domain_identity_gate(L):
    B, H, D = 2, 1, 3
    C = H * D
    q, k, v, _ = _mk(B, L, C, seed=L)
    G = torch.ones(H, L // 2 + 1)
    out = oracle.spectre_out(q, k, v, G, H=H, F=L // 2 + 1)
    for b in range(B):
        for c in range(C):
            ref = _time_domain_out(q[b, :, c].double().numpy(), k[b, :, c].double().numpy(),
                                   v[b, :, c].double().numpy(), None)
            err = np.max(np.abs(out[b, :, c] - ref)) / np.max(np.abs(ref))
            assert err < 1e-12, (b, c, err)


@pytest.mark.parametrize("L,F", [(16, 3), (24, 13), (64, 33), (96, 20), (256, 129), (256, 37),
                                 (384, 1), (512, 100)])
def test_mixer_matches_time_domain_general_gate(L, F):
    B, H, D = 1, 3, 2
    C = H * D
    q, k, v, _ = _mk(B, L, C, seed=1000 + L + F)
    G = torch.rand(H, L // 2 + 1, generator=torch.Generator().manual_seed(F))
    out = oracle.spectre_out(q, k, v, G, H=H, F=F)
    for c in range(C):
        h = c // D
        gk = _gate_kernel(G[h].double().numpy(), F, L)
        ref = _time_domain_out(q[0, :, c].double().numpy(), k[0, :, c].double().numpy(),
                               v[0, :, c].double().numpy(), gk)
        err = np.max(np.abs(out[0, :, c] - ref)) / max(np.max(np.abs(ref)), 1e-300)
        assert err < 1e-11, (c, err)


def _complex_gate_kernel(Grow, F, L):
    """g'[n] = (1/L) sum_f G'_f e^{2 pi i f n / L} for a complex gate given on
    f <= L/2 (truncated at F), extended Hermitian-symmetrically
    (G'_{L-f} = conj G'_f) with the imaginary parts at DC and Nyquist
    dropped: a direct sum of cosines and sines."""
    n = np.arange(L)
    g = np.zeros(L)
    for f in range(L // 2 + 1):
        if f >= F:
            continue
        edge = f == 0 or (L % 2 == 0 and f == L // 2)
        ph = 2 * np.pi * f * n / L
        if edge:
            g += Grow[f].real * np.cos(ph)
        else:
            g += 2.0 * (Grow[f].real * np.cos(ph) - Grow[f].imag * np.sin(ph))
    return g / L


@pytest.mark.parametrize("L,F", [(16, 9), (48, 11), (64, 33), (96, 20)])
def test_complex_gate_matches_time_domain(L, F):
    """A complex (phase-carrying) gate against the O(L^2) time-domain form."""
    B, H, D = 1, 2, 2
    C = H * D
    q, k, v, _ = _mk(B, L, C, seed=2000 + L + F)
    g = torch.Generator().manual_seed(L + F)
    G = torch.complex(torch.rand(H, L // 2 + 1, generator=g), torch.randn(H, L // 2 + 1, generator=g))
    out = oracle.spectre_out(q, k, v, G, H=H, F=F)
    for c in range(C):
        gk = _complex_gate_kernel(G[c // D].to(torch.complex128).numpy(), F, L)
        ref = _time_domain_out(q[0, :, c].double().numpy(), k[0, :, c].double().numpy(),
                               v[0, :, c].double().numpy(), gk)
        err = np.max(np.abs(out[0, :, c] - ref)) / max(np.max(np.abs(ref)), 1e-300)
        assert err < 1e-11, (c, err)


def test_complex_gate_with_zero_phase_equals_real_gate():
    B, L, H, D = 2, 64, 2, 3
    C = H * D
    q, k, v, _ = _mk(B, L, C, seed=31)
    G = torch.rand(H, L // 2 + 1, generator=torch.Generator().manual_seed(2))
    out_r = oracle.spectre_out(q, k, v, G, H=H, F=20)
    out_c = oracle.spectre_out(q, k, v, torch.complex(G, torch.zeros_like(G)), H=H, F=20)
    assert np.array_equal(out_r, out_c)


@pytest.mark.parametrize("s", [1, 5, 17])
def test_complex_gate_pure_delay_shifts_the_output(s):
    """G_f = e^{-2 pi i f s / L}, no truncation: the gate kernel is a delta at
    s, so the output is the identity-gate output delayed by s tokens."""
    B, L, H, D = 1, 64, 1, 3
    C = H * D
    q, k, v, _ = _mk(B, L, C, seed=40 + s)
    f = np.arange(L // 2 + 1)
    ph = torch.from_numpy(np.exp(-2j * np.pi * f * s / L)).to(torch.complex64)[None, :]
    out_1 = oracle.spectre_out(q, k, v, torch.ones(H, L // 2 + 1), H=H, F=L // 2 + 1)
    out_s = oracle.spectre_out(q, k, v, ph, H=H, F=L // 2 + 1)
    ref = np.roll(out_1, s, axis=1)
    assert np.max(np.abs(out_s - ref)) < 1e-4 * np.max(np.abs(ref))


def test_zero_gate_gives_layernorm_of_x():
    B, L, H, D = 2, 64, 2, 8
    C = H * D
    q, k, v, x = _mk(B, L, C, seed=5)
    G = torch.zeros(H, L // 2 + 1)
    gamma = torch.randn(C, generator=torch.Generator().manual_seed(1))
    beta = torch.randn(C, generator=torch.Generator().manual_seed(2))
    out, y = oracle.spectre_mix(q, k, v, x, G, gamma, beta, H=H, F=L // 2 + 1)
    assert np.all(out == 0.0)
    ref = torch.nn.functional.layer_norm(x.double(), (C,), gamma.double(), beta.double(),
                                         eps=float(np.float32(1e-5))).numpy()
    assert np.max(np.abs(y - ref)) < 1e-12


@pytest.mark.parametrize("L", [16, 48, 256])
def test_delta_q_gives_convolution_of_reversed_k_with_v(L):
    B, H, D = 1, 1, 2
    C = H * D
    _, k, v, _ = _mk(B, L, C, seed=L + 3)
    q = torch.zeros(B, L, C)
    q[:, 0, :] = 1.0
    G = torch.ones(H, L // 2 + 1)
    out = oracle.spectre_out(q, k, v, G, H=H, F=L // 2 + 1)
    for c in range(C):
        kk = k[0, :, c].double().numpy()
        vv = v[0, :, c].double().numpy()
        krev = np.array([kk[(-t) % L] for t in range(L)])
        ref = np.array([sum(krev[s] * vv[(t - s) % L] for s in range(L)) for t in range(L)])
        assert np.max(np.abs(out[0, :, c] - ref)) < 1e-11 * max(1.0, np.max(np.abs(ref)))


def test_constant_inputs_closed_form():
    B, L, H, D = 1, 96, 2, 2
    C = H * D
    q = torch.ones(B, L, C)
    G = torch.rand(H, L // 2 + 1, generator=torch.Generator().manual_seed(9))
    out = oracle.spectre_out(q, q, q, G, H=H, F=5)
    for c in range(C):
        expect = L * L * float(G[c // D, 0])
        assert np.max(np.abs(out[0, :, c] - expect)) < 1e-9 * expect


@pytest.mark.parametrize("L,F", [(64, 9), (96, 17), (256, 33)])
def test_single_tone_closed_form_and_truncation_edge(L, F):
    """q = k = v = cos(2 pi a t / L): out = (L^2/4) G[a] cos(2 pi a t / L) when
    a < F, else 0.  Checked at a = F-1 and a = F (the truncation edge)."""
    H, D = 1, 1
    G = torch.rand(H, L // 2 + 1, generator=torch.Generator().manual_seed(L))
    t = np.arange(L)
    for a in (1, F - 1, F, L // 2 - 1):
        col = np.cos(2 * np.pi * a * t / L)
        q = torch.from_numpy(col.astype(np.float32)).reshape(1, L, 1)
        out = oracle.spectre_out(q, q, q, G, H=H, F=F)[0, :, 0]
        # the oracle reads the fp32-rounded tone, so compare with the tone the
        # oracle actually received: scale is exact up to that rounding
        col32 = q[0, :, 0].double().numpy()
        if a < F:
            expect = (L * L / 4) * float(G[0, a]) * col32
            assert np.max(np.abs(out - expect)) < 1e-5 * (L * L / 4)
        else:
            assert np.max(np.abs(out)) < 1e-5 * (L * L / 4)


def test_shift_equivariance_and_trilinearity():
    B, L, H, D = 1, 48, 1, 3
    C = H * D
    q, k, v, _ = _mk(B, L, C, seed=77)
    G = torch.rand(H, L // 2 + 1, generator=torch.Generator().manual_seed(3))
    F = 17
    base = oracle.spectre_out(q, k, v, G, H=H, F=F)
    s = 11
    same = oracle.spectre_out(torch.roll(q, s, 1), torch.roll(k, s, 1), v, G, H=H, F=F)
    assert np.max(np.abs(same - base)) < 1e-12 * np.max(np.abs(base))
    shifted = oracle.spectre_out(q, k, torch.roll(v, s, 1), G, H=H, F=F)
    assert np.max(np.abs(shifted - np.roll(base, s, axis=1))) < 1e-12 * np.max(np.abs(base))
    scaled = oracle.spectre_out(q * 2.0, k, v, G, H=H, F=F)
    assert np.max(np.abs(scaled - 2.0 * base)) < 1e-12 * np.max(np.abs(base))


@pytest.mark.parametrize("norm", ["pre_ln", "post_rms", "pre_rms"])
def test_norm_variants_match_torch_on_oracle_out(norm):
    """The norm-order and RMSNorm variants (walk-through §3.3) against torch's
    layer_norm / rms_norm applied to the oracle's own pre-norm output; out
    itself does not depend on the variant."""
    B, L, H, D = 2, 32, 2, 5
    C = H * D
    q, k, v, x = _mk(B, L, C, seed=13)
    G = torch.rand(H, L // 2 + 1, generator=torch.Generator().manual_seed(7))
    gamma = torch.randn(C, generator=torch.Generator().manual_seed(8))
    beta = torch.randn(C, generator=torch.Generator().manual_seed(9))
    out0, _ = oracle.spectre_mix(q, k, v, x, G, gamma, beta, H=H, F=11)
    out, y = oracle.spectre_mix(q, k, v, x, G, gamma, beta, H=H, F=11, norm=norm)
    assert np.array_equal(out, out0)
    eps = float(np.float32(1e-5))
    o = torch.from_numpy(out)
    xd, g, bt = x.double(), gamma.double(), beta.double()
    F_ = torch.nn.functional
    if norm == "pre_ln":
        ref = F_.layer_norm(o, (C,), g, bt, eps=eps) + xd
    elif norm == "post_rms":
        ref = F_.rms_norm(o + xd, (C,), g, eps=eps) + bt
    else:
        ref = F_.rms_norm(o, (C,), g, eps=eps) + bt + xd
    assert np.max(np.abs(y - ref.numpy())) < 1e-12


def test_rmsnorm_equals_layernorm_on_zero_mean_tokens():
    """With x chosen so that every token's z = out + x has zero channel mean,
    RMS(z) and LN(z) coincide: pins the one step in which they differ."""
    B, L, H, D = 1, 64, 2, 4
    C = H * D
    q, k, v, x = _mk(B, L, C, seed=21)
    q, k, v, x = q.double(), k.double(), v.double(), x.double()
    G = torch.rand(H, L // 2 + 1, generator=torch.Generator().manual_seed(3), dtype=torch.float64)
    gamma = torch.randn(C, generator=torch.Generator().manual_seed(4))
    beta = torch.randn(C, generator=torch.Generator().manual_seed(5))
    out, _ = oracle.spectre_mix(q.float(), k.float(), v.float(), x.float(), G.float(), gamma, beta,
                                H=H, F=L // 2 + 1)
    z = torch.from_numpy(out) + x
    x0 = (x - z.mean(dim=-1, keepdim=True)).float()     # z + (x0 - x) has mean ~ 0
    _, y_ln = oracle.spectre_mix(q.float(), k.float(), v.float(), x0, G.float(), gamma, beta,
                                 H=H, F=L // 2 + 1, norm="post_ln")
    _, y_rms = oracle.spectre_mix(q.float(), k.float(), v.float(), x0, G.float(), gamma, beta,
                                  H=H, F=L // 2 + 1, norm="post_rms")
    assert np.max(np.abs(y_ln - y_rms)) < 1e-5


def test_layernorm_matches_torch_on_oracle_z():
    B, L, H, D = 2, 32, 2, 5
    C = H * D
    q, k, v, x = _mk(B, L, C, seed=12)
    G = torch.rand(H, L // 2 + 1, generator=torch.Generator().manual_seed(4))
    gamma = torch.randn(C, generator=torch.Generator().manual_seed(5))
    beta = torch.randn(C, generator=torch.Generator().manual_seed(6))
    out, y = oracle.spectre_mix(q, k, v, x, G, gamma, beta, H=H, F=11)
    z = torch.from_numpy(out) + x.double()
    ref = torch.nn.functional.layer_norm(z, (C,), gamma.double(), beta.double(),
                                         eps=float(np.float32(1e-5))).numpy()
    assert np.max(np.abs(y - ref)) < 1e-12


def test_token_selection_matches_full_output():
    B, L, H, D = 2, 64, 2, 4
    C = H * D
    q, k, v, x = _mk(B, L, C, seed=21)
    G = torch.rand(H, L // 2 + 1, generator=torch.Generator().manual_seed(8))
    gamma = torch.ones(C)
    beta = torch.zeros(C)
    out_all, y_all = oracle.spectre_mix(q, k, v, x, G, gamma, beta, H=H, F=20)
    toks = [0, 5, 63, 17]
    out_s, y_s = oracle.spectre_mix(q, k, v, x, G, gamma, beta, H=H, F=20, tokens=toks)
    assert np.array_equal(out_s, out_all[:, toks, :])
    assert np.array_equal(y_s, y_all[:, toks, :])
    full = oracle.spectre_out(q, k, v, G, H=H, F=20)
    assert np.allclose(full, out_all, rtol=0, atol=1e-13 * np.max(np.abs(full)))
    part = oracle.spectre_out(q, k, v, G, H=H, F=20, c0=3, c1=6)
    assert np.array_equal(part, full[:, :, 3:6])


def test_bf16_inputs_are_widened_exactly():
    B, L, H, D = 1, 96, 2, 3
    C = H * D
    q, k, v, x = _mk(B, L, C, seed=31, dtype=torch.bfloat16)
    G = torch.rand(H, L // 2 + 1, generator=torch.Generator().manual_seed(2))
    gamma, beta = torch.ones(C), torch.zeros(C)
    o16, y16 = oracle.spectre_mix(q, k, v, x, G, gamma, beta, H=H, F=30)
    o32, y32 = oracle.spectre_mix(q.float(), k.float(), v.float(), x.float(), G, gamma, beta,
                                  H=H, F=30)
    assert np.array_equal(o16, o32) and np.array_equal(y16, y32)


def test_rejects_bad_arguments():
    q = torch.zeros(1, 16, 2)
    G = torch.ones(1, 9)
    with pytest.raises(RuntimeError):
        oracle.spectre_out(q, q, q, G, H=1, F=10)   # F > L/2 + 1
    with pytest.raises(RuntimeError):
        oracle.spectre_out(q, q, q, G, H=1, F=0)
