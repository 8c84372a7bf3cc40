"""Double-precision CPU oracles: SPECTRE frequency-domain token mixing, and
per-token DCT mixing with spectral-entropy routing.

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the CPU-baseline
leg of ``bench.py`` are the only callers.  The CUDA library never imports,
links or calls anything here, and nothing here imports the CUDA library.

The arithmetic lives in ``spectre_oracle.c`` and ``dct_oracle.c`` (plain C,
fp64, OpenMP over channels or tokens).  This module only marshals arrays
through ctypes.

What the oracle computes follows the SPECTRE walk-through
(hotelren.com/news/5925787): §2.2 pseudocode (FFT of q, k, v along the
sequence, ``Q_f * conj(K_f)`` gated by ``G``, times ``V_f``, inverse FFT,
``layer_norm(out + x)``) and §2.3 (keep only the low-frequency bins f < F).
The DCT mix follows the Chiaroscuro Attention summary
(paper.rainbus.top/paper/2606.08327): the orthonormal Type-II DCT of each
token, its normalised spectral entropy H(x), the routing rule H(x) <= tau,
and DCTMix without its feed-forward layer, LayerNorm(x + iDCT(DCT(x) * w)).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = [os.path.join(_HERE, "spectre_oracle.c"), os.path.join(_HERE, "dct_oracle.c")]
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle's C sources into ``liboracle.so`` beside them."""
    newest = max(os.path.getmtime(s) for s in _SRCS)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", _LIB, *_SRCS, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        vp = ctypes.c_void_p
        lib.oracle_fft.argtypes = [ctypes.c_long, dp, dp, dp, dp, ctypes.c_int]
        lib.oracle_fft.restype = ctypes.c_int
        lib.oracle_spectre_out.argtypes = [
            ctypes.c_int, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            vp, vp, vp, vp, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, ctypes.c_int]
        lib.oracle_spectre_out.restype = ctypes.c_int
        lib.oracle_spectre_mix.argtypes = [
            ctypes.c_int, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_double, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_long, vp, vp, ctypes.c_int,
            ctypes.c_int, ctypes.c_int]
        lib.oracle_spectre_mix.restype = ctypes.c_int
        for name in ("oracle_dct2", "oracle_dct3"):
            getattr(lib, name).argtypes = [ctypes.c_long, ctypes.c_long, vp, vp]
            getattr(lib, name).restype = ctypes.c_int
        lib.oracle_dct_mix.argtypes = [
            ctypes.c_long, ctypes.c_long, ctypes.c_int, vp, vp, vp, vp, ctypes.c_double,
            ctypes.c_double, vp, vp, vp, vp, ctypes.c_int]
        lib.oracle_dct_mix.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _as_stored(t):
    """Return (numpy array of the stored bits, dtype code).

    fp32 tensors pass as float32; bf16 tensors pass as their raw 16-bit
    patterns, which the C side widens exactly to double.
    """
    import torch

    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy(), 1
        if t.dtype == torch.float32:
            return t.numpy(), 0
        raise TypeError(f"unsupported dtype {t.dtype}")
    a = np.ascontiguousarray(t)
    if a.dtype == np.float32:
        return a, 0
    raise TypeError(f"unsupported dtype {a.dtype}")


def _gate(G):
    """(float32 array, cgate): a real gate [H, L/2+1], or a complex one as
    [H, L/2+1, 2] (re, im) pairs with cgate = 1."""
    import torch

    if isinstance(G, torch.Tensor) and G.is_complex():
        return np.ascontiguousarray(torch.view_as_real(G.to(torch.complex64)).numpy()), 1
    if isinstance(G, np.ndarray) and np.iscomplexobj(G):
        a = np.stack([G.real, G.imag], axis=-1).astype(np.float32)
        return np.ascontiguousarray(a), 1
    return _f32(G), 0


def _f32(t) -> np.ndarray:
    import torch

    if isinstance(t, torch.Tensor):
        return t.detach().cpu().to(torch.float32).contiguous().numpy()
    return np.ascontiguousarray(t, dtype=np.float32)


def fft(x: np.ndarray, sign: int = -1) -> np.ndarray:
    """Complex DFT (unscaled) of a 1-D array with the oracle's own FFT."""
    x = np.asarray(x, dtype=np.complex128)
    n = x.shape[0]
    re = np.ascontiguousarray(x.real)
    im = np.ascontiguousarray(x.imag)
    ore = np.empty(n)
    oim = np.empty(n)
    dp = ctypes.POINTER(ctypes.c_double)
    rc = _load().oracle_fft(n, re.ctypes.data_as(dp), im.ctypes.data_as(dp),
                            ore.ctypes.data_as(dp), oim.ctypes.data_as(dp), int(sign))
    if rc != 0:
        raise RuntimeError("oracle_fft failed")
    return ore + 1j * oim


def spectre_out(q, k, v, G, H: int, F: int, c0: int = 0, c1: Optional[int] = None,
                nthreads: int = 0) -> np.ndarray:
    """Pre-LayerNorm output ``out[B, L, c0:c1]`` in float64."""
    qa, dt = _as_stored(q)
    ka, dk = _as_stored(k)
    va, dv = _as_stored(v)
    if not (dt == dk == dv):
        raise TypeError("q, k, v must share a dtype")
    B, L, C = qa.shape
    if C % H:
        raise ValueError("C must be a multiple of H")
    D = C // H
    c1 = C if c1 is None else c1
    Ga, cg = _gate(G)
    out = np.empty((B, L, c1 - c0), dtype=np.float64)
    rc = _load().oracle_spectre_out(B, L, H, D, F, dt, _ptr(qa), _ptr(ka), _ptr(va), _ptr(Ga),
                                    c0, c1, _ptr(out), nthreads, cg)
    if rc != 0:
        raise RuntimeError("oracle_spectre_out failed")
    return out


NORM_MODES = {"post_ln": 0, "pre_ln": 1, "post_rms": 2, "pre_rms": 3}


def spectre_mix(q, k, v, x, G, gamma, beta, H: int, F: int, eps: float = 1e-5,
                tokens: Optional[Sequence[int]] = None, nthreads: int = 0, norm: str = "post_ln"):
    """Return ``(out, y)`` in float64 at the selected tokens (all if None).

    Shapes: ``out`` and ``y`` are ``[B, ntok, C]``.  ``eps`` is taken as the
    fp32 value the library receives, widened to double.  ``norm``: "post_ln"
    y = LN(out + x) (walk-through §2.2), "pre_ln" y = LN(out) + x, "post_rms"
    y = RMS(out + x), "pre_rms" y = RMS(out) + x (the §3.3 variants), with
    RMS(z) = z / sqrt(mean(z^2) + eps) * gamma + beta.
    """
    qa, dt = _as_stored(q)
    ka, _ = _as_stored(k)
    va, _ = _as_stored(v)
    xa, dx = _as_stored(x)
    if dx != dt:
        raise TypeError("x must share q's dtype")
    B, L, C = qa.shape
    D = C // H
    Ga, cg = _gate(G)
    ga = _f32(gamma)
    ba = _f32(beta)
    if tokens is None:
        tok = None
        ntok = L
    else:
        tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64))
        ntok = tok.shape[0]
    out = np.empty((B, ntok, C), dtype=np.float64)
    y = np.empty((B, ntok, C), dtype=np.float64)
    eps64 = float(np.float32(eps))
    rc = _load().oracle_spectre_mix(B, L, H, D, F, dt, eps64, _ptr(qa), _ptr(ka), _ptr(va),
                                    _ptr(xa), _ptr(Ga), _ptr(ga), _ptr(ba),
                                    None if tok is None else _ptr(tok), ntok,
                                    _ptr(out), _ptr(y), nthreads, NORM_MODES[norm], cg)
    if rc != 0:
        raise RuntimeError("oracle_spectre_mix failed")
    return out, y


# ---------------------------------------------------------------------------
# per-token DCT mixing (Chiaroscuro Attention summary)
# ---------------------------------------------------------------------------
def _rows64(a) -> np.ndarray:
    import torch

    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def dct2(x) -> np.ndarray:
    """Orthonormal Type-II DCT along the last axis ("Prerequisites: DCT")."""
    a = _rows64(x)
    d = a.shape[-1]
    out = np.empty_like(a)
    if _load().oracle_dct2(a.size // d, d, _ptr(a), _ptr(out)) != 0:
        raise RuntimeError("oracle_dct2 failed")
    return out


def idct2(X) -> np.ndarray:
    """Inverse of ``dct2`` (the orthonormal Type-III DCT) along the last axis."""
    a = _rows64(X)
    d = a.shape[-1]
    out = np.empty_like(a)
    if _load().oracle_dct3(a.size // d, d, _ptr(a), _ptr(out)) != 0:
        raise RuntimeError("oracle_dct3 failed")
    return out


def dct_mix(x, w, gamma, beta, eps: float = 1e-5, tau: float = 0.8954, nthreads: int = 0):
    """The DCT mix of token rows ``x[..., d]`` (fp32 or bf16, widened exactly).

    Returns a dict of float64 ``mix`` (iDCT(DCT(x) * w), before the residual),
    ``y`` (LayerNorm_d(x + mix; gamma, beta, eps)), ``H`` (normalised spectral
    entropy per token) and uint8 ``route`` (1 where H <= tau).  ``eps`` and
    ``tau`` are taken as the fp32 values the library receives.
    """
    xa, dt = _as_stored(x)
    shape = xa.shape
    d = shape[-1]
    T = xa.size // d
    mix = np.empty(shape, dtype=np.float64)
    y = np.empty(shape, dtype=np.float64)
    H = np.empty(shape[:-1], dtype=np.float64)
    route = np.empty(shape[:-1], dtype=np.uint8)
    wa, ga, ba = _f32(w), _f32(gamma), _f32(beta)
    if wa.size != d or ga.size != d or ba.size != d:
        raise ValueError("w, gamma and beta must hold d values")
    rc = _load().oracle_dct_mix(T, d, dt, _ptr(xa), _ptr(wa), _ptr(ga), _ptr(ba),
                                float(np.float32(eps)), float(np.float32(tau)), _ptr(mix),
                                _ptr(y), _ptr(H), _ptr(route), nthreads)
    if rc != 0:
        raise RuntimeError("oracle_dct_mix failed")
    return {"mix": mix, "y": y, "H": H, "route": route}
