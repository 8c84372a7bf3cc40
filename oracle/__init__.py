"""Double-precision CPU oracle for SPECTRE frequency-domain token mixing.

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the CPU-baseline
leg of ``bench.py`` are the only callers.  The CUDA library never imports,
links or calls anything here, and nothing here imports the CUDA library.

The arithmetic lives in ``spectre_oracle.c`` (plain C, fp64, OpenMP over
channels).  This module only marshals arrays through ctypes.

What the oracle computes follows the SPECTRE walk-through
(hotelren.com/news/5925787): §2.2 pseudocode (FFT of q, k, v along the
sequence, ``Q_f * conj(K_f)`` gated by ``G``, times ``V_f``, inverse FFT,
``layer_norm(out + x)``) and §2.3 (keep only the low-frequency bins f < F).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spectre_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile ``spectre_oracle.c`` into ``liboracle.so`` beside it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", _LIB, _SRC, "-lm"]
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
