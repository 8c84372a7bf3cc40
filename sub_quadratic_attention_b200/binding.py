"""ctypes binding of libspectre_mix (C ABI in include/spectre_mix.h and
include/dct_mix.h).

Argument marshalling only: every step of the mix runs in the library's CUDA
kernels.  The functions carry the C names; :class:`SpectreMix` and
:class:`DctMix` wrap a handle for use with torch tensors.  Importing this module loads the library and
raises if it has not been built -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspectre_mix.so")

SPECTRE_F32 = 0
SPECTRE_BF16 = 1

SPECTRE_OK = 0
SPECTRE_ERR_ARG = -1
SPECTRE_ERR_UNSUPPORTED_L = -2
SPECTRE_ERR_ALIGN = -3
SPECTRE_ERR_CUDA = -4
SPECTRE_ERR_NOMEM = -5
SPECTRE_ERR_DEVICE = -6
SPECTRE_ERR_SCRATCH = -7
SPECTRE_ERR_TIMEOUT = -8

SPECTRE_OPT_TENSOR_CORES = 1
SPECTRE_OPT_NORM = 2
SPECTRE_OPT_COMPLEX_GATE = 3
SPECTRE_OPT_TEST_WAIT_TIMEOUT = 4
SPECTRE_OPT_ROW_TENSOR_CORES = 5
SPECTRE_OPT_GRAPH = 6

# enum spectre_norm, keyed as in the oracle
SPECTRE_NORM = {"post_ln": 0, "pre_ln": 1, "post_rms": 2, "pre_rms": 3}

SPECTRE_SLICE_CUDA_CORES = 0
SPECTRE_SLICE_TENSOR_CORES = 1

# fixed device scratch behind spectre_mix_run_noalloc (SPECTRE_NOALLOC_SCRATCH_BYTES)
SPECTRE_NOALLOC_SCRATCH_BYTES = 64 << 20

# every entry point the header declares, with its ctypes signature
_vp = ctypes.c_void_p
_i = ctypes.c_int
SIGNATURES = {
    "spectre_mix_create": (_i, [ctypes.POINTER(_vp), _i, _i, _i, _i, _i, _i, ctypes.c_float]),
    "spectre_mix_run": (_i, [_vp] * 10),
    "spectre_mix_run_debug": (_i, [_vp] * 11),
    "spectre_mix_run_host": (_i, [_vp] * 10),
    "spectre_mix_run_profiled": (_i, [_vp] * 10 + [_i, _vp]),
    "spectre_mix_run_noalloc": (_i, [_i] * 6 + [ctypes.c_float] + [_vp] * 9),
    "spectre_mix_destroy": (_i, [_vp]),
    "spectre_mix_device_status": (_i, [_vp, _vp]),
    "spectre_mix_set_option": (_i, [_vp, _i, _i]),
    "spectre_mix_slice_pass": (_i, [_vp]),
    "spectre_mix_error_string": (ctypes.c_char_p, [_i]),
    "spectre_mix_workspace_bytes": (ctypes.c_size_t, [_vp]),
    "spectre_mix_plan_info": (_i, [_vp] + [ctypes.POINTER(_i)] * 5),
    "dct_mix_create": (_i, [ctypes.POINTER(_vp), _i, _i, ctypes.c_float]),
    "dct_mix_run": (_i, [_vp, ctypes.c_longlong] + [_vp] * 4 + [ctypes.c_float] + [_vp] * 4),
    "dct_mix_run_debug": (_i, [_vp, ctypes.c_longlong] + [_vp] * 4 + [ctypes.c_float] + [_vp] * 5),
    "dct_mix_run_host": (_i, [_vp, ctypes.c_longlong] + [_vp] * 4 + [ctypes.c_float] + [_vp] * 4),
    "dct_mix_destroy": (_i, [_vp]),
}


class SpectreMixError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {spectre_mix_error_string(code)} (status {code})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libspectre_mix.so not found at {LIB_PATH}; build it with "
            "`python -m sub_quadratic_attention_b200.build_lib` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _ptr(t) -> Optional[int]:
    """Device or host address of a tensor, an int address, or None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to libspectre_mix must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(code: int, where: str) -> None:
    if code != SPECTRE_OK:
        raise SpectreMixError(code, where)


def spectre_mix_error_string(code: int) -> str:
    return _lib.spectre_mix_error_string(int(code)).decode()


def spectre_mix_create(B: int, L: int, H: int, D: int, F: int, dtype: int, eps: float = 1e-5) -> int:
    h = _vp()
    _check(_lib.spectre_mix_create(ctypes.byref(h), B, L, H, D, F, dtype, eps), "spectre_mix_create")
    return h.value


def spectre_mix_create_status(B: int, L: int, H: int, D: int, F: int, dtype: int,
                              eps: float = 1e-5) -> Tuple[int, Optional[int]]:
    """Raw status and handle (for tests of the error paths)."""
    h = _vp()
    code = _lib.spectre_mix_create(ctypes.byref(h), B, L, H, D, F, dtype, eps)
    return code, h.value


def spectre_mix_run(h: int, q, k, v, x, G, gamma, beta, y, stream=None) -> None:
    _check(_lib.spectre_mix_run(h, _ptr(q), _ptr(k), _ptr(v), _ptr(x), _ptr(G), _ptr(gamma),
                                _ptr(beta), _ptr(y), _stream(stream)), "spectre_mix_run")


def spectre_mix_run_status(h: int, q, k, v, x, G, gamma, beta, y, stream=None) -> int:
    return _lib.spectre_mix_run(h, _ptr(q), _ptr(k), _ptr(v), _ptr(x), _ptr(G), _ptr(gamma),
                                _ptr(beta), _ptr(y), _stream(stream))


def spectre_mix_run_debug(h: int, q, k, v, x, G, gamma, beta, y, out_f32, stream=None) -> None:
    _check(_lib.spectre_mix_run_debug(h, _ptr(q), _ptr(k), _ptr(v), _ptr(x), _ptr(G), _ptr(gamma),
                                      _ptr(beta), _ptr(y), _ptr(out_f32), _stream(stream)),
           "spectre_mix_run_debug")


def spectre_mix_run_host(h: int, q, k, v, x, G, gamma, beta, y, stream=None) -> None:
    _check(_lib.spectre_mix_run_host(h, _ptr(q), _ptr(k), _ptr(v), _ptr(x), _ptr(G), _ptr(gamma),
                                     _ptr(beta), _ptr(y), _stream(stream)), "spectre_mix_run_host")


def spectre_mix_run_profiled(h: int, q, k, v, x, G, gamma, beta, y, events, stream=None) -> None:
    """``events``: launches + 1 ``torch.cuda.Event(enable_timing=True)`` (already
    created), recorded before every kernel launch and after the last."""
    arr = (_vp * len(events))(*[e.cuda_event for e in events])
    _check(_lib.spectre_mix_run_profiled(h, _ptr(q), _ptr(k), _ptr(v), _ptr(x), _ptr(G),
                                         _ptr(gamma), _ptr(beta), _ptr(y),
                                         ctypes.cast(arr, _vp), len(events), _stream(stream)),
           "spectre_mix_run_profiled")


def spectre_mix_run_noalloc_status(B: int, L: int, H: int, D: int, F: int, dtype: int, eps: float,
                                   q, k, v, x, G, gamma, beta, y, stream=None) -> int:
    """One mix with no device allocation (the library's fixed 64 MiB scratch);
    for callers that may not call cudaMalloc.  Returns the raw status."""
    return _lib.spectre_mix_run_noalloc(B, L, H, D, F, dtype, eps, _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(x), _ptr(G), _ptr(gamma), _ptr(beta), _ptr(y),
                                        _stream(stream))


def spectre_mix_run_noalloc(B: int, L: int, H: int, D: int, F: int, dtype: int, eps: float,
                            q, k, v, x, G, gamma, beta, y, stream=None) -> None:
    _check(spectre_mix_run_noalloc_status(B, L, H, D, F, dtype, eps, q, k, v, x, G, gamma, beta,
                                          y, stream), "spectre_mix_run_noalloc")


def spectre_mix_set_option(h: int, option: int, value: int) -> None:
    _check(_lib.spectre_mix_set_option(h, option, value), "spectre_mix_set_option")


def spectre_mix_slice_pass(h: int) -> int:
    """SPECTRE_SLICE_TENSOR_CORES or SPECTRE_SLICE_CUDA_CORES for the plan's runs."""
    st = _lib.spectre_mix_slice_pass(h)
    if st < 0:
        _check(st, "spectre_mix_slice_pass")
    return st


def spectre_mix_device_status(h: int, stream=None) -> int:
    """Synchronise and return SPECTRE_OK or SPECTRE_ERR_TIMEOUT for earlier runs."""
    return _lib.spectre_mix_device_status(h, _stream(stream))


def spectre_mix_destroy(h: Optional[int]) -> None:
    _check(_lib.spectre_mix_destroy(h), "spectre_mix_destroy")


def spectre_mix_workspace_bytes(h: Optional[int]) -> int:
    return int(_lib.spectre_mix_workspace_bytes(h))


def spectre_mix_plan_info(h: int) -> Tuple[int, int, int, int, int]:
    """(R, M, slices per channel, channels per wave, kernel launches per run)."""
    vals = [_i() for _ in range(5)]
    _check(_lib.spectre_mix_plan_info(h, *[ctypes.byref(v) for v in vals]), "spectre_mix_plan_info")
    return tuple(v.value for v in vals)


def check_arguments(B, L, H, C, plan_L, dtype_code, q, k, v, x, G, gamma, beta, y, out=None):
    """Sizes and element types of one run's tensors, checked on the host: the
    library reads raw pointers, so a short buffer would be read out of bounds.
    q, k, v, x, y hold B * L * C values of the plan's type (bf16 or fp32); G
    holds H * (plan_L / 2 + 1) fp32 values (complex64 for a complex gate);
    gamma, beta hold C fp32 values; out (optional) B * L * C fp32 values."""
    import torch

    n = B * L * C
    tok_type = torch.float32 if dtype_code == SPECTRE_F32 else torch.bfloat16
    for name, t in (("q", q), ("k", k), ("v", v), ("x", x), ("y", y)):
        if t.numel() != n or t.dtype != tok_type:
            raise ValueError(f"{name} must hold B * L * C = {n} values of {tok_type}")
    if out is not None and (out.numel() != n or out.dtype != torch.float32):
        raise ValueError(f"out must hold B * L * C = {n} fp32 values")
    nb = plan_L // 2 + 1
    if G.numel() != H * nb or G.dtype not in (torch.float32, torch.complex64, torch.complex128):
        raise ValueError(f"G must be [H, {nb}], fp32 (or complex for a complex gate)")
    for name, t in (("gamma", gamma), ("beta", beta)):
        if t.numel() != C or t.dtype != torch.float32:
            raise ValueError(f"{name} must hold C = {C} fp32 values")


class SpectreMix:
    """A plan for one shape, usable with torch CUDA tensors.

    ``mix(q, k, v, x, G, gamma, beta)`` returns y; pass ``out=`` (fp32
    [B, L, C]) to also receive the pre-LayerNorm mixer output.

    ``block_len``: blockwise mode (walk-through §3.2, ``fft_len``): the mix runs
    within each block of block_len consecutive tokens, as B * L / block_len
    independent sequences of length block_len.  A [B, L, C] tensor is already
    laid out as [B * L / block_len, block_len, C], so only the plan's shape
    changes; G is then [H, block_len / 2 + 1] and F counts the block's bins.
    (The pages leave the exchange between blocks unspecified; none is done.)
    """

    def __init__(self, B: int, L: int, H: int, D: int, F: Optional[int] = None,
                 dtype: str = "bf16", eps: float = 1e-5, tensor_cores: Optional[bool] = None,
                 norm: Optional[str] = None, complex_gate: bool = False,
                 block_len: Optional[int] = None, row_tensor_cores: bool = False,
                 graph: Optional[bool] = None):
        self.B, self.L, self.H, self.D = B, L, H, D
        self.C = H * D
        if block_len is not None and (block_len < 1 or L % block_len):
            raise ValueError("block_len must divide L")
        self.block_len = block_len
        self.plan_B, self.plan_L = (B * (L // block_len), block_len) if block_len else (B, L)
        self.F = self.plan_L // 2 + 1 if F is None else F
        self.dtype_code = SPECTRE_F32 if dtype in ("f32", "float32", "fp32") else SPECTRE_BF16
        self.eps = eps
        self.handle = spectre_mix_create(self.plan_B, self.plan_L, H, D, self.F, self.dtype_code, eps)
        if tensor_cores is not None:   # None keeps the library's default (on)
            spectre_mix_set_option(self.handle, SPECTRE_OPT_TENSOR_CORES, 1 if tensor_cores else 0)
        if norm is not None:           # None keeps the default, "post_ln": LayerNorm(out + x)
            spectre_mix_set_option(self.handle, SPECTRE_OPT_NORM, SPECTRE_NORM[norm])
        self.complex_gate = complex_gate
        if complex_gate:               # G: complex [H, L/2+1] (a relative-position phase)
            spectre_mix_set_option(self.handle, SPECTRE_OPT_COMPLEX_GATE, 1)
        if row_tensor_cores:           # the row pass on the tensor cores (where it applies)
            spectre_mix_set_option(self.handle, SPECTRE_OPT_ROW_TENSOR_CORES, 1)
        if graph is not None:          # None keeps the library's default
            spectre_mix_set_option(self.handle, SPECTRE_OPT_GRAPH, 1 if graph else 0)
        self._gate_ref = None

    def _check_shapes(self, q, k, v, x, G, gamma, beta, y, out):
        check_arguments(self.B, self.L, self.H, self.C, self.plan_L, self.dtype_code,
                        q, k, v, x, G, gamma, beta, y, out)

    def _gate(self, G):
        """G as the library reads it: a real gate as given, a complex one as its
        (re, im) fp32 pairs.  The converted tensor stays referenced until the
        next call, since runs are asynchronous."""
        if G.is_complex():
            if not self.complex_gate:
                raise ValueError("a complex G needs a plan made with complex_gate=True")
            import torch

            G = torch.view_as_real(G.to(torch.complex64)).contiguous()
        elif self.complex_gate:
            raise ValueError("this plan expects a complex G")
        self._gate_ref = G
        return G

    def __call__(self, q, k, v, x, G, gamma, beta, y=None, out=None, stream=None):
        import torch

        if y is None:
            y = torch.empty_like(x)
        self._check_shapes(q, k, v, x, G, gamma, beta, y, out)
        G = self._gate(G)
        if out is None:
            spectre_mix_run(self.handle, q, k, v, x, G, gamma, beta, y, stream)
        else:
            spectre_mix_run_debug(self.handle, q, k, v, x, G, gamma, beta, y, out, stream)
        return y

    def run_host(self, q, k, v, x, G, gamma, beta, y, stream=None):
        self._check_shapes(q, k, v, x, G, gamma, beta, y, None)
        G = self._gate(G)
        spectre_mix_run_host(self.handle, q, k, v, x, G, gamma, beta, y, stream)
        return y

    @property
    def workspace_bytes(self) -> int:
        return spectre_mix_workspace_bytes(self.handle)

    @property
    def plan(self) -> Tuple[int, int, int, int, int]:
        return spectre_mix_plan_info(self.handle)

    @property
    def slice_pass(self) -> str:
        """'tensor_cores' or 'cuda_cores': the slice pass runs of this plan launch."""
        sp = spectre_mix_slice_pass(self.handle)
        return "tensor_cores" if sp == SPECTRE_SLICE_TENSOR_CORES else "cuda_cores"

    def close(self) -> None:
        if self.handle is not None:
            h, self.handle = self.handle, None
            spectre_mix_destroy(h)

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---------------------------------------------------------------------------
# per-token DCT mix with spectral-entropy routing (include/dct_mix.h)
# ---------------------------------------------------------------------------
def dct_mix_create_status(d: int, dtype: int, eps: float = 1e-5) -> Tuple[int, Optional[int]]:
    h = _vp()
    code = _lib.dct_mix_create(ctypes.byref(h), d, dtype, eps)
    return code, h.value


def dct_mix_create(d: int, dtype: int, eps: float = 1e-5) -> int:
    code, h = dct_mix_create_status(d, dtype, eps)
    _check(code, "dct_mix_create")
    return h


def dct_mix_run(h: int, T: int, x, w, gamma, beta, tau: float, y, H, route, stream=None) -> None:
    _check(_lib.dct_mix_run(h, T, _ptr(x), _ptr(w), _ptr(gamma), _ptr(beta), tau, _ptr(y),
                            _ptr(H), _ptr(route), _stream(stream)), "dct_mix_run")


def dct_mix_run_debug(h: int, T: int, x, w, gamma, beta, tau: float, y, H, route, mix,
                      stream=None) -> None:
    _check(_lib.dct_mix_run_debug(h, T, _ptr(x), _ptr(w), _ptr(gamma), _ptr(beta), tau, _ptr(y),
                                  _ptr(H), _ptr(route), _ptr(mix), _stream(stream)),
           "dct_mix_run_debug")


def dct_mix_run_host(h: int, T: int, x, w, gamma, beta, tau: float, y, H, route,
                     stream=None) -> None:
    _check(_lib.dct_mix_run_host(h, T, _ptr(x), _ptr(w), _ptr(gamma), _ptr(beta), tau, _ptr(y),
                                 _ptr(H), _ptr(route), _stream(stream)), "dct_mix_run_host")


def dct_mix_destroy(h: Optional[int]) -> None:
    _check(_lib.dct_mix_destroy(h), "dct_mix_destroy")


def check_dct_arguments(d, dtype_code, x, w, gamma, beta, y, H, route, mix=None) -> int:
    """Sizes and types of one DCT-mix run's tensors; returns T (token rows).
    x and y hold T * d values of the plan's type; w, gamma, beta d fp32
    values; H T fp32 values; route T uint8 values; mix (optional) T * d fp32."""
    import torch

    if x.numel() % d:
        raise ValueError(f"x must hold whole rows of d = {d} values")
    T = x.numel() // d
    tok_type = torch.float32 if dtype_code == SPECTRE_F32 else torch.bfloat16
    for name, t in (("x", x), ("y", y)):
        if t.numel() != T * d or t.dtype != tok_type:
            raise ValueError(f"{name} must hold T * d = {T * d} values of {tok_type}")
    for name, t in (("w", w), ("gamma", gamma), ("beta", beta)):
        if t.numel() != d or t.dtype != torch.float32:
            raise ValueError(f"{name} must hold d = {d} fp32 values")
    if H.numel() != T or H.dtype != torch.float32:
        raise ValueError(f"H must hold T = {T} fp32 values")
    if route.numel() != T or route.dtype != torch.uint8:
        raise ValueError(f"route must hold T = {T} uint8 values")
    if mix is not None and (mix.numel() != T * d or mix.dtype != torch.float32):
        raise ValueError(f"mix must hold T * d = {T * d} fp32 values")
    return T


class DctMix:
    """A DCT-mix plan for token rows of length d (Chiaroscuro Attention
    summary: the orthonormal Type-II DCT of each token, its normalised
    spectral entropy H, the route H <= tau, and LayerNorm(x + iDCT(DCT(x) * w))).

    ``mix(x, w, gamma, beta, tau)`` takes x [..., d] on the GPU and returns
    (y, H, route) shaped [..., d], [...], [...]; pass ``mix_out=`` (fp32, the
    shape of x) to also receive iDCT(DCT(x) * w).
    """

    def __init__(self, d: int, dtype: str = "bf16", eps: float = 1e-5):
        self.d = d
        self.dtype_code = SPECTRE_F32 if dtype in ("f32", "float32", "fp32") else SPECTRE_BF16
        self.eps = eps
        self.handle = dct_mix_create(d, self.dtype_code, eps)

    def __call__(self, x, w, gamma, beta, tau: float, y=None, H=None, route=None, mix_out=None,
                 stream=None):
        import torch

        lead = tuple(x.shape[:-1])
        if y is None:
            y = torch.empty_like(x)
        if H is None:
            H = torch.empty(lead, dtype=torch.float32, device=x.device)
        if route is None:
            route = torch.empty(lead, dtype=torch.uint8, device=x.device)
        T = check_dct_arguments(self.d, self.dtype_code, x, w, gamma, beta, y, H, route, mix_out)
        if mix_out is None:
            dct_mix_run(self.handle, T, x, w, gamma, beta, tau, y, H, route, stream)
        else:
            dct_mix_run_debug(self.handle, T, x, w, gamma, beta, tau, y, H, route, mix_out, stream)
        return y, H, route

    def run_host(self, x, w, gamma, beta, tau: float, y, H, route, stream=None):
        T = check_dct_arguments(self.d, self.dtype_code, x, w, gamma, beta, y, H, route)
        dct_mix_run_host(self.handle, T, x, w, gamma, beta, tau, y, H, route, stream)
        return y, H, route

    def close(self) -> None:
        if self.handle is not None:
            h, self.handle = self.handle, None
            dct_mix_destroy(h)

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
