"""Seeded synthetic workloads for the spectral mixer.

This module only draws random inputs.  It holds none of the mixer's arithmetic,
so both the CUDA path's tests and the CPU oracle can take their inputs from it.

The five named workloads carry the shapes and value distributions of the
benchmark configurations (tiny fp32, fp32 mid, bf16 long, bf16 mixed-radix,
bf16 very long).  The pages measure on no public dataset for this path; these
synthetic inputs are the workloads.

Recipe, per workload ``i`` (its position in ``WORKLOADS``):
  * a CPU ``torch.Generator`` seeded with ``1000 + i``;
  * draw order q, k, v, x, G, gamma, beta (constant gamma/beta are not drawn);
  * every draw in fp32, then scaled, then cast to the storage dtype
    (q, k, v, x only; G, gamma, beta stay fp32).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    L: int
    H: int
    D: int
    F: int
    dtype: str            # "f32" or "bf16": storage of q, k, v, x and y
    qkv_scale: str        # "unit" -> N(0,1); "invsqrtL" -> N(0,1)/sqrt(L)
    x_scale: str
    gate: str             # "u0.5_1.5", "u0_1", "exp2048"
    gamma: str            # "one" or "n1_0.1"
    beta: str             # "zero" or "n0_0.1"
    eps: float = 1e-5

    @property
    def C(self) -> int:
        return self.H * self.D

    @property
    def nbins(self) -> int:
        return self.L // 2 + 1

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def algorithmic_bytes(self) -> int:
        """Bytes the method must move: q, k, v, x read, G[:, :F] read,
        gamma and beta read, y written."""
        n = self.B * self.L * self.C
        return 5 * n * self.elem_bytes + self.H * self.F * 4 + 2 * self.C * 4


WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("tiny_fp32", 0, B=1, L=256, H=1, D=16, F=129, dtype="f32",
             qkv_scale="unit", x_scale="unit", gate="u0.5_1.5", gamma="one", beta="zero"),
    Workload("fp32_mid", 1, B=2, L=4096, H=8, D=64, F=2049, dtype="f32",
             qkv_scale="invsqrtL", x_scale="invsqrtL", gate="u0_1", gamma="n1_0.1", beta="n0_0.1"),
    Workload("bf16_long", 2, B=1, L=65536, H=8, D=64, F=8192, dtype="bf16",
             qkv_scale="invsqrtL", x_scale="invsqrtL", gate="u0_1", gamma="one", beta="zero"),
    Workload("bf16_mixed_radix", 3, B=4, L=12288, H=16, D=128, F=6145, dtype="bf16",
             qkv_scale="invsqrtL", x_scale="unit", gate="exp2048", gamma="n1_0.1", beta="zero"),
    Workload("bf16_very_long", 4, B=1, L=1048576, H=8, D=64, F=65536, dtype="bf16",
             qkv_scale="invsqrtL", x_scale="invsqrtL", gate="u0_1", gamma="one", beta="zero"),
]}


def custom(B: int, L: int, H: int, D: int, F: Optional[int] = None, dtype: str = "f32",
           qkv_scale: str = "invsqrtL", x_scale: str = "invsqrtL", gate: str = "u0_1",
           gamma: str = "n1_0.1", beta: str = "n0_0.1", name: str = "custom",
           index: int = 100) -> Workload:
    """A workload of any shape with one of the recipes above (for sweeps)."""
    return Workload(name, index, B=B, L=L, H=H, D=D, F=(L // 2 + 1) if F is None else F,
                    dtype=dtype, qkv_scale=qkv_scale, x_scale=x_scale, gate=gate,
                    gamma=gamma, beta=beta)


def _scale(kind: str, L: int) -> float:
    return 1.0 if kind == "unit" else 1.0 / math.sqrt(L)


def make_inputs(w: Workload, seed_offset: int = 0) -> Dict[str, torch.Tensor]:
    """Draw q, k, v, x, G, gamma, beta on the CPU for workload ``w``.

    ``seed_offset`` shifts the seed (used to give each rank of a multi-GPU
    run its own batch).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(1000 + w.index + seed_offset)
    shape = (w.B, w.L, w.C)
    out: Dict[str, torch.Tensor] = {}
    for name, kind in (("q", w.qkv_scale), ("k", w.qkv_scale), ("v", w.qkv_scale),
                       ("x", w.x_scale)):
        t = torch.randn(shape, generator=g, dtype=torch.float32)
        s = _scale(kind, w.L)
        if s != 1.0:
            t.mul_(s)
        out[name] = t.to(w.torch_dtype)
        del t
    nb = w.nbins
    if w.gate == "u0.5_1.5":
        G = torch.rand((w.H, nb), generator=g, dtype=torch.float32) + 0.5
    elif w.gate == "u0_1":
        G = torch.rand((w.H, nb), generator=g, dtype=torch.float32)
    elif w.gate == "exp2048":
        u = torch.rand((w.H, nb), generator=g, dtype=torch.float32) * 0.5 + 0.5
        f = torch.arange(nb, dtype=torch.float32)
        G = torch.exp(-f / 2048.0)[None, :] * u
    else:
        raise ValueError(w.gate)
    out["G"] = G.contiguous()
    if w.gamma == "one":
        out["gamma"] = torch.ones(w.C, dtype=torch.float32)
    else:
        out["gamma"] = torch.randn(w.C, generator=g, dtype=torch.float32) * 0.1 + 1.0
    if w.beta == "zero":
        out["beta"] = torch.zeros(w.C, dtype=torch.float32)
    else:
        out["beta"] = torch.randn(w.C, generator=g, dtype=torch.float32) * 0.1
    return out


# ---------------------------------------------------------------------------
# per-token DCT mix workloads
# ---------------------------------------------------------------------------
@dataclass(frozen=True)
class DctWorkload:
    """Token rows x[B, L, d] for the DCT mix.

    Recipe (``make_dct_inputs``): a CPU generator seeded with ``2000 + index``;
    draw order: the smooth/white choice per token, white rows, smooth-row
    noise, w, gamma, beta.  Each token is, with probability 1/2, white
    (N(0,1) i.i.d. over d) or smooth (a circular moving average of N(0,1)
    noise over a window of d/16 along d, scaled back to unit variance), so
    the spectral entropies spread over both sides of tau.  w ~ U(0,1),
    gamma ~ N(1, 0.1), beta ~ N(0, 0.1); eps = 1e-5.  tau = 0.8954 at
    d = 1024 (the threshold the page quotes for its 400M model, whose width
    is 1024); the page gives none for d = 256, where 0.75 splits the smooth
    rows (H about 0.5 to 0.6) from the white ones (about 0.87).
    """
    name: str
    index: int
    B: int
    L: int
    d: int
    dtype: str
    eps: float = 1e-5
    tau: float = 0.8954

    @property
    def T(self) -> int:
        return self.B * self.L

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def algorithmic_bytes(self) -> int:
        """x read, y written, H (fp32) and route (1 byte) written per token,
        w, gamma, beta read once."""
        return self.T * (2 * self.d * self.elem_bytes + 5) + 3 * self.d * 4


DCT_WORKLOADS: Dict[str, DctWorkload] = {w.name: w for w in [
    DctWorkload("dct_tiny_fp32", 0, B=1, L=37, d=64, dtype="f32", tau=0.75),
    # the two model widths the page gives (d = 256 and 1024), sequence length 256
    DctWorkload("dct_d256", 1, B=2048, L=256, d=256, dtype="bf16", tau=0.75),
    DctWorkload("dct_d1024", 2, B=512, L=256, d=1024, dtype="bf16"),
]}


def dct_custom(B: int, L: int, d: int, dtype: str = "f32", index: int = 100,
               tau: float = 0.8954) -> DctWorkload:
    return DctWorkload("dct_custom", index, B=B, L=L, d=d, dtype=dtype, tau=tau)


def make_dct_inputs(w: DctWorkload, seed_offset: int = 0) -> Dict[str, torch.Tensor]:
    """Draw x [B, L, d], w, gamma, beta [d] on the CPU for workload ``w``
    (``seed_offset`` gives each rank of a multi-GPU run its own tokens)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(2000 + w.index + seed_offset)
    T, d = w.T, w.d
    smooth = torch.rand(T, generator=g) < 0.5
    x = torch.randn((T, d), generator=g, dtype=torch.float32)
    ns = int(smooth.sum())
    if ns:
        win = max(1, d // 16)
        e = torch.randn((ns, d), generator=g, dtype=torch.float32)
        c = torch.cumsum(torch.cat([e, e[:, :win]], dim=1), dim=1)
        avg = (c[:, win - 1:win - 1 + d] - torch.cat([torch.zeros(ns, 1), c[:, :d - 1]], dim=1))
        x[smooth] = avg / math.sqrt(win)
    out = {"x": x.reshape(w.B, w.L, d).to(w.torch_dtype)}
    out["w"] = torch.rand(d, generator=g, dtype=torch.float32)
    out["gamma"] = torch.randn(d, generator=g, dtype=torch.float32) * 0.1 + 1.0
    out["beta"] = torch.randn(d, generator=g, dtype=torch.float32) * 0.1
    return out
