"""Seeded synthetic KV-cache workloads.

This module only draws data: it holds none of the codec or attention
arithmetic, so both the fp64 oracle (``oracle/``) and the CUDA path may take
their inputs from it.

Workload recipe (the pages measure on real model KV and on an undefined
"random-walk autocorrelated signal"; these AR(1) streams stand in for both):

* ``gen = torch.Generator('cpu').manual_seed(seed)``.
* Draw order: K innovations, V innovations, queries, then outlier channels.
* K and V are AR(1) along the sequence axis: ``x_0 = e_0`` and
  ``x_t = rho * x_{t-1} + e_t`` with ``e ~ N(0, 1)`` (unit innovations, no
  variance normalisation), shape ``(B, Hk, T, D)``, computed in float64 and
  rounded to float32.
* Outliers (when ``outlier_frac > 0``): ``max(1, round(outlier_frac * D))``
  channels per (batch, kv head), picked with ``torch.randperm`` from the same
  generator; that channel of K and of V is multiplied by ``outlier_gain``.
* Queries are ``N(0, 1)`` of shape ``(B, Hq, 1, D)`` (``(steps, B, Hq, 1, D)``
  for streaming workloads, one query per decode step).
* Finally everything is cast to the workload's input dtype (bfloat16 with
  round-to-nearest-even, or float32).
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np
import torch

try:
    from scipy.signal import lfilter as _lfilter
except Exception:  # pragma: no cover - scipy is part of the image
    _lfilter = None


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and codec settings of one synthetic decode-attention workload.

    ``T`` is the total sequence length seen by decode attention (archived
    blocks plus the raw tail). For streaming workloads ``T`` is the prefill
    length and ``steps`` single-token appends follow it.
    """

    name: str
    B: int
    Hq: int
    Hk: int
    D: int
    T: int
    R: int
    S: int
    k_coeff: str = "i8"      # "i8" (int8 codes + fp32 scales), "f32", "bf16"
    v_coeff: str = "i8"
    in_dtype: str = "bf16"   # dtype of K/V tokens, tail and q: "bf16" or "f32"
    rho: float = 0.9
    outlier_frac: float = 0.0
    outlier_gain: float = 8.0
    seed: int = 0
    steps: int = 0           # decode_step appends after the prefill

    @property
    def G(self) -> int:
        return self.Hq // self.Hk

    @property
    def T_total(self) -> int:
        return self.T + self.steps

    @property
    def n_blocks(self) -> int:
        return self.T // self.R

    @property
    def n_tail(self) -> int:
        return self.T - self.n_blocks * self.R

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five published workloads (names follow the codec's vocabulary).
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", B=1, Hq=4, Hk=4, D=64, T=256, R=8, S=2,
                     k_coeff="f32", v_coeff="f32", in_dtype="f32",
                     rho=0.9, seed=0),
    "gqa": Workload("gqa", B=8, Hq=32, Hk=8, D=128, T=4096 + 5, R=8, S=2,
                    rho=0.9, seed=1),
    "long": Workload("long", B=1, Hq=32, Hk=8, D=128, T=131072 + 3, R=16,
                     S=4, rho=0.95, outlier_frac=0.01, seed=2),
    "large": Workload("large", B=64, Hq=64, Hk=8, D=128, T=8192 + 7, R=8,
                      S=3, k_coeff="i8", v_coeff="bf16", rho=0.85, seed=3),
    "stream": Workload("stream", B=4, Hq=32, Hk=8, D=128, T=32768, R=8, S=2,
                       rho=0.9, seed=4, steps=256),
}


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def _ar1_rows(eps: np.ndarray, rho: float) -> np.ndarray:
    """AR(1) filter along axis -2 of a float64 array (x_0 = e_0)."""
    if _lfilter is not None:
        return _lfilter([1.0], [1.0, -rho], eps, axis=-2)
    out = np.empty_like(eps)
    acc = np.zeros(eps.shape[:-2] + eps.shape[-1:], dtype=np.float64)
    for t in range(eps.shape[-2]):
        acc = rho * acc + eps[..., t, :]
        out[..., t, :] = acc
    return out


def ar1(gen: torch.Generator, shape, rho: float) -> torch.Tensor:
    """Seeded AR(1) stream of ``shape = (B, H, T, D)`` in float32."""
    eps = torch.randn(shape, generator=gen, dtype=torch.float32)
    out = torch.empty(shape, dtype=torch.float32)
    # float64 filtering one batch row at a time bounds host memory
    for b in range(shape[0]):
        x = _ar1_rows(eps[b].numpy().astype(np.float64), rho)
        out[b] = torch.from_numpy(x.astype(np.float32))
    return out


def generate(w: Workload, q_steps: Optional[int] = None):
    """Draw the workload's K, V (B, Hk, T_total, D) and queries.

    Returns a dict with ``k``, ``v`` (input dtype, CPU), ``q`` (input dtype,
    ``(B, Hq, 1, D)``, or ``(steps, B, Hq, 1, D)`` for streaming workloads)
    and ``outlier_channels`` (``(B, Hk, n)`` int64, empty when unused).
    """
    gen = torch.Generator("cpu").manual_seed(w.seed)
    shape = (w.B, w.Hk, w.T_total, w.D)
    k = ar1(gen, shape, w.rho)
    v = ar1(gen, shape, w.rho)
    n_q = w.steps if q_steps is None else q_steps
    if n_q:
        q = torch.randn((n_q, w.B, w.Hq, 1, w.D), generator=gen)
    else:
        q = torch.randn((w.B, w.Hq, 1, w.D), generator=gen)
    chans = torch.empty((w.B, w.Hk, 0), dtype=torch.int64)
    if w.outlier_frac > 0:
        n_out = max(1, int(round(w.outlier_frac * w.D)))
        chans = torch.empty((w.B, w.Hk, n_out), dtype=torch.int64)
        for b in range(w.B):
            for h in range(w.Hk):
                c = torch.randperm(w.D, generator=gen)[:n_out]
                chans[b, h] = c
                k[b, h, :, c] *= w.outlier_gain
                v[b, h, :, c] *= w.outlier_gain
    dt = torch_dtype(w.in_dtype)
    return {"k": k.to(dt), "v": v.to(dt), "q": q.to(dt),
            "outlier_channels": chans}


def small(name: str, **overrides) -> Workload:
    """A reduced copy of a published workload for oracle-sized parity runs."""
    return WORKLOADS[name].replace(**overrides)
