"""Seeded synthetic inputs for the delta-rule prefill and decode step.

This module holds only input recipes (random draws, normalisation of the draws,
rounding to the storage dtype) and the comparison metric.  It contains none
of the delta rule's arithmetic and imports neither the CUDA library nor the
oracle, so both sides of a parity check can draw the same inputs from it.

Recipe (all draws from one ``torch.Generator`` on the CPU, in the order
q, k, v, beta, g, S0):

* ``q`` ~ N(0, 1); L2-normalised per token when ``q_norm`` (the caller then
  passes ``scale = d_k ** -0.5``), left raw otherwise.
* ``k`` ~ N(0, 1), L2-normalised per token, ``x / max(|x|, 1e-12)``.
* ``v`` ~ N(0, 1).
* ``beta = sigmoid(N(0, 1))``, fp32.
* ``g = -softplus(N(0, 1) + shift)``, fp32: ``[B,H,T]`` for a scalar gate,
  ``[B,H,T,d_k]`` for a per-key gate, absent for no gate.
* ``S0 ~ N(0, s0_std^2)``, fp32, when ``s0_std`` is given.

q, k and v are drawn in fp32, normalised in fp32 and then rounded to the
storage dtype (round to nearest even); everything downstream, oracle included,
sees the rounded values.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch

GATES = ("none", "scalar", "per_key")


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    dtype: str            # "f32" | "bf16"  (q, k, v and o)
    gate: str             # "none" | "scalar" | "per_key"
    chunk: int
    seed: int
    q_norm: bool
    g_shift: float = 2.0
    s0_std: Optional[float] = None

    @property
    def scale(self) -> float:
        return self.dk ** -0.5 if self.q_norm else 1.0


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    H: int
    dk: int
    dv: int
    dtype: str
    gate: str
    seed: int
    steps: int
    s_std: float = 0.1
    g_shift: float = 2.0
    bank: int = 16        # distinct token sets, reused cyclically over the steps

    @property
    def scale(self) -> float:
        return self.dk ** -0.5


# The five workloads of the method, named by what they are.
DELTANET_SMALL = PrefillConfig("deltanet_f32_B1_H1_T512_d64", 1, 1, 512, 64, 64,
                               "f32", "none", 64, 0, q_norm=False)
GDN_PREFILL = PrefillConfig("gated_deltanet_bf16_B4_H16_T4096_d128", 4, 16, 4096,
                            128, 128, "bf16", "scalar", 64, 1, q_norm=True)
GDN_LONG = PrefillConfig("gated_deltanet_bf16_B1_H32_T65536_d128_S0", 1, 32, 65536,
                         128, 128, "bf16", "scalar", 64, 2, q_norm=True, s0_std=0.1)
DECODE = DecodeConfig("decode_step_bf16_B256_H32_d128", 256, 32, 128, 128, "bf16",
                      "scalar", 3, steps=1000)
KDA_PREFILL = PrefillConfig("kda_bf16_B2_H16_T8192_d128", 2, 16, 8192, 128, 128,
                            "bf16", "per_key", 64, 4, q_norm=True, g_shift=3.0)

PREFILL_CONFIGS = {c.name: c for c in (DELTANET_SMALL, GDN_PREFILL, GDN_LONG, KDA_PREFILL)}


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def gen_prefill(B: int, H: int, T: int, dk: int, dv: int, *, dtype: str = "bf16",
                gate: str = "scalar", seed: int = 0, q_norm: bool = True,
                g_shift: float = 2.0, s0_std: Optional[float] = None) -> dict:
    """Draw one prefill problem on the CPU; returns a dict of torch tensors
    ``q, k, v`` (storage dtype), ``beta`` fp32, ``g`` fp32 or None,
    ``S0`` fp32 or None."""
    assert gate in GATES
    gen = torch.Generator().manual_seed(seed)
    td = torch_dtype(dtype)
    q = torch.randn(B, H, T, dk, generator=gen)
    if q_norm:
        q = _l2norm(q)
    k = _l2norm(torch.randn(B, H, T, dk, generator=gen))
    v = torch.randn(B, H, T, dv, generator=gen)
    beta = torch.sigmoid(torch.randn(B, H, T, generator=gen))
    g = None
    if gate == "scalar":
        g = -torch.nn.functional.softplus(torch.randn(B, H, T, generator=gen) + g_shift)
    elif gate == "per_key":
        g = -torch.nn.functional.softplus(torch.randn(B, H, T, dk, generator=gen) + g_shift)
    S0 = None
    if s0_std is not None:
        S0 = torch.randn(B, H, dk, dv, generator=gen) * s0_std
    return {"q": q.to(td).contiguous(), "k": k.to(td).contiguous(),
            "v": v.to(td).contiguous(), "beta": beta.contiguous(),
            "g": None if g is None else g.contiguous(),
            "S0": None if S0 is None else S0.contiguous()}


def gen_prefill_config(cfg: PrefillConfig, **overrides) -> dict:
    kw = dict(dtype=cfg.dtype, gate=cfg.gate, seed=cfg.seed, q_norm=cfg.q_norm,
              g_shift=cfg.g_shift, s0_std=cfg.s0_std)
    shape = dict(B=cfg.B, H=cfg.H, T=cfg.T, dk=cfg.dk, dv=cfg.dv)
    for key in list(overrides):
        if key in shape:
            shape[key] = overrides.pop(key)
    kw.update(overrides)
    return gen_prefill(**shape, **kw)


def gen_decode(cfg: DecodeConfig, *, B: Optional[int] = None, H: Optional[int] = None,
               bank: Optional[int] = None) -> dict:
    """Draw the decode workload: the fp32 state ``S [B,H,dk,dv]`` and a bank
    of ``bank`` token sets ``q, k, v [bank,B,H,d]``, ``beta [bank,B,H]``,
    ``g [bank,B,H]`` (scalar gate) or ``[bank,B,H,dk]`` (per-key gate).
    Step ``s`` uses token set ``s % bank``."""
    B = cfg.B if B is None else B
    H = cfg.H if H is None else H
    n = cfg.bank if bank is None else bank
    gen = torch.Generator().manual_seed(cfg.seed)
    td = torch_dtype(cfg.dtype)
    S = torch.randn(B, H, cfg.dk, cfg.dv, generator=gen) * cfg.s_std
    q = _l2norm(torch.randn(n, B, H, cfg.dk, generator=gen))
    k = _l2norm(torch.randn(n, B, H, cfg.dk, generator=gen))
    v = torch.randn(n, B, H, cfg.dv, generator=gen)
    beta = torch.sigmoid(torch.randn(n, B, H, generator=gen))
    g = None
    if cfg.gate == "scalar":
        g = -torch.nn.functional.softplus(torch.randn(n, B, H, generator=gen) + cfg.g_shift)
    elif cfg.gate == "per_key":
        g = -torch.nn.functional.softplus(torch.randn(n, B, H, cfg.dk, generator=gen) + cfg.g_shift)
    return {"S": S.contiguous(), "q": q.to(td).contiguous(), "k": k.to(td).contiguous(),
            "v": v.to(td).contiguous(), "beta": beta.contiguous(),
            "g": None if g is None else g.contiguous()}


def max_rel_err(x, ref) -> float:
    """Largest, over (b, h) slices, of ``max|x - ref| / max|ref|`` (absolute
    error where a reference slice is all zero).  ``x`` and ``ref`` have the
    same shape with (b, h) leading (any further dims are flattened)."""
    import numpy as np
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if x.size == 0:
        return 0.0
    lead = x.shape[0] * x.shape[1] if x.ndim >= 2 else 1
    xd = x.reshape(lead, -1)
    rd = ref.reshape(lead, -1)
    if xd.shape[1] == 0:
        return 0.0
    num = np.abs(xd - rd).max(axis=1)
    den = np.abs(rd).max(axis=1)
    rel = np.where(den > 0, num / np.where(den > 0, den, 1.0), num)
    if not np.all(np.isfinite(xd)):
        return float("inf")
    return float(rel.max())
