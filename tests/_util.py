"""Shared helpers for the parity tests (test infrastructure)."""
import numpy as np
import torch

import oracle
from delta_rule_recurrent_02_b200.workloads import max_rel_err

# Tolerances on max relative error (per (b, h) slice, max over slices):
# fp32 token inputs 1e-4, bf16 token inputs 2e-2, on o and on the final state.
TOL = {"f32": 1e-4, "bf16": 2e-2}


def f64(t):
    if t is None:
        return None
    return t.detach().to("cpu", torch.float64).numpy()


def to_dev(inp, device="cuda"):
    return {k: (None if v is None else v.to(device)) for k, v in inp.items()}


def oracle_prefill(inp, scale, bh=None, nthreads=0):
    """Oracle on all (b, h) or on a subset given as a list of (b, h) pairs."""
    q, k, v, beta, g, S0 = (inp[n] for n in ("q", "k", "v", "beta", "g", "S0"))
    if bh is not None:
        sel = lambda t: None if t is None else torch.stack([t[b, h] for b, h in bh])[None]
        q, k, v, beta, g, S0 = (sel(t) for t in (q, k, v, beta, g, S0))
    return oracle.delta_rule(f64(q), f64(k), f64(v), f64(beta), f64(g), f64(S0),
                             scale=scale, nthreads=nthreads)


def pick(t, bh):
    return torch.stack([t[b, h] for b, h in bh])[None]


def assert_close(got, ref, dtype, what=""):
    err = max_rel_err(f64(got) if torch.is_tensor(got) else got, ref)
    assert err <= TOL[dtype], f"{what}: max relative error {err:.3e} > {TOL[dtype]:.0e}"
    return err
