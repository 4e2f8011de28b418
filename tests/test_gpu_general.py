"""The generalised delta rule of RWKV-7 ("DeltaNet: Memory That Edits", D2L
12.5, "The generalized delta rule") on the GPU against the fp64 oracle:
S_t = (diag(w_t) - (a_t * kappa_t) kappa_t^T) S_{t-1} + k_t v_t^T, o_t = S_t^T
(scale q_t), with a removal key kappa that differs from the write key k."""
import numpy as np
import pytest
import torch

import delta_rule_recurrent_02_b200 as dn
import oracle
from _util import assert_close, f64, oracle_prefill

pytestmark = pytest.mark.gpu


def _inputs(B, H, T, d, dtype, seed, s0_std=0.3, decay_shift=-1.0):
    """RWKV-7-like draws: unit removal keys, removal rates sigmoid(N(0,1)), write
    keys N(0,1)/sqrt(d), log-decays -exp(N(0,1) + shift) (decays in (0, 1))."""
    gen = torch.Generator().manual_seed(seed)
    unit = lambda x: x / x.norm(dim=-1, keepdim=True)
    q = torch.randn(B, H, T, d, generator=gen)
    wlog = -torch.exp(torch.randn(B, H, T, d, generator=gen) + decay_shift)
    kappa = unit(torch.randn(B, H, T, d, generator=gen))
    a = torch.sigmoid(torch.randn(B, H, T, d, generator=gen))
    k = torch.randn(B, H, T, d, generator=gen) / d ** 0.5
    v = torch.randn(B, H, T, d, generator=gen)
    S0 = s0_std * torch.randn(B, H, d, d, generator=gen) if s0_std else None
    cast = lambda t: t.to(dtype)
    return dict(q=cast(q), wlog=wlog, kappa=cast(kappa), a=a, k=cast(k), v=cast(v), S0=S0)


def _run(inp, chunk, scale):
    d = {n: (None if t is None else t.cuda()) for n, t in inp.items()}
    B, H, T, dk = d["q"].shape
    o = torch.full((B, H, T, d["v"].shape[-1]), float("nan"), dtype=d["q"].dtype, device="cuda")
    S = torch.full((B, H, dk, d["v"].shape[-1]), float("nan"), device="cuda")
    dn.dn_chunk_fwd_general(d["q"], d["wlog"], d["kappa"], d["a"], d["k"], d["v"], d["S0"], o, S, chunk=chunk,
                            scale=scale)
    dn.dn_device_status()
    return o, S


def _oracle(inp, scale):
    return oracle.generalized_delta_rule(f64(inp["q"]), np.exp(f64(inp["wlog"])), f64(inp["kappa"]), f64(inp["a"]),
                                         f64(inp["k"]), f64(inp["v"]), f64(inp["S0"]), scale=scale)


@pytest.mark.parametrize("dtype,kind", [(torch.float32, "f32"), (torch.bfloat16, "bf16")])
@pytest.mark.parametrize("chunk", [1, 5, 16, 32])
@pytest.mark.parametrize("d", [64, 128])
def test_general_t37_matches_oracle(cuda_device, dtype, kind, chunk, d):
    # the chunk test of "The chunked form" (ch. 28): 37 tokens, several chunk sizes,
    # a non-zero initial state; removal and write keys unrelated
    inp = _inputs(2, 2, 37, d, dtype, seed=100 + chunk + d)
    sc = d ** -0.5
    o, S = _run(inp, chunk, sc)
    ro, rS = _oracle(inp, sc)
    assert_close(o, ro, kind, "o")
    assert_close(S, rS, kind, "S_T")


@pytest.mark.parametrize("dtype,kind", [(torch.float32, "f32"), (torch.bfloat16, "bf16")])
def test_general_long_sequence(cuda_device, dtype, kind):
    inp = _inputs(1, 3, 1000, 128, dtype, seed=7, decay_shift=-2.0)
    sc = 128 ** -0.5
    o, S = _run(inp, 32, sc)
    ro, rS = _oracle(inp, sc)
    assert_close(o, ro, kind, "o")
    assert_close(S, rS, kind, "S_T")


def test_general_tied_is_deltanet(cuda_device):
    # the page: with w = 1, kappa = k', a = beta (every channel) and k = beta k' the
    # generalised rule is DeltaNet; compared with the oracle's DeltaNet recurrence
    B, H, T, d = 2, 2, 90, 64
    gen = torch.Generator().manual_seed(3)
    kp = torch.randn(B, H, T, d, generator=gen)
    kp = kp / kp.norm(dim=-1, keepdim=True)
    beta = torch.sigmoid(torch.randn(B, H, T, generator=gen))
    q = torch.randn(B, H, T, d, generator=gen)
    v = torch.randn(B, H, T, d, generator=gen)
    S0 = 0.3 * torch.randn(B, H, d, d, generator=gen)
    inp = dict(q=q, wlog=torch.zeros(B, H, T, d), kappa=kp, a=beta[..., None].expand(B, H, T, d).contiguous(),
               k=(beta[..., None] * kp).contiguous(), v=v, S0=S0)
    o, S = _run(inp, 16, 1.0)
    ro, rS = oracle_prefill(dict(q=q, k=kp, v=v, beta=beta, g=None, S0=S0), 1.0)
    assert_close(o, ro, "f32", "o")
    assert_close(S, rS, "f32", "S_T")


def test_general_rejects(cuda_device):
    inp = _inputs(1, 1, 8, 128, torch.float32, seed=1)
    d = {n: (None if t is None else t.cuda()) for n, t in inp.items()}
    o = torch.empty(1, 1, 8, 128, device="cuda")
    with pytest.raises(dn.DNError) as ei:             # chunks above 32 are not covered
        dn.dn_chunk_fwd_general(d["q"], d["wlog"], d["kappa"], d["a"], d["k"], d["v"], None, o, None, chunk=64)
    assert ei.value.status == dn.DN_ERR_UNSUPPORTED
