"""Grouped value heads on the GPU against the fp64 oracle ("Linear attention and
Gated DeltaNet", ch. 28, "The full layer", step 3: the layer has fewer key
heads than value heads, and each key head's q and k serve H / H_k value heads;
value head h reads key head h // (H / H_k))."""
import numpy as np
import pytest
import torch

import delta_rule_recurrent_02_b200 as dn
import oracle
from _util import assert_close, f64

pytestmark = pytest.mark.gpu


def _gva_inputs(B, Hk, H, T, seed, gate="scalar", s0_std=0.1):
    gen = torch.Generator().manual_seed(seed)
    unit = lambda x: x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    q = unit(torch.randn(B, Hk, T, 128, generator=gen)).to(torch.bfloat16)
    k = unit(torch.randn(B, Hk, T, 128, generator=gen)).to(torch.bfloat16)
    v = torch.randn(B, H, T, 128, generator=gen).to(torch.bfloat16)
    beta = torch.sigmoid(torch.randn(B, H, T, generator=gen))
    g = -torch.nn.functional.softplus(torch.randn(B, H, T, generator=gen) + 2) if gate == "scalar" else None
    S0 = s0_std * torch.randn(B, H, 128, 128, generator=gen) if s0_std else None
    return dict(q=q, k=k, v=v, beta=beta, g=g, S0=S0)


def _oracle(inp, scale):
    return oracle.gva_delta_rule(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["beta"]), f64(inp["g"]),
                                 f64(inp["S0"]), scale=scale)


@pytest.mark.parametrize("B,Hk,H,T,gate", [
    (2, 2, 6, 200, "scalar"),      # three value heads per key head, a ragged last chunk
    (1, 4, 16, 333, "none"),
    (1, 16, 48, 130, "scalar"),    # the layer's 16 key : 48 value heads
    (2, 8, 32, 64, "scalar"),      # 64 value heads: the single launch
    (3, 32, 64, 100, "scalar"),    # 192 value heads: the two-launch form
])
def test_chunk_fwd_gva_matches_oracle(cuda_device, B, Hk, H, T, gate):
    inp = _gva_inputs(B, Hk, H, T, seed=B * 1000 + H + T, gate=gate)
    d = {n: (None if t is None else t.cuda()) for n, t in inp.items()}
    sc = 128 ** -0.5
    o = torch.full((B, H, T, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    S = torch.full((B, H, 128, 128), float("nan"), device="cuda")
    dn.dn_chunk_fwd_gva(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], o, S, scale=sc, gate=gate)
    dn.dn_device_status()
    ro, rS = _oracle(inp, sc)
    assert_close(o, ro, "bf16", "o")
    assert_close(S, rS, "bf16", "S_T")


def test_chunk_fwd_gva_equals_repeated_heads(cuda_device):
    # the grouped call gives what dn_chunk_fwd gives on q and k repeated per value head
    B, Hk, H, T = 2, 4, 12, 257
    inp = _gva_inputs(B, Hk, H, T, seed=5)
    d = {n: (None if t is None else t.cuda()) for n, t in inp.items()}
    sc = 128 ** -0.5
    o = torch.empty((B, H, T, 128), dtype=torch.bfloat16, device="cuda")
    S = torch.empty((B, H, 128, 128), device="cuda")
    dn.dn_chunk_fwd_gva(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], o, S, scale=sc)
    r = H // Hk
    o2, S2 = dn.chunk_fwd(d["q"].repeat_interleave(r, 1).contiguous(), d["k"].repeat_interleave(r, 1).contiguous(),
                          d["v"], d["beta"], d["g"], d["S0"], scale=sc, path="tc")
    dn.dn_device_status()
    # the same kernels on the same values: identical results
    assert torch.equal(o, o2) and torch.equal(S, S2)


def test_chunk_fwd_gva_rejects(cuda_device):
    inp = _gva_inputs(1, 3, 8, 64, seed=1)
    d = {n: (None if t is None else t.cuda()) for n, t in inp.items()}
    o = torch.empty((1, 8, 64, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dn.DNError) as ei:          # 8 value heads are not a multiple of 3 key heads
        dn.dn_chunk_fwd_gva(d["q"], d["k"], d["v"], d["beta"], d["g"], None, o, None)
    assert ei.value.status == dn.DN_ERR_INVALID
    q32 = d["q"][:, :2].float().contiguous()
    with pytest.raises(dn.DNError) as ei:          # fp32 tokens: the tensor-core path only
        dn.dn_chunk_fwd_gva(q32, q32, d["v"].float(), d["beta"], d["g"], None, o.float(), None)
    assert ei.value.status == dn.DN_ERR_UNSUPPORTED


@pytest.mark.parametrize("gate", ["none", "scalar", "per_key"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_step_gva_matches_oracle(cuda_device, gate, dtype):
    B, Hk, H, d = 3, 4, 12, 128
    gen = torch.Generator().manual_seed(11)
    unit = lambda x: x / x.norm(dim=-1, keepdim=True)
    q = unit(torch.randn(B, Hk, d, generator=gen)).to(dtype)
    k = unit(torch.randn(B, Hk, d, generator=gen)).to(dtype)
    v = torch.randn(B, H, d, generator=gen).to(dtype)
    beta = torch.sigmoid(torch.randn(B, H, generator=gen))
    g = {"none": None, "scalar": -torch.rand(B, H, generator=gen),
         "per_key": -torch.rand(B, H, d, generator=gen)}[gate]
    S0 = 0.1 * torch.randn(B, H, d, d, generator=gen)
    S = S0.cuda()
    o = torch.empty(B, H, d, dtype=dtype, device="cuda")
    dn.dn_decode_step_gva(q.cuda(), k.cuda(), v.cuda(), beta.cuda(), None if g is None else g.cuda(), S, o,
                          scale=d ** -0.5)
    dn.dn_device_status()
    t = lambda x: None if x is None else f64(x)[:, :, None]
    ro, rS = oracle.gva_delta_rule(t(q), t(k), t(v), t(beta), t(g), f64(S0), scale=d ** -0.5)
    kind = "f32" if dtype == torch.float32 else "bf16"
    assert_close(o, ro[:, :, 0], kind, "o")
    assert_close(S, rS, kind, "S")
