"""Decode step on the GPU against the fp64 oracle ("Linear attention and Gated
DeltaNet", ch. 28, "The recurrent form"; KDA's recurrence in "A walk through of
the DeltaNet family")."""
import numpy as np
import pytest
import torch

import delta_rule_recurrent_02_b200 as dn
import oracle
from delta_rule_recurrent_02_b200 import workloads as W
from _util import TOL, assert_close, f64

pytestmark = pytest.mark.gpu


def run_steps(S, q, k, v, beta, g, scale, gate):
    """Run len(q) decode steps on the GPU (S updated in place); outputs [steps,B,H,dv]."""
    outs = []
    for s in range(q.shape[0]):
        outs.append(dn.decode_step(q[s], k[s], v[s], beta[s], S, None if g is None else g[s],
                                   scale=scale, gate=gate).clone())
    return torch.stack(outs)


def oracle_steps(S0, q, k, v, beta, g, scale):
    # steps become the time axis of one recurrence: [B,H,steps,d]
    tr = lambda t: None if t is None else f64(t).transpose((1, 2, 0) + tuple(range(3, t.dim())))
    return oracle.delta_rule(tr(q), tr(k), tr(v), tr(beta), tr(g), f64(S0), scale=scale)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("gate", ["none", "scalar", "per_key"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (128, 64), (64, 128)])
def test_decode_parity(cuda_device, dtype, gate, dk, dv):
    cfg = W.DecodeConfig("t", B=3, H=5, dk=dk, dv=dv, dtype=dtype, gate=gate, seed=21, steps=12, bank=12)
    inp = W.gen_decode(cfg)
    d = {k_: (None if v_ is None else v_.cuda()) for k_, v_ in inp.items()}
    S = d["S"].clone()
    o = run_steps(S, d["q"], d["k"], d["v"], d["beta"], d["g"], cfg.scale, gate)
    ro, rS = oracle_steps(inp["S"], inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], cfg.scale)
    assert_close(o.permute(1, 2, 0, 3), ro, dtype, "o")
    assert_close(S, rS, dtype, "S")


def test_decode_worked_example(cuda_device):
    # ch. 28 worked example at d = 64: k = q = e_1, v = (2, 4, 0, ...), beta 0.5 then 1
    for dtype, td in (("f32", torch.float32), ("bf16", torch.bfloat16)):
        d = 64
        q = torch.zeros(1, 1, d, dtype=td, device="cuda"); q[0, 0, 0] = 1
        v = torch.zeros(1, 1, d, dtype=td, device="cuda"); v[0, 0, 0] = 2; v[0, 0, 1] = 4
        S = torch.zeros(1, 1, d, d, device="cuda")
        o1 = dn.decode_step(q, q, v, torch.full((1, 1), 0.5, device="cuda"), S)
        assert o1[0, 0, :2].float().tolist() == [1.0, 2.0] and torch.all(o1[0, 0, 2:] == 0)
        assert S[0, 0, 0, :2].tolist() == [1.0, 2.0]
        o2 = dn.decode_step(q, q, v, torch.ones(1, 1, device="cuda"), S)
        assert o2[0, 0, :2].float().tolist() == [2.0, 4.0]
        assert S[0, 0, 0, :2].tolist() == [2.0, 4.0] and torch.count_nonzero(S) == 2


def test_decode_full_size(cuda_device):
    """B=256, H=32, d=128 fp32 state, bf16 tokens, scalar decay: every head for the
    first 4 steps, then 64 seeded-sampled heads over 1000 steps (heads are
    independent, so a subset check is exact).  Step s uses token set s % 16."""
    cfg = W.DECODE
    inp = W.gen_decode(cfg)
    d = {k_: (None if v_ is None else v_.cuda()) for k_, v_ in inp.items()}
    S = d["S"].clone()
    n_all = 4
    o = run_steps(S, d["q"][:n_all], d["k"][:n_all], d["v"][:n_all], d["beta"][:n_all],
                  d["g"][:n_all], cfg.scale, "scalar")
    ro, rS = oracle_steps(inp["S"], inp["q"][:n_all], inp["k"][:n_all], inp["v"][:n_all],
                          inp["beta"][:n_all], inp["g"][:n_all], cfg.scale)
    assert_close(o.permute(1, 2, 0, 3), ro, "bf16", "o (all heads, 4 steps)")
    assert_close(S, rS, "bf16", "S (all heads, 4 steps)")
    # continue to 1000 steps on the GPU, all heads
    steps = cfg.steps
    o_hist = []
    gen = torch.Generator().manual_seed(99)
    flat = torch.randperm(cfg.B * cfg.H, generator=gen)[:64]
    sb, sh = (flat // cfg.H).tolist(), (flat % cfg.H).tolist()
    for s in range(n_all, steps):
        j = s % cfg.bank
        o_s = dn.decode_step(d["q"][j], d["k"][j], d["v"][j], d["beta"][j], S, d["g"][j], scale=cfg.scale)
        o_hist.append(o_s[sb, sh].float().cpu())
    torch.cuda.synchronize()
    # oracle on the sampled heads, from the 4-step state, over the same cyclic tokens
    idx = [s % cfg.bank for s in range(n_all, steps)]
    sel = lambda t: t[:, sb, sh][idx]          # [steps, 64, ...]
    q, k, v, beta, g = (sel(inp[n]) for n in ("q", "k", "v", "beta", "g"))
    tr = lambda t: f64(t).transpose((1, 0) + tuple(range(2, t.dim())))[None]
    ro2, rS2 = oracle.delta_rule(tr(q), tr(k), tr(v), tr(beta), tr(g),
                                 np.asarray(rS)[sb, sh][None], scale=cfg.scale)
    got_o = torch.stack(o_hist, dim=1)[None]     # [1, 64, steps, dv]
    assert_close(got_o, ro2, "bf16", "o (64 heads, 1000 steps)")
    assert_close(S[sb, sh][None], rS2, "bf16", "S (64 heads, 1000 steps)")


def test_decode_after_prefill_equals_longer_prefill(cuda_device):
    inp = W.gen_prefill(2, 3, 70, 128, 128, dtype="bf16", gate="scalar", seed=5, s0_std=0.1)
    d = {k_: (None if v_ is None else v_.cuda()) for k_, v_ in inp.items()}
    sc = 128 ** -0.5
    o_full, S_full = dn.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], scale=sc, path="simt")
    sl = slice(0, 69)
    o_pre, S = dn.chunk_fwd(d["q"][:, :, sl].contiguous(), d["k"][:, :, sl].contiguous(),
                            d["v"][:, :, sl].contiguous(), d["beta"][:, :, sl].contiguous(),
                            d["g"][:, :, sl].contiguous(), d["S0"], scale=sc, path="simt")
    o_last = dn.decode_step(d["q"][:, :, 69].contiguous(), d["k"][:, :, 69].contiguous(),
                            d["v"][:, :, 69].contiguous(), d["beta"][:, :, 69].contiguous(), S,
                            d["g"][:, :, 69].contiguous(), scale=sc)
    err_o = W.max_rel_err(f64(o_last), f64(o_full[:, :, 69]))
    err_s = W.max_rel_err(f64(S), f64(S_full))
    assert err_o <= 1e-2 and err_s <= 1e-4, (err_o, err_s)


def test_decode_empty_and_errors(cuda_device):
    q = torch.zeros(0, 4, 128, dtype=torch.bfloat16, device="cuda")
    S = torch.zeros(0, 4, 128, 128, device="cuda")
    o = dn.decode_step(q, q, torch.zeros(0, 4, 128, dtype=torch.bfloat16, device="cuda"),
                       torch.zeros(0, 4, device="cuda"), S, torch.zeros(0, 4, device="cuda"))
    assert o.shape == (0, 4, 128)
    q = torch.zeros(1, 1, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dn.DNError) as ei:
        dn.decode_step(q, q, q, torch.zeros(1, 1, device="cuda"), torch.zeros(1, 1, 96, 96, device="cuda"))
    assert ei.value.status == dn.DN_ERR_UNSUPPORTED


@pytest.mark.parametrize("neg", [False, True])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)])
def test_decode_layer_prologue(cuda_device, dtype, dk, dv, neg):
    # dn_decode_step_gdn: raw q and k (varied norms, one zero row), raw b and a with the
    # per-head A_log and dt_bias, against the oracle prologue then the oracle recurrence
    B, H, steps = 3, 5, 8
    gen = torch.Generator().manual_seed(55 + dk)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    q = (torch.randn(steps, B, H, dk, generator=gen) * (0.2 + 3 * torch.rand(steps, B, H, 1, generator=gen))).to(td)
    k = (torch.randn(steps, B, H, dk, generator=gen) * (0.2 + 3 * torch.rand(steps, B, H, 1, generator=gen))).to(td)
    q[2, 1, 3] = 0
    v = torch.randn(steps, B, H, dv, generator=gen).to(td)
    b = torch.randn(steps, B, H, generator=gen)
    a = torch.randn(steps, B, H, generator=gen)
    A_log = torch.log(1 + 15 * torch.rand(H, generator=gen))
    dt_bias = 0.5 * torch.randn(H, generator=gen)
    S0 = 0.1 * torch.randn(B, H, dk, dv, generator=gen)
    sc = dk ** -0.5
    S = S0.cuda().clone()
    outs = []
    for s in range(steps):
        o = torch.empty((B, H, dv), dtype=td, device="cuda")
        if neg:
            # beta = 2 sigmoid(b) ("DeltaNet: Memory That Edits", "The reflection hiding in the delta rule")
            dn.dn_decode_step_gdn_ex(q[s].cuda(), k[s].cuda(), v[s].cuda(), b[s].cuda(), a[s].cuda(), A_log.cuda(),
                                     dt_bias.cuda(), S, o, scale=sc, allow_neg_eigval=True)
        else:
            dn.dn_decode_step_gdn(q[s].cuda(), k[s].cuda(), v[s].cuda(), b[s].cuda(), a[s].cuda(), A_log.cuda(),
                                  dt_bias.cuda(), S, o, scale=sc)
        outs.append(o)
    dn.dn_device_status()
    # the prologue on [B,H,steps,...] (steps become the time axis)
    tr = lambda t: f64(t).transpose((1, 2, 0) + tuple(range(3, t.dim())))
    qn, kn, beta, g = oracle.gdn_prologue(tr(q), tr(k), tr(b), tr(a), f64(A_log), f64(dt_bias), allow_neg_eigval=neg)
    ro, rS = oracle.delta_rule(qn, kn, tr(v), beta, g, f64(S0), scale=sc)
    assert_close(torch.stack(outs).permute(1, 2, 0, 3), ro, dtype, "o")
    assert_close(S, rS, dtype, "S")


@pytest.mark.parametrize("activation", ["silu", "sigmoid"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64)])
def test_decode_prologue_and_gated_norm(cuda_device, activation, dtype, dk, dv):
    # dn_decode_step_gdn_ex with z: the layer's prologue, the step and its gated RMSNorm
    # ("The full layer", steps 4-7) in one kernel, against oracle.rms_norm_gated applied
    # to the oracle recurrence's read-out
    B, H, steps = 3, 4, 5
    gen = torch.Generator().manual_seed(77 + dk + dv)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    q = (torch.randn(steps, B, H, dk, generator=gen) * 2).to(td)
    k = (torch.randn(steps, B, H, dk, generator=gen) * 2).to(td)
    v = torch.randn(steps, B, H, dv, generator=gen).to(td)
    z = (2 * torch.randn(steps, B, H, dv, generator=gen)).to(td)
    b = torch.randn(steps, B, H, generator=gen)
    a = torch.randn(steps, B, H, generator=gen)
    A_log = torch.log(1 + 15 * torch.rand(H, generator=gen))
    dt_bias = 0.5 * torch.randn(H, generator=gen)
    w = 1 + 0.5 * torch.randn(dv, generator=gen)
    S0 = 0.1 * torch.randn(B, H, dk, dv, generator=gen)
    sc = dk ** -0.5
    S = S0.cuda().clone()
    outs = []
    for s in range(steps):
        o = torch.empty((B, H, dv), dtype=td, device="cuda")
        dn.dn_decode_step_gdn_ex(q[s].cuda(), k[s].cuda(), v[s].cuda(), b[s].cuda(), a[s].cuda(), A_log.cuda(),
                                 dt_bias.cuda(), S, o, scale=sc, z=z[s].cuda(), norm_weight=w.cuda(), eps=1e-6,
                                 norm_activation=activation)
        outs.append(o)
    dn.dn_device_status()
    tr = lambda t: f64(t).transpose((1, 2, 0) + tuple(range(3, t.dim())))
    qn, kn, beta, g = oracle.gdn_prologue(tr(q), tr(k), tr(b), tr(a), f64(A_log), f64(dt_bias))
    ro, rS = oracle.delta_rule(qn, kn, tr(v), beta, g, f64(S0), scale=sc)
    ry = oracle.rms_norm_gated(ro, tr(z), f64(w), eps=1e-6, activation=activation)
    assert_close(torch.stack(outs).permute(1, 2, 0, 3), ry, dtype, "y")
    assert_close(S, rS, dtype, "S")
