"""Parity of the layer's causal conv (dn_causal_conv1d) and gated RMSNorm
(dn_rms_norm_gated) with the fp64 oracle, element by element.

Tolerances, from the arithmetic: both kernels compute in fp32 from inputs that
are exact in fp32 and round once at the store.  The fp32 part is a few
operations deep (at most K = 4 products and a sum; a 128-term sum of squares, a
root, a division and one exp), so its relative error stays below 1e-6.  A bf16
store then adds at most half an ulp, 2^-9 relative: hence 2^-8 relative for
bf16 outputs and 1e-5 for fp32 outputs, plus an absolute 1e-5 (conv) or 1e-6
(norm) for outputs that cancel to near zero.  The carried conv state is a copy
of inputs and must match exactly."""
import numpy as np
import pytest
import torch

import delta_rule_recurrent_02_b200 as dn
import oracle

RTOL = {torch.bfloat16: 2.0 ** -8, torch.float32: 1e-5}


def f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def check(got, ref, dtype, atol, what):
    g = f64(got)
    err = np.abs(g - ref) - (RTOL[dtype] * np.abs(ref) + atol)
    worst = np.unravel_index(np.argmax(err), err.shape) if err.size else None
    assert err.size == 0 or err.max() <= 0, \
        f"{what}: at {worst} got {g[worst]!r}, oracle {ref[worst]!r} (rtol {RTOL[dtype]}, atol {atol})"


def conv_inputs(B, T, C, K, dtype, seed, with_state=True, ld=None):
    gen = torch.Generator().manual_seed(seed)
    ld = C if ld is None else ld
    wide = torch.randn(B, T, ld, generator=gen).to(dtype)
    x = wide[:, :, :C]
    w = (torch.randn(C, K, generator=gen) * 0.5).float()
    s = torch.randn(B, K - 1, C, generator=gen).to(dtype) if with_state else None
    return wide, x, w, s


def head_major(y, B, T, C, hd):
    """[B, C / hd, T, hd] -> [B, T, C]"""
    return y.reshape(B, C // hd, T, hd).permute(0, 2, 1, 3).reshape(B, T, C)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,T,C,K,hd,ld,act,state", [
    (2, 37, 256, 4, 128, None, True, True),     # several row tiles, ragged tail, 16-byte path
    (1, 16, 64, 4, 64, None, True, True),       # exactly one tile
    (3, 100, 48, 3, 16, None, False, True),     # no activation, K = 3
    (2, 50, 40, 4, 20, None, True, True),       # C and head_dim not multiples of 8: one channel per thread
    (2, 33, 128, 2, 32, 384, True, True),       # x a column slice of a wider row (ld_x = 384)
    (2, 21, 64, 1, 64, None, True, True),       # K = 1: no history
    (2, 19, 96, 4, 96, None, True, False),      # no carried state: zeros
    (1, 2, 64, 4, 64, None, True, True),        # T < K - 1: the new state keeps old rows
    (2, 70, 320, 4, 64, 448, True, True),       # several channel blocks (the last partial), 3 row tiles
])
def test_causal_conv1d_matches_oracle(cuda_device, dtype, B, T, C, K, hd, ld, act, state):
    wide, x, w, s = conv_inputs(B, T, C, K, dtype, seed=B * 1000 + T + C + K, with_state=state, ld=ld)
    y_ref, s_ref = oracle.causal_conv1d(f64(x), f64(w), f64(s), activation=act)
    wide_d = wide.cuda()
    x_d = wide_d[:, :, :C]
    y = torch.full((B, C // hd, T, hd), float("nan"), dtype=dtype, device="cuda")
    s_out = torch.full((B, K - 1, C), float("nan"), dtype=dtype, device="cuda")
    dn.dn_causal_conv1d(x_d, w.cuda(), y, None if s is None else s.cuda(), s_out, head_dim=hd, activation=act)
    dn.dn_device_status()
    check(head_major(y.cpu(), B, T, C, hd), y_ref, dtype, 1e-5, "y")
    assert np.array_equal(f64(s_out), s_ref), "carried state"


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_causal_conv1d_decode_steps_in_place(cuda_device, dtype):
    """Token-by-token steps (T = 1) with the state updated in place equal one
    prefill over the whole sequence; so does a prefill split at 5 and 23 with the
    carried state (T > 16 writes a separate state buffer)."""
    B, T, C, K = 3, 29, 256, 4
    _, x, w, s = conv_inputs(B, T, C, K, dtype, seed=77)
    y_ref, s_ref = oracle.causal_conv1d(f64(x), f64(w), f64(s))
    x_d, w_d = x.contiguous().cuda(), w.cuda()
    st = s.cuda().clone()
    ys = []
    for t in range(T):
        y = torch.empty((B, 1, C), dtype=dtype, device="cuda")
        dn.dn_causal_conv1d(x_d[:, t:t + 1], w_d, y, st, st)
        ys.append(y)
    dn.dn_device_status()
    check(torch.cat(ys, dim=1).cpu(), y_ref, dtype, 1e-5, "decode steps")
    assert np.array_equal(f64(st), s_ref), "in-place state after T steps"
    cur = s.cuda()
    parts = []
    for a, b in ((0, 5), (5, 23), (23, T)):
        y = torch.empty((B, b - a, C), dtype=dtype, device="cuda")
        nxt = torch.empty_like(cur)
        dn.dn_causal_conv1d(x_d[:, a:b].contiguous(), w_d, y, cur, nxt)
        parts.append(y)
        cur = nxt
    dn.dn_device_status()
    check(torch.cat(parts, dim=1).cpu(), y_ref, dtype, 1e-5, "split prefill")
    assert np.array_equal(f64(cur), s_ref), "state after split prefill"


@pytest.mark.gpu
def test_causal_conv1d_empty_sequence_copies_state(cuda_device):
    B, C, K = 2, 64, 4
    _, _, w, s = conv_inputs(B, 1, C, K, torch.bfloat16, seed=5)
    s_out = torch.full((B, K - 1, C), float("nan"), dtype=torch.bfloat16, device="cuda")
    x = torch.empty((B, 0, C), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((B, 0, C), dtype=torch.bfloat16, device="cuda")
    dn.dn_causal_conv1d(x, w.cuda(), y, s.cuda(), s_out)
    dn.dn_device_status()
    assert torch.equal(s_out.cpu(), s)


@pytest.mark.gpu
def test_causal_conv1d_layer_size_sampled(cuda_device):
    """The q, k, v convs of a B=4, T=4096 layer with 16 heads of 128 (C = 6144 in
    one projection row, three calls on its column slices, head-major outputs),
    checked on 96 sampled channels against the oracle; the states in full."""
    B, T, H, d, K = 4, 4096, 16, 128, 4
    C3 = 3 * H * d
    gen = torch.Generator().manual_seed(4096)
    proj = torch.randn(B, T, C3, generator=gen).to(torch.bfloat16)
    w = (torch.randn(C3, K, generator=gen) * 0.5).float()
    s = torch.randn(B, K - 1, C3, generator=gen).to(torch.bfloat16)
    proj_d, w_d, s_d = proj.cuda(), w.cuda(), s.cuda()
    outs, states = [], []
    for part in range(3):
        lo = part * H * d
        y = torch.empty((B, H, T, d), dtype=torch.bfloat16, device="cuda")
        so = torch.empty((B, K - 1, H * d), dtype=torch.bfloat16, device="cuda")
        dn.dn_causal_conv1d(proj_d[:, :, lo:lo + H * d], w_d[lo:lo + H * d].contiguous(), y,
                            s_d[:, :, lo:lo + H * d].contiguous(), so, head_dim=d)
        outs.append(y)
        states.append(so)
    dn.dn_device_status()
    rng = np.random.default_rng(9)
    ch = np.sort(rng.choice(C3, 96, replace=False))
    y_ref, s_ref = oracle.causal_conv1d(f64(proj[:, :, ch]), f64(w[ch]), f64(s[:, :, ch]))
    got = torch.stack([outs[c // (H * d)][:, (c % (H * d)) // d, :, c % d] for c in ch], dim=-1)
    check(got.cpu(), y_ref, torch.bfloat16, 1e-5, "sampled channels")
    s_all = torch.cat(states, dim=-1).cpu()
    assert torch.equal(s_all, proj[:, T - K + 1:, :])


# ---- gated RMSNorm -----------------------------------------------------------------------

def norm_inputs(B, T, H, D, dtype, seed):
    gen = torch.Generator().manual_seed(seed)
    o = (torch.randn(B, H, T, D, generator=gen) * 3).to(dtype)
    z = torch.randn(B, T, H, D, generator=gen).to(dtype)
    w = (1 + 0.5 * torch.randn(D, generator=gen)).float()
    return o, z, w


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,T,H,D,act,head_major_x", [
    (2, 33, 4, 128, "silu", True),
    (1, 5, 3, 64, "silu", False),
    (2, 7, 2, 256, "sigmoid", True),
    (3, 1, 5, 128, "sigmoid", False),     # a decode step's output, T = 1
])
def test_rms_norm_gated_matches_oracle(cuda_device, dtype, B, T, H, D, act, head_major_x):
    o, z, w = norm_inputs(B, T, H, D, dtype, seed=B + 10 * T + 100 * H + D)
    o[0, 0, 0] = 0                                     # a zero row stays zero
    x = o if head_major_x else o.permute(0, 2, 1, 3).contiguous()
    x_tm = o.permute(0, 2, 1, 3)                       # [B, T, H, D] for the oracle
    ref = oracle.rms_norm_gated(f64(x_tm), f64(z), f64(w), eps=1e-6, activation=act)
    y = torch.full((B, T, H, D), float("nan"), dtype=dtype, device="cuda")
    dn.dn_rms_norm_gated(x.cuda(), z.cuda(), w.cuda(), y, eps=1e-6, x_head_major=head_major_x, activation=act)
    dn.dn_device_status()
    check(y.cpu(), ref, dtype, 1e-6, "y")
    assert not y[0, 0, 0].any()


@pytest.mark.gpu
def test_rms_norm_gated_layer_size_sampled(cuda_device):
    """The bench layer's output, o [4, 16, 4096, 128] bf16 head-major, against the
    oracle on 2048 sampled rows."""
    B, T, H, D = 4, 4096, 16, 128
    o, z, w = norm_inputs(B, T, H, D, torch.bfloat16, seed=31)
    y = torch.empty((B, T, H, D), dtype=torch.bfloat16, device="cuda")
    dn.dn_rms_norm_gated(o.cuda(), z.cuda(), w.cuda(), y)
    dn.dn_device_status()
    rng = np.random.default_rng(10)
    b, t, h = rng.integers(0, B, 2048), rng.integers(0, T, 2048), rng.integers(0, H, 2048)
    ref = oracle.rms_norm_gated(f64(o[b, h, t]), f64(z[b, t, h]), f64(w))
    check(y.cpu()[b, t, h], ref, torch.bfloat16, 1e-6, "sampled rows")
