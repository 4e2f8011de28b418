"""Packed batches of sequences on the GPU against the fp64 oracle ("Linear
attention and Gated DeltaNet", ch. 28, "The state a request carries": every
request carries its own fixed-size state, so a batch of ragged requests is N
independent runs, each from its own initial state to its own final state)."""
import numpy as np
import pytest
import torch

import delta_rule_recurrent_02_b200 as dn
import oracle
from _util import assert_close, f64

pytestmark = pytest.mark.gpu


def _packed(lens, H, seed, gate="scalar", s0_std=0.2):
    T = int(sum(lens))
    gen = torch.Generator().manual_seed(seed)
    unit = lambda x: x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    q = unit(torch.randn(1, H, T, 128, generator=gen)).to(torch.bfloat16)
    k = unit(torch.randn(1, H, T, 128, generator=gen)).to(torch.bfloat16)
    v = torch.randn(1, H, T, 128, generator=gen).to(torch.bfloat16)
    beta = torch.sigmoid(torch.randn(1, H, T, generator=gen))
    g = -torch.nn.functional.softplus(torch.randn(1, H, T, generator=gen) + 2) if gate == "scalar" else None
    N = len(lens)
    S0 = s0_std * torch.randn(N, H, 128, 128, generator=gen) if s0_std else None
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return dict(q=q, k=k, v=v, beta=beta, g=g, S0=S0, cu=cu)


def _run(inp, scale, gate, workspace=True):
    d = {n: (None if t is None else t.cuda()) for n, t in inp.items()}
    H, T = d["q"].shape[1], d["q"].shape[2]
    N = d["cu"].numel() - 1
    o = torch.full((1, H, T, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    S = torch.full((N, H, 128, 128), float("nan"), device="cuda")
    ws = None
    if workspace:
        nb = dn.dn_chunk_fwd_varlen_workspace_size(N, T, H, 128, 128, gate=gate)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    dn.dn_chunk_fwd_varlen(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], o, S, d["cu"], scale=scale,
                           gate=gate, workspace=ws)
    return o, S


def _oracle(inp, scale):
    return oracle.varlen_delta_rule(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["beta"]), f64(inp["g"]),
                                    inp["cu"].tolist(), f64(inp["S0"]), scale=scale)


@pytest.mark.parametrize("lens,H,gate", [
    ([300, 1, 64, 0, 129], 3, "scalar"),     # a 1-token and an empty sequence, ragged chunks
    ([64, 64, 64], 2, "none"),               # whole chunks only
    ([1000, 37, 517, 2, 65], 4, "scalar"),
    ([0, 0, 200], 2, "scalar"),              # leading empty sequences
    ([4096] * 3 + [1500, 2596], 8, "scalar"),
])
def test_varlen_matches_oracle(cuda_device, lens, H, gate):
    inp = _packed(lens, H, seed=sum(lens) + H, gate=gate)
    sc = 128 ** -0.5
    o, S = _run(inp, sc, gate)
    dn.dn_device_status()
    ro, rS = _oracle(inp, sc)
    assert_close(o, ro, "bf16", "o")
    assert_close(S, rS, "bf16", "S_T")


def test_varlen_equals_separate_calls(cuda_device):
    # each packed sequence gives what dn_chunk_fwd gives on it alone
    lens = [333, 64, 1, 700]
    inp = _packed(lens, 3, seed=9)
    sc = 128 ** -0.5
    o, S = _run(inp, sc, "scalar", workspace=False)     # the library allocates the workspace
    cu = inp["cu"].tolist()
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        part = {n: inp[n][:, :, a:b].contiguous().cuda() for n in ("q", "k", "v", "beta", "g")}
        o1, S1 = dn.chunk_fwd(part["q"], part["k"], part["v"], part["beta"], part["g"], inp["S0"][s:s + 1].cuda(),
                              scale=sc, path="tc")
        assert torch.equal(o[:, :, a:b], o1), f"sequence {s}: o"
        assert torch.equal(S[s:s + 1], S1), f"sequence {s}: S_T"
    dn.dn_device_status()


def test_varlen_no_initial_state(cuda_device):
    inp = _packed([130, 0, 70], 2, seed=4, s0_std=None)
    sc = 128 ** -0.5
    o, S = _run(inp, sc, "scalar")
    dn.dn_device_status()
    ro, rS = _oracle(inp, sc)
    assert_close(o, ro, "bf16", "o")
    assert_close(S, rS, "bf16", "S_T")
    assert torch.count_nonzero(S[1]) == 0      # the empty sequence's state is the zero initial state


def test_varlen_bad_offsets_reported(cuda_device):
    # offsets that do not rise from 0 to T: checked on the device (no host sync), nothing
    # is computed, every S_T is S0, and dn_device_status reports DN_ERR_INVALID
    inp = _packed([100, 100], 2, seed=5)
    inp["cu"] = torch.tensor([0, 150, 120], dtype=torch.int32)
    o, S = _run(inp, 1.0, "scalar")
    with pytest.raises(dn.DNError) as ei:
        dn.dn_device_status()
    assert ei.value.status == dn.DN_ERR_INVALID
    assert torch.equal(S.cpu(), inp["S0"])
    assert torch.isnan(o).all()
    # the context stays usable
    inp2 = _packed([50, 60], 2, seed=6)
    o2, S2 = _run(inp2, 1.0, "scalar")
    dn.dn_device_status()
    ro, rS = _oracle(inp2, 1.0)
    assert_close(o2, ro, "bf16", "o")


def test_varlen_rejects(cuda_device):
    inp = _packed([64, 64], 2, seed=1)
    d = {n: (None if t is None else t.cuda()) for n, t in inp.items()}
    o = torch.empty((1, 2, 128, 128), dtype=torch.bfloat16, device="cuda")
    S = torch.empty((2, 2, 128, 128), device="cuda")
    g_pk = torch.zeros(1, 2, 128, 128, device="cuda")
    with pytest.raises(dn.DNError) as ei:            # per-key gate: not on this path
        dn.dn_chunk_fwd_varlen(d["q"], d["k"], d["v"], d["beta"], g_pk, None, o, S, d["cu"], gate="per_key")
    assert ei.value.status == dn.DN_ERR_UNSUPPORTED
    q32 = d["q"].float()
    with pytest.raises(dn.DNError) as ei:            # fp32 tokens
        dn.dn_chunk_fwd_varlen(q32, q32, d["v"].float(), d["beta"], d["g"], None, o.float(), S, d["cu"])
    assert ei.value.status == dn.DN_ERR_UNSUPPORTED
