"""Chunked prefill on the GPU against the fp64 oracle ("Linear attention and
Gated DeltaNet", ch. 28, "The chunked form": same contract and result as the
recurrent form; its test plan: chunk sizes 1, 5, 8 and 64 on 37 tokens with a
non-zero initial state, because a chunk size of 1 hides a wrong triangle)."""
import numpy as np
import pytest
import torch

import delta_rule_recurrent_02_b200 as dn
import oracle
from delta_rule_recurrent_02_b200 import workloads as W
from _util import TOL, assert_close, f64, oracle_prefill, pick, to_dev

pytestmark = pytest.mark.gpu

PATHS = ["simt", "tc"]
# the tensor-core path covers bf16, chunk 64, d_k = d_v = 128 and every gate
TC_GATES = ("none", "scalar", "per_key")


def skip_unsupported(path, gate):
    if path == "tc" and gate not in TC_GATES:
        pytest.skip(f"{gate} gate runs on the SIMT path")


def run(d, scale, chunk=64, path="simt", gate=None):
    return dn.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], chunk=chunk,
                        scale=scale, path=path, gate=gate)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("gate", ["none", "scalar", "per_key"])
@pytest.mark.parametrize("chunk", [1, 5, 8, 16, 64])
@pytest.mark.parametrize("d", [64, 128])
def test_chunk_t37_nonzero_state(cuda_device, dtype, gate, chunk, d):
    inp = W.gen_prefill(2, 3, 37, d, d, dtype=dtype, gate=gate, seed=100 + chunk, s0_std=0.5,
                        g_shift=0.5)
    sc = d ** -0.5
    o, S = run(to_dev(inp), sc, chunk=chunk, path="simt")
    ro, rS = oracle_prefill(inp, sc)
    assert_close(o, ro, dtype, "o")
    assert_close(S, rS, dtype, "S_T")


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 517])
@pytest.mark.parametrize("gate", ["none", "scalar", "per_key"])
def test_chunk_ragged_lengths(cuda_device, path, T, gate):
    skip_unsupported(path, gate)
    inp = W.gen_prefill(2, 2, T, 128, 128, dtype="bf16", gate=gate, seed=T, s0_std=0.1)
    sc = 128 ** -0.5
    o, S = run(to_dev(inp), sc, path=path)
    ro, rS = oracle_prefill(inp, sc)
    assert_close(o, ro, "bf16", "o")
    assert_close(S, rS, "bf16", "S_T")


@pytest.mark.parametrize("path", PATHS)
def test_chunk_worked_example(cuda_device, path):
    # ch. 28 worked example, embedded at d = 128 (and 64 for SIMT): exact
    dims = [128] if path == "tc" else [64, 128]
    dts = [torch.bfloat16] if path == "tc" else [torch.float32, torch.bfloat16]
    for d in dims:
        for td in dts:
            q = torch.zeros(1, 1, 2, d, dtype=td, device="cuda"); q[0, 0, :, 0] = 1
            v = torch.zeros(1, 1, 2, d, dtype=td, device="cuda"); v[0, 0, :, 0] = 2; v[0, 0, :, 1] = 4
            beta = torch.tensor([[[0.5, 1.0]]], device="cuda")
            o, S = dn.chunk_fwd(q, q, v, beta, None, None, path=path)
            assert o[0, 0, 0, :2].float().tolist() == [1.0, 2.0]
            assert o[0, 0, 1, :2].float().tolist() == [2.0, 4.0]
            assert torch.count_nonzero(o[0, 0, :, 2:]) == 0
            assert S[0, 0, 0, :2].tolist() == [2.0, 4.0] and torch.count_nonzero(S) == 2


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T", [8, 24, 64, 200])
def test_chunk_reflection_parity_exact(cuda_device, path, T):
    # D2L 12.5, "The reflection hiding in the delta rule": k = e_1, S0 = e_1 e_1^T,
    # v = 0, beta_t = 2 x_t, q = e_1: o_t[0] = (-1)^(x_1 + ... + x_t), exactly.
    d = 128
    gen = torch.Generator().manual_seed(T)
    x = torch.randint(0, 2, (T,), generator=gen)
    td = torch.bfloat16
    k = torch.zeros(1, 1, T, d, dtype=td); k[..., 0] = 1
    v = torch.zeros(1, 1, T, d, dtype=td)
    S0 = torch.zeros(1, 1, d, d); S0[0, 0, 0, 0] = 1
    beta = (2.0 * x).float().reshape(1, 1, T)
    o, S = dn.chunk_fwd(k.cuda(), k.cuda(), v.cuda(), beta.cuda(), None, S0.cuda(), path=path)
    want = (-1.0) ** torch.cumsum(x, 0).double()
    assert torch.equal(o[0, 0, :, 0].double().cpu(), want)
    assert torch.count_nonzero(o[0, 0, :, 1:]) == 0


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("gate", ["scalar", "per_key"])
def test_chunk_beta_zero_pure_decay(cuda_device, path, gate):
    skip_unsupported(path, gate)
    # beta = 0: o_t = (Diag(e^Gamma_t) S0)^T (scale q_t), S_T = Diag(e^Gamma_T) S0.
    # A mild decay (g ~ -softplus(N(0,1) - 1)) keeps e^Gamma_T inside the fp32 range.
    inp = W.gen_prefill(1, 2, 100, 128, 128, dtype="bf16", gate=gate, seed=7, s0_std=0.1, g_shift=-1.0)
    inp["beta"].zero_()
    sc = 128 ** -0.5
    o, S = run(to_dev(inp), sc, path=path)
    g = f64(inp["g"])
    lg = np.repeat(g[..., None], 128, -1) if g.ndim == 3 else g
    Gam = np.cumsum(lg, axis=2)
    want_o = np.einsum("bhtc,bhcj,bhtc->bhtj", np.exp(Gam), f64(inp["S0"]), sc * f64(inp["q"]))
    assert_close(o, want_o, "bf16", "o")
    assert_close(S, np.exp(Gam[:, :, -1])[..., None] * f64(inp["S0"]), "f32", "S_T")


@pytest.mark.parametrize("path", PATHS)
def test_chunk_resume_through_state(cuda_device, path):
    inp = W.gen_prefill(2, 4, 300, 128, 128, dtype="bf16", gate="scalar", seed=9, s0_std=0.1)
    d = to_dev(inp)
    sc = 128 ** -0.5
    o, S = run(d, sc, path=path)
    cut = 128
    first = {n: (None if t is None or n == "S0" else t[:, :, :cut].contiguous()) for n, t in d.items()}
    first["S0"] = d["S0"]
    second = {n: (None if t is None or n == "S0" else t[:, :, cut:].contiguous()) for n, t in d.items()}
    o1, S1 = run(first, sc, path=path)
    second["S0"] = S1
    o2, S2 = run(second, sc, path=path)
    ro, rS = oracle_prefill(inp, sc)
    assert_close(torch.cat([o1, o2], dim=2), ro, "bf16", "o (resumed)")
    assert_close(S2, rS, "bf16", "S_T (resumed)")
    # in-place continuation: S_T may be the same buffer as S0
    S_inplace = S1.clone()
    dn.dn_chunk_fwd(second["q"], second["k"], second["v"], second["beta"], second["g"], S_inplace,
                    torch.empty_like(o2), S_inplace, scale=sc, path=path)
    assert_close(S_inplace, rS, "bf16", "S_T (in place)")


@pytest.mark.parametrize("path", PATHS)
def test_chunk_overwrites_poisoned_outputs(cuda_device, path):
    inp = W.gen_prefill(2, 3, 130, 128, 128, dtype="bf16", gate="scalar", seed=11)
    d = to_dev(inp)
    o = torch.full((2, 3, 130, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    S = torch.full((2, 3, 128, 128), float("nan"), device="cuda")
    dn.dn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], None, o, S, scale=0.1, path=path)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()


def test_tc_workspace_caller_internal_and_poisoned(cuda_device):
    # the tensor-core path keeps -W, u^T and P of every chunk in a workspace: a
    # caller's buffer (poisoned with NaN first: it is scratch, nothing is read
    # before it is written) and the library's own stream-ordered allocation
    # give bit-identical results, which match the oracle
    inp = W.gen_prefill(2, 3, 200, 128, 128, dtype="bf16", gate="scalar", seed=12, s0_std=0.2)
    d = to_dev(inp)
    sc = 128 ** -0.5
    nbytes = dn.dn_chunk_fwd_workspace_size(2, 200, 3, 128, 128, path="tc")
    assert nbytes == 2 * 3 * 4 * 41216 + 256
    ws = torch.full((nbytes // 2,), float("nan"), dtype=torch.bfloat16, device="cuda")
    outs = []
    for w in (ws, None):
        o = torch.empty((2, 3, 200, 128), dtype=torch.bfloat16, device="cuda")
        S = torch.empty((2, 3, 128, 128), device="cuda")
        dn.dn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], o, S, scale=sc, path="tc",
                        workspace=w)
        outs.append((o, S))
    dn.dn_device_status()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    ro, rS = oracle_prefill(inp, sc)
    assert_close(outs[0][0], ro, "bf16", "o")
    assert_close(outs[0][1], rS, "bf16", "S_T")
    with pytest.raises(dn.DNError) as ei:
        dn.dn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], outs[0][0], outs[0][1], scale=sc,
                        path="tc", workspace=ws[: nbytes // 4])
    assert ei.value.status == dn.DN_ERR_INVALID


@pytest.mark.parametrize("gate", ["none", "scalar", "per_key"])
def test_tc_workspace_reused_back_to_back(cuda_device, gate):
    # one caller workspace for calls A, B, A on the same stream: each call clears its ready
    # flags and tile counter, its WY groups load the next tile's K and Q ahead, and its
    # state passes drop the tiles they consumed from L2, so nothing of one call may leak
    # into the next: the repeated A is bit-identical to the first, and both match the oracle
    B, H, T = 2, 8, 1000
    sc = 128 ** -0.5
    nb = dn.dn_chunk_fwd_workspace_size(B, T, H, 128, 128, gate=gate, path="tc")
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    ins = [W.gen_prefill(B, H, T, 128, 128, dtype="bf16", gate=gate, seed=s, s0_std=0.3) for s in (21, 22)]
    outs = []
    for which in (0, 1, 0):
        d = to_dev(ins[which])
        o = torch.full((B, H, T, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        S = torch.full((B, H, 128, 128), float("nan"), device="cuda")
        dn.dn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], o, S, scale=sc, path="tc",
                        gate=gate, workspace=ws)
        outs.append((o, S))
    dn.dn_device_status()
    assert torch.equal(outs[0][0], outs[2][0]) and torch.equal(outs[0][1], outs[2][1])
    for which, (o, S) in zip((0, 1), outs[:2]):
        ro, rS = oracle_prefill(ins[which], sc)
        assert_close(o, ro, "bf16", "o")
        assert_close(S, rS, "bf16", "S_T")


@pytest.mark.parametrize("B,H,T", [(3, 32, 200), (4, 32, 130)])
@pytest.mark.parametrize("gate", ["scalar", "per_key"])
def test_tc_many_heads(cuda_device, B, H, T, gate):
    # 96 heads: the single launch (scalar gate: each state-pass CTA also hosts a
    # WY group); 128 heads: the two launches (WY kernel, then state pass)
    inp = W.gen_prefill(B, H, T, 128, 128, dtype="bf16", gate=gate, seed=B * H + T, s0_std=0.2)
    sc = 128 ** -0.5
    o, S = run(to_dev(inp), sc, path="tc")
    dn.dn_device_status()
    bh = [(0, 0), (1, 7), (B - 1, H - 1), (B // 2, H // 2)]
    ro, rS = oracle_prefill(inp, sc, bh=bh)
    assert_close(pick(o, bh), ro, "bf16", "o")
    assert_close(pick(S, bh), rS, "bf16", "S_T")


@pytest.mark.parametrize("B,H,T,path,kernels", [
    (4, 16, 4096, "tc", 1),      # the cooperative launch: WY groups beside the state pass
    (3, 32, 200, "tc", 1),       # the same, each state-pass CTA hosting a WY group
    (4, 32, 130, "tc", 2),       # too many heads for one launch: WY kernel, then state pass
    (2, 3, 200, "simt", 1),
])
@pytest.mark.parametrize("gate", ["scalar", "per_key"])
def test_chunk_kernel_launch_count(cuda_device, B, H, T, path, kernels, gate):
    inp = W.gen_prefill(B, H, T, 128, 128, dtype="bf16", gate=gate, seed=5, s0_std=0.2)
    d = to_dev(inp)
    torch.cuda.synchronize()
    before = dn.dn_kernel_launches()
    run(d, 0.1, path=path)
    assert dn.dn_kernel_launches() - before == kernels
    dn.dn_device_status()


def test_chunk_empty_inputs(cuda_device):
    # T = 0: no output rows; S_T = S0 (or zeros).  B = 0: nothing at all.
    S0 = torch.randn(2, 3, 64, 64, device="cuda")
    z = lambda *s, dt=torch.float32: torch.zeros(*s, dtype=dt, device="cuda")
    S_T = torch.full_like(S0, float("nan"))
    dn.dn_chunk_fwd(z(2, 3, 0, 64), z(2, 3, 0, 64), z(2, 3, 0, 64), z(2, 3, 0), None, S0,
                    z(2, 3, 0, 64), S_T, chunk=16)
    assert torch.equal(S_T, S0)
    dn.dn_chunk_fwd(z(2, 3, 0, 64), z(2, 3, 0, 64), z(2, 3, 0, 64), z(2, 3, 0), None, None,
                    z(2, 3, 0, 64), S_T, chunk=16)
    assert torch.count_nonzero(S_T) == 0
    o, S = dn.chunk_fwd(z(0, 3, 5, 64), z(0, 3, 5, 64), z(0, 3, 5, 64), z(0, 3, 5), None, None)
    assert o.shape == (0, 3, 5, 64)


def test_chunk_errors_on_device(cuda_device):
    q = torch.zeros(1, 1, 8, 64, device="cuda")
    beta = torch.zeros(1, 1, 8, device="cuda")
    with pytest.raises(dn.DNError) as ei:
        dn.chunk_fwd(q, q, q, beta, None, None, chunk=65, path="simt")
    assert ei.value.status == dn.DN_ERR_UNSUPPORTED
    with pytest.raises(dn.DNError) as ei:
        dn.chunk_fwd(q, q, q, beta, None, None, path="tc")   # fp32 is not on the tensor-core path
    assert ei.value.status == dn.DN_ERR_UNSUPPORTED
    with pytest.raises(dn.DNError) as ei:
        dn.chunk_fwd(q, q, q, beta, None, None, gate="scalar")   # gate without g
    assert ei.value.status == dn.DN_ERR_INVALID


# --- the five workloads at full size -----------------------------------------

def test_deltanet_small_full(cuda_device):
    cfg = W.DELTANET_SMALL
    inp = W.gen_prefill_config(cfg)
    o, S = run(to_dev(inp), cfg.scale, chunk=cfg.chunk, path="simt")
    ro, rS = oracle_prefill(inp, cfg.scale)
    assert_close(o, ro, "f32", "o")
    assert_close(S, rS, "f32", "S_T")


@pytest.mark.parametrize("path", PATHS)
def test_gated_deltanet_full(cuda_device, path):
    cfg = W.GDN_PREFILL
    inp = W.gen_prefill_config(cfg)
    o, S = run(to_dev(inp), cfg.scale, chunk=cfg.chunk, path=path)
    ro, rS = oracle_prefill(inp, cfg.scale)
    assert_close(o, ro, "bf16", "o")
    assert_close(S, rS, "bf16", "S_T")


_FULL_ORACLE = {}


def _full_oracle(cfg):
    """Inputs and the oracle's o, S_T on every head of a workload, computed once
    per test session and shared by both kernel paths."""
    if cfg.name not in _FULL_ORACLE:
        inp = W.gen_prefill_config(cfg)
        _FULL_ORACLE.clear()                # one workload's arrays at a time
        _FULL_ORACLE[cfg.name] = (inp, oracle_prefill(inp, cfg.scale))
    return _FULL_ORACLE[cfg.name]


def _every_head(cfg, path):
    # every (b, h) of the workload against the oracle: the kernels hand tiles to their
    # groups from a shared counter, so a fault in that scheduling could hit any head
    inp, (ro, rS) = _full_oracle(cfg)
    o, S = run(to_dev(inp), cfg.scale, chunk=cfg.chunk, path=path)
    dn.dn_device_status()
    assert_close(o, ro, "bf16", "o (every head)")
    assert_close(S, rS, "bf16", "S_T (every head)")


@pytest.mark.parametrize("path", ["tc", "simt"])
def test_gated_deltanet_long_full(cuda_device, path):
    _every_head(W.GDN_LONG, path)


@pytest.mark.parametrize("path", ["tc", "simt"])
def test_kda_full(cuda_device, path):
    _every_head(W.KDA_PREFILL, path)


@pytest.mark.parametrize("g_shift", [-1.0, 8.0])
def test_kda_tc_weak_and_strong_decay(cuda_device, g_shift):
    # per-key gate on tensor cores: g = -softplus(N(0,1) + shift) per channel; shift 8
    # decays each channel by about e^-64 over 8 tokens, near the e^-80 bound of the
    # gram's split around each 16-token block's middle; shift -1 barely decays
    inp = W.gen_prefill(2, 3, 200, 128, 128, dtype="bf16", gate="per_key", seed=31, s0_std=0.2,
                        g_shift=g_shift)
    sc = 128 ** -0.5
    o, S = run(to_dev(inp), sc, path="tc")
    dn.dn_device_status()
    ro, rS = oracle_prefill(inp, sc)
    assert_close(o, ro, "bf16", "o")
    assert_close(S, rS, "bf16", "S_T")


def test_kda_tc_matches_simt_path(cuda_device):
    # the two kernels share no code: the tensor-core and fp32 paths agree to bf16 rounding
    inp = W.gen_prefill(1, 4, 333, 128, 128, dtype="bf16", gate="per_key", seed=7, s0_std=0.3, g_shift=3.0)
    sc = 128 ** -0.5
    d = to_dev(inp)
    o1, S1 = run(d, sc, path="tc")
    o2, S2 = run(d, sc, path="simt")
    dn.dn_device_status()
    assert_close(o1, f64(o2), "bf16", "o (tc vs simt)")
    assert_close(S1, f64(S2), "bf16", "S_T (tc vs simt)")


def _prefix(inp, t_end):
    """The same problem cut to its first t_end tokens (S0 unchanged)."""
    out = {}
    for name, t in inp.items():
        out[name] = None if t is None or name == "S0" else t[:, :, :t_end].contiguous()
    out["S0"] = inp["S0"]
    return out


@pytest.mark.parametrize("path,gate,chunk", [("simt", "scalar", 16), ("simt", "per_key", 64), ("tc", "none", 64),
                                             ("tc", "scalar", 64), ("tc", "per_key", 64)])
@pytest.mark.parametrize("T,every", [(300, 2), (256, 1)])
def test_chunk_state_snapshots(cuda_device, path, gate, chunk, T, every):
    # snapshot s is the state after the first (s + 1) * every * chunk tokens, i.e. the
    # final state of that prefix (the oracle's S_T on the cut problem); a partial last
    # chunk has none.  With T = 256 and every = 1 the last snapshot is S_T itself.
    inp = W.gen_prefill(2, 3, T, 128, 128, dtype="bf16", gate=gate, seed=T + every, s0_std=0.2)
    d = to_dev(inp)
    sc = 128 ** -0.5
    n_snap = T // (every * chunk)
    snaps = torch.full((2, 3, n_snap, 128, 128), float("nan"), device="cuda")
    o = torch.empty((2, 3, T, 128), dtype=torch.bfloat16, device="cuda")
    S = torch.empty((2, 3, 128, 128), device="cuda")
    dn.dn_chunk_fwd_snapshots(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], o, S, snaps, every,
                              chunk=chunk, scale=sc, path=path)
    dn.dn_device_status()
    ro, rS = oracle_prefill(inp, sc)
    assert_close(o, ro, "bf16", "o")
    assert_close(S, rS, "bf16", "S_T")
    for s in range(n_snap):
        _, rs = oracle_prefill(_prefix(inp, (s + 1) * every * chunk), sc)
        assert_close(snaps[:, :, s], rs, "bf16", f"snapshot {s}")
    if T % (every * chunk) == 0:
        assert torch.equal(snaps[:, :, -1], S)


def _gdn_raw(B, H, T, seed, zero_rows=False):
    """Raw layer inputs: q and k of varied norms (not normalised), b and a ~ N(0,1),
    A_log = log U(1, 16), dt_bias ~ N(0, 0.5)."""
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, T, 128, generator=gen) * (0.2 + 3 * torch.rand(B, H, T, 1, generator=gen))
    k = torch.randn(B, H, T, 128, generator=gen) * (0.2 + 3 * torch.rand(B, H, T, 1, generator=gen))
    if zero_rows:
        q[0, 0, 5] = 0.0
        k[0, 0, 7] = 0.0
    v = torch.randn(B, H, T, 128, generator=gen)
    b = torch.randn(B, H, T, generator=gen)
    a = torch.randn(B, H, T, generator=gen)
    A_log = torch.log(1 + 15 * torch.rand(H, generator=gen))
    dt_bias = 0.5 * torch.randn(H, generator=gen)
    S0 = 0.2 * torch.randn(B, H, 128, 128, generator=gen)
    return {"q": q.to(torch.bfloat16), "k": k.to(torch.bfloat16), "v": v.to(torch.bfloat16), "b": b, "a": a,
            "A_log": A_log, "dt_bias": dt_bias, "S0": S0}


def _gdn_oracle(raw, scale, bh=None):
    qn, kn, beta, g = oracle.gdn_prologue(f64(raw["q"]), f64(raw["k"]), f64(raw["b"]), f64(raw["a"]),
                                          f64(raw["A_log"]), f64(raw["dt_bias"]))
    inp = {"q": torch.from_numpy(qn), "k": torch.from_numpy(kn), "v": raw["v"], "beta": torch.from_numpy(beta),
           "g": torch.from_numpy(g), "S0": raw["S0"]}
    return oracle_prefill(inp, scale, bh=bh)


@pytest.mark.parametrize("B,H,T", [(2, 3, 200), (1, 2, 64), (3, 32, 200), (4, 32, 130)])
def test_gdn_layer_prologue(cuda_device, B, H, T):
    # 6 heads and 2 heads: the single launch; 96 heads: hosted WY groups; 128 heads: two launches
    raw = _gdn_raw(B, H, T, seed=B * 100 + H + T, zero_rows=True)
    d = to_dev(raw)
    sc = 128 ** -0.5
    o = torch.full((B, H, T, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    S = torch.full((B, H, 128, 128), float("nan"), device="cuda")
    dn.dn_chunk_fwd_gdn(d["q"], d["k"], d["v"], d["b"], d["a"], d["A_log"], d["dt_bias"], d["S0"], o, S, scale=sc)
    dn.dn_device_status()
    ro, rS = _gdn_oracle(raw, sc)
    assert_close(o, ro, "bf16", "o")
    assert_close(S, rS, "bf16", "S_T")


def test_gdn_layer_prologue_full_size(cuda_device):
    B, H, T = 4, 16, 4096
    raw = _gdn_raw(B, H, T, seed=9)
    d = to_dev(raw)
    sc = 128 ** -0.5
    o = torch.empty((B, H, T, 128), dtype=torch.bfloat16, device="cuda")
    S = torch.empty((B, H, 128, 128), device="cuda")
    dn.dn_chunk_fwd_gdn(d["q"], d["k"], d["v"], d["b"], d["a"], d["A_log"], d["dt_bias"], d["S0"], o, S, scale=sc)
    dn.dn_device_status()
    # every head
    ro, rS = _gdn_oracle(raw, sc)
    assert_close(o, ro, "bf16", "o (every head)")
    assert_close(S, rS, "bf16", "S_T (every head)")


def _gdn_raw_d(B, H, T, d, dtype, seed):
    """As _gdn_raw, at head size d and token dtype `dtype`."""
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, T, d, generator=gen) * (0.2 + 3 * torch.rand(B, H, T, 1, generator=gen))
    k = torch.randn(B, H, T, d, generator=gen) * (0.2 + 3 * torch.rand(B, H, T, 1, generator=gen))
    q[0, 0, 3] = 0.0
    k[-1, -1, T // 2] = 0.0
    v = torch.randn(B, H, T, d, generator=gen)
    b = torch.randn(B, H, T, generator=gen)
    a = torch.randn(B, H, T, generator=gen) - 1.0
    A_log = torch.log(1 + 3 * torch.rand(H, generator=gen))
    dt_bias = 0.5 * torch.randn(H, generator=gen)
    S0 = 0.2 * torch.randn(B, H, d, d, generator=gen)
    return {"q": q.to(dtype), "k": k.to(dtype), "v": v.to(dtype), "b": b, "a": a, "A_log": A_log,
            "dt_bias": dt_bias, "S0": S0}


@pytest.mark.parametrize("neg", [False, True])
@pytest.mark.parametrize("path,dtype,d,chunk", [
    ("tc", torch.bfloat16, 128, 64),
    ("simt", torch.float32, 64, 64),
    ("simt", torch.float32, 128, 16),
    ("simt", torch.bfloat16, 128, 64),
    ("simt", torch.bfloat16, 64, 5),
])
def test_gdn_prologue_ex_both_paths(cuda_device, neg, path, dtype, d, chunk):
    # dn_chunk_fwd_gdn_ex: the layer's prologue on the tensor-core kernels and on the
    # fp32 CUDA-core kernel; with allow_neg_eigval, beta = 2 sigmoid(b) ("DeltaNet:
    # Memory That Edits", "The reflection hiding in the delta rule")
    B, H, T = 2, 3, 150
    raw = _gdn_raw_d(B, H, T, d, dtype, seed=1000 + d + chunk + 7 * neg)
    dd = to_dev(raw)
    sc = d ** -0.5
    o = torch.full((B, H, T, d), float("nan"), dtype=dtype, device="cuda")
    S = torch.full((B, H, d, d), float("nan"), device="cuda")
    nb = dn.dn_chunk_fwd_workspace_size(B, T, H, d, d, chunk=chunk, dtype="bf16" if dtype == torch.bfloat16 else "f32",
                                        gate="scalar", path=path)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda") if nb else None
    dn.dn_chunk_fwd_gdn_ex(dd["q"], dd["k"], dd["v"], dd["b"], dd["a"], dd["A_log"], dd["dt_bias"], dd["S0"], o, S,
                           chunk=chunk, scale=sc, path=path, allow_neg_eigval=neg, workspace=ws)
    dn.dn_device_status()
    qn, kn, beta, g = oracle.gdn_prologue(f64(raw["q"]), f64(raw["k"]), f64(raw["b"]), f64(raw["a"]),
                                          f64(raw["A_log"]), f64(raw["dt_bias"]), allow_neg_eigval=neg)
    ro, rS = oracle.delta_rule(qn, kn, f64(raw["v"]), beta, g, f64(raw["S0"]), scale=sc)
    kind = "f32" if dtype == torch.float32 else "bf16"
    assert_close(o, ro, kind, "o")
    assert_close(S, rS, kind, "S_T")


def test_gdn_prologue_ex_rejects_unknown_flags(cuda_device):
    raw = _gdn_raw_d(1, 1, 8, 128, torch.bfloat16, seed=3)
    dd = to_dev(raw)
    o = torch.empty((1, 1, 8, 128), dtype=torch.bfloat16, device="cuda")
    lib = dn.load_library()
    st = lib.dn_chunk_fwd_gdn_ex(dd["q"].data_ptr(), dd["k"].data_ptr(), dd["v"].data_ptr(), dd["b"].data_ptr(),
                                 dd["a"].data_ptr(), dd["A_log"].data_ptr(), dd["dt_bias"].data_ptr(), None,
                                 o.data_ptr(), None, 1, 8, 1, 128, 128, 64, 1.0, 1, 0, 4, None, None, 0.0, None, 0,
                                 None)
    assert st == dn.DN_ERR_INVALID


@pytest.mark.parametrize("activation", ["silu", "sigmoid"])
@pytest.mark.parametrize("B,H,T", [(2, 3, 150), (1, 2, 64), (3, 32, 100), (4, 16, 1024), (4, 32, 130)])
def test_gdn_prologue_and_gated_norm(cuda_device, activation, B, H, T):
    # dn_chunk_fwd_gdn_ex with z: the layer's prologue, the rule and the gated RMSNorm
    # ("The full layer", steps 4-7) in the tensor-core kernels, against
    # oracle.rms_norm_gated on the oracle recurrence's read-out (token-major y);
    # 6 and 2 heads: the single launch; 96 heads: hosted WY groups; 64 heads, long
    raw = _gdn_raw(B, H, T, seed=B * 7 + H + T, zero_rows=True)
    gen = torch.Generator().manual_seed(T + H)
    z = (2 * torch.randn(B, T, H, 128, generator=gen)).to(torch.bfloat16)
    w = 1 + 0.5 * torch.randn(128, generator=gen)
    d = to_dev(raw)
    sc = 128 ** -0.5
    y = torch.full((B, T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    S = torch.full((B, H, 128, 128), float("nan"), device="cuda")
    dn.dn_chunk_fwd_gdn_ex(d["q"], d["k"], d["v"], d["b"], d["a"], d["A_log"], d["dt_bias"], d["S0"], y, S,
                           scale=sc, path="tc", z=z.cuda(), norm_weight=w.cuda(), eps=1e-6,
                           norm_activation=activation)
    dn.dn_device_status()
    ro, rS = _gdn_oracle(raw, sc)
    ry = oracle.rms_norm_gated(ro.transpose(0, 2, 1, 3), f64(z), f64(w), eps=1e-6, activation=activation)
    assert_close(y.permute(0, 2, 1, 3), ry.transpose(0, 2, 1, 3), "bf16", "y")
    assert_close(S, rS, "bf16", "S_T")


def test_gdn_norm_needs_tensor_cores(cuda_device):
    raw = _gdn_raw_d(1, 1, 8, 64, torch.float32, seed=2)
    d = to_dev(raw)
    y = torch.empty((1, 8, 1, 64), device="cuda")
    with pytest.raises(dn.DNError) as ei:
        dn.dn_chunk_fwd_gdn_ex(d["q"], d["k"], d["v"], d["b"], d["a"], d["A_log"], d["dt_bias"], None, y, None,
                               path="simt", z=torch.zeros(1, 8, 1, 64, device="cuda"),
                               norm_weight=torch.ones(64, device="cuda"))
    assert ei.value.status == dn.DN_ERR_UNSUPPORTED
