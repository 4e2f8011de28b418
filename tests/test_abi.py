"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point ``include/dn.h`` declares, and rejects bad arguments before
touching the device."""
import ctypes
import os
import re

import pytest

import delta_rule_recurrent_02_b200 as dn
from delta_rule_recurrent_02_b200 import build as dn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    dn_build.build()
    return dn.load_library()


def declared_symbols():
    with open(os.path.join(ROOT, "include", "dn.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"DN_API\s+[\w\s\*]+?\b(dn_\w+)\s*\(", text)))


def test_header_declares_abi():
    assert declared_symbols() == sorted(dn.ABI_SYMBOLS)


def test_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert lib.dn_version() >> 16 == 2 and lib.dn_version() & 0xffff >= 2
    for code in range(5):
        assert lib.dn_status_str(code).startswith(b"DN_")
    assert lib.dn_status_str(99) == b"unknown dn_status"


# Fake, never dereferenced addresses: validation must fail before any CUDA call.
A = 0x10000000
STEP = 0x01000000


def chunk_call(lib, **over):
    args = dict(q=A, k=A + STEP, v=A + 2 * STEP, beta=A + 3 * STEP, g=A + 4 * STEP, S0=None,
                o=A + 5 * STEP, S_T=A + 6 * STEP, B=1, T=8, H=1, dk=64, dv=64, chunk=8,
                scale=1.0, dtype=0, gate=1, path=0, ws=None, ws_bytes=0)
    args.update(over)
    return lib.dn_chunk_fwd_ex(args["q"], args["k"], args["v"], args["beta"], args["g"], args["S0"],
                               args["o"], args["S_T"], args["B"], args["T"], args["H"], args["dk"],
                               args["dv"], args["chunk"], args["scale"], args["dtype"], args["gate"],
                               args["path"], args["ws"], args["ws_bytes"], None)


# a request the tensor-core path covers (bf16, chunk 64, d_k = d_v = 128)
TC = dict(dtype=1, dk=128, dv=128, chunk=64, path=2)
WS = A + 8 * STEP


@pytest.mark.parametrize("over,code", [
    (dict(B=-1), dn.DN_ERR_INVALID),
    (dict(T=-3), dn.DN_ERR_INVALID),
    (dict(q=None), dn.DN_ERR_INVALID),
    (dict(o=None), dn.DN_ERR_INVALID),
    (dict(g=None), dn.DN_ERR_INVALID),                       # scalar gate needs g
    (dict(gate=0), dn.DN_ERR_INVALID),                       # no gate but g given
    (dict(gate=7), dn.DN_ERR_INVALID),
    (dict(dtype=5), dn.DN_ERR_INVALID),
    (dict(path=9), dn.DN_ERR_INVALID),
    (dict(chunk=0), dn.DN_ERR_INVALID),
    (dict(scale=float("nan")), dn.DN_ERR_INVALID),
    (dict(q=A + 8), dn.DN_ERR_INVALID),                       # not 16-byte aligned
    (dict(beta=A + 3 * STEP + 2), dn.DN_ERR_INVALID),         # not 4-byte aligned
    (dict(gate=2, g=A + 4 * STEP + 4), dn.DN_ERR_INVALID),    # per-key g not 16-byte aligned
    (dict(o=A + 64), dn.DN_ERR_INVALID),                      # o overlaps q
    (dict(S_T=A + 2 * STEP), dn.DN_ERR_INVALID),              # S_T overlaps v
    (dict(S0=A + 7 * STEP, S_T=A + 7 * STEP + 256), dn.DN_ERR_INVALID),  # partial overlap
    (dict(dk=96), dn.DN_ERR_UNSUPPORTED),
    (dict(dv=256), dn.DN_ERR_UNSUPPORTED),
    (dict(path=2), dn.DN_ERR_UNSUPPORTED),                    # tensor-core path needs bf16, d = 128
    (dict(path=3), dn.DN_ERR_UNSUPPORTED),                    # so does its self-test
    (dict(TC, ws=WS, ws_bytes=41216 + 255), dn.DN_ERR_INVALID),     # workspace smaller than one chunk's tiles
    (dict(TC, ws=WS + 128, ws_bytes=1 << 20), dn.DN_ERR_INVALID),   # not 256-byte aligned
    (dict(TC, ws=A + 256, ws_bytes=1 << 20), dn.DN_ERR_INVALID),    # overlaps q
    (dict(TC, ws=A + 6 * STEP, ws_bytes=1 << 20), dn.DN_ERR_INVALID),  # overlaps S_T
])
def test_chunk_fwd_rejects(lib, over, code):
    before = lib.dn_kernel_launches()
    assert chunk_call(lib, **over) == code
    assert lib.dn_last_error() != b""
    assert lib.dn_kernel_launches() == before        # refused before any launch


def ws_size(lib, B=2, T=130, H=3, dk=128, dv=128, chunk=64, dtype=1, gate=1, path=0):
    out = ctypes.c_size_t(12345)
    st = lib.dn_chunk_fwd_workspace_size(B, T, H, dk, dv, chunk, dtype, gate, path, ctypes.byref(out))
    return st, out.value


def test_workspace_size():
    lib = dn.load_library()
    # -W and u^T (bf16, 64 x 128 each), P (bf16, 64 x 64) and 1 / ||q|| (fp32, 64) per (b, h, chunk), then
    # a 4-byte ready flag per chunk rounded up to 256 bytes: ceil(130 / 64) = 3 chunks
    tiles = 2 * 3 * 3
    assert ws_size(lib) == (dn.DN_OK, tiles * ((2 * 64 * 128 + 64 * 64) * 2 + 64 * 4) + 256)
    assert ws_size(lib, path=2) == (dn.DN_OK, tiles * 41216 + 256)
    # per-key gate: also K~ and Qh (bf16, 64 x 128 each) and e^Gamma_last (fp32, 128) per chunk
    assert ws_size(lib, gate=2, path=2) == (dn.DN_OK, tiles * (41216 + 2 * 16384 + 512) + 256)
    assert ws_size(lib, gate=2, path=1) == (dn.DN_OK, 0)
    assert ws_size(lib, T=0) == (dn.DN_OK, 0)
    assert ws_size(lib, path=1) == (dn.DN_OK, 0)             # SIMT needs none
    assert ws_size(lib, dtype=0) == (dn.DN_OK, 0)            # fp32 runs on SIMT under auto
    assert ws_size(lib, gate=2) == ws_size(lib, gate=2, path=2)   # the per-key gate runs on tensor cores
    assert ws_size(lib, dtype=0, path=2)[0] == dn.DN_ERR_UNSUPPORTED
    assert ws_size(lib, B=-1) == (dn.DN_ERR_INVALID, 12345)  # not written on failure
    assert lib.dn_chunk_fwd_workspace_size(1, 8, 1, 128, 128, 64, 1, 1, 0, None) == dn.DN_ERR_INVALID
    assert dn.dn_chunk_fwd_workspace_size(1, 64, 1, 128, 128) == 41216 + 256


def test_chunk_fwd_empty_batch_is_ok_without_device(lib):
    assert chunk_call(lib, B=0) == dn.DN_OK
    assert chunk_call(lib, H=0, q=None, k=None, v=None, beta=None, g=None, o=None) == dn.DN_OK


def decode_call(lib, **over):
    args = dict(q=A, k=A + STEP, v=A + 2 * STEP, beta=A + 3 * STEP, g=A + 4 * STEP,
                S=A + 5 * STEP, o=A + 6 * STEP, B=2, H=3, dk=128, dv=128, scale=1.0, dtype=1, gate=1)
    args.update(over)
    return lib.dn_decode_step(args["q"], args["k"], args["v"], args["beta"], args["g"], args["S"],
                              args["o"], args["B"], args["H"], args["dk"], args["dv"], args["scale"],
                              args["dtype"], args["gate"], None)


@pytest.mark.parametrize("over,code", [
    (dict(B=-2), dn.DN_ERR_INVALID),
    (dict(S=None), dn.DN_ERR_INVALID),
    (dict(g=None), dn.DN_ERR_INVALID),
    (dict(o=A + 5 * STEP + 4096), dn.DN_ERR_INVALID),         # o inside S
    (dict(S=A + 32), dn.DN_ERR_INVALID),                      # S overlaps q
    (dict(k=A + STEP + 4), dn.DN_ERR_INVALID),
    (dict(dk=32), dn.DN_ERR_UNSUPPORTED),
])
def test_decode_rejects(lib, over, code):
    assert decode_call(lib, **over) == code


def test_decode_empty_is_ok(lib):
    assert decode_call(lib, B=0) == dn.DN_OK


def test_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 1, 8, 64)
    with pytest.raises(ValueError):
        dn.dn_chunk_fwd(q, q, q, torch.zeros(1, 1, 8), None, None, torch.zeros(1, 1, 8, 64), None)


def snap_call(lib, snaps, every, **over):
    args = dict(q=A, k=A + STEP, v=A + 2 * STEP, beta=A + 3 * STEP, g=A + 4 * STEP, S0=None,
                o=A + 5 * STEP, S_T=A + 6 * STEP, B=1, T=128, H=1, dk=64, dv=64, chunk=16,
                scale=1.0, dtype=0, gate=1, path=1)
    args.update(over)
    return lib.dn_chunk_fwd_snapshots(args["q"], args["k"], args["v"], args["beta"], args["g"], args["S0"],
                                      args["o"], args["S_T"], snaps, every, args["B"], args["T"], args["H"],
                                      args["dk"], args["dv"], args["chunk"], args["scale"], args["dtype"],
                                      args["gate"], args["path"], None, 0, None)


@pytest.mark.parametrize("snaps,every,what", [
    (A + 9 * STEP, 0, "every"),              # every must be >= 1
    (A + 9 * STEP + 8, 1, "aligned"),        # not 16-byte aligned
    (A + 2 * STEP + 64, 1, "overlaps"),      # overlaps v
    (A + 6 * STEP, 2, "overlaps"),           # overlaps S_T
])
def test_chunk_snapshots_rejects(lib, snaps, every, what):
    before = lib.dn_kernel_launches()
    assert snap_call(lib, snaps, every) == dn.DN_ERR_INVALID
    assert what in lib.dn_last_error().decode()
    assert lib.dn_kernel_launches() == before


def gdn_call(lib, **over):
    args = dict(q=A, k=A + STEP, v=A + 2 * STEP, b=A + 3 * STEP, a=A + 4 * STEP, A_log=A + 10 * STEP,
                dt_bias=A + 11 * STEP, S0=None, o=A + 5 * STEP, S_T=A + 6 * STEP, B=1, T=128, H=2, dk=128, dv=128)
    args.update(over)
    return lib.dn_chunk_fwd_gdn(args["q"], args["k"], args["v"], args["b"], args["a"], args["A_log"],
                                args["dt_bias"], args["S0"], args["o"], args["S_T"], args["B"], args["T"],
                                args["H"], args["dk"], args["dv"], 1.0, None, 0, None)


@pytest.mark.parametrize("over,code", [
    (dict(A_log=None), dn.DN_ERR_INVALID),
    (dict(dt_bias=None), dn.DN_ERR_INVALID),
    (dict(A_log=A + 10 * STEP + 2), dn.DN_ERR_INVALID),     # not 4-byte aligned
    (dict(dt_bias=A + 5 * STEP + 4), dn.DN_ERR_INVALID),    # inside o
    (dict(dk=64, dv=64), dn.DN_ERR_UNSUPPORTED),            # tensor-core path only
    (dict(a=None), dn.DN_ERR_INVALID),                      # the raw decay input is required
])
def test_gdn_layer_rejects(lib, over, code):
    before = lib.dn_kernel_launches()
    assert gdn_call(lib, **over) == code
    assert lib.dn_last_error() != b""
    assert lib.dn_kernel_launches() == before


def test_decode_layer_rejects_missing_params(lib):
    A0 = 0x10000000
    st = lib.dn_decode_step_gdn(A0, A0 + STEP, A0 + 2 * STEP, A0 + 3 * STEP, A0 + 4 * STEP, None, None,
                                A0 + 5 * STEP, A0 + 6 * STEP, 2, 3, 128, 128, 1.0, 1, None)
    assert st == dn.DN_ERR_INVALID and b"A_log" in lib.dn_last_error()


def conv_call(lib, **over):
    args = dict(x=A, ld_x=256, w=A + STEP, s_in=None, y=A + 2 * STEP, s_out=None, B=2, T=40, C=256, K=4,
                hd=128, act=1, dtype=1)
    args.update(over)
    return lib.dn_causal_conv1d(args["x"], args["ld_x"], args["w"], args["s_in"], args["y"], args["s_out"],
                                args["B"], args["T"], args["C"], args["K"], args["hd"], args["act"], args["dtype"],
                                None)


@pytest.mark.parametrize("over,code", [
    (dict(K=5), dn.DN_ERR_UNSUPPORTED),
    (dict(K=0), dn.DN_ERR_UNSUPPORTED),
    (dict(T=-1), dn.DN_ERR_INVALID),
    (dict(dtype=7), dn.DN_ERR_INVALID),
    (dict(act=2), dn.DN_ERR_INVALID),
    (dict(ld_x=100), dn.DN_ERR_INVALID),                  # ld_x < C
    (dict(hd=100), dn.DN_ERR_INVALID),                    # does not divide C
    (dict(hd=0), dn.DN_ERR_INVALID),
    (dict(w=None), dn.DN_ERR_INVALID),
    (dict(y=None), dn.DN_ERR_INVALID),
    (dict(x=None), dn.DN_ERR_INVALID),
    (dict(x=A + 1), dn.DN_ERR_INVALID),                   # bf16 needs 2-byte alignment
    (dict(w=A + STEP + 2), dn.DN_ERR_INVALID),
    (dict(y=A + 100), dn.DN_ERR_INVALID),                 # y overlaps x
    (dict(s_out=A + 64), dn.DN_ERR_INVALID),              # state_out overlaps x
    (dict(s_in=A + 3 * STEP, s_out=A + 3 * STEP), dn.DN_ERR_INVALID),        # in place needs T <= 16
    (dict(s_in=A + 3 * STEP, s_out=A + 3 * STEP + 512), dn.DN_ERR_INVALID),  # partial overlap
    (dict(T=16 * 65535 + 1), dn.DN_ERR_UNSUPPORTED),
])
def test_causal_conv1d_rejects(lib, over, code):
    assert conv_call(lib, **over) == code, lib.dn_last_error()


def test_causal_conv1d_empty_is_ok(lib):
    assert conv_call(lib, B=0) == dn.DN_OK
    assert conv_call(lib, C=0, ld_x=0, hd=1) == dn.DN_OK
    assert conv_call(lib, T=0, x=None) == dn.DN_OK           # no state out: nothing to do
    assert conv_call(lib, K=1, T=0, s_out=A + 3 * STEP) == dn.DN_OK


def norm_call(lib, **over):
    args = dict(x=A, z=A + STEP, w=A + 2 * STEP, y=A + 3 * STEP, B=2, T=10, H=4, D=128, eps=1e-6, hm=1, act=1,
                dtype=1)
    args.update(over)
    return lib.dn_rms_norm_gated(args["x"], args["z"], args["w"], args["y"], args["B"], args["T"], args["H"],
                                 args["D"], args["eps"], args["hm"], args["act"], args["dtype"], None)


@pytest.mark.parametrize("over,code", [
    (dict(D=96), dn.DN_ERR_UNSUPPORTED),
    (dict(D=512), dn.DN_ERR_UNSUPPORTED),
    (dict(B=-1), dn.DN_ERR_INVALID),
    (dict(eps=-1.0), dn.DN_ERR_INVALID),
    (dict(eps=float("nan")), dn.DN_ERR_INVALID),
    (dict(eps=float("inf")), dn.DN_ERR_INVALID),
    (dict(hm=2), dn.DN_ERR_INVALID),
    (dict(act=3), dn.DN_ERR_INVALID),
    (dict(dtype=5), dn.DN_ERR_INVALID),
    (dict(z=None), dn.DN_ERR_INVALID),
    (dict(x=A + 8), dn.DN_ERR_INVALID),                   # 16-byte alignment
    (dict(w=A + 2 * STEP + 2), dn.DN_ERR_INVALID),
    (dict(y=A + STEP + 4096), dn.DN_ERR_INVALID),         # y overlaps z
    (dict(y=A), dn.DN_ERR_INVALID),                       # y is x: not in place
])
def test_rms_norm_gated_rejects(lib, over, code):
    assert norm_call(lib, **over) == code, lib.dn_last_error()


def test_rms_norm_gated_empty_is_ok(lib):
    assert norm_call(lib, T=0) == dn.DN_OK
    assert norm_call(lib, H=0, x=None, z=None, y=None) == dn.DN_OK


def test_layer_op_bindings_check_shapes_before_any_device_call():
    """The C ABI sees only pointers and sizes, so the binding checks that the tensors
    agree: a mismatch raises before the library is called.  (CPU tensors that pass the
    checks are then refused as not on a CUDA device.)"""
    import torch
    bf = torch.bfloat16
    x = torch.zeros(2, 10, 64, dtype=bf)
    w = torch.zeros(64, 4)
    s = torch.zeros(2, 3, 64, dtype=bf)
    y = torch.zeros(2, 2, 10, 32, dtype=bf)
    bad = [
        dict(w=torch.zeros(32, 4)),                      # channels disagree
        dict(y=torch.zeros(2, 2, 10, 31, dtype=bf)),     # wrong output size
        dict(y=torch.zeros(2, 10, 2, 32, dtype=bf)),     # token-major given for head-major
        dict(s_in=torch.zeros(2, 2, 64, dtype=bf)),      # K - 1 rows
        dict(s_out=torch.zeros(2, 3, 64)),               # dtype
        dict(hd=24),                                     # does not divide C
    ]
    for over in bad:
        a = dict(x=x, w=w, y=y, s_in=s, s_out=s, hd=32)
        a.update(over)
        with pytest.raises(ValueError, match=r"^dn: (?!tensors must be CUDA)"):
            dn.dn_causal_conv1d(a["x"], a["w"], a["y"], a["s_in"], a["s_out"], head_dim=a["hd"])
    with pytest.raises(ValueError, match="CUDA"):
        dn.dn_causal_conv1d(x, w, y, s, s, head_dim=32)

    o = torch.zeros(2, 4, 10, 128, dtype=bf)             # head-major [B, H, T, D]
    z = torch.zeros(2, 10, 4, 128, dtype=bf)
    yn = torch.zeros(2, 10, 4, 128, dtype=bf)
    nw = torch.zeros(128)
    bad = [
        dict(x=z.clone()),                               # token-major given as head-major
        dict(y=torch.zeros(2, 4, 10, 128, dtype=bf)),
        dict(w=torch.zeros(64)),
        dict(x=torch.zeros(2, 4, 10, 128)),              # dtype
    ]
    for over in bad:
        a = dict(x=o, z=z, w=nw, y=yn)
        a.update(over)
        with pytest.raises(ValueError, match=r"^dn: (?!tensors must be CUDA)"):
            dn.dn_rms_norm_gated(a["x"], a["z"], a["w"], a["y"])
    with pytest.raises(ValueError, match="CUDA"):
        dn.dn_rms_norm_gated(o, z, nw, yn)
    with pytest.raises(ValueError, match="CUDA"):
        dn.dn_rms_norm_gated(z, z, nw, yn, x_head_major=False)


# ---- entry points added with grouped heads, packed batches and the 2 sigmoid gate ----

def test_gva_rejects_before_device_work(lib):
    # 8 value heads over 3 key heads: not a whole group per key head
    st = lib.dn_chunk_fwd_gva(A, A + STEP, A + 2 * STEP, A + 3 * STEP, A + 4 * STEP, None, A + 5 * STEP, None,
                              1, 64, 3, 8, 128, 128, 1.0, 1, 1, None, 0, None)
    assert st == dn.DN_ERR_INVALID
    # fp32 tokens: grouped heads run on the tensor-core kernels only
    st = lib.dn_chunk_fwd_gva(A, A + STEP, A + 2 * STEP, A + 3 * STEP, A + 4 * STEP, None, A + 5 * STEP, None,
                              1, 64, 2, 8, 128, 128, 1.0, 0, 1, None, 0, None)
    assert st == dn.DN_ERR_UNSUPPORTED
    st = lib.dn_decode_step_gva(A, A + STEP, A + 2 * STEP, A + 3 * STEP, None, A + 4 * STEP, A + 5 * STEP,
                                2, 3, 8, 128, 128, 1.0, 1, 0, None)
    assert st == dn.DN_ERR_INVALID


def varlen_call(lib, **over):
    args = dict(q=A, k=A + STEP, v=A + 2 * STEP, beta=A + 3 * STEP, g=A + 4 * STEP, S0=None, o=A + 5 * STEP,
                S_T=A + 6 * STEP, cu=A + 7 * STEP, N=3, T=200, H=2, dk=128, dv=128, dtype=1, gate=1)
    args.update(over)
    return lib.dn_chunk_fwd_varlen(args["q"], args["k"], args["v"], args["beta"], args["g"], args["S0"], args["o"],
                                   args["S_T"], args["cu"], args["N"], args["T"], args["H"], args["dk"], args["dv"],
                                   1.0, args["dtype"], args["gate"], None, 0, None)


@pytest.mark.parametrize("over,code", [
    (dict(cu=None), dn.DN_ERR_INVALID),
    (dict(N=0), dn.DN_ERR_INVALID),
    (dict(cu=A + 7 * STEP + 2), dn.DN_ERR_INVALID),          # not 4-byte aligned
    (dict(o=A + 7 * STEP), dn.DN_ERR_INVALID),               # o overlaps cu_seqlens
    (dict(gate=2), dn.DN_ERR_UNSUPPORTED),                   # per-key gate
    (dict(dtype=0), dn.DN_ERR_UNSUPPORTED),                  # fp32 tokens
    (dict(dk=64, dv=64), dn.DN_ERR_UNSUPPORTED),
])
def test_varlen_rejects_before_device_work(lib, over, code):
    assert varlen_call(lib, **over) == code


def test_varlen_workspace_size_depends_on_N_and_T(lib):
    out = ctypes.c_size_t(0)
    assert lib.dn_chunk_fwd_varlen_workspace_size(3, 200, 2, 128, 128, 1, 1, ctypes.byref(out)) == dn.DN_OK
    # at most 200 / 64 + 3 = 6 chunks per head: 12 tiles of 40.25 KiB, their flags, then the tables
    tiles = 2 * (200 // 64 + 3)
    assert out.value >= tiles * 41216 + 4 * (tiles + 1)
    big = ctypes.c_size_t(0)
    assert lib.dn_chunk_fwd_varlen_workspace_size(30, 200, 2, 128, 128, 1, 1, ctypes.byref(big)) == dn.DN_OK
    assert big.value > out.value


def test_gdn_ex_rejects_unknown_flags(lib):
    st = lib.dn_chunk_fwd_gdn_ex(A, A + STEP, A + 2 * STEP, A + 3 * STEP, A + 4 * STEP, A + 5 * STEP,
                                 A + 5 * STEP + 256, None, A + 6 * STEP, None, 1, 8, 1, 128, 128, 64, 1.0, 1, 0, 4,
                                 None, None, 0.0, None, 0, None)
    assert st == dn.DN_ERR_INVALID
    st = lib.dn_decode_step_gdn_ex(A, A + STEP, A + 2 * STEP, A + 3 * STEP, A + 4 * STEP, A + 5 * STEP,
                                   A + 5 * STEP + 256, A + 6 * STEP, A + 7 * STEP, 1, 1, 128, 128, 1.0, 1, 8, None,
                                   None, 0.0, None)
    assert st == dn.DN_ERR_INVALID
    # the norm needs z and its weight, and a positive eps
    base = (A, A + STEP, A + 2 * STEP, A + 3 * STEP, A + 4 * STEP, A + 5 * STEP, A + 5 * STEP + 256, A + 6 * STEP,
            A + 7 * STEP, 1, 1, 128, 128, 1.0, 1)
    assert lib.dn_decode_step_gdn_ex(*base, 2, None, None, 0.0, None) == dn.DN_ERR_INVALID
    assert lib.dn_decode_step_gdn_ex(*base, 0, A + 8 * STEP, None, 1e-6, None) == dn.DN_ERR_INVALID
    assert lib.dn_decode_step_gdn_ex(*base, 0, A + 8 * STEP, A + 9 * STEP, 0.0, None) == dn.DN_ERR_INVALID
