"""dn_chunk_fwd_noalloc: the prefill for callers that cannot allocate device
memory (a process that reserved the device's memory for its own pools, or an
allocator that must see every byte).  It takes the tensor-core path's scratch
workspace from a fixed area inside the library instead of allocating it.

The file is named to be collected last: a failure here comes after every
other test has run."""
import ctypes

import pytest
import torch

import delta_rule_recurrent_02_b200 as dn
from delta_rule_recurrent_02_b200 import workloads as W
from _util import assert_close, to_dev


def noalloc_fn():
    lib = dn.load_library()
    f = lib.dn_chunk_fwd_noalloc
    vp, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    f.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, I, I, I, I, I, I, F, I, I, vp]
    f.restype = I
    return lib, f


def ptr(t):
    return None if t is None else t.data_ptr()


@pytest.mark.gpu
def test_noalloc_matches_dn_chunk_fwd_on_two_calls(cuda_device):
    lib, f = noalloc_fn()
    stream = torch.cuda.current_stream()
    sc = 128 ** -0.5
    # two different requests in a row: the second reuses the scratch area the
    # first left behind
    for B, H, T, seed in ((2, 4, 300, 71), (1, 3, 1000, 72)):
        inp = W.gen_prefill(B, H, T, 128, 128, dtype="bf16", gate="scalar", seed=seed, s0_std=0.2)
        d = to_dev(inp)
        need = dn.dn_chunk_fwd_workspace_size(B, T, H, 128, 128)
        assert 0 < need <= 64 << 20
        o = torch.full((B, H, T, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        S = torch.full((B, H, 128, 128), float("nan"), device="cuda")
        st = f(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["beta"]), ptr(d["g"]), ptr(d["S0"]), ptr(o), ptr(S),
               B, T, H, 128, 128, 64, sc, 1, 1, ctypes.c_void_p(stream.cuda_stream))
        assert st == dn.DN_OK, lib.dn_last_error()
        o_ref = torch.empty_like(o)
        S_ref = torch.empty_like(S)
        dn.dn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], o_ref, S_ref, scale=sc)
        dn.dn_device_status()
        assert_close(o, o_ref.double().cpu().numpy(), "bf16", f"o (T={T})")
        assert_close(S, S_ref.double().cpu().numpy(), "bf16", f"S_T (T={T})")


def test_noalloc_rejects_requests_above_its_scratch_area():
    # 32 heads x 1024 chunks x 40 KiB, plus a 4-byte flag per chunk and a tile counter, is
    # 1.25 GiB of scratch, above the fixed 64 MiB: refused before any device work (the fake
    # addresses are never used)
    lib, f = noalloc_fn()
    A, STEP = 0x10000000, 0x40000000
    st = f(A, A + STEP, A + 2 * STEP, A + 3 * STEP, A + 4 * STEP, None, A + 5 * STEP, None,
           1, 65536, 32, 128, 128, 64, 1.0, 1, 1, None)
    assert st == dn.DN_ERR_UNSUPPORTED
    msg = lib.dn_last_error().decode()
    n = 32 * 1024
    need = n * 40960 + (4 * (n + 1) + 255) // 256 * 256
    assert str(need) in msg and str(64 << 20) in msg
