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


class DefaultPoolMeter:
    """High-water mark of the device's default memory pool, the pool that
    stream-ordered allocations (cudaMallocAsync) draw from when no other pool is
    named, read through the driver API.  torch's caching allocator does not use
    that pool, so between two reads it sees only the library's allocations."""

    def __init__(self, device: int = 0):
        from cuda.bindings import driver as cu
        self.cu = cu
        err, = cu.cuInit(0)
        assert err == cu.CUresult.CUDA_SUCCESS, err
        err, dev = cu.cuDeviceGet(device)
        assert err == cu.CUresult.CUDA_SUCCESS, err
        err, self.pool = cu.cuDeviceGetDefaultMemPool(dev)
        assert err == cu.CUresult.CUDA_SUCCESS, err
        self.attr = cu.CUmemPool_attribute.CU_MEMPOOL_ATTR_USED_MEM_HIGH

    def reset(self):
        err, = self.cu.cuMemPoolSetAttribute(self.pool, self.attr, self.cu.cuuint64_t(0))
        assert err == self.cu.CUresult.CUDA_SUCCESS, err

    def high(self) -> int:
        err, v = self.cu.cuMemPoolGetAttribute(self.pool, self.attr)
        assert err == self.cu.CUresult.CUDA_SUCCESS, err
        return int(v)


@pytest.mark.gpu
@pytest.mark.parametrize("gate", ["scalar", "per_key"])
def test_noalloc_matches_dn_chunk_fwd_on_two_calls(cuda_device, gate):
    lib, f = noalloc_fn()
    stream = torch.cuda.current_stream()
    meter = DefaultPoolMeter(torch.cuda.current_device())
    sc = 128 ** -0.5
    gate_code = 1 if gate == "scalar" else 2
    # two different requests in a row: the second reuses the scratch area the
    # first left behind (the per-key gate lays its tiles, gamma table and flags
    # out differently, so both layouts run against the shared area)
    for B, H, T, seed in ((2, 4, 300, 71), (1, 3, 1000, 72)):
        inp = W.gen_prefill(B, H, T, 128, 128, dtype="bf16", gate=gate, seed=seed, s0_std=0.2,
                            g_shift=2.0 if gate == "scalar" else 3.0)
        d = to_dev(inp)
        need = dn.dn_chunk_fwd_workspace_size(B, T, H, 128, 128, gate=gate)
        assert 0 < need <= 64 << 20
        o = torch.full((B, H, T, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        S = torch.full((B, H, 128, 128), float("nan"), device="cuda")
        torch.cuda.synchronize()
        meter.reset()
        st = f(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["beta"]), ptr(d["g"]), ptr(d["S0"]), ptr(o), ptr(S),
               B, T, H, 128, 128, 64, sc, 1, gate_code, ctypes.c_void_p(stream.cuda_stream))
        assert st == dn.DN_OK, lib.dn_last_error()
        torch.cuda.synchronize()
        assert meter.high() == 0, "dn_chunk_fwd_noalloc drew memory from the default pool"
        o_ref = torch.empty_like(o)
        S_ref = torch.empty_like(S)
        # the allocating entry point (no workspace given) does move the meter: the
        # check above can see a stream-ordered allocation
        meter.reset()
        dn.dn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], o_ref, S_ref, scale=sc, gate=gate)
        torch.cuda.synchronize()
        assert meter.high() >= need
        dn.dn_device_status()
        assert_close(o, o_ref.double().cpu().numpy(), "bf16", f"o (T={T}, {gate})")
        assert_close(S, S_ref.double().cpu().numpy(), "bf16", f"S_T (T={T}, {gate})")


def test_noalloc_rejects_requests_above_its_scratch_area():
    # 32 heads x 1024 chunks x 40.25 KiB, plus a 4-byte flag per chunk and a tile counter, is
    # 1.25 GiB of scratch, above the fixed 64 MiB: refused before any device work (the fake
    # addresses are never used)
    lib, f = noalloc_fn()
    A, STEP = 0x10000000, 0x40000000
    st = f(A, A + STEP, A + 2 * STEP, A + 3 * STEP, A + 4 * STEP, None, A + 5 * STEP, None,
           1, 65536, 32, 128, 128, 64, 1.0, 1, 1, None)
    assert st == dn.DN_ERR_UNSUPPORTED
    msg = lib.dn_last_error().decode()
    n = 32 * 1024
    need = n * 41216 + (4 * (n + 1) + 255) // 256 * 256
    assert str(need) in msg and str(64 << 20) in msg
