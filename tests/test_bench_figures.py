"""The roofline numerators bench.py reports, against their per-unit
definitions worked out by hand (no GPU): counted FLOPs of the chunked form,
algorithmic HBM bytes of the prefill, the decode step and the layer ops."""
import types

import pytest
import torch

import bench


def test_prefill_flops_per_chunk():
    # 5 C^2 d_k + 3 C^2 d_v + 6 C d_k d_v at C = 64, d = 128: 10,485,760 per chunk
    per_chunk = 5 * 64 * 64 * 128 + 3 * 64 * 64 * 128 + 6 * 64 * 128 * 128
    assert per_chunk == 10_485_760
    assert bench.prefill_flops(1, 1, 64, 128, 128) == per_chunk
    # bench prefill: B=4 H=16 T=4096 -> 4096 chunks, 4.295e10 FLOP; a ragged tail counts a whole chunk
    assert bench.prefill_flops(4, 16, 4096, 128, 128) == 4096 * per_chunk
    assert bench.prefill_flops(1, 1, 65, 128, 128) == 2 * per_chunk


def test_prefill_bytes_per_token_head():
    # bf16 q, k, v, o (2 B x 4 x 128) + fp32 beta and g: 1032 B per token-head
    assert bench.prefill_bytes(1, 1, 1, 128, 128, st=False) == 1032
    # plus S_T fp32 once: 64 KiB per head
    assert bench.prefill_bytes(1, 1, 1, 128, 128) == 1032 + 65536
    # bench prefill: 274.7 MB
    assert bench.prefill_bytes(4, 16, 4096, 128, 128) == 4 * 16 * 4096 * 1032 + 64 * 65536
    # per-key gate: g is [.., d_k] fp32; S0 read adds another state
    assert bench.prefill_bytes(1, 1, 1, 128, 128, gate_per_key=True, st=False) == 1024 + 4 + 512
    assert bench.prefill_bytes(1, 1, 1, 128, 128, s0=True) == 1032 + 2 * 65536


def test_decode_bytes_per_head():
    # the fp32 state in and out (2 x 64 KiB) + bf16 q, k, v, o + fp32 beta and g
    assert bench.decode_bytes(1, 1, 128, 128) == 2 * 65536 + 1024 + 8
    assert bench.decode_bytes(256, 32, 128, 128) == 256 * 32 * 132104          # 1.0822 GB


def test_layer_op_bytes(monkeypatch):
    """measure_layer_ops at a small shape with the library calls and CUDA events
    replaced: its byte counts follow the stated per-call formulas."""
    class Ev:
        def __init__(self, **k):
            pass

        def record(self, s=None):
            pass

        def synchronize(self):
            pass

        def elapsed_time(self, other):
            return 1.0

    monkeypatch.setattr(torch.cuda, "Event", Ev)
    monkeypatch.setattr(torch.cuda, "empty_cache", lambda: None)
    dn = types.SimpleNamespace(dn_causal_conv1d=lambda *a, **k: None, dn_rms_norm_gated=lambda *a, **k: None,
                               dn_device_status=lambda *a, **k: None)
    B, H, T, d = 2, 3, 32, 128
    W = types.SimpleNamespace(GDN_PREFILL=types.SimpleNamespace(B=B, H=H, T=T, dk=d, dv=d, seed=1))
    out = bench.measure_layer_ops(dn, torch, W, {"hbm_gbs": 1000.0}, "cpu", None)
    C3, K = 3 * H * d, 4
    conv = out[f"causal_conv1d_qkv_bf16_B{B}_T{T}_C{C3}_K{K}"]
    norm = out[f"rms_norm_gated_bf16_B{B}_T{T}_H{H}_d{d}"]
    # conv: x in and y out in bf16, the fp32 filters, the carried state in and out in bf16
    assert conv["algorithmic_bytes"] == 2 * B * T * C3 * 2 + C3 * K * 4 + 2 * B * (K - 1) * C3 * 2
    # norm: o and z in, y out, in bf16, plus the fp32 weight
    assert norm["algorithmic_bytes"] == 3 * B * T * H * d * 2 + d * 4
    assert conv["kernel_launches_per_call"] == 3 and norm["kernel_launches_per_call"] == 1
    assert norm["hbm_gbs"] == pytest.approx(norm["algorithmic_bytes"] / 1e-3 / 1e9)
