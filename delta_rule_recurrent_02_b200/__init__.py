"""B200 (sm_100a) causal delta-rule layer: chunked prefill and decode step.

A thin Python binding over the C ABI of ``include/dn.h`` (``libdn.so``, built
in-tree by ``delta_rule_recurrent_02_b200/build.py``).  The binding only
marshals arguments: torch tensors supply device pointers and streams, and
every arithmetic step runs in the library's CUDA kernels.  There is no CPU
path: if the library is missing, or a tensor is not on a CUDA device, the
call raises.

Functions with the ABI's names take preallocated outputs:

    dn_chunk_fwd(q, k, v, beta, g, S0, o, S_T, chunk=64, scale=1.0, workspace=None, ...)
    dn_chunk_fwd_workspace_size(B, T, H, d_k, d_v, chunk=64, dtype="bf16", gate="scalar", path="auto")
    dn_chunk_fwd_snapshots(q, k, v, beta, g, S0, o, S_T, snaps, every, ...)
    dn_chunk_fwd_gdn(q, k, v, b, a, A_log, dt_bias, S0, o, S_T, scale=1.0, ...)   # layer prologue fused in
    dn_chunk_fwd_gdn_ex(..., chunk=64, path="auto", allow_neg_eigval=False, ...)  # either path; beta = 2 sigmoid(b)
    dn_chunk_fwd_gva(q, k, v, beta, g, S0, o, S_T, scale=1.0, ...)   # H_k key heads, H value heads
    dn_chunk_fwd_varlen(q, k, v, beta, g, S0, o, S_T, cu_seqlens, scale=1.0, ...)   # packed sequences
    dn_chunk_fwd_varlen_workspace_size(N, T, H, d_k, d_v, dtype="bf16", gate="scalar")
    dn_chunk_fwd_general(q, w_log, kappa, a, k, v, S0, o, S_T, chunk=32, scale=1.0)   # RWKV-7's rule
    dn_decode_step(q, k, v, beta, g, S, o, scale=1.0, ...)
    dn_decode_step_gva(q, k, v, beta, g, S, o, scale=1.0, ...)
    dn_decode_step_gdn(q, k, v, b, a, A_log, dt_bias, S, o, scale=1.0, ...)
    dn_decode_step_gdn_ex(..., allow_neg_eigval=False, ...)
    dn_causal_conv1d(x, weight, y, state_in=None, state_out=None, head_dim=None, activation=True)
    dn_rms_norm_gated(x, z, weight, y, eps=1e-6, x_head_major=True, activation="silu")
    dn_device_status(stream=None)
    dn_kernel_launches()

and two conveniences allocate the outputs (and the prefill's workspace) with torch:

    o, S_T = chunk_fwd(q, k, v, beta, g=None, S0=None, chunk=64, scale=1.0)
    o      = decode_step(q, k, v, beta, S, g=None, scale=1.0)
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["DNError", "load_library", "library_path", "dn_chunk_fwd", "dn_chunk_fwd_workspace_size",
           "dn_chunk_fwd_snapshots", "dn_chunk_fwd_gdn", "dn_decode_step_gdn", "dn_chunk_fwd_gva",
           "dn_decode_step_gva", "dn_chunk_fwd_gdn_ex", "dn_decode_step_gdn_ex", "DN_GDN_BETA_2SIGMOID",
           "dn_chunk_fwd_varlen", "dn_chunk_fwd_varlen_workspace_size", "dn_chunk_fwd_general", "dn_decode_step", "dn_kernel_launches", "dn_causal_conv1d", "dn_rms_norm_gated",
           "dn_device_status", "chunk_fwd", "decode_step", "ABI_SYMBOLS",
           "DN_OK", "DN_ERR_INVALID", "DN_ERR_UNSUPPORTED", "DN_ERR_CUDA", "DN_ERR_TIMEOUT"]

DN_OK, DN_ERR_INVALID, DN_ERR_UNSUPPORTED, DN_ERR_CUDA, DN_ERR_TIMEOUT = 0, 1, 2, 3, 4
DN_GDN_BETA_2SIGMOID = 1
DN_GDN_NORM_SIGMOID = 2
_DTYPES = {"f32": 0, "bf16": 1}
_GATES = {"none": 0, "scalar": 1, "per_key": 2}
_PATHS = {"auto": 0, "simt": 1, "tc": 2, "tc_stall_test": 3}

ABI_SYMBOLS = ("dn_chunk_fwd", "dn_chunk_fwd_ex", "dn_chunk_fwd_workspace_size", "dn_chunk_fwd_noalloc",
               "dn_chunk_fwd_snapshots", "dn_chunk_fwd_gdn", "dn_decode_step_gdn", "dn_chunk_fwd_gva",
               "dn_decode_step_gva", "dn_chunk_fwd_gdn_ex", "dn_decode_step_gdn_ex", "dn_chunk_fwd_varlen",
               "dn_chunk_fwd_varlen_workspace_size", "dn_chunk_fwd_general", "dn_decode_step", "dn_device_status", "dn_status_str",
               "dn_last_error", "dn_version", "dn_kernel_launches", "dn_causal_conv1d", "dn_rms_norm_gated")

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None


class DNError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} [status {status}]")
        self.status = status


def library_path() -> str:
    return os.path.join(_HERE, "libdn.so")


def load_library():
    """Load ``libdn.so`` and declare the ABI's signatures.  Raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m delta_rule_recurrent_02_b200.build` "
                           "(there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    vp, fp, I, F, Z = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.dn_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, I, I, I, I, I, I, F, I, I, vp]
    lib.dn_chunk_fwd.restype = I
    lib.dn_chunk_fwd_ex.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, I, I, I, I, I, I, F, I, I, I, vp, Z, vp]
    lib.dn_chunk_fwd_ex.restype = I
    lib.dn_chunk_fwd_snapshots.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, fp, I, I, I, I, I, I, I, F, I, I, I,
                                           vp, Z, vp]
    lib.dn_chunk_fwd_snapshots.restype = I
    lib.dn_chunk_fwd_gdn.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, vp, fp, I, I, I, I, I, F, vp, Z, vp]
    lib.dn_chunk_fwd_gdn.restype = I
    lib.dn_decode_step_gdn.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, vp, I, I, I, I, F, I, vp]
    lib.dn_decode_step_gdn.restype = I
    lib.dn_chunk_fwd_gdn_ex.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, vp, fp, I, I, I, I, I, I, F, I, I, I, vp,
                                        fp, F, vp, Z, vp]
    lib.dn_chunk_fwd_gdn_ex.restype = I
    lib.dn_decode_step_gdn_ex.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, vp, I, I, I, I, F, I, I, vp, fp, F, vp]
    lib.dn_decode_step_gdn_ex.restype = I
    lib.dn_chunk_fwd_gva.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, I, I, I, I, I, I, F, I, I, vp, Z, vp]
    lib.dn_chunk_fwd_gva.restype = I
    lib.dn_decode_step_gva.argtypes = [vp, vp, vp, fp, fp, fp, vp, I, I, I, I, I, F, I, I, vp]
    lib.dn_decode_step_gva.restype = I
    lib.dn_chunk_fwd_varlen.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, vp, I, I, I, I, I, F, I, I, vp, Z, vp]
    lib.dn_chunk_fwd_varlen.restype = I
    lib.dn_chunk_fwd_varlen_workspace_size.argtypes = [I, I, I, I, I, I, I, ctypes.POINTER(Z)]
    lib.dn_chunk_fwd_varlen_workspace_size.restype = I
    lib.dn_chunk_fwd_general.argtypes = [vp, fp, vp, fp, vp, vp, fp, vp, fp, I, I, I, I, I, I, F, I, vp]
    lib.dn_chunk_fwd_general.restype = I
    lib.dn_chunk_fwd_workspace_size.argtypes = [I, I, I, I, I, I, I, I, I, ctypes.POINTER(Z)]
    lib.dn_chunk_fwd_workspace_size.restype = I
    lib.dn_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, vp, I, I, I, I, F, I, I, vp]
    lib.dn_decode_step.restype = I
    lib.dn_device_status.argtypes = [vp]
    lib.dn_device_status.restype = I
    lib.dn_status_str.argtypes = [I]
    lib.dn_status_str.restype = ctypes.c_char_p
    lib.dn_last_error.argtypes = []
    lib.dn_last_error.restype = ctypes.c_char_p
    lib.dn_version.argtypes = []
    lib.dn_version.restype = I
    lib.dn_causal_conv1d.argtypes = [vp, I, fp, vp, vp, vp, I, I, I, I, I, I, I, vp]
    lib.dn_causal_conv1d.restype = I
    lib.dn_rms_norm_gated.argtypes = [vp, vp, fp, vp, I, I, I, I, F, I, I, I, vp]
    lib.dn_rms_norm_gated.restype = I
    lib.dn_kernel_launches.argtypes = []
    lib.dn_kernel_launches.restype = ctypes.c_ulonglong
    _lib = lib
    return lib


def dn_kernel_launches() -> int:
    """Kernels the library has launched in this process so far (all threads
    and devices); the difference of two reads counts a region's launches."""
    return int(load_library().dn_kernel_launches())


def _check(lib, status: int):
    if status != DN_OK:
        msg = (lib.dn_last_error() or b"").decode() or lib.dn_status_str(status).decode()
        raise DNError(status, msg)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("dn: tensors must be CUDA tensors (the library takes device pointers)")
    if not t.is_contiguous():
        raise ValueError("dn: tensors must be contiguous")
    return t.data_ptr()


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return _DTYPES["f32"]
    if t.dtype == torch.bfloat16:
        return _DTYPES["bf16"]
    raise ValueError(f"dn: unsupported token dtype {t.dtype}")


def _gate_code(gate, g, lead_shape) -> int:
    if gate is not None:
        return _GATES[gate]
    if g is None:
        return _GATES["none"]
    return _GATES["scalar"] if tuple(g.shape) == tuple(lead_shape) else _GATES["per_key"]


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _f32(t):
    import torch
    if t is not None and t.dtype != torch.float32:
        raise ValueError("dn: beta, g and states must be float32")
    return t


def dn_chunk_fwd_workspace_size(B: int, T: int, H: int, d_k: int, d_v: int, *, chunk: int = 64,
                                dtype: str = "bf16", gate: str = "scalar", path: str = "auto") -> int:
    """Bytes of workspace ``dn_chunk_fwd`` needs for this request (0 if none)."""
    lib = load_library()
    out = ctypes.c_size_t(0)
    _check(lib, lib.dn_chunk_fwd_workspace_size(B, T, H, d_k, d_v, int(chunk), _DTYPES[dtype], _GATES[gate],
                                                _PATHS[path], ctypes.byref(out)))
    return out.value


def dn_chunk_fwd(q, k, v, beta, g, S0, o, S_T, *, chunk: int = 64, scale: float = 1.0,
                 gate: str | None = None, path: str = "auto", workspace=None, stream=None) -> None:
    """Chunked prefill through ``dn_chunk_fwd_ex``; writes ``o`` and ``S_T``.

    ``workspace`` is a CUDA tensor of at least ``dn_chunk_fwd_workspace_size``
    bytes, or None (the library then allocates one stream-ordered for the call).
    """
    lib = load_library()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    for t in (beta, g, S0, S_T):
        _f32(t)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.dn_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S0), _ptr(o),
                             _ptr(S_T), B, T, H, dk, dv, int(chunk), float(scale), _dtype_code(q),
                             _gate_code(gate, g, (B, H, T)), _PATHS[path], _ptr(workspace), ws_bytes,
                             _stream(stream))
    _check(lib, st)


def dn_chunk_fwd_snapshots(q, k, v, beta, g, S0, o, S_T, snaps, every: int, *, chunk: int = 64,
                           scale: float = 1.0, gate: str | None = None, path: str = "auto", workspace=None,
                           stream=None) -> None:
    """``dn_chunk_fwd`` that also writes ``snaps`` [B, H, n_snap, d_k, d_v] fp32, the
    state after every ``every`` chunks (n_snap = T // (every * chunk)), through
    ``dn_chunk_fwd_snapshots``."""
    lib = load_library()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    for t in (beta, g, S0, S_T, snaps):
        _f32(t)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.dn_chunk_fwd_snapshots(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S0), _ptr(o),
                                    _ptr(S_T), _ptr(snaps), int(every), B, T, H, dk, dv, int(chunk), float(scale),
                                    _dtype_code(q), _gate_code(gate, g, (B, H, T)), _PATHS[path],
                                    _ptr(workspace), ws_bytes, _stream(stream))
    _check(lib, st)


def dn_chunk_fwd_gdn(q, k, v, b, a, A_log, dt_bias, S0, o, S_T, *, scale: float = 1.0, workspace=None,
                     stream=None) -> None:
    """Gated DeltaNet prefill with the layer's prologue fused in, through
    ``dn_chunk_fwd_gdn``: q and k raw (normalised inside), b and a [B, H, T] the
    raw write-strength and decay inputs, A_log and dt_bias [H]."""
    lib = load_library()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    for t in (b, a, A_log, dt_bias, S0, S_T):
        _f32(t)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.dn_chunk_fwd_gdn(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(a), _ptr(A_log), _ptr(dt_bias), _ptr(S0),
                              _ptr(o), _ptr(S_T), B, T, H, dk, dv, float(scale), _ptr(workspace), ws_bytes,
                              _stream(stream))
    _check(lib, st)


def dn_chunk_fwd_gdn_ex(q, k, v, b, a, A_log, dt_bias, S0, o, S_T, *, chunk: int = 64, scale: float = 1.0,
                        path: str = "auto", allow_neg_eigval: bool = False, z=None, norm_weight=None,
                        eps: float = 1e-6, norm_activation: str = "silu", workspace=None, stream=None) -> None:
    """``dn_chunk_fwd_gdn`` on either kernel path (``dn_chunk_fwd_gdn_ex``): fp32 or
    bf16 tokens, d in {64, 128}, chunk 1..64 on the CUDA-core path;
    ``allow_neg_eigval`` takes beta = 2 sigmoid(b); with ``z`` [B, T, H, d_v] and
    ``norm_weight`` [d_v], ``o`` [B, T, H, d_v] receives the gated RMSNorm of the
    read-out (tensor-core path)."""
    lib = load_library()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    for t in (b, a, A_log, dt_bias, S0, S_T, norm_weight):
        _f32(t)
    if z is not None and (tuple(z.shape) != (B, T, H, dv) or z.dtype != q.dtype or tuple(o.shape) != (B, T, H, dv)):
        raise ValueError("dn: z and o must be [B, T, H, d_v] in the token dtype")
    flags = (DN_GDN_BETA_2SIGMOID if allow_neg_eigval else 0) | \
        (DN_GDN_NORM_SIGMOID if z is not None and norm_activation == "sigmoid" else 0)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.dn_chunk_fwd_gdn_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(a), _ptr(A_log), _ptr(dt_bias),
                                 _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv, int(chunk), float(scale),
                                 _dtype_code(q), _PATHS[path], flags, _ptr(z), _ptr(norm_weight), float(eps),
                                 _ptr(workspace), ws_bytes, _stream(stream))
    _check(lib, st)


def dn_decode_step_gdn_ex(q, k, v, b, a, A_log, dt_bias, S, o, *, scale: float = 1.0,
                          allow_neg_eigval: bool = False, z=None, norm_weight=None, eps: float = 1e-6,
                          norm_activation: str = "silu", stream=None) -> None:
    """``dn_decode_step_gdn`` with flags (``dn_decode_step_gdn_ex``):
    ``allow_neg_eigval`` takes beta = 2 sigmoid(b); with ``z`` [B, H, d_v] and
    ``norm_weight`` [d_v], ``o`` receives the gated RMSNorm of the read-out."""
    lib = load_library()
    B, H, dk = q.shape
    dv = v.shape[-1]
    for t in (b, a, A_log, dt_bias, S, norm_weight):
        _f32(t)
    if z is not None and (tuple(z.shape) != (B, H, dv) or z.dtype != q.dtype):
        raise ValueError("dn: z must be [B, H, d_v] in the token dtype")
    flags = (DN_GDN_BETA_2SIGMOID if allow_neg_eigval else 0) | \
        (DN_GDN_NORM_SIGMOID if z is not None and norm_activation == "sigmoid" else 0)
    st = lib.dn_decode_step_gdn_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(a), _ptr(A_log), _ptr(dt_bias),
                                   _ptr(S), _ptr(o), B, H, dk, dv, float(scale), _dtype_code(q), flags, _ptr(z),
                                   _ptr(norm_weight), float(eps), _stream(stream))
    _check(lib, st)


def dn_decode_step_gdn(q, k, v, b, a, A_log, dt_bias, S, o, *, scale: float = 1.0, stream=None) -> None:
    """One decode step with the Gated DeltaNet layer's prologue fused in, through
    ``dn_decode_step_gdn``: q and k [B, H, d] raw, b and a [B, H] raw, A_log and
    dt_bias [H]; updates S in place and writes o."""
    lib = load_library()
    B, H, dk = q.shape
    dv = v.shape[-1]
    for t in (b, a, A_log, dt_bias, S):
        _f32(t)
    st = lib.dn_decode_step_gdn(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(a), _ptr(A_log), _ptr(dt_bias), _ptr(S),
                                _ptr(o), B, H, dk, dv, float(scale), _dtype_code(q), _stream(stream))
    _check(lib, st)


def dn_chunk_fwd_gva(q, k, v, beta, g, S0, o, S_T, *, scale: float = 1.0, gate: str | None = None,
                     workspace=None, stream=None) -> None:
    """Prefill with grouped value heads through ``dn_chunk_fwd_gva``: q and k
    [B, H_k, T, d_k], v and o [B, H, T, d_v], beta and g [B, H, T], states
    [B, H, d_k, d_v]; value head h reads key head h // (H // H_k)."""
    lib = load_library()
    B, Hk, T, dk = q.shape
    H, dv = v.shape[1], v.shape[-1]
    if tuple(k.shape) != tuple(q.shape) or tuple(v.shape[:3]) != (B, H, T):
        raise ValueError("dn: q, k must be [B, H_k, T, d_k] and v [B, H, T, d_v]")
    for t in (beta, g, S0, S_T):
        _f32(t)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.dn_chunk_fwd_gva(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S0), _ptr(o), _ptr(S_T),
                              B, T, Hk, H, dk, dv, float(scale), _dtype_code(q), _gate_code(gate, g, (B, H, T)),
                              _ptr(workspace), ws_bytes, _stream(stream))
    _check(lib, st)


def dn_chunk_fwd_varlen_workspace_size(N: int, T: int, H: int, d_k: int, d_v: int, *, dtype: str = "bf16",
                                       gate: str = "scalar") -> int:
    """Bytes of workspace ``dn_chunk_fwd_varlen`` needs for N sequences of T tokens in all."""
    lib = load_library()
    out = ctypes.c_size_t(0)
    _check(lib, lib.dn_chunk_fwd_varlen_workspace_size(N, T, H, d_k, d_v, _DTYPES[dtype], _GATES[gate],
                                                       ctypes.byref(out)))
    return out.value


def dn_chunk_fwd_varlen(q, k, v, beta, g, S0, o, S_T, cu_seqlens, *, scale: float = 1.0, gate: str | None = None,
                        workspace=None, stream=None) -> None:
    """Prefill of N packed sequences through ``dn_chunk_fwd_varlen``: q, k, v, o
    [1, H, T, d] (or [H, T, d]), beta and g [1, H, T] (or [H, T]), cu_seqlens a
    CUDA int32 tensor [N + 1], states [N, H, d_k, d_v]."""
    import torch
    lib = load_library()
    H, T, dk = q.shape[-3:]
    dv = v.shape[-1]
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("dn: cu_seqlens must be int32")
    N = cu_seqlens.numel() - 1
    for t in (beta, g, S0, S_T):
        _f32(t)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.dn_chunk_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S0), _ptr(o), _ptr(S_T),
                                 _ptr(cu_seqlens), N, T, H, dk, dv, float(scale), _dtype_code(q),
                                 _gate_code(gate, g, tuple(beta.shape)), _ptr(workspace), ws_bytes, _stream(stream))
    _check(lib, st)


def dn_chunk_fwd_general(q, w_log, kappa, a, k, v, S0, o, S_T, *, chunk: int = 32, scale: float = 1.0,
                         stream=None) -> None:
    """The generalised delta rule of RWKV-7 through ``dn_chunk_fwd_general``:
    q, kappa, k [B, H, T, d_k] and v [B, H, T, d_v] in the token dtype; w_log
    (log of the per-channel decay) and a [B, H, T, d_k] fp32; states
    [B, H, d_k, d_v] fp32."""
    lib = load_library()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    for t in (w_log, a, S0, S_T):
        _f32(t)
    st = lib.dn_chunk_fwd_general(_ptr(q), _ptr(w_log), _ptr(kappa), _ptr(a), _ptr(k), _ptr(v), _ptr(S0), _ptr(o),
                                  _ptr(S_T), B, T, H, dk, dv, int(chunk), float(scale), _dtype_code(q),
                                  _stream(stream))
    _check(lib, st)


def dn_decode_step_gva(q, k, v, beta, g, S, o, *, scale: float = 1.0, gate: str | None = None,
                       stream=None) -> None:
    """One decode step with grouped value heads through ``dn_decode_step_gva``:
    q and k [B, H_k, d_k], v and o [B, H, d_v], beta [B, H], S [B, H, d_k, d_v]."""
    lib = load_library()
    B, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[-1]
    if tuple(k.shape) != tuple(q.shape) or tuple(v.shape[:2]) != (B, H):
        raise ValueError("dn: q, k must be [B, H_k, d_k] and v [B, H, d_v]")
    for t in (beta, g, S):
        _f32(t)
    st = lib.dn_decode_step_gva(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S), _ptr(o),
                                B, Hk, H, dk, dv, float(scale), _dtype_code(q), _gate_code(gate, g, (B, H)),
                                _stream(stream))
    _check(lib, st)


def dn_decode_step(q, k, v, beta, g, S, o, *, scale: float = 1.0, gate: str | None = None,
                   stream=None) -> None:
    """One decode step through ``dn_decode_step``; updates ``S`` in place, writes ``o``."""
    lib = load_library()
    B, H, dk = q.shape
    dv = v.shape[-1]
    for t in (beta, g, S):
        _f32(t)
    st = lib.dn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S), _ptr(o),
                            B, H, dk, dv, float(scale), _dtype_code(q),
                            _gate_code(gate, g, (B, H)), _stream(stream))
    _check(lib, st)


def _conv_check(x, weight, y, state_in, state_out, head_dim):
    """Shapes and dtypes of a dn_causal_conv1d call (the C ABI cannot see them)."""
    if x.dim() != 3 or weight.dim() != 2:
        raise ValueError("dn: x must be [B, T, C] and weight [C, K]")
    B, T, C = x.shape
    K = weight.shape[1]
    hd = C if head_dim is None else int(head_dim)
    if weight.shape[0] != C:
        raise ValueError(f"dn: weight has {weight.shape[0]} channels, x has {C}")
    if hd <= 0 or C % hd:
        raise ValueError(f"dn: head_dim {hd} must divide C = {C}")
    if y.numel() != B * T * C or (y.dim() == 4 and tuple(y.shape) != (B, C // hd, T, hd)):
        raise ValueError(f"dn: y must be [B, C // head_dim, T, head_dim] = {(B, C // hd, T, hd)}")
    for name, t in (("state_in", state_in), ("state_out", state_out)):
        if t is not None and tuple(t.shape) != (B, K - 1, C):
            raise ValueError(f"dn: {name} must be [B, K - 1, C] = {(B, K - 1, C)}, got {tuple(t.shape)}")
    for t in (y, state_in, state_out):
        if t is not None and t.dtype != x.dtype:
            raise ValueError("dn: y and the states must have x's dtype")


def _norm_check(x, z, weight, y, x_head_major):
    """Shapes and dtypes of a dn_rms_norm_gated call."""
    if z.dim() != 4:
        raise ValueError("dn: z must be [B, T, H, D]")
    B, T, H, D = z.shape
    want_x = (B, H, T, D) if x_head_major else (B, T, H, D)
    if tuple(x.shape) != want_x:
        raise ValueError(f"dn: x must be {want_x}, got {tuple(x.shape)}")
    if tuple(y.shape) != (B, T, H, D):
        raise ValueError(f"dn: y must be [B, T, H, D] = {(B, T, H, D)}")
    if tuple(weight.shape) != (D,):
        raise ValueError(f"dn: weight must be [D] = ({D},)")
    if x.dtype != z.dtype or y.dtype != z.dtype:
        raise ValueError("dn: x, z and y must share one dtype")


def dn_causal_conv1d(x, weight, y, state_in=None, state_out=None, *, head_dim: int | None = None,
                     activation: bool = True, stream=None) -> None:
    """Depthwise causal conv over time with carried history, through
    ``dn_causal_conv1d``: x [B, T, C] (its rows may be a column slice of a wider
    tensor: unit stride over channels, any row stride), weight [C, K] fp32,
    states [B, K-1, C] in x's dtype, y [B, C // head_dim, T, head_dim]
    (head_dim defaults to C: y is then [B, T, C] in effect)."""
    _conv_check(x, weight, y, state_in, state_out, head_dim)
    lib = load_library()
    B, T, C = x.shape
    K = weight.shape[-1]
    if not x.is_cuda:
        raise ValueError("dn: tensors must be CUDA tensors (the library takes device pointers)")
    if x.stride(2) != 1 or (T > 1 and B > 1 and x.stride(0) != T * x.stride(1)):
        raise ValueError("dn: x needs unit channel stride and rows evenly spaced across the batch")
    ld_x = x.stride(1) if T > 1 else (x.stride(0) if B > 1 else C)
    _f32(weight)
    st = lib.dn_causal_conv1d(x.data_ptr(), ld_x, _ptr(weight), _ptr(state_in), _ptr(y), _ptr(state_out),
                              B, T, C, K, C if head_dim is None else head_dim, 1 if activation else 0,
                              _dtype_code(x), _stream(stream))
    _check(lib, st)


def dn_rms_norm_gated(x, z, weight, y, *, eps: float = 1e-6, x_head_major: bool = True,
                      activation: str = "silu", stream=None) -> None:
    """Gated RMSNorm of each head's output row, through ``dn_rms_norm_gated``:
    x [B, H, T, D] (x_head_major) or [B, T, H, D]; z and y [B, T, H, D];
    weight [D] fp32; activation "silu" or "sigmoid"."""
    _norm_check(x, z, weight, y, x_head_major)
    lib = load_library()
    B, T, H, D = z.shape
    _f32(weight)
    st = lib.dn_rms_norm_gated(_ptr(x), _ptr(z), _ptr(weight), _ptr(y), B, T, H, D, float(eps),
                               1 if x_head_major else 0, {"silu": 1, "sigmoid": 0}[activation],
                               _dtype_code(x), _stream(stream))
    _check(lib, st)


def dn_device_status(stream=None) -> None:
    """Synchronise the stream and raise DNError(DN_ERR_TIMEOUT) if a kernel gave up."""
    lib = load_library()
    _check(lib, lib.dn_device_status(_stream(stream)))


def chunk_fwd(q, k, v, beta, g=None, S0=None, *, chunk: int = 64, scale: float = 1.0,
              gate: str | None = None, path: str = "auto", want_state: bool = True, stream=None):
    """Allocate ``o`` (dtype of q), ``S_T`` (fp32) and the workspace, run the prefill, return (o, S_T)."""
    import torch
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    o = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if want_state else None
    gcode = _gate_code(gate, g, (B, H, T))
    gname = {v2: k2 for k2, v2 in _GATES.items()}[gcode]
    dname = {v2: k2 for k2, v2 in _DTYPES.items()}[_dtype_code(q)]
    nbytes = dn_chunk_fwd_workspace_size(B, T, H, dk, dv, chunk=chunk, dtype=dname, gate=gname, path=path)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None
    dn_chunk_fwd(q, k, v, beta, g, S0, o, S_T, chunk=chunk, scale=scale, gate=gname, path=path,
                 workspace=ws, stream=stream)
    return o, S_T


def decode_step(q, k, v, beta, S, g=None, *, scale: float = 1.0, gate: str | None = None,
                stream=None):
    """Allocate ``o``, run one decode step (S updated in place), return ``o``."""
    import torch
    B, H, _ = q.shape
    o = torch.empty((B, H, v.shape[-1]), dtype=q.dtype, device=q.device)
    dn_decode_step(q, k, v, beta, g, S, o, scale=scale, gate=gate, stream=stream)
    return o
