"""B200-native gated delta rule (KDA / Gated DeltaNet): Python binding.

A thin ctypes layer over ``libgdr.so`` (the C ABI declared in
``include/gdr.h``).  It only marshals arguments: it checks dtypes, devices
and contiguity, allocates outputs with PyTorch, passes raw device pointers
and the current CUDA stream, and raises on a non-OK status.  Every step of
the computation runs in the library's CUDA kernels; there is no fallback.
If the library has not been built, importing the functions raises.

Host tensors are accepted too: they are copied to the current CUDA device,
processed, and the outputs are copied back to host memory (this is what the
end-to-end measurement times).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = ["chunk_fwd", "recurrent_step", "chunk_fwd_workspace_size", "chunk_fwd_prologue", "chunk_fwd_gdr2",
           "chunk_fwd_gated", "chunk_bwd",
           "recurrent_step_gdr2", "GDRError", "library_path",
           "last_launch_count", "device_status", "GATE_PER_CHANNEL", "GATE_SCALAR"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libgdr.so")
_lib = None

GDR_OK = 0
GATE_PER_CHANNEL = 0
GATE_SCALAR = 1
_DTYPES = {torch.float32: 0, torch.bfloat16: 1}


class GDRError(RuntimeError):
    pass


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libgdr.so (raises ImportError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"libgdr.so is not built ({_LIB_PATH}); run "
                              "`python -m gated_delta_rule_89_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.gdr_chunk_fwd.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, Z, P]
        L.gdr_chunk_fwd.restype = I
        L.gdr_chunk_fwd_prologue.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, Z, P]
        L.gdr_chunk_fwd_prologue.restype = I
        L.gdr_recurrent_step.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, P]
        L.gdr_recurrent_step.restype = I
        L.gdr_chunk_fwd_workspace_size.argtypes = [I, I, I, I, I, I, I, I]
        L.gdr_chunk_fwd_workspace_size.restype = Z
        L.gdr_chunk_bwd.argtypes = [P] * 14 + [I] * 8 + [P, Z, P]
        L.gdr_chunk_bwd.restype = I
        L.gdr_chunk_bwd_workspace_size.argtypes = [I] * 8
        L.gdr_chunk_bwd_workspace_size.restype = Z
        L.gdr_chunk_fwd_gated.argtypes = [P, P, P, P, P, P, P, ctypes.c_float, P, P, P, I, I, I, I, I, I, I, I,
                                          P, Z, P]
        L.gdr_chunk_fwd_gated.restype = I
        L.gdr2_chunk_fwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, Z, P]
        L.gdr2_chunk_fwd.restype = I
        L.gdr2_chunk_fwd_workspace_size.argtypes = [I, I, I, I, I, I, I, I]
        L.gdr2_chunk_fwd_workspace_size.restype = Z
        L.gdr2_recurrent_step.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, P]
        L.gdr2_recurrent_step.restype = I
        L.gdr_status_string.argtypes = [I]
        L.gdr_status_string.restype = ctypes.c_char_p
        L.gdr_last_cuda_error.restype = I
        L.gdr_last_launch_count.restype = I
        L.gdr_device_status.argtypes = [P]
        L.gdr_device_status.restype = I
        L.gdr_debug_set_wait_budget.argtypes = [ctypes.c_longlong]
        L.gdr_debug_set_wait_budget.restype = None
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != GDR_OK:
        L = lib()
        name = L.gdr_status_string(status).decode()
        extra = f" (cudaError {L.gdr_last_cuda_error()})" if name == "GDR_ERR_CUDA" else ""
        raise GDRError(f"{what}: {name}{extra}")


def last_launch_count() -> int:
    """Kernels launched by this thread's last successful library call."""
    return int(lib().gdr_last_launch_count())


def device_status(device=None, stream=None) -> int:
    """Synchronize the stream and return (and clear) the library's device
    status word: 0 unless a kernel ran out of a bounded wait (GDR_ERR_TIMEOUT)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return int(lib().gdr_device_status(_stream_handle(dev, stream)))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device: torch.device, stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    h = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return ctypes.c_void_p(h)


def _need(t: torch.Tensor, name: str, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def chunk_fwd_workspace_size(B, H, T, dk, dv, C=64, gate="per_channel", dtype=torch.bfloat16) -> int:
    g = GATE_PER_CHANNEL if gate == "per_channel" else GATE_SCALAR
    return int(lib().gdr_chunk_fwd_workspace_size(B, H, T, dk, dv, C, g, _DTYPES[dtype]))


def _to_device(x, device):
    return None if x is None else x.to(device, non_blocking=True)


def _to_host(x):
    """Device tensor -> page-locked host tensor.  The device is synchronized
    first (the kernels may run on a stream other than the current one); the
    copy into pinned memory then runs at the full DMA rate."""
    if x is None:
        return None
    torch.cuda.synchronize(x.device)
    h = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    h.copy_(x)
    return h


def chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
              S0: Optional[torch.Tensor] = None, C: int = 64, gate: Optional[str] = None,
              O: Optional[torch.Tensor] = None, S_T: Optional[torch.Tensor] = None,
              final_state: bool = True, workspace: Optional[torch.Tensor] = None,
              stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise forward of the gated delta rule (``gdr_chunk_fwd``).

    q, k [B,H,T,dk] and v [B,H,T,dv] (fp32 or bf16, same dtype); g fp32
    [B,H,T,dk] (per-channel, KDA) or [B,H,T] (scalar, Gated DeltaNet);
    beta fp32 [B,H,T]; S0 fp32 [B,H,dv,dk] or None (zeros).  Returns
    (O [B,H,T,dv] in v's dtype, S_T [B,H,dv,dk] fp32 or None).
    """
    host = not q.is_cuda
    if host:
        dev = torch.device("cuda", torch.cuda.current_device())
        q, k, v, g, beta, S0 = (_to_device(x, dev) for x in (q, k, v, g, beta, S0))
    dev = q.device
    if gate is None:
        gate = "per_channel" if g.dim() == 4 else "scalar"
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DTYPES:
        raise TypeError("q, k, v must be float32 or bfloat16")
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dt, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    if tuple(k.shape) != (B, H, T, dk) or tuple(v.shape[:3]) != (B, H, T) or tuple(beta.shape) != (B, H, T):
        raise ValueError("inconsistent shapes")
    if gate == "per_channel" and tuple(g.shape) != (B, H, T, dk):
        raise ValueError("per-channel g must be [B,H,T,dk]")
    if gate == "scalar" and tuple(g.shape) != (B, H, T):
        raise ValueError("scalar g must be [B,H,T]")
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (B, H, dv, dk):
            raise ValueError("S0 must be [B,H,dv,dk]")
    if O is None:
        O = torch.empty(B, H, T, dv, dtype=dt, device=dev)
    _need(O, "O", dt, dev)
    if S_T is None and final_state:
        S_T = torch.empty(B, H, dv, dk, dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, dev)
    gm = GATE_PER_CHANNEL if gate == "per_channel" else GATE_SCALAR
    L = lib()
    ws_bytes = int(L.gdr_chunk_fwd_workspace_size(B, H, T, dk, dv, C, gm, _DTYPES[dt]))
    if ws_bytes and (workspace is None or workspace.numel() * workspace.element_size() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = L.gdr_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(O), _ptr(S_T),
                         B, H, T, dk, dv, C, gm, _DTYPES[dt],
                         _ptr(workspace) if ws_bytes else None, ws_bytes, _stream_handle(dev, stream))
    _check(st, "gdr_chunk_fwd")
    if host:
        O = _to_host(O)
        S_T = _to_host(S_T)
    return O, S_T


def chunk_fwd_prologue(q_raw: torch.Tensor, k_raw: torch.Tensor, v: torch.Tensor, a: torch.Tensor,
                       A_log: torch.Tensor, dt_bias: torch.Tensor, b_logit: torch.Tensor,
                       S0: Optional[torch.Tensor] = None, C: int = 64, gate: Optional[str] = None,
                       O: Optional[torch.Tensor] = None, S_T: Optional[torch.Tensor] = None,
                       final_state: bool = True, workspace: Optional[torch.Tensor] = None,
                       stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise forward with the input prologue fused in (``gdr_chunk_fwd_prologue``).

    q_raw, k_raw [B,H,T,dk] and v [B,H,T,dv] bf16 (q, k not normalised);
    gate pre-activation a bf16 [B,H,T,dk] (per-channel) or [B,H,T] (scalar);
    A_log fp32 [H]; dt_bias fp32 [H,dk] or [H]; b_logit fp32 [B,H,T]; S0 fp32
    [B,H,dv,dk] or None.  Returns (O [B,H,T,dv] bf16, S_T fp32 or None).
    """
    host = not q_raw.is_cuda
    if host:
        dev = torch.device("cuda", torch.cuda.current_device())
        q_raw, k_raw, v, a, A_log, dt_bias, b_logit, S0 = (_to_device(x, dev) for x in
                                                           (q_raw, k_raw, v, a, A_log, dt_bias, b_logit, S0))
    dev = q_raw.device
    if gate is None:
        gate = "per_channel" if a.dim() == 4 else "scalar"
    B, H, T, dk = q_raw.shape
    dv = v.shape[-1]
    dt = q_raw.dtype
    if dt != torch.bfloat16:
        raise TypeError("the prologue forward takes bf16 q, k, v, a")
    for t, n in ((q_raw, "q_raw"), (k_raw, "k_raw"), (v, "v"), (a, "a")):
        _need(t, n, dt, dev)
    for t, n in ((A_log, "A_log"), (dt_bias, "dt_bias"), (b_logit, "b_logit")):
        _need(t, n, torch.float32, dev)
    if tuple(k_raw.shape) != (B, H, T, dk) or tuple(v.shape[:3]) != (B, H, T) or tuple(b_logit.shape) != (B, H, T):
        raise ValueError("inconsistent shapes")
    if tuple(A_log.shape) != (H,):
        raise ValueError("A_log must be [H]")
    if gate == "per_channel" and (tuple(a.shape) != (B, H, T, dk) or tuple(dt_bias.shape) != (H, dk)):
        raise ValueError("per-channel gate: a [B,H,T,dk], dt_bias [H,dk]")
    if gate == "scalar" and (tuple(a.shape) != (B, H, T) or tuple(dt_bias.shape) != (H,)):
        raise ValueError("scalar gate: a [B,H,T], dt_bias [H]")
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (B, H, dv, dk):
            raise ValueError("S0 must be [B,H,dv,dk]")
    if O is None:
        O = torch.empty(B, H, T, dv, dtype=dt, device=dev)
    _need(O, "O", dt, dev)
    if S_T is None and final_state:
        S_T = torch.empty(B, H, dv, dk, dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, dev)
    gm = GATE_PER_CHANNEL if gate == "per_channel" else GATE_SCALAR
    L = lib()
    ws_bytes = int(L.gdr_chunk_fwd_workspace_size(B, H, T, dk, dv, C, gm, _DTYPES[dt]))
    if ws_bytes and (workspace is None or workspace.numel() * workspace.element_size() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = L.gdr_chunk_fwd_prologue(_ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(a), _ptr(A_log), _ptr(dt_bias),
                                  _ptr(b_logit), _ptr(S0), _ptr(O), _ptr(S_T), B, H, T, dk, dv, C, gm, _DTYPES[dt],
                                  _ptr(workspace) if ws_bytes else None, ws_bytes, _stream_handle(dev, stream))
    _check(st, "gdr_chunk_fwd_prologue")
    if host:
        O = _to_host(O)
        S_T = _to_host(S_T)
    return O, S_T


def recurrent_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
                   S: torch.Tensor, o: Optional[torch.Tensor] = None, gate: Optional[str] = None,
                   stream=None) -> torch.Tensor:
    """One decode step (``gdr_recurrent_step``); S [B,H,dv,dk] fp32 is updated in place.

    q, k [B,H,dk], v [B,H,dv] (fp32 or bf16); g fp32 [B,H,dk] (per-channel)
    or [B,H] (scalar); beta fp32 [B,H].  Returns o [B,H,dv] in v's dtype.
    """
    dev = S.device
    if gate is None:
        gate = "per_channel" if g.dim() == 3 else "scalar"
    B, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DTYPES:
        raise TypeError("q, k, v must be float32 or bfloat16")
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dt, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(S, "S", torch.float32, dev)
    if tuple(S.shape) != (B, H, dv, dk) or tuple(beta.shape) != (B, H):
        raise ValueError("inconsistent shapes")
    if o is None:
        o = torch.empty(B, H, dv, dtype=dt, device=dev)
    _need(o, "o", dt, dev)
    gm = GATE_PER_CHANNEL if gate == "per_channel" else GATE_SCALAR
    st = lib().gdr_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o),
                                  B, H, dk, dv, gm, _DTYPES[dt], _stream_handle(dev, stream))
    _check(st, "gdr_recurrent_step")
    return o


def chunk_fwd_gdr2(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, b: torch.Tensor,
                   w: torch.Tensor, S0: Optional[torch.Tensor] = None, C: int = 64, gate: Optional[str] = None,
                   O: Optional[torch.Tensor] = None, S_T: Optional[torch.Tensor] = None,
                   final_state: bool = True, workspace: Optional[torch.Tensor] = None,
                   stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise Gated Delta Rule-2 forward (``gdr2_chunk_fwd``).

    q, k, b [B,H,T,dk] and v, w [B,H,T,dv] bf16 (b: erase gate, w: write
    gate); g fp32 [B,H,T,dk] (per-channel) or [B,H,T] (scalar); S0 fp32
    [B,H,dv,dk] or None.  Returns (O [B,H,T,dv] bf16, S_T fp32 or None).
    """
    host = not q.is_cuda
    if host:
        dev = torch.device("cuda", torch.cuda.current_device())
        q, k, v, g, b, w, S0 = (_to_device(x, dev) for x in (q, k, v, g, b, w, S0))
    dev = q.device
    if gate is None:
        gate = "per_channel" if g.dim() == 4 else "scalar"
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt != torch.bfloat16:
        raise TypeError("the Gated Delta Rule-2 forward takes bf16 q, k, v, b, w")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (b, "b"), (w, "w")):
        _need(t, n, dt, dev)
    _need(g, "g", torch.float32, dev)
    if tuple(k.shape) != (B, H, T, dk) or tuple(b.shape) != (B, H, T, dk) or tuple(v.shape[:3]) != (B, H, T) \
            or tuple(w.shape) != (B, H, T, dv):
        raise ValueError("inconsistent shapes")
    if gate == "per_channel" and tuple(g.shape) != (B, H, T, dk):
        raise ValueError("per-channel g must be [B,H,T,dk]")
    if gate == "scalar" and tuple(g.shape) != (B, H, T):
        raise ValueError("scalar g must be [B,H,T]")
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (B, H, dv, dk):
            raise ValueError("S0 must be [B,H,dv,dk]")
    if O is None:
        O = torch.empty(B, H, T, dv, dtype=dt, device=dev)
    _need(O, "O", dt, dev)
    if S_T is None and final_state:
        S_T = torch.empty(B, H, dv, dk, dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, dev)
    gm = GATE_PER_CHANNEL if gate == "per_channel" else GATE_SCALAR
    L = lib()
    ws_bytes = int(L.gdr2_chunk_fwd_workspace_size(B, H, T, dk, dv, C, gm, _DTYPES[dt]))
    if ws_bytes and (workspace is None or workspace.numel() * workspace.element_size() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = L.gdr2_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0), _ptr(O), _ptr(S_T),
                          B, H, T, dk, dv, C, gm, _DTYPES[dt],
                          _ptr(workspace) if ws_bytes else None, ws_bytes, _stream_handle(dev, stream))
    _check(st, "gdr2_chunk_fwd")
    if host:
        O = _to_host(O)
        S_T = _to_host(S_T)
    return O, S_T


def recurrent_step_gdr2(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, b: torch.Tensor,
                        w: torch.Tensor, S: torch.Tensor, o: Optional[torch.Tensor] = None,
                        gate: Optional[str] = None, stream=None) -> torch.Tensor:
    """One Gated Delta Rule-2 decode step (``gdr2_recurrent_step``); S is updated in place.

    q, k, b [B,H,dk], v, w [B,H,dv] (fp32 or bf16, one dtype); g fp32
    [B,H,dk] or [B,H].  Returns o [B,H,dv] in v's dtype.
    """
    dev = S.device
    if gate is None:
        gate = "per_channel" if g.dim() == 3 else "scalar"
    B, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DTYPES:
        raise TypeError("q, k, v, b, w must be float32 or bfloat16")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (b, "b"), (w, "w")):
        _need(t, n, dt, dev)
    _need(g, "g", torch.float32, dev)
    _need(S, "S", torch.float32, dev)
    if tuple(S.shape) != (B, H, dv, dk) or tuple(b.shape) != (B, H, dk) or tuple(w.shape) != (B, H, dv):
        raise ValueError("inconsistent shapes")
    if o is None:
        o = torch.empty(B, H, dv, dtype=dt, device=dev)
    _need(o, "o", dt, dev)
    gm = GATE_PER_CHANNEL if gate == "per_channel" else GATE_SCALAR
    st = lib().gdr2_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S), _ptr(o),
                                   B, H, dk, dv, gm, _DTYPES[dt], _stream_handle(dev, stream))
    _check(st, "gdr2_recurrent_step")
    return o


def chunk_fwd_gated(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
                    gate: torch.Tensor, norm_w: torch.Tensor, eps: float = 1e-6,
                    S0: Optional[torch.Tensor] = None, C: int = 64, gate_mode: Optional[str] = None,
                    Y: Optional[torch.Tensor] = None, S_T: Optional[torch.Tensor] = None,
                    final_state: bool = True, workspace: Optional[torch.Tensor] = None,
                    stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise forward with the output epilogue fused in (``gdr_chunk_fwd_gated``):
    Y = Sigmoid(gate) * RMSNorm(o) per head and token.

    q, k [B,H,T,dk], v and gate [B,H,T,dv] bf16; g, beta, S0 as ``chunk_fwd``;
    norm_w fp32 [dv].  Returns (Y [B,H,T,dv] bf16, S_T fp32 or None).
    """
    host = not q.is_cuda
    if host:
        dev = torch.device("cuda", torch.cuda.current_device())
        q, k, v, g, beta, gate, norm_w, S0 = (_to_device(x, dev) for x in (q, k, v, g, beta, gate, norm_w, S0))
    dev = q.device
    if gate_mode is None:
        gate_mode = "per_channel" if g.dim() == 4 else "scalar"
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt != torch.bfloat16:
        raise TypeError("the gated-output forward takes bf16 q, k, v, gate")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (gate, "gate")):
        _need(t, n, dt, dev)
    for t, n in ((g, "g"), (beta, "beta"), (norm_w, "norm_w")):
        _need(t, n, torch.float32, dev)
    if tuple(k.shape) != (B, H, T, dk) or tuple(v.shape[:3]) != (B, H, T) or tuple(beta.shape) != (B, H, T) \
            or tuple(gate.shape) != (B, H, T, dv) or tuple(norm_w.shape) != (dv,):
        raise ValueError("inconsistent shapes")
    if gate_mode == "per_channel" and tuple(g.shape) != (B, H, T, dk):
        raise ValueError("per-channel g must be [B,H,T,dk]")
    if gate_mode == "scalar" and tuple(g.shape) != (B, H, T):
        raise ValueError("scalar g must be [B,H,T]")
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (B, H, dv, dk):
            raise ValueError("S0 must be [B,H,dv,dk]")
    if Y is None:
        Y = torch.empty(B, H, T, dv, dtype=dt, device=dev)
    _need(Y, "Y", dt, dev)
    if S_T is None and final_state:
        S_T = torch.empty(B, H, dv, dk, dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, dev)
    gm = GATE_PER_CHANNEL if gate_mode == "per_channel" else GATE_SCALAR
    L = lib()
    ws_bytes = int(L.gdr_chunk_fwd_workspace_size(B, H, T, dk, dv, C, gm, _DTYPES[dt]))
    if ws_bytes and (workspace is None or workspace.numel() * workspace.element_size() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = L.gdr_chunk_fwd_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(gate), _ptr(norm_w), float(eps),
                               _ptr(S0), _ptr(Y), _ptr(S_T), B, H, T, dk, dv, C, gm, _DTYPES[dt],
                               _ptr(workspace) if ws_bytes else None, ws_bytes, _stream_handle(dev, stream))
    _check(st, "gdr_chunk_fwd_gated")
    if host:
        Y = _to_host(Y)
        S_T = _to_host(S_T)
    return Y, S_T


def chunk_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
              dO: torch.Tensor, S0: Optional[torch.Tensor] = None, dS_T: Optional[torch.Tensor] = None,
              C: int = 64, gate: Optional[str] = None, want_dS0: bool = True,
              workspace: Optional[torch.Tensor] = None, stream=None):
    """Backward of the chunkwise forward (``gdr_chunk_bwd``): the gradients of
    <dO, O> + <dS_T, S_T> with respect to q, k, v, g, beta and S0.

    Inputs as ``chunk_fwd`` plus dO [B,H,T,dv] (dtype of v) and dS_T fp32
    [B,H,dv,dk] or None.  Returns (dq, dk, dv, dg, dbeta, dS0 or None).
    Host tensors are copied to the current device and the gradients back.
    """
    host = not q.is_cuda
    if host:
        d = torch.device("cuda", torch.cuda.current_device())
        q, k, v, g, beta, dO, S0, dS_T = (_to_device(x, d) for x in (q, k, v, g, beta, dO, S0, dS_T))
    dev = q.device
    if gate is None:
        gate = "per_channel" if g.dim() == 4 else "scalar"
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DTYPES:
        raise TypeError("q, k, v must be float32 or bfloat16")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dO, "dO")):
        _need(t, n, dt, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    if tuple(k.shape) != (B, H, T, dk) or tuple(v.shape[:3]) != (B, H, T) or tuple(beta.shape) != (B, H, T) \
            or tuple(dO.shape) != tuple(v.shape):
        raise ValueError("inconsistent shapes")
    for t, n in ((S0, "S0"), (dS_T, "dS_T")):
        if t is not None:
            _need(t, n, torch.float32, dev)
            if tuple(t.shape) != (B, H, dv, dk):
                raise ValueError(f"{n} must be [B,H,dv,dk]")
    dq, dk_, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dg, dbeta = torch.empty_like(g), torch.empty_like(beta)
    dS0 = torch.empty(B, H, dv, dk, dtype=torch.float32, device=dev) if want_dS0 else None
    gm = GATE_PER_CHANNEL if gate == "per_channel" else GATE_SCALAR
    L = lib()
    ws_bytes = int(L.gdr_chunk_bwd_workspace_size(B, H, T, dk, dv, C, gm, _DTYPES[dt]))
    if ws_bytes and (workspace is None or workspace.numel() * workspace.element_size() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = L.gdr_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(dO), _ptr(dS_T),
                         _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dg), _ptr(dbeta), _ptr(dS0),
                         B, H, T, dk, dv, C, gm, _DTYPES[dt],
                         _ptr(workspace) if ws_bytes else None, ws_bytes, _stream_handle(dev, stream))
    _check(st, "gdr_chunk_bwd")
    out = (dq, dk_, dv_, dg, dbeta, dS0)
    if host:
        out = tuple(_to_host(t) for t in out)
    return out


def chunk_bwd_workspace_size(B, H, T, dk, dv, C=64, gate="per_channel", dtype=torch.bfloat16) -> int:
    g = GATE_PER_CHANNEL if gate == "per_channel" else GATE_SCALAR
    return int(lib().gdr_chunk_bwd_workspace_size(B, H, T, dk, dv, C, g, _DTYPES[dtype]))
