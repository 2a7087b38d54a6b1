"""fp64 CPU oracle of the gated delta rule -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  The CUDA library never imports,
links or calls it, and it never imports the CUDA library.  It shares with the
GPU side only the seeded input generator (``gdr_workloads``), which holds none
of the method's arithmetic.

Contents
  * ``forward``   -- the token-by-token fp64 recurrence (``gdr_oracle.c``),
    the parity reference for the chunked forward and the decode step.
  * ``decode``    -- the same recurrence driven one decode step per token.
  * ``forward_gdr2`` / ``decode_gdr2`` -- Gated Delta Rule-2 (per-channel erase
    gate b on the key side, write gate w on the value side), the reference of
    the GDR-2 entry points.
  * ``prologue`` / ``forward_prologue`` -- the input prologue (L2-normalised
    q, k; softplus gate with the -5 bound; sigmoid beta) and the forward fed
    by it, the reference of the fused-prologue entry point.
  * ``backward``  -- reverse mode through the same token recurrence (the
    gradients of <dO, O> + <dS_T, S_T>), the reference of the chunked backward.
  * ``output_gate`` / ``forward_gated`` -- the output epilogue of the layer
    (per-head RMSNorm of o_t, times a sigmoid output gate), the reference of
    the gated-output entry point.
  * ``chunk_form`` (module) -- an fp64 restatement of the chunkwise WY/UT
    equations, used only to pin ``forward`` (it is not a parity reference).

Every function reads exactly the values the GPU receives: bf16 and fp32
tensors are widened to fp64 exactly before the recurrence runs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.gdr_oracle_forward.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I]
            lib.gdr_oracle_forward.restype = I
            lib.gdr_oracle_backward.argtypes = [P] * 14 + [I] * 8
            lib.gdr_oracle_backward.restype = I
            lib.gdr2_oracle_forward.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I]
            lib.gdr2_oracle_forward.restype = I
            lib.gdr_oracle_online_cores.restype = I
            _lib = lib
    return _lib


def online_cores() -> int:
    return int(_load().gdr_oracle_online_cores())


def _f64(x) -> Optional[np.ndarray]:
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        x = x.detach().to("cpu").to(torch.float64).contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def forward(q, k, v, g, beta, S0=None, gate: str = "per_channel", erase=None, write=None,
            clamp: bool = True, threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 recurrence over T tokens.

    Shapes: q, k [B,H,T,dk]; v [B,H,T,dv]; g [B,H,T,dk] (per_channel) or
    [B,H,T] (scalar); beta [B,H,T]; S0 [B,H,dv,dk] or None.
    ``erase`` / ``write`` ([B,H,T]) replace beta on the erase and write sides
    (pins only).  Returns (O [B,H,T,dv], S_T [B,H,dv,dk]) as fp64 numpy arrays.
    """
    qa, ka, va, ga = _f64(q), _f64(k), _f64(v), _f64(g)
    ba = _f64(beta)
    ea, wa = _f64(erase), _f64(write)
    B, H, T, dk = qa.shape
    dv = va.shape[-1]
    assert ka.shape == (B, H, T, dk) and va.shape == (B, H, T, dv)
    if gate == "per_channel":
        assert ga.shape == (B, H, T, dk)
    elif gate == "scalar":
        assert ga.shape == (B, H, T)
    else:
        raise ValueError(gate)
    for x in (ba, ea, wa):
        assert x is None or x.shape == (B, H, T)
    s0 = _f64(S0)
    if s0 is not None:
        assert s0.shape == (B, H, dv, dk)
    O = np.empty((B, H, T, dv), dtype=np.float64)
    ST = np.empty((B, H, dv, dk), dtype=np.float64)
    rc = _load().gdr_oracle_forward(_ptr(qa), _ptr(ka), _ptr(va), _ptr(ga), _ptr(ba), _ptr(ea), _ptr(wa),
                                    _ptr(s0), _ptr(O), _ptr(ST), B, H, T, dk, dv,
                                    1 if gate == "scalar" else 0, 1 if clamp else 0, int(threads))
    if rc != 0:
        raise RuntimeError("oracle forward failed")
    return O, ST


def backward(q, k, v, g, beta, S0, dO, dS_T=None, gate: str = "per_channel", clamp: bool = True,
             threads: int = 0):
    """fp64 gradients of L = <dO, O> + <dS_T, S_T> through the token recurrence
    of ``forward`` (reverse mode, token by token, states recomputed from
    checkpoints).  The per-channel -5 bound passes the gradient where
    g >= -5.  Returns (dq, dk, dv, dg, dbeta, dS0) as fp64 numpy arrays
    shaped like q, k, v, g, beta and the state.
    """
    qa, ka, va, ga, ba, oa = _f64(q), _f64(k), _f64(v), _f64(g), _f64(beta), _f64(dO)
    B, H, T, dk = qa.shape
    dv = va.shape[-1]
    assert ka.shape == qa.shape and oa.shape == va.shape and ba.shape == (B, H, T)
    assert ga.shape == ((B, H, T, dk) if gate == "per_channel" else (B, H, T))
    s0, dst = _f64(S0), _f64(dS_T)
    for x in (s0, dst):
        assert x is None or x.shape == (B, H, dv, dk)
    outs = [np.zeros_like(qa), np.zeros_like(ka), np.zeros_like(va), np.zeros_like(ga), np.zeros_like(ba),
            np.zeros((B, H, dv, dk))]
    rc = _load().gdr_oracle_backward(_ptr(qa), _ptr(ka), _ptr(va), _ptr(ga), _ptr(ba), _ptr(s0), _ptr(oa), _ptr(dst),
                                     *[_ptr(o) for o in outs], B, H, T, dk, dv, 1 if gate == "scalar" else 0,
                                     1 if clamp else 0, int(threads))
    if rc != 0:
        raise RuntimeError("oracle backward failed")
    return tuple(outs)


def forward_gdr2(q, k, v, g, b, w, S0=None, gate: str = "per_channel", clamp: bool = True,
                 threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 Gated Delta Rule-2 over T tokens ("Token Mixer I", section "Gated
    DeltaNet-2: Decoupling Erase and Write in Linear Attention", eq. (10)):
    the state is read along b_t * k_t and the delta w_t * v_t - S~ (b_t * k_t)
    is written along k_t.

    Shapes: q, k, b [B,H,T,dk]; v, w [B,H,T,dv]; g as in ``forward``.  The
    -5 bound applies to a per-channel gate when ``clamp`` (as in ``forward``).
    Returns (O [B,H,T,dv], S_T [B,H,dv,dk]) as fp64 numpy arrays.
    """
    qa, ka, va, ga, ba, wa = _f64(q), _f64(k), _f64(v), _f64(g), _f64(b), _f64(w)
    B, H, T, dk = qa.shape
    dv = va.shape[-1]
    assert ka.shape == (B, H, T, dk) and ba.shape == (B, H, T, dk)
    assert va.shape == (B, H, T, dv) and wa.shape == (B, H, T, dv)
    if gate == "per_channel":
        assert ga.shape == (B, H, T, dk)
    elif gate == "scalar":
        assert ga.shape == (B, H, T)
    else:
        raise ValueError(gate)
    s0 = _f64(S0)
    if s0 is not None:
        assert s0.shape == (B, H, dv, dk)
    O = np.empty((B, H, T, dv), dtype=np.float64)
    ST = np.empty((B, H, dv, dk), dtype=np.float64)
    rc = _load().gdr2_oracle_forward(_ptr(qa), _ptr(ka), _ptr(va), _ptr(ga), _ptr(ba), _ptr(wa), _ptr(s0),
                                     _ptr(O), _ptr(ST), B, H, T, dk, dv, 1 if gate == "scalar" else 0,
                                     1 if clamp else 0, int(threads))
    if rc != 0:
        raise RuntimeError("oracle forward_gdr2 failed")
    return O, ST


L2NORM_EPS = 1e-6   # the pages do not give the epsilon of L2Norm; see the reading in the design notes


def prologue(q_raw, k_raw, a, A_log, dt_bias, b_logit, gate: str = "per_channel"):
    """The input prologue of a KDA / Gated DeltaNet layer, in fp64.

    "Token Mixer I", section "Kimi Delta Attention", Neural
    Parameterization: q and k are L2-normalised per head and token, and
    beta = Sigmoid(logit).  "Kimi Linear paper notes", gate paragraph: the
    log-decay is -exp(A_log) * softplus(a + dt_bias), with A_log per head and
    dt_bias per head and key channel (per head for a scalar gate); KDA bounds
    the per-channel log-decay below by g_min = -5 ("KDA engineering notes",
    lower-bounded decay).

    Shapes: q_raw, k_raw [B,H,T,dk]; a [B,H,T,dk] or [B,H,T]; A_log [H];
    dt_bias [H,dk] or [H]; b_logit [B,H,T].  Returns fp64 (q, k, g, beta).
    """
    q = _f64(q_raw)
    k = _f64(k_raw)
    q = q / np.sqrt((q * q).sum(-1, keepdims=True) + L2NORM_EPS)
    k = k / np.sqrt((k * k).sum(-1, keepdims=True) + L2NORM_EPS)
    A = np.exp(_f64(A_log))                       # [H]
    z = _f64(a)
    dtb = _f64(dt_bias)
    if gate == "per_channel":
        z = z + dtb[None, :, None, :]
        sp = np.logaddexp(0.0, z)                 # softplus(z) = log(1 + e^z)
        g = np.maximum(-A[None, :, None, None] * sp, -5.0)
    elif gate == "scalar":
        z = z + dtb[None, :, None]
        g = -A[None, :, None] * np.logaddexp(0.0, z)
    else:
        raise ValueError(gate)
    beta = 1.0 / (1.0 + np.exp(-_f64(b_logit)))
    return q, k, g, beta


def forward_prologue(q_raw, k_raw, v, a, A_log, dt_bias, b_logit, S0=None, gate: str = "per_channel",
                     threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """``prologue`` then ``forward``: the reference of the fused-prologue forward."""
    q, k, g, beta = prologue(q_raw, k_raw, a, A_log, dt_bias, b_logit, gate)
    return forward(q, k, v, g, beta, S0, gate=gate, clamp=False, threads=threads)


def decode(q, k, v, g, beta, S, gate: str = "per_channel", threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """``steps`` consecutive single-token updates.

    q, k [steps,B,H,dk]; v [steps,B,H,dv]; g [steps,B,H,dk] or [steps,B,H];
    beta [steps,B,H]; S [B,H,dv,dk].  A decode step is one token of the
    recurrence, so this runs ``forward`` with the steps as the token axis.
    Returns (o [steps,B,H,dv], S_final [B,H,dv,dk]).
    """
    mv = lambda x: _f64(x).transpose(1, 2, 0, *range(3, _f64(x).ndim)).copy()
    O, ST = forward(mv(q), mv(k), mv(v), mv(g), mv(beta), S0=S, gate=gate, threads=threads)
    return O.transpose(2, 0, 1, 3).copy(), ST


def decode_gdr2(q, k, v, g, b, w, S, gate: str = "per_channel", threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """``steps`` consecutive Gated Delta Rule-2 single-token updates: q, k, b
    [steps,B,H,dk]; v, w [steps,B,H,dv]; g [steps,B,H,dk] or [steps,B,H];
    S [B,H,dv,dk].  Returns (o [steps,B,H,dv], S_final)."""
    mv = lambda x: _f64(x).transpose(1, 2, 0, *range(3, _f64(x).ndim)).copy()
    O, ST = forward_gdr2(mv(q), mv(k), mv(v), mv(g), mv(b), mv(w), S0=S, gate=gate, threads=threads)
    return O.transpose(2, 0, 1, 3).copy(), ST


def output_gate(O, gate, norm_w, eps: float):
    """The output epilogue of a KDA layer, in fp64: "Token Mixer I", section
    "The Kimi Linear Model Architecture" -- before the output projection W_o,
    each head's output o_t is normalised by a per-head RMSNorm and multiplied
    by a data-dependent sigmoid gate:

        y_t = Sigmoid(gate_t) * RMSNorm(o_t),
        RMSNorm(x) = x / sqrt(mean_c x_c^2 + eps) * norm_w      (over the d_v channels)

    O, gate [B,H,T,dv]; norm_w [dv] (one weight vector shared by the heads).
    Returns y [B,H,T,dv] (fp64).
    """
    o = _f64(O)
    z = _f64(gate)
    wv = _f64(norm_w)
    ms = (o * o).mean(-1, keepdims=True)
    return o / np.sqrt(ms + eps) * wv * (1.0 / (1.0 + np.exp(-z)))


def forward_gated(q, k, v, g, beta, gate, norm_w, eps: float, S0=None, gate_mode: str = "per_channel",
                  threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """``forward`` then ``output_gate``: returns (y [B,H,T,dv], S_T)."""
    O, ST = forward(q, k, v, g, beta, S0, gate=gate_mode, threads=threads)
    return output_gate(O, gate, norm_w, eps), ST
