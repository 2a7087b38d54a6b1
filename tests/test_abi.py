"""The C ABI library loads, exports every symbol include/gdr.h declares, and
rejects bad arguments on the host before any device work (no GPU needed)."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_89_b200 as gdr
from gated_delta_rule_89_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, UNSUPPORTED, ALIGN = 0, 1, 2, 3


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return gdr.lib()


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"\b(gdr_[a-z0-9_]+)\s*\(", txt)
    return sorted(set(names))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "gdr_chunk_fwd" in names and "gdr_recurrent_step" in names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    assert L.gdr_status_string(0) == b"GDR_OK"
    assert L.gdr_status_string(3) == b"GDR_ERR_ALIGNMENT"
    assert L.gdr_status_string(99) == b"GDR_ERR_UNKNOWN"


P = ctypes.c_void_p
GOOD = P(0x100000)      # never dereferenced: every case below fails validation first
ODD = P(0x100008)


def chunk(L, B=1, H=1, T=64, dk=128, dv=128, C=64, gate=0, dtype=1, ptr=GOOD, S0=None, ST=None,
          ws=1 << 40, wsp=GOOD):
    return L.gdr_chunk_fwd(ptr, ptr, ptr, ptr, ptr, S0, ptr, ST, B, H, T, dk, dv, C, gate, dtype, wsp, ws, None)


def test_chunk_argument_validation(L):
    assert chunk(L, B=-1) == INVALID
    assert chunk(L, T=-3) == INVALID
    assert chunk(L, gate=2) == INVALID
    assert chunk(L, dtype=5) == INVALID
    assert chunk(L, dk=0) == INVALID
    assert chunk(L, dk=96) == UNSUPPORTED
    assert chunk(L, dv=256) == UNSUPPORTED
    assert chunk(L, C=48) == UNSUPPORTED
    assert chunk(L, ptr=ODD) == ALIGN
    assert chunk(L, ptr=None) == INVALID
    assert chunk(L, ST=ODD) == ALIGN
    assert chunk(L, wsp=ODD) == ALIGN
    # the tensor-core path needs its workspace; a short or missing one is refused
    need = L.gdr_chunk_fwd_workspace_size(1, 1, 64, 128, 128, 64, 0, 1)
    assert need > 0
    assert chunk(L, ws=need - 1) == INVALID
    assert chunk(L, wsp=None) == INVALID
    # empty problems succeed without touching the device
    assert chunk(L, B=0) == OK and L.gdr_last_launch_count() == 0
    assert chunk(L, H=0) == OK
    assert chunk(L, T=0) == OK          # no S_T requested: nothing to do


def prologue(L, B=1, H=1, T=64, dk=128, dv=128, C=64, gate=0, dtype=1, ptr=GOOD, a=GOOD, alog=GOOD,
             blog=GOOD, ST=None, ws=1 << 40, wsp=GOOD):
    return L.gdr_chunk_fwd_prologue(ptr, ptr, ptr, a, alog, ptr, blog, None, ptr, ST, B, H, T, dk, dv, C, gate,
                                    dtype, wsp, ws, None)


def test_prologue_argument_validation(L):
    assert prologue(L, B=-1) == INVALID
    assert prologue(L, gate=3) == INVALID
    # the fused prologue runs on the tensor-core configuration only
    assert prologue(L, dtype=0) == UNSUPPORTED
    assert prologue(L, dk=64, dv=64) == UNSUPPORTED
    assert prologue(L, C=32) == UNSUPPORTED
    assert prologue(L, a=None) == INVALID
    assert prologue(L, alog=None) == INVALID
    assert prologue(L, blog=None) == INVALID
    assert prologue(L, a=ODD) == ALIGN
    assert prologue(L, alog=P(0x100002)) == ALIGN
    assert prologue(L, wsp=None) == INVALID
    assert prologue(L, B=0) == OK and L.gdr_last_launch_count() == 0
    assert prologue(L, T=0) == OK


def gdr2(L, B=1, H=1, T=64, dk=128, dv=128, C=64, gate=0, dtype=1, ptr=GOOD, b=GOOD, w=GOOD, ws=1 << 40, wsp=GOOD):
    return L.gdr2_chunk_fwd(ptr, ptr, ptr, ptr, b, w, None, ptr, None, B, H, T, dk, dv, C, gate, dtype, wsp, ws, None)


def test_gdr2_argument_validation(L):
    assert gdr2(L, B=-1) == INVALID
    assert gdr2(L, gate=2) == INVALID
    assert gdr2(L, dtype=0) == UNSUPPORTED          # the tensor-core configuration only
    assert gdr2(L, dk=64, dv=64) == UNSUPPORTED
    assert gdr2(L, b=None) == INVALID
    assert gdr2(L, w=None) == INVALID
    assert gdr2(L, w=ODD) == ALIGN
    need = L.gdr2_chunk_fwd_workspace_size(1, 1, 64, 128, 128, 64, 0, 1)
    assert need == _tc_workspace(1, 1, 64) + 64 * 128 * 2   # plus w * v, bf16 per token
    assert gdr2(L, ws=need - 1) == INVALID
    assert gdr2(L, B=0) == OK and L.gdr_last_launch_count() == 0
    assert gdr2(L, T=0) == OK

    def step(dk=128, dv=128, b=GOOD, w=GOOD, ptr=GOOD):
        return L.gdr2_recurrent_step(ptr, ptr, ptr, ptr, b, w, ptr, ptr, 2, 2, dk, dv, 0, 1, None)
    assert step(dk=32) == UNSUPPORTED
    assert step(b=None) == INVALID
    assert step(w=ODD) == ALIGN


def gated(L, B=1, H=1, T=64, dk=128, dv=128, C=64, gate=0, dtype=1, ptr=GOOD, og=GOOD, nw=GOOD, eps=1e-6,
          ws=1 << 40, wsp=GOOD):
    return L.gdr_chunk_fwd_gated(ptr, ptr, ptr, ptr, ptr, og, nw, eps, None, ptr, None, B, H, T, dk, dv, C, gate,
                                 dtype, wsp, ws, None)


def test_gated_argument_validation(L):
    assert gated(L, B=-1) == INVALID
    assert gated(L, eps=-1.0) == INVALID
    assert gated(L, eps=float("nan")) == INVALID
    assert gated(L, dtype=0) == UNSUPPORTED
    assert gated(L, C=32) == UNSUPPORTED
    assert gated(L, og=None) == INVALID
    assert gated(L, nw=None) == INVALID
    assert gated(L, og=ODD) == ALIGN
    assert gated(L, nw=P(0x100002)) == ALIGN
    assert gated(L, wsp=None) == INVALID
    assert gated(L, B=0) == OK and L.gdr_last_launch_count() == 0
    assert gated(L, T=0) == OK


def bwd(L, B=1, H=1, T=64, d=128, C=64, gate=0, dtype=1, ptr=GOOD, dST=None, dS0=None, ws=1 << 40, wsp=GOOD):
    return L.gdr_chunk_bwd(ptr, ptr, ptr, ptr, ptr, None, ptr, dST, ptr, ptr, ptr, ptr, ptr, dS0,
                           B, H, T, d, d, C, gate, dtype, wsp, ws, None)


def test_backward_argument_validation(L):
    assert bwd(L, B=-1) == INVALID
    assert bwd(L, gate=2) == INVALID
    assert bwd(L, dtype=3) == INVALID
    assert bwd(L, d=96) == UNSUPPORTED
    assert bwd(L, C=32) == UNSUPPORTED
    assert L.gdr_chunk_bwd(GOOD, GOOD, GOOD, GOOD, GOOD, None, GOOD, None, GOOD, GOOD, GOOD, GOOD, GOOD, None,
                           1, 1, 64, 128, 64, 64, 0, 1, GOOD, 1 << 40, None) == UNSUPPORTED   # d_k != d_v
    assert bwd(L, ptr=ODD) == ALIGN
    assert bwd(L, dS0=ODD) == ALIGN
    assert bwd(L, wsp=None) == INVALID
    need = L.gdr_chunk_bwd_workspace_size(1, 1, 64, 128, 128, 64, 0, 1)
    # per 64-token chunk: G, W, U, V_new, dV_new, K_tail, Q<- (64 x 128 fp32 each),
    # (I + A)^{-1} and Aqk (64 x 64 fp32), the state and its gradient (128 x 128 fp32)
    assert need == 4 * (7 * 64 * 128 + 2 * 64 * 64 + 2 * 128 * 128)
    assert bwd(L, ws=need - 1) == INVALID
    assert L.gdr_chunk_bwd_workspace_size(1, 1, 64, 128, 128, 32, 0, 1) == 0
    assert bwd(L, B=0) == OK and L.gdr_last_launch_count() == 0


def test_step_argument_validation(L):
    def step(B=2, H=2, dk=128, dv=128, gate=0, dtype=1, ptr=GOOD):
        return L.gdr_recurrent_step(ptr, ptr, ptr, ptr, ptr, ptr, ptr, B, H, dk, dv, gate, dtype, None)
    assert step(B=-1) == INVALID
    assert step(gate=7) == INVALID
    assert step(dk=32) == UNSUPPORTED
    assert step(ptr=ODD) == ALIGN
    assert step(ptr=None) == INVALID
    assert step(B=0) == OK


def _tc_workspace(B, H, T):
    # per chunk: T' and Aqk (2 x 64 x 64 bf16), -W and K_tail^T (2 x 64 x 128
    # bf16, whole chunks) and gamma_C (128 fp32); per token: Q<- (128 bf16)
    nch = (T + 63) // 64
    return B * H * (nch * (2 * 64 * 64 * 2 + 2 * 128 * 64 * 2 + 128 * 4) + T * 128 * 2)


def test_workspace_query(L):
    assert L.gdr_chunk_fwd_workspace_size(2, 32, 8192, 128, 128, 64, 0, 1) == _tc_workspace(2, 32, 8192)
    assert L.gdr_chunk_fwd_workspace_size(1, 1, 65, 128, 128, 64, 1, 1) == _tc_workspace(1, 1, 65)
    # fp32 inputs or other sizes run on the CUDA-core path, which needs none
    assert L.gdr_chunk_fwd_workspace_size(1, 2, 256, 64, 64, 64, 0, 0) == 0
    assert L.gdr_chunk_fwd_workspace_size(1, 2, 256, 128, 128, 32, 0, 1) == 0
    assert L.gdr2_chunk_fwd_workspace_size(2, 32, 8192, 128, 128, 64, 0, 1) == \
        _tc_workspace(2, 32, 8192) + 2 * 32 * 8192 * 128 * 2
    assert L.gdr2_chunk_fwd_workspace_size(1, 2, 256, 64, 64, 64, 0, 0) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(gdr, "_lib", None)
    monkeypatch.setattr(gdr, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        gdr.lib()
