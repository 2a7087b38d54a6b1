"""The allocation-free chunked forward (gdr_chunk_fwd_noalloc), called
through the C ABI, against the regular entry point (gdr_chunk_fwd).

It exists for callers that cannot allocate device memory (allocator-free
serving loops, regions recorded as graphs, foreign memory owners): its scratch
is a fixed array inside the library.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_delta_rule_89_b200 as gdr
import gdr_workloads as W
import oracle

pytestmark = pytest.mark.gpu

GDR_OK, GDR_ERR_UNSUPPORTED = 0, 2


def _noalloc():
    L = gdr.lib()
    f = L.gdr_chunk_fwd_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P]
    f.restype = I
    return f


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _case(seed, gate, T):
    recipe = "softplus_n02_clamp5" if gate == "per_channel" else "scalar_softplus_n01_plus2"
    w = W.small_chunk_case(2, 3, T, 128, 128, gate, torch.bfloat16, g_recipe=recipe, seed=seed)
    return w, {k: v.cuda() for k, v in W.generate(w).items()}


def test_noalloc_matches_regular_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    f = _noalloc()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # Calls in a row with different inputs and gates: the shared scratch still
    # holds the previous call's data when the next one runs.  The first call is
    # the largest, so its leftovers lie under the later calls' ragged last
    # chunks.  Both entry points run the same deterministic kernels, so the
    # results must be bitwise equal.
    for seed, gate, T in ((21, "per_channel", 1000), (22, "scalar", 517), (23, "per_channel", 70)):
        w, d = _case(seed, gate, T)
        B, H, dk, dv = w.B, w.H, w.dk, w.dv
        assert 0 < gdr.chunk_fwd_workspace_size(B, H, T, dk, dv, 64, gate) <= 32 * 1024 * 1024
        O = torch.full((B, H, T, dv), float("nan"), dtype=torch.bfloat16, device="cuda")
        S = torch.full((B, H, dv, dk), float("nan"), dtype=torch.float32, device="cuda")
        st = f(_ptr(d["q"]), _ptr(d["k"]), _ptr(d["v"]), _ptr(d["g"]), _ptr(d["beta"]), _ptr(d["S0"]),
               _ptr(O), _ptr(S), B, H, T, dk, dv, 64, 0 if gate == "per_channel" else 1, 1, stream)
        assert st == GDR_OK
        O_ref, S_ref = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], C=64, gate=gate)
        torch.cuda.synchronize()
        assert gdr.device_status() == 0
        assert bool(torch.isfinite(O).all()) and bool(torch.isfinite(S).all())
        assert torch.equal(O, O_ref) and torch.equal(S, S_ref), (seed, gate, T)
        # and against the fp64 oracle, at the bf16 tolerance of the parity tests
        c = {k: v.cpu() for k, v in d.items()}
        Oo, So = oracle.forward(c["q"], c["k"], c["v"], c["g"], c["beta"], c["S0"], gate=gate)
        for x, ref in ((O, Oo), (S, So)):
            err = float(np.max(np.abs(x.double().cpu().numpy() - ref)) / np.max(np.abs(ref)))
            assert err <= 2e-2, (seed, gate, T, err)


def test_noalloc_rejects_problems_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    f = _noalloc()
    # 4 x 32 heads x 64 chunks = 8192 chunks need 128 MiB > 32 MiB; refused on the host,
    # before any pointer is touched
    fake = ctypes.c_void_p(0x100000)
    st = f(fake, fake, fake, fake, fake, None, fake, None, 4, 32, 4096, 128, 128, 64, 0, 1, None)
    assert st == GDR_ERR_UNSUPPORTED
