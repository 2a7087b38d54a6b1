"""GPU parity of the chunked backward (gdr_chunk_bwd) against the fp64
oracle's reverse-mode ``backward`` on the same inputs.  Every gradient is
compared element by element: max|X - X_ref| / max|X_ref| <= 2e-2 for bf16
inputs (dq, dk, dv leave in bf16; the arithmetic is fp32) and <= 1e-4 for
fp32 inputs."""
import numpy as np
import pytest
import torch

import gated_delta_rule_89_b200 as gdr
import gdr_workloads as W
import oracle

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dS0")


def relerr(x, ref):
    x = np.asarray(x.detach().double().cpu() if isinstance(x, torch.Tensor) else x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-30))


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gdr.lib()
    yield


def check(w, tol, with_dST=True, with_S0=True):
    x = W.generate(w)
    gr = W.generate_grads(w)
    S0 = x["S0"] if with_S0 else None
    dST = gr["dS_T"] if with_dST else None
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], S0, gr["dO"], dST, gate=w.gate)
    d = {k: v.cuda() for k, v in x.items()}
    got = gdr.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], gr["dO"].cuda(),
                        S0=d["S0"] if with_S0 else None, dS_T=dST.cuda() if with_dST else None, gate=w.gate)
    torch.cuda.synchronize()
    assert gdr.last_launch_count() == 4
    errs = {n: relerr(a, b) for n, a, b in zip(NAMES, got, ref)}
    assert all(e <= tol for e in errs.values()), errs
    return errs


CASES = [
    # B, H, T, d, gate, dtype, recipe
    (1, 2, 64, 128, "per_channel", torch.bfloat16, "softplus_n02_clamp5"),
    (1, 2, 200, 128, "per_channel", torch.bfloat16, "softplus_n02_clamp5"),
    (2, 1, 130, 128, "per_channel", torch.bfloat16, "softplus_n02_unbounded"),
    (1, 2, 150, 128, "scalar", torch.bfloat16, "scalar_softplus_n01_plus2"),
    (1, 1, 1, 128, "per_channel", torch.bfloat16, "softplus_n02_clamp5"),
    (2, 1, 300, 128, "per_channel", torch.bfloat16, "long_context_mix"),
    (1, 2, 150, 64, "per_channel", torch.float32, "softplus_n01_plus1_clamp5"),
    (1, 1, 130, 128, "per_channel", torch.float32, "softplus_n02_clamp5"),   # d = 128 fp32: CUDA-core products
    (1, 1, 97, 64, "scalar", torch.float32, "scalar_softplus_n01_plus2"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}H{c[1]}T{c[2]}d{c[3]}-{c[4]}-{str(c[5])[6:]}-{c[6]}")
def test_backward_cases(case):
    B, H, T, d, gate, dt, recipe = case
    w = W.small_chunk_case(B, H, T, d, d, gate, dt, g_recipe=recipe)
    check(w, 1e-4 if dt == torch.float32 else 2e-2)


def test_without_state_gradients():
    w = W.small_chunk_case(1, 2, 100, 128, 128, "per_channel", torch.bfloat16)
    check(w, 2e-2, with_dST=False, with_S0=False)


def test_full_size_sampled():
    w = W.WORKLOADS["kda_d128_t8192"]
    heads = [0, 45]
    d = W.generate(w, device="cuda")
    gr = W.generate_grads(w, device="cuda")
    got = gdr.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], gr["dO"], S0=d["S0"], dS_T=gr["dS_T"])
    torch.cuda.synchronize()
    for t in got:
        assert bool(torch.isfinite(t).all())
    H = w.H
    sel = lambda t: torch.stack([t[h // H, h % H] for h in heads])[:, None].cpu()
    ref = oracle.backward(sel(d["q"]), sel(d["k"]), sel(d["v"]), sel(d["g"]), sel(d["beta"]), sel(d["S0"]),
                          sel(gr["dO"]), sel(gr["dS_T"]))
    errs = {n: relerr(sel(a), b) for n, a, b in zip(NAMES, got, ref)}
    assert all(e <= 2e-2 for e in errs.values()), errs


def test_empty_problems():
    dev = torch.device("cuda")
    # T = 0: S_T = S0, so dS0 = dS_T (zeros without dS_T)
    e = torch.empty(1, 2, 0, 128, dtype=torch.bfloat16, device=dev)
    g = torch.empty(1, 2, 0, 128, device=dev)
    b = torch.empty(1, 2, 0, device=dev)
    dST = torch.randn(1, 2, 128, 128, device=dev)
    out = gdr.chunk_bwd(e, e, e, g, b, e, dS_T=dST)
    torch.cuda.synchronize()
    assert torch.equal(out[5], dST) and out[0].numel() == 0
    out = gdr.chunk_bwd(e, e, e, g, b, e)
    torch.cuda.synchronize()
    assert float(out[5].abs().max()) == 0.0
    # B = 0
    z = torch.empty(0, 2, 64, 128, dtype=torch.bfloat16, device=dev)
    out = gdr.chunk_bwd(z, z, z, torch.empty(0, 2, 64, 128, device=dev), torch.empty(0, 2, 64, device=dev), z)
    assert out[0].shape == (0, 2, 64, 128)
