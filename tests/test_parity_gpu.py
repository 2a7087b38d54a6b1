"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle.

Inputs come from the seeded generator and are identical on both sides (the
oracle reads the exact bf16 / fp32 values the device receives).  Metric:
max|X - X_ref| / max|X_ref| over every element of O and S_T, with the
tolerances the workloads state: 1e-5 for fp32 inputs, 2e-2 for bf16 inputs
with an fp32 state.  Full-size workloads run exactly as bench.py launches
them and are compared on sampled heads, plus finiteness everywhere.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_89_b200 as gdr
import gdr_workloads as W
import oracle

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2}


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


def to_dev(x):
    return {k: v.cuda() for k, v in x.items()}


def check_chunk(w, C=None, S0_none=False):
    x = W.generate(w)
    O_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], None if S0_none else x["S0"],
                                  gate=w.gate)
    d = to_dev(x)
    O, S = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None if S0_none else d["S0"],
                         C=C or w.C, gate=w.gate)
    torch.cuda.synchronize()
    assert gdr.last_launch_count() >= 1
    assert gdr.device_status() == 0
    eo, es = relerr(O, O_ref), relerr(S, S_ref)
    tol = TOL[w.dtype]
    assert eo <= tol and es <= tol, (w.name, eo, es)
    return eo, es


def test_tiny_fp32_workload():
    eo, es = check_chunk(W.WORKLOADS["kda_tiny_fp32"])
    assert eo <= 1e-5 and es <= 1e-5


CASES = [
    # B, H, T, dk, dv, gate, dtype, recipe, C
    (1, 2, 200, 128, 128, "per_channel", torch.bfloat16, "softplus_n02_clamp5", 64),
    (1, 2, 200, 128, 128, "scalar", torch.bfloat16, "scalar_softplus_n01_plus2", 64),
    (2, 1, 300, 128, 128, "per_channel", torch.bfloat16, "long_context_mix", 64),
    (1, 2, 130, 128, 128, "per_channel", torch.bfloat16, "softplus_n02_unbounded", 64),
    (1, 2, 150, 64, 64, "per_channel", torch.bfloat16, "softplus_n01_plus1_clamp5", 64),
    (1, 1, 150, 64, 128, "per_channel", torch.float32, "softplus_n01_plus1_clamp5", 64),
    (1, 1, 150, 128, 64, "scalar", torch.float32, "scalar_softplus_n01_plus2", 64),
    (1, 1, 97, 128, 128, "per_channel", torch.float32, "softplus_n02_unbounded", 32),
    (1, 1, 97, 64, 64, "per_channel", torch.bfloat16, "softplus_n02_clamp5", 16),
    (1, 2, 1, 128, 128, "per_channel", torch.bfloat16, "softplus_n02_clamp5", 64),
    (1, 2, 63, 128, 128, "per_channel", torch.bfloat16, "softplus_n02_clamp5", 64),
    (1, 2, 65, 128, 128, "scalar", torch.bfloat16, "scalar_softplus_n01_plus2", 64),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}H{c[1]}T{c[2]}d{c[3]}x{c[4]}-{c[5]}-{str(c[6])[6:]}-{c[7]}-C{c[8]}")
def test_chunk_cases(case):
    B, H, T, dk, dv, gate, dt, recipe, C = case
    w = W.small_chunk_case(B, H, T, dk, dv, gate, dt, g_recipe=recipe, C=C)
    check_chunk(w)


def test_zero_initial_state_pointer():
    w = W.small_chunk_case(1, 2, 100, 128, 128, "per_channel", torch.bfloat16)
    check_chunk(w, S0_none=True)


def test_empty_and_degenerate():
    dev = torch.device("cuda")
    # T = 0: S_T is S0 (copied) or zeros
    S0 = torch.randn(1, 2, 128, 128, device=dev)
    e = torch.empty(1, 2, 0, 128, dtype=torch.bfloat16, device=dev)
    O, S = gdr.chunk_fwd(e, e, e, torch.empty(1, 2, 0, 128, device=dev), torch.empty(1, 2, 0, device=dev), S0)
    torch.cuda.synchronize()
    assert O.numel() == 0 and torch.equal(S, S0)
    O, S = gdr.chunk_fwd(e, e, e, torch.empty(1, 2, 0, 128, device=dev), torch.empty(1, 2, 0, device=dev), None)
    torch.cuda.synchronize()
    assert float(S.abs().max()) == 0.0
    # B = 0
    z = torch.empty(0, 2, 64, 128, dtype=torch.bfloat16, device=dev)
    O, S = gdr.chunk_fwd(z, z, z, torch.empty(0, 2, 64, 128, device=dev), torch.empty(0, 2, 64, device=dev))
    assert O.shape == (0, 2, 64, 128)
    # beta = 0 everywhere: nothing is written, O = S0 Diag(gamma_t) q_t
    w = W.small_chunk_case(1, 1, 70, 128, 128, "per_channel", torch.bfloat16)
    x = W.generate(w)
    x["beta"].zero_()
    O_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    d = to_dev(x)
    O, S = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert relerr(O, O_ref) <= 2e-2 and relerr(S, S_ref) <= 2e-2


def test_in_place_state_and_guard_bands():
    w = W.small_chunk_case(1, 2, 150, 128, 128, "per_channel", torch.bfloat16)
    x = W.generate(w)
    O_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    d = to_dev(x)
    # outputs live inside larger buffers filled with a canary value
    canary = 12345.0
    n_o = d["v"].numel()
    obuf = torch.full((n_o + 4096,), canary, dtype=torch.bfloat16, device="cuda")
    O = obuf[2048:2048 + n_o].view_as(d["v"])
    n_s = d["S0"].numel()
    sbuf = torch.full((n_s + 4096,), canary, dtype=torch.float32, device="cuda")
    S = sbuf[2048:2048 + n_s].view_as(d["S0"])
    S.copy_(d["S0"])
    gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S, O=O, S_T=S)  # in place: S_T is S0
    torch.cuda.synchronize()
    assert relerr(O, O_ref) <= 2e-2 and relerr(S, S_ref) <= 2e-2
    assert bool((obuf[:2048] == canary).all()) and bool((obuf[2048 + n_o:] == canary).all())
    assert bool((sbuf[:2048] == canary).all()) and bool((sbuf[2048 + n_s:] == canary).all())


def test_host_buffers_round_trip():
    w = W.small_chunk_case(1, 2, 100, 128, 128, "scalar", torch.bfloat16, g_recipe="scalar_softplus_n01_plus2")
    x = W.generate(w)
    O_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], gate="scalar")
    O, S = gdr.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    assert O.device.type == "cpu" and S.device.type == "cpu"
    assert relerr(O, O_ref) <= 2e-2 and relerr(S, S_ref) <= 2e-2


@pytest.mark.parametrize("name,heads", [("gdn_scalar_t4096", [0, 17, 40, 63]),
                                        ("kda_d128_t8192", [0, 31, 50]),
                                        ("kda_long_t65536", [5, 30])])
def test_full_size_sampled(name, heads):
    w = W.WORKLOADS[name]
    d = W.generate(w, device="cuda")
    O, S = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], C=w.C, gate=w.gate)
    torch.cuda.synchronize()
    assert gdr.device_status() == 0
    assert bool(torch.isfinite(O).all()) and bool(torch.isfinite(S).all())
    H = w.H
    sel = lambda t: torch.stack([t[h // H, h % H] for h in heads])[:, None].cpu()
    O_ref, S_ref = oracle.forward(sel(d["q"]), sel(d["k"]), sel(d["v"]), sel(d["g"]), sel(d["beta"]),
                                  sel(d["S0"]), gate=w.gate)
    eo, es = relerr(sel(O), O_ref), relerr(sel(S), S_ref)
    assert eo <= 2e-2 and es <= 2e-2, (name, eo, es)


# ---------------------------------------------------------------- decode step

@pytest.mark.parametrize("dk,dv,gate,dt", [(128, 128, "per_channel", torch.bfloat16),
                                           (64, 64, "scalar", torch.float32),
                                           (64, 128, "per_channel", torch.float32),
                                           (128, 64, "scalar", torch.bfloat16)])
def test_decode_small(dk, dv, gate, dt):
    steps = 20
    w = W.small_chunk_case(3, 2, steps, dk, dv, gate, dt,
                           g_recipe="softplus_n02_unbounded" if gate == "per_channel" else "scalar_softplus_n01_plus2")
    x = W.generate(w)  # [B,H,T,...]: use the token axis as the step axis
    O_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], gate=gate)
    d = to_dev(x)
    S = d["S0"].clone()
    outs = []
    for t in range(steps):
        gt = d["g"][:, :, t].contiguous()
        outs.append(gdr.recurrent_step(d["q"][:, :, t].contiguous(), d["k"][:, :, t].contiguous(),
                                       d["v"][:, :, t].contiguous(), gt, d["beta"][:, :, t].contiguous(), S,
                                       gate=gate))
    O = torch.stack(outs, dim=2)
    torch.cuda.synchronize()
    tol = TOL[dt]
    assert relerr(O, O_ref) <= tol and relerr(S, S_ref) <= tol


def test_decode_full_size_sampled():
    w = W.WORKLOADS["kda_decode_b256"]
    heads = [0, 1, 777, 4096, 8191]
    steps = w.T
    d0 = W.generate(w, device="cuda", steps=1, step0=0)
    S = d0["S0"].clone()
    sel_hist = {k: [] for k in ("q", "k", "v", "g", "beta", "o")}
    H = w.H
    pick = lambda t: torch.stack([t[h // H, h % H] for h in heads])
    for s in range(steps):
        x = W.generate(w, device="cuda", steps=1, step0=s)
        o = gdr.recurrent_step(x["q"][0], x["k"][0], x["v"][0], x["g"][0], x["beta"][0], S)
        for key in ("q", "k", "v", "g", "beta"):
            sel_hist[key].append(pick(x[key][0]))
        sel_hist["o"].append(pick(o))
    torch.cuda.synchronize()
    assert bool(torch.isfinite(S).all())
    st = lambda key: torch.stack(sel_hist[key])[:, :, None].cpu()   # [steps, nh, 1, ...]
    o_ref, S_ref = oracle.decode(st("q"), st("k"), st("v"), st("g"), st("beta"), pick(d0["S0"])[:, None].cpu())
    eo = relerr(torch.stack(sel_hist["o"]), o_ref[:, :, 0])
    es = relerr(pick(S), S_ref[:, 0])
    assert eo <= 2e-2 and es <= 2e-2, (eo, es)


# A slowly decaying gate keeps the state alive across chunks, so a wrong state
# read at a chunk boundary shows in every later output (a fast gate hides it).
# Repeated runs must also be bitwise identical.
@pytest.mark.parametrize("gate", ["per_channel", "scalar"])
def test_state_carry_and_repeatability(gate):
    recipe = "slow_decay" if gate == "per_channel" else "scalar_softplus_n01_plus2"
    w = W.small_chunk_case(2, 4, 300, 128, 128, gate, torch.bfloat16, g_recipe=recipe, seed=31)
    x = W.generate(w)
    if gate == "scalar":
        x["g"] = x["g"] * 0.02   # slow scalar decay too
    O_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], gate=gate)
    d = to_dev(x)
    junk = torch.empty(1 << 26, dtype=torch.uint8, device="cuda")
    first = None
    for it in range(12):
        junk.random_()   # vary the timing of the runs
        O, S = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], C=64, gate=gate)
        torch.cuda.synchronize()
        assert gdr.device_status() == 0
        eo, es = relerr(O, O_ref), relerr(S, S_ref)
        assert eo <= 2e-2 and es <= 2e-2, (it, eo, es)
        if first is None:
            first = (O.clone(), S.clone())
        else:
            assert torch.equal(O, first[0]) and torch.equal(S, first[1]), it
