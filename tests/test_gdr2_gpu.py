"""GPU parity of the Gated Delta Rule-2 entry points (gdr2_chunk_fwd,
gdr2_recurrent_step) against the fp64 oracle's ``forward_gdr2``.

Same metric and tolerance as the tied-gate parity tests: max|X - X_ref| /
max|X_ref| over every element of O and S_T, 2e-2 for bf16 inputs with an fp32
state (1e-5 for the fp32 decode step).
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


CASES = [
    # B, H, T, gate, recipe
    (1, 2, 64, "per_channel", "softplus_n02_clamp5"),
    (1, 2, 200, "per_channel", "softplus_n02_clamp5"),
    (2, 3, 333, "per_channel", "long_context_mix"),
    (1, 2, 130, "per_channel", "softplus_n02_unbounded"),
    (1, 2, 200, "scalar", "scalar_softplus_n01_plus2"),
    (1, 1, 1, "per_channel", "softplus_n02_clamp5"),
    (1, 2, 65, "scalar", "scalar_softplus_n01_plus2"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}H{c[1]}T{c[2]}-{c[3]}-{c[4]}")
def test_chunk_cases(case):
    B, H, T, gate, recipe = case
    w = W.small_chunk_case(B, H, T, 128, 128, gate, torch.bfloat16, g_recipe=recipe, rule="gdr2")
    x = W.generate(w)
    O_ref, S_ref = oracle.forward_gdr2(x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], x["S0"], gate=gate)
    d = {k: v.cuda() for k, v in x.items()}
    O, S = gdr.chunk_fwd_gdr2(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], gate=gate)
    torch.cuda.synchronize()
    assert gdr.last_launch_count() == 2
    assert gdr.device_status() == 0
    eo, es = relerr(O, O_ref), relerr(S, S_ref)
    assert eo <= 2e-2 and es <= 2e-2, (eo, es)


def test_extreme_gates():
    # b = 1 everywhere (full erase along k), w = 0 on half the value channels
    w = W.small_chunk_case(1, 2, 150, 128, 128, "per_channel", torch.bfloat16, rule="gdr2")
    x = W.generate(w)
    x["b"].fill_(1.0)
    x["w"][..., ::2] = 0.0
    O_ref, S_ref = oracle.forward_gdr2(x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], x["S0"])
    d = {k: v.cuda() for k, v in x.items()}
    O, S = gdr.chunk_fwd_gdr2(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"])
    torch.cuda.synchronize()
    assert relerr(O, O_ref) <= 2e-2 and relerr(S, S_ref) <= 2e-2


def test_tied_gates_match_the_tied_forward():
    # b = w = beta (as bf16) is the tied rule: both entry points agree
    w = W.small_chunk_case(1, 2, 190, 128, 128, "per_channel", torch.bfloat16, rule="gdr2")
    x = {k: v.cuda() for k, v in W.generate(w).items()}
    beta = x["beta"].to(torch.bfloat16)
    b = beta[..., None].expand(-1, -1, -1, 128).contiguous()
    O2, S2 = gdr.chunk_fwd_gdr2(x["q"], x["k"], x["v"], x["g"], b, b, x["S0"])
    O1, S1 = gdr.chunk_fwd(x["q"], x["k"], x["v"], x["g"], beta.float(), x["S0"])
    torch.cuda.synchronize()
    assert relerr(O2, O1.double().cpu()) <= 1e-2 and relerr(S2, S1.double().cpu()) <= 1e-2


def test_full_size_sampled():
    w = W.WORKLOADS["gdr2_d128_t8192"]
    heads = [0, 33, 63]
    d = W.generate(w, device="cuda")
    O, S = gdr.chunk_fwd_gdr2(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], C=w.C, gate=w.gate)
    torch.cuda.synchronize()
    assert gdr.device_status() == 0
    assert bool(torch.isfinite(O).all()) and bool(torch.isfinite(S).all())
    H = w.H
    sel = lambda t: torch.stack([t[h // H, h % H] for h in heads])[:, None].cpu()
    O_ref, S_ref = oracle.forward_gdr2(sel(d["q"]), sel(d["k"]), sel(d["v"]), sel(d["g"]), sel(d["b"]),
                                       sel(d["w"]), sel(d["S0"]), gate=w.gate)
    eo, es = relerr(sel(O), O_ref), relerr(sel(S), S_ref)
    assert eo <= 2e-2 and es <= 2e-2, (eo, es)


def test_argument_errors():
    w = W.small_chunk_case(1, 1, 64, 128, 128, "per_channel", torch.bfloat16, rule="gdr2")
    x = {k: v.cuda() for k, v in W.generate(w).items()}
    with pytest.raises(TypeError):   # fp32 inputs: the GDR-2 forward runs the bf16 configuration
        gdr.chunk_fwd_gdr2(*(x[n].float() for n in ("q", "k", "v")), x["g"], x["b"].float(), x["w"].float())
    with pytest.raises(ValueError):
        gdr.chunk_fwd_gdr2(x["q"], x["k"], x["v"], x["g"], x["b"][..., :64].contiguous(), x["w"])


@pytest.mark.parametrize("dk,dv,gate,dt", [(128, 128, "per_channel", torch.bfloat16),
                                           (64, 64, "scalar", torch.float32),
                                           (64, 128, "per_channel", torch.float32),
                                           (128, 64, "scalar", torch.bfloat16)])
def test_decode_small(dk, dv, gate, dt):
    steps = 20
    w = W.small_chunk_case(3, 2, steps, dk, dv, gate, dt, rule="gdr2",
                           g_recipe="softplus_n02_unbounded" if gate == "per_channel" else "scalar_softplus_n01_plus2")
    x = W.generate(w)
    O_ref, S_ref = oracle.forward_gdr2(x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], x["S0"], gate=gate)
    d = {k: v.cuda() for k, v in x.items()}
    S = d["S0"].clone()
    outs = []
    at = lambda n, t: d[n][:, :, t].contiguous()
    for t in range(steps):
        outs.append(gdr.recurrent_step_gdr2(at("q", t), at("k", t), at("v", t), at("g", t), at("b", t), at("w", t),
                                            S, gate=gate))
    O = torch.stack(outs, dim=2)
    torch.cuda.synchronize()
    tol = TOL[dt]
    assert relerr(O, O_ref) <= tol and relerr(S, S_ref) <= tol


def test_decode_full_size_sampled():
    w = W.WORKLOADS["gdr2_decode_b256"]
    heads = [0, 4097, 8191]
    steps = 50
    d0 = W.generate(w, device="cuda", steps=1, step0=0)
    S = d0["S0"].clone()
    H = w.H
    pick = lambda t: torch.stack([t[h // H, h % H] for h in heads])
    hist = {k: [] for k in ("q", "k", "v", "g", "b", "w", "o")}
    for s in range(steps):
        x = W.generate(w, device="cuda", steps=1, step0=s)
        o = gdr.recurrent_step_gdr2(x["q"][0], x["k"][0], x["v"][0], x["g"][0], x["b"][0], x["w"][0], S)
        for n in ("q", "k", "v", "g", "b", "w"):
            hist[n].append(pick(x[n][0]).cpu())
        hist["o"].append(pick(o).cpu())
    torch.cuda.synchronize()
    st = lambda n: torch.stack(hist[n])[:, :, None]            # [steps, heads, 1, ...]
    o_ref, S_ref = oracle.decode_gdr2(st("q"), st("k"), st("v"), st("g"), st("b"), st("w"),
                                      pick(d0["S0"]).cpu()[:, None])
    assert relerr(torch.stack(hist["o"]), o_ref[:, :, 0]) <= 2e-2
    assert relerr(pick(S).cpu(), S_ref[:, 0]) <= 2e-2


def test_empty_problems():
    dev = torch.device("cuda")
    S0 = torch.randn(1, 2, 128, 128, device=dev)
    e = torch.empty(1, 2, 0, 128, dtype=torch.bfloat16, device=dev)
    O, S = gdr.chunk_fwd_gdr2(e, e, e, torch.empty(1, 2, 0, 128, device=dev), e, e, S0)
    torch.cuda.synchronize()
    assert O.numel() == 0 and torch.equal(S, S0)
