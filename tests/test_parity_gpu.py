"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle.

Inputs come from the seeded generator and are identical on both sides (the
oracle reads the exact bf16 / fp32 values the device receives).  Metric:
max|X - X_ref| / max|X_ref| over every element of O and S_T, with the
tolerances the workloads state: 1e-5 for fp32 inputs, 2e-2 for bf16 inputs
with an fp32 state.  Full-size workloads run exactly as bench.py launches
them and are compared over every element (the oracle runs over batches of
heads).  The special cases the pages reduce the method to (no decay with
beta = 1 and orthonormal keys, the -5 gate bound on every channel, beta = 1)
run on the device too.
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


def _orthonormal_keys(n, dk, seed):
    """n <= dk orthonormal rows (fp64 QR of a seeded Gaussian matrix)."""
    gen = torch.Generator().manual_seed(seed)
    m = torch.randn(dk, dk, generator=gen, dtype=torch.float64)
    qm, _ = torch.linalg.qr(m)
    return qm[:n]


# The reductions the pages state, on the device.  "retrieval": no decay
# (g = 0), beta = 1, orthonormal keys and S0 = 0, so every write overwrites its
# own key direction and S_T k_i returns v_i ("Token Mixer I", the DeltaNet
# section, and the overwrite property of "Gated DeltaNet-2", Preliminary).
# "gmin": every channel and token at the KDA bound g = -5 (and below it,
# clamped), the largest decay spread a 16-token sub-block can see.  "beta1":
# full-strength writes.  "alpha1": no decay with random writes, so the state
# carries across every chunk.
EDGE = [
    # name, B, H, T, dk, dtype, gate
    ("retrieval", 1, 2, 128, 128, torch.bfloat16, "per_channel"),
    ("retrieval", 1, 2, 100, 128, torch.bfloat16, "scalar"),
    ("retrieval", 1, 1, 64, 64, torch.float32, "per_channel"),
    ("retrieval", 1, 1, 128, 128, torch.float32, "scalar"),
    ("gmin", 1, 2, 293, 128, torch.bfloat16, "per_channel"),
    ("gmin_below", 1, 2, 256, 128, torch.bfloat16, "per_channel"),
    ("gmin", 1, 1, 150, 64, torch.float32, "per_channel"),
    ("beta1", 1, 2, 200, 128, torch.bfloat16, "per_channel"),
    ("beta1", 1, 2, 200, 128, torch.bfloat16, "scalar"),
    ("alpha1", 2, 1, 300, 128, torch.bfloat16, "per_channel"),
    ("alpha1", 1, 2, 300, 128, torch.bfloat16, "scalar"),
]


@pytest.mark.parametrize("case", EDGE, ids=lambda c: f"{c[0]}-B{c[1]}H{c[2]}T{c[3]}d{c[4]}-{str(c[5])[6:]}-{c[6]}")
def test_reductions_on_device(case):
    kind, B, H, T, dk, dt, gate = case
    recipe = "softplus_n02_clamp5" if gate == "per_channel" else "scalar_softplus_n01_plus2"
    w = W.small_chunk_case(B, H, T, dk, dk, gate, dt, g_recipe=recipe, seed=41)
    x = W.generate(w)
    if kind == "retrieval":
        keys = torch.stack([_orthonormal_keys(T, dk, 100 + h) for h in range(B * H)]).view(B, H, T, dk)
        x["k"] = W.to_dtype(keys, dt)
        x["g"].zero_()
        x["beta"].fill_(1.0)
        x["S0"].zero_()
    elif kind in ("gmin", "gmin_below"):
        x["g"].fill_(-5.0 if kind == "gmin" else -9.0)
    elif kind == "beta1":
        x["beta"].fill_(1.0)
    elif kind == "alpha1":
        x["g"].zero_()
    O_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], gate=gate)
    d = to_dev(x)
    O, S = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], C=64, gate=gate)
    torch.cuda.synchronize()
    assert gdr.device_status() == 0
    tol = TOL[dt]
    eo, es = relerr(O, O_ref), relerr(S, S_ref)
    assert eo <= tol and es <= tol, (case, eo, es)
    if kind == "retrieval" and dt == torch.float32:
        # S_T k_i = v_i for every written key, to the fp32 tolerance
        got = torch.einsum("bhvk,bhtk->bhtv", S.double().cpu(), x["k"].double())
        assert relerr(got, x["v"].double().numpy()) <= 1e-5


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


def _parity_accumulate(acc, x, ref):
    """Running max|X - X_ref| and max|X_ref| over batches of heads."""
    x = np.asarray(x.detach().double().cpu() if isinstance(x, torch.Tensor) else x, np.float64)
    ref = np.asarray(ref, np.float64)
    acc[0] = max(acc[0], float(np.max(np.abs(x - ref))))
    acc[1] = max(acc[1], float(np.max(np.abs(ref))))


# Every element of the three full-size chunk workloads, launched exactly as
# bench.py launches them.  The oracle runs over batches of heads (one thread
# per head) so that its fp64 copies stay a few GB.
@pytest.mark.parametrize("name,batch", [("gdn_scalar_t4096", 64), ("kda_d128_t8192", 64),
                                        ("kda_long_t65536", 16)])
def test_full_size_every_element(name, batch):
    w = W.WORKLOADS[name]
    d = W.generate(w, device="cuda")
    O, S = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], C=w.C, gate=w.gate)
    torch.cuda.synchronize()
    assert gdr.device_status() == 0
    BH = w.B * w.H
    flat = lambda t: t.reshape(BH, 1, *t.shape[2:])
    eo, es = [0.0, 0.0], [0.0, 0.0]
    for h0 in range(0, BH, batch):
        sl = lambda t: flat(t)[h0:h0 + batch].cpu()
        O_ref, S_ref = oracle.forward(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["beta"]),
                                      sl(d["S0"]), gate=w.gate)
        _parity_accumulate(eo, sl(O), O_ref)
        _parity_accumulate(es, sl(S), S_ref)
        del O_ref, S_ref
    ro, rs = eo[0] / eo[1], es[0] / es[1]
    assert ro <= 2e-2 and rs <= 2e-2, (name, ro, rs)


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


def test_decode_full_size_every_element():
    """All 8192 heads of the decode workload over its 1000 steps: every o_t and
    the final state against the oracle (heads in batches on the host)."""
    w = W.WORKLOADS["kda_decode_b256"]
    steps, BH = w.T, w.B * w.H
    d0 = W.generate(w, device="cuda", steps=1, step0=0)
    S = d0["S0"].clone()
    outs = torch.empty(steps, w.B, w.H, w.dv, dtype=w.dtype, device="cuda")
    for s in range(steps):
        x = W.generate(w, device="cuda", steps=1, step0=s)
        gdr.recurrent_step(x["q"][0], x["k"][0], x["v"][0], x["g"][0], x["beta"][0], S, o=outs[s])
    torch.cuda.synchronize()
    assert gdr.device_status() == 0
    S0 = d0["S0"].reshape(BH, 1, w.dv, w.dk)
    outs = outs.reshape(steps, BH, 1, w.dv)
    Sf = S.reshape(BH, 1, w.dv, w.dk)
    eo, es = [0.0, 0.0], [0.0, 0.0]
    batch = 512
    for h0 in range(0, BH, batch):
        heads = list(range(h0, min(BH, h0 + batch)))
        x = W.generate(w, device="cuda", heads=heads, steps=steps, step0=0)   # [steps, nh, 1, ...]
        cpu = lambda t: t.cpu()
        o_ref, S_ref = oracle.decode(cpu(x["q"]), cpu(x["k"]), cpu(x["v"]), cpu(x["g"]), cpu(x["beta"]),
                                     S0[h0:h0 + batch].cpu())
        _parity_accumulate(eo, outs[:, h0:h0 + batch].cpu(), o_ref)
        _parity_accumulate(es, Sf[h0:h0 + batch].cpu(), S_ref)
        del x, o_ref, S_ref
    ro, rs = eo[0] / eo[1], es[0] / es[1]
    assert ro <= 2e-2 and rs <= 2e-2, (ro, rs)


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
