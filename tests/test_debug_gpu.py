"""Debug mode (GDR_DEBUG): the gate-range check of every entry point that
takes a log-decay g.  The library reads the variable once per process, so
each check runs in a fresh Python process with GDR_DEBUG=1 set."""
import os
import subprocess
import sys
import textwrap

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = textwrap.dedent("""
    import math, sys
    import numpy as np
    import torch
    sys.path.insert(0, ROOT)
    import gated_delta_rule_89_b200 as gdr
    import gdr_workloads as W
    import oracle

    def status_of(fn):
        try:
            fn()
            return "GDR_OK"
        except gdr.GDRError as e:
            return str(e).split(": ")[-1].split(" ")[0]

    dev = torch.device("cuda")
    for gate, recipe in (("per_channel", "softplus_n02_clamp5"), ("scalar", "scalar_softplus_n01_plus2")):
        for dt in (torch.bfloat16, torch.float32):
            w = W.small_chunk_case(1, 2, 77, 128, 128, gate, dt, g_recipe=recipe)
            x = {k: v.to(dev) for k, v in W.generate(w).items()}
            run = lambda g: gdr.chunk_fwd(x["q"], x["k"], x["v"], g, x["beta"], x["S0"], gate=gate)
            # a valid gate runs and matches the oracle; below -5 is legal (clamped)
            g_ok = x["g"].clone()
            g_ok.view(-1)[3] = -40.0
            O, S = run(g_ok)
            xr = {k: v.cpu() for k, v in x.items()}
            O_ref, S_ref = oracle.forward(xr["q"], xr["k"], xr["v"], g_ok.cpu(), xr["beta"], xr["S0"], gate=gate)
            err = float(np.max(np.abs(O.double().cpu().numpy() - O_ref)) / np.max(np.abs(O_ref)))
            assert err <= (2e-2 if dt == torch.bfloat16 else 1e-5), (gate, dt, err)
            for bad in (0.25, float("nan"), float("inf"), -float("inf")):
                gb = x["g"].clone()
                gb.view(-1)[gb.numel() - 1] = bad       # the last element: the scalar tail of the check
                st = status_of(lambda: run(gb))
                assert st == "GDR_ERR_GATE_RANGE", (gate, dt, bad, st)
    # the decode step
    w = W.small_chunk_case(2, 2, 1, 128, 128, "per_channel", torch.bfloat16)
    x = {k: v.to(dev) for k, v in W.generate(w).items()}
    S = x["S0"].clone()
    g = x["g"][:, :, 0].contiguous()
    assert status_of(lambda: gdr.recurrent_step(x["q"][:, :, 0].contiguous(), x["k"][:, :, 0].contiguous(),
                                                x["v"][:, :, 0].contiguous(), g, x["beta"][:, :, 0].contiguous(),
                                                S)) == "GDR_OK"
    g[1, 0, 5] = 1e-3
    assert status_of(lambda: gdr.recurrent_step(x["q"][:, :, 0].contiguous(), x["k"][:, :, 0].contiguous(),
                                                x["v"][:, :, 0].contiguous(), g, x["beta"][:, :, 0].contiguous(),
                                                S)) == "GDR_ERR_GATE_RANGE"
    print("debug checks ok")
""")


def test_gate_range_check_in_debug_mode():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, GDR_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + SCRIPT], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "debug checks ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
