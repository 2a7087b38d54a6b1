"""The timeout path of the bounded device waits, without a fault: with a wait
budget far below the time the pipeline's hand-offs take, the state scan's
waits run out; the kernel records GDR_ERR_TIMEOUT, drains what it issued,
frees its tensor memory and returns, and the next call on the same stream is
correct again."""
import numpy as np
import pytest
import torch

import gated_delta_rule_89_b200 as gdr
import gdr_workloads as W
import oracle

pytestmark = pytest.mark.gpu

GDR_ERR_TIMEOUT = 6


def _rel(x, ref):
    return float(np.max(np.abs(x.double().cpu().numpy() - ref)) / np.max(np.abs(ref)))


@pytest.mark.parametrize("gate", ["per_channel", "scalar"])
def test_waits_run_out_then_the_next_call_is_clean(gate):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = gdr.lib()
    recipe = "softplus_n02_clamp5" if gate == "per_channel" else "scalar_softplus_n01_plus2"
    w = W.small_chunk_case(1, 2, 256, 128, 128, gate, torch.bfloat16, g_recipe=recipe, seed=5)
    x = W.generate(w)
    d = {k: v.cuda() for k, v in x.items()}
    assert gdr.device_status() == 0
    L.gdr_debug_set_wait_budget(300)       # ~150 ns: far below a TMA round trip
    try:
        gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], C=64, gate=gate)
        status = gdr.device_status()      # synchronizes the stream
    finally:
        L.gdr_debug_set_wait_budget(0)
    assert status == GDR_ERR_TIMEOUT
    assert gdr.device_status() == 0       # read and cleared
    O_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], gate=gate)
    O, S = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], C=64, gate=gate)
    torch.cuda.synchronize()
    assert gdr.device_status() == 0
    assert _rel(O, O_ref) <= 2e-2 and _rel(S, S_ref) <= 2e-2
