"""GPU parity of the fused-prologue forward (gdr_chunk_fwd_prologue) with the
fp64 oracle (prologue, then the recurrence), on the same seeded inputs."""
import numpy as np
import pytest
import torch

import gated_delta_rule_89_b200 as gdr
import gdr_workloads as W
import oracle

pytestmark = pytest.mark.gpu

TOL = 2e-2   # bf16 operands: max |X - X_ref| / max |X_ref|


def relerr(x, ref):
    x = x.double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x)
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-30))


def _run(w):
    x = W.generate_prologue(w)
    d = {k: v.cuda() for k, v in x.items()}
    O, S = gdr.chunk_fwd_prologue(d["q_raw"], d["k_raw"], d["v"], d["a"], d["A_log"], d["dt_bias"], d["b_logit"],
                                  d["S0"], C=64, gate=w.gate)
    torch.cuda.synchronize()
    assert gdr.device_status() == 0
    Or, Sr = oracle.forward_prologue(x["q_raw"], x["k_raw"], x["v"], x["a"], x["A_log"], x["dt_bias"],
                                     x["b_logit"], x["S0"], gate=w.gate)
    return O, S, Or, Sr


@pytest.mark.parametrize("gate,T,B,H,seed", [("per_channel", 300, 2, 3, 31), ("per_channel", 64, 1, 2, 32),
                                             ("per_channel", 1, 1, 1, 33), ("scalar", 517, 2, 2, 34),
                                             ("scalar", 129, 1, 3, 35), ("per_channel", 2048, 1, 4, 36)])
def test_prologue_forward_matches_oracle(gate, T, B, H, seed):
    w = W.small_chunk_case(B, H, T, 128, 128, gate, torch.bfloat16, seed=seed)
    O, S, Or, Sr = _run(w)
    assert bool(torch.isfinite(O).all()) and bool(torch.isfinite(S).all())
    assert relerr(O, Or) <= TOL, relerr(O, Or)
    assert relerr(S, Sr) <= TOL, relerr(S, Sr)


def test_prologue_equals_plain_forward_on_prenormalised_inputs():
    # fed with the oracle's own prologue outputs (rounded as the plain entry point takes them), the
    # plain forward and the prologue forward solve the same problem
    w = W.small_chunk_case(1, 2, 200, 128, 128, "per_channel", torch.bfloat16, seed=37)
    x = W.generate_prologue(w)
    q, k, g, beta = oracle.prologue(x["q_raw"], x["k_raw"], x["a"], x["A_log"], x["dt_bias"], x["b_logit"])
    d = {k_: v.cuda() for k_, v in x.items()}
    O1, S1 = gdr.chunk_fwd_prologue(d["q_raw"], d["k_raw"], d["v"], d["a"], d["A_log"], d["dt_bias"],
                                    d["b_logit"], d["S0"])
    O2, S2 = gdr.chunk_fwd(torch.from_numpy(q).to(torch.bfloat16).cuda(), torch.from_numpy(k).to(torch.bfloat16).cuda(),
                           d["v"], torch.from_numpy(g).float().cuda(), torch.from_numpy(beta).float().cuda(), d["S0"])
    torch.cuda.synchronize()
    assert relerr(O1, O2.double().cpu().numpy()) <= TOL
    assert relerr(S1, S2.double().cpu().numpy()) <= TOL
