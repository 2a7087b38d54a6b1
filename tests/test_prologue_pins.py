"""Pins of the oracle's input prologue (L2-normalised q, k; softplus gate
with the -5 bound; sigmoid beta) against closed forms and invariants, and of
its composition with the forward on one-token cases with closed forms.
"""
import math

import numpy as np
import pytest
import torch

import gdr_workloads as W
import oracle


def _raw(B=1, H=2, T=5, dk=8, seed=3):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((B, H, T, dk))


def test_l2norm_gives_unit_vectors_parallel_to_the_input():
    x = _raw()
    q, k, _, _ = oracle.prologue(x, 2.5 * x, np.zeros(x.shape), np.zeros(2), np.zeros((2, 8)), np.zeros(x.shape[:3]))
    n = np.linalg.norm(q, axis=-1)
    assert np.allclose(n, 1.0, atol=1e-7)          # eps = 1e-6 against sum(x^2) of order 8
    cos = (q * x).sum(-1) / (np.linalg.norm(x, axis=-1))
    assert np.allclose(cos, 1.0, atol=1e-7)        # same direction
    assert np.allclose(k, q, atol=1e-7)            # invariant to a positive scale


@pytest.mark.parametrize("A_log,alpha", [(0.0, 0.5), (math.log(2.0), 0.25), (math.log(3.0), 0.125)])
def test_gate_closed_form_at_zero_preactivation(A_log, alpha):
    # a + dt_bias = 0: softplus(0) = ln 2, so g = -exp(A_log) ln 2 and alpha = 2^-exp(A_log)
    a = np.full((1, 1, 3, 4), 0.75)
    dtb = np.full((1, 4), -0.75)
    _, _, g, _ = oracle.prologue(np.ones((1, 1, 3, 4)), np.ones((1, 1, 3, 4)), a, np.array([A_log]), dtb,
                                 np.zeros((1, 1, 3)))
    assert np.allclose(np.exp(g), alpha, rtol=1e-13)


def test_gate_bounds_and_tails():
    ones = np.ones((1, 1, 2, 3))
    big = np.full((1, 1, 2, 3), 40.0)
    _, _, g, _ = oracle.prologue(ones, ones, big, np.zeros(1), np.zeros((1, 3)), np.zeros((1, 1, 2)))
    assert np.all(g == -5.0)                       # per-channel lower bound g_min = -5
    _, _, gs, _ = oracle.prologue(ones, ones, big[..., 0], np.zeros(1), np.zeros(1), np.zeros((1, 1, 2)),
                                  gate="scalar")
    assert np.allclose(gs, -40.0, rtol=1e-15)      # scalar gate: softplus(40) = 40 + O(e^-40), no bound
    _, _, gt, _ = oracle.prologue(ones, ones, -big, np.zeros(1), np.zeros((1, 3)), np.zeros((1, 1, 2)))
    assert np.all(gt < 0) and np.allclose(gt, -math.exp(-40.0), rtol=1e-12)   # softplus(-40) = e^-40


def test_beta_is_the_logistic_function():
    b = np.array([[[0.0, math.log(3.0), -math.log(3.0), 50.0]]])
    ones = np.ones((1, 1, 4, 2))
    _, _, _, beta = oracle.prologue(ones, ones, np.zeros((1, 1, 4, 2)), np.zeros(1), np.zeros((1, 2)), b)
    assert np.allclose(beta[0, 0], [0.5, 0.75, 0.25, 1.0], rtol=1e-14)


def test_one_token_forward_with_prologue_closed_form():
    # k_raw = 3 e1, q_raw = 5 e1 -> k = q = e1 (up to eps); alpha = 1/2 on every channel
    # (A_log = 0, a + dt_bias = 0), beta = 1/2 (logit 0).  With S0 given:
    #   S1 = S0 Diag(1/2) (I - 1/2 e1 e1^T) + 1/2 v e1^T,  o = S1 e1 = S0[:, 0] / 4 + v / 2
    dk, dv = 4, 3
    rng = np.random.default_rng(7)
    S0 = rng.standard_normal((1, 1, dv, dk))
    v = rng.standard_normal((1, 1, 1, dv))
    e1 = np.zeros((1, 1, 1, dk))
    e1[..., 0] = 1.0
    O, ST = oracle.forward_prologue(5.0 * e1, 3.0 * e1, v, np.full((1, 1, 1, dk), 0.2), np.zeros(1),
                                    np.full((1, dk), -0.2), np.zeros((1, 1, 1)), S0)
    assert np.allclose(O[0, 0, 0], S0[0, 0, :, 0] / 4 + v[0, 0, 0] / 2, rtol=1e-7, atol=1e-12)
    expect = S0[0, 0] / 2
    expect[:, 0] = S0[0, 0, :, 0] / 4 + v[0, 0, 0] / 2
    assert np.allclose(ST[0, 0], expect, rtol=1e-7, atol=1e-12)


def test_generator_draws_raw_prologue_inputs():
    w = W.small_chunk_case(1, 2, 70, 16, 8, "per_channel", torch.bfloat16)
    x = W.generate_prologue(w)
    assert x["q_raw"].shape == (1, 2, 70, 16) and x["a"].shape == (1, 2, 70, 16)
    assert x["A_log"].shape == (2,) and x["dt_bias"].shape == (2, 16) and x["b_logit"].shape == (1, 2, 70)
    n = x["q_raw"].double().norm(dim=-1)
    assert n.min() > 1.5                           # not normalised: the prologue does that
    assert torch.equal(x["v"], W.generate(w)["v"]) # same value stream as the plain inputs
    assert torch.all(x["A_log"].abs() <= 1)
    y = W.generate_prologue(w)
    assert all(torch.equal(x[k], y[k]) for k in x)  # seeded
