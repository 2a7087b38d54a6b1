"""Pins of the oracle's output epilogue ("Token Mixer I", section "The Kimi
Linear Model Architecture": y_t = Sigmoid(gate_t) * RMSNorm(o_t), per head,
before the output projection).

Expected values come from closed forms, invariants and torch's own RMSNorm
(a library routine, run in fp64), not from the oracle's formula.
"""
import numpy as np
import torch

import oracle


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def test_matches_torch_rms_norm():
    rng = np.random.default_rng(30)
    O = rng.standard_normal((2, 3, 17, 16))
    gate = rng.standard_normal((2, 3, 17, 16))
    w = rng.uniform(0.5, 1.5, 16)
    y = oracle.output_gate(O, gate, w, 1e-6)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(O), (16,), weight=torch.from_numpy(w), eps=1e-6)
    ref = ref * torch.sigmoid(torch.from_numpy(gate))
    assert rel(y, ref.numpy()) < 1e-13


def test_constant_row_closed_form():
    # o = c * 1: RMSNorm gives c / sqrt(c^2 + eps) per channel; gate 0 halves it
    c, eps = -0.37, 1e-6
    O = np.full((1, 1, 1, 8), c)
    y = oracle.output_gate(O, np.zeros_like(O), np.ones(8), eps)
    assert rel(y, np.full_like(O, 0.5 * c / np.sqrt(c * c + eps))) < 1e-14


def test_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(31)
    O = rng.standard_normal((1, 2, 9, 32))
    big = 40.0 * np.ones_like(O)                 # sigmoid(40) = 1 to fp64 rounding
    y = oracle.output_gate(O, big, np.ones(32), 0.0)
    assert np.allclose(np.sqrt((y * y).mean(-1)), 1.0, rtol=1e-13, atol=0)
    y2 = oracle.output_gate(1e3 * O, big, np.ones(32), 0.0)
    assert rel(y2, y) < 1e-13


def test_gate_and_weight_are_per_channel():
    rng = np.random.default_rng(32)
    O = rng.standard_normal((1, 1, 5, 6))
    gate = rng.standard_normal((1, 1, 5, 6))
    w = rng.uniform(0.1, 2.0, 6)
    base = oracle.output_gate(O, np.full_like(gate, 40.0), np.ones(6), 1e-6)
    y = oracle.output_gate(O, gate, w, 1e-6)
    assert rel(y, base * w / (1.0 + np.exp(-gate))) < 1e-13
