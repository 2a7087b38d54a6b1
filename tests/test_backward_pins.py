"""Pins of the oracle's backward pass (reverse mode through the token
recurrence): the gradients of L = <dO, O> + <dS_T, S_T> are checked against
central finite differences of the oracle's own forward in fp64, against the
exact linearity of the output in (v, S0), and against closed forms.
"""
import numpy as np
import pytest

import oracle


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def case(rng, B=1, H=2, T=70, dk=4, dv=3, gate="per_channel", g_lo=-1.5):
    q = unit(rng.standard_normal((B, H, T, dk)))
    k = unit(rng.standard_normal((B, H, T, dk)))
    v = rng.standard_normal((B, H, T, dv))
    g = rng.uniform(g_lo, 0.0, (B, H, T, dk) if gate == "per_channel" else (B, H, T))
    beta = rng.uniform(0.0, 1.0, (B, H, T))
    S0 = 0.3 * rng.standard_normal((B, H, dv, dk))
    dO = rng.standard_normal((B, H, T, dv))
    dST = rng.standard_normal((B, H, dv, dk))
    return [q, k, v, g, beta, S0], dO, dST


def loss(args, dO, dST, gate):
    O, S = oracle.forward(*args, gate=gate)
    return float((O * dO).sum() + (S * dST).sum())


# Central differences, 6 random coordinates of every input; T = 70 crosses the
# 64-token checkpoint of the reverse sweep, and g down to -7 puts entries on
# both sides of the -5 bound (the bound's kink is avoided by the sampling).
@pytest.mark.parametrize("gate", ["per_channel", "scalar"])
def test_finite_differences(gate):
    rng = np.random.default_rng(40)
    args, dO, dST = case(rng, gate=gate, g_lo=-7.0 if gate == "per_channel" else -1.5)
    grads = oracle.backward(*args, dO, dST, gate=gate)
    h = 1e-6
    for ai, gr in enumerate(grads):
        x = args[ai]
        for _ in range(6):
            ix = tuple(int(rng.integers(0, s)) for s in x.shape)
            if ai == 3 and gate == "per_channel" and abs(x[ix] + 5.0) < 2 * h:
                continue
            xp, xm = x.copy(), x.copy()
            xp[ix] += h
            xm[ix] -= h
            ap, am = list(args), list(args)
            ap[ai], am[ai] = xp, xm
            fd = (loss(ap, dO, dST, gate) - loss(am, dO, dST, gate)) / (2 * h)
            assert abs(fd - gr[ix]) <= 1e-6 * max(1.0, abs(fd)), (ai, ix, fd, gr[ix])


def test_clamped_gate_has_no_gradient():
    rng = np.random.default_rng(41)
    args, dO, dST = case(rng, g_lo=-9.0)
    dg = oracle.backward(*args, dO, dST)[3]
    below = args[3] < -5.0
    assert below.any() and np.all(dg[below] == 0.0) and np.any(dg[~below] != 0.0)


# O and S_T are linear in (v, S0) jointly: the directional change of L along
# (Dv, DS0) equals the gradient's inner product with it, exactly.
def test_linearity_in_v_and_S0():
    rng = np.random.default_rng(42)
    args, dO, dST = case(rng, T=50)
    _, _, dv, _, _, dS0 = oracle.backward(*args, dO, dST)
    Dv = rng.standard_normal(args[2].shape)
    DS = rng.standard_normal(args[5].shape)
    moved = list(args)
    moved[2] = args[2] + Dv
    moved[5] = args[5] + DS
    change = loss(moved, dO, dST, "per_channel") - loss(args, dO, dST, "per_channel")
    assert abs(change - (np.sum(dv * Dv) + np.sum(dS0 * DS))) < 1e-10 * max(1.0, abs(change))


# beta = 0 and dO = 0: S_T = S0 Diag(prod_t alpha_t), so dS0 = dS_T Diag(prod alpha)
# and dg_{t,c} = sum_i dS_T[i,c] S0[i,c] prod_t alpha_{t,c} for every token t.
def test_closed_form_without_writes():
    rng = np.random.default_rng(43)
    args, dO, dST = case(rng, T=20)
    args[4][:] = 0.0
    dO[:] = 0.0
    _, _, _, dg, _, dS0 = oracle.backward(*args, dO, dST)
    P = np.exp(args[3].sum(axis=2))                       # [B,H,dk]
    assert np.allclose(dS0, dST * P[:, :, None, :], rtol=1e-12, atol=1e-14)
    expect = (dST * args[5]).sum(axis=2) * P               # [B,H,dk]
    assert np.allclose(dg, np.repeat(expect[:, :, None, :], 20, axis=2), rtol=1e-12, atol=1e-14)


# A scalar gate is the per-channel gate broadcast over the channels, so its
# gradient is the per-channel gradient summed over them (for g >= -5).
def test_scalar_gradient_is_channel_sum():
    rng = np.random.default_rng(44)
    args, dO, dST = case(rng, gate="scalar", g_lo=-4.0)
    gs = oracle.backward(*args, dO, dST, gate="scalar")
    pc = list(args)
    pc[3] = np.repeat(args[3][..., None], args[0].shape[-1], -1)
    gp = oracle.backward(*pc, dO, dST, gate="per_channel")
    for a, b in zip(gs[:3] + gs[4:], gp[:3] + gp[4:]):
        assert np.allclose(a, b, rtol=1e-12, atol=1e-13)
    assert np.allclose(gs[3], gp[3].sum(-1), rtol=1e-12, atol=1e-13)
