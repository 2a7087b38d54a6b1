"""Pins of the Gated Delta Rule-2 oracle ("Token Mixer I", section "Gated
DeltaNet-2: Decoupling Erase and Write in Linear Attention").

The erase gate b_t in [0,1]^dk weights the key coordinates the old content is
read along; the write gate w_t in [0,1]^dv weights the value coordinates
written.  Each pin takes its expected value from something other than the
oracle's token loop: the reduction to KDA the section states, the section's
chunkwise equations, closed forms for basis keys and for a zero erase gate,
and the section's update written as explicit d_k x d_k transition matrices in
its own (d_k x d_v) orientation.
"""
import numpy as np
import pytest

import oracle
from oracle import chunk_form

RTOL = 1e-12


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def unit(x, axis=-1):
    return x / np.linalg.norm(x, axis=axis, keepdims=True)


def rand_case(rng, B=1, H=2, T=20, dk=5, dv=3, gate="per_channel", g_lo=-1.5):
    q = unit(rng.standard_normal((B, H, T, dk)))
    k = unit(rng.standard_normal((B, H, T, dk)))
    v = rng.standard_normal((B, H, T, dv))
    g = rng.uniform(g_lo, 0.0, (B, H, T, dk) if gate == "per_channel" else (B, H, T))
    b = rng.uniform(0.0, 1.0, (B, H, T, dk))
    w = rng.uniform(0.0, 1.0, (B, H, T, dv))
    S0 = 0.3 * rng.standard_normal((B, H, dv, dk))
    return q, k, v, g, b, w, S0


# The section: with b_t = beta_t 1 and w_t = beta_t 1 the rule is exactly KDA
# (and, with a scalar decay, Gated DeltaNet).
@pytest.mark.parametrize("gate", ["per_channel", "scalar"])
def test_tied_gates_reduce_to_kda(gate):
    rng = np.random.default_rng(11)
    q, k, v, g, _, _, S0 = rand_case(rng, T=29, dk=6, dv=4, gate=gate, g_lo=-7.0)
    beta = rng.uniform(0.0, 1.0, q.shape[:3])
    b = np.repeat(beta[..., None], q.shape[-1], -1)
    w = np.repeat(beta[..., None], v.shape[-1], -1)
    O2, S2 = oracle.forward_gdr2(q, k, v, g, b, w, S0, gate=gate)
    O1, S1 = oracle.forward(q, k, v, g, beta, S0, gate=gate)
    assert rel(O2, O1) < RTOL and rel(S2, S1) < RTOL


# Subsection "Chunkwise parallel training": the chunk equations (erase-side
# auxiliary Y, write-side auxiliary U, K_tail, the masked output) agree with
# the token recurrence for every chunk size, with a ragged last chunk.
@pytest.mark.parametrize("C", [1, 2, 3, 8, 16, 64])
@pytest.mark.parametrize("gate,glo", [("per_channel", -1.0), ("per_channel", -9.0), ("scalar", -1.0)])
def test_chunk_form_equals_recurrence(C, gate, glo):
    rng = np.random.default_rng(100 + C)
    q, k, v, g, b, w, S0 = rand_case(rng, B=1, H=2, T=75, dk=6, dv=5, gate=gate, g_lo=glo)
    O, ST = oracle.forward_gdr2(q, k, v, g, b, w, S0, gate=gate)
    for h in range(2):
        Oc, Sc = chunk_form.chunk_forward_gdr2(q[0, h], k[0, h], v[0, h], g[0, h], b[0, h], w[0, h], S0[0, h],
                                               C=C, gate=gate)
        assert rel(Oc, O[0, h]) < 1e-11 and rel(Sc, ST[0, h]) < 1e-11


# Basis keys k_t = e_{c_t}: the read along b_t * e_c picks b_{t,c} S~[:, c], so
# column c of the state follows s <- (1 - b_{t,c}) alpha_{t,c} s + w_t * v_t
# when token t writes it and s <- alpha_{t,c} s otherwise; no other entry of
# b_t matters.  Channels are reused, so the erase term is exercised.
def test_basis_keys_closed_form():
    rng = np.random.default_rng(12)
    B, H, T, dk, dv = 1, 1, 24, 5, 3
    _, _, v, g, b, w, S0 = rand_case(rng, B, H, T, dk, dv, g_lo=-7.0)
    ch = rng.integers(0, dk, T)
    k = np.zeros((B, H, T, dk))
    k[0, 0, np.arange(T), ch] = 1.0
    q = unit(rng.standard_normal((B, H, T, dk)))
    O, ST = oracle.forward_gdr2(q, k, v, g, b, w, S0)
    alpha = np.exp(np.maximum(g[0, 0], -5.0))
    S = S0[0, 0].copy()
    for t in range(T):
        for c in range(dk):
            if c == ch[t]:
                S[:, c] = (1.0 - b[0, 0, t, c]) * alpha[t, c] * S[:, c] + w[0, 0, t] * v[0, 0, t]
            else:
                S[:, c] = alpha[t, c] * S[:, c]
        assert rel(O[0, 0, t], S @ q[0, 0, t]) < RTOL
    assert rel(ST[0, 0], S) < RTOL


# b = 0 erases nothing: gated linear attention with the write gate,
# o_t = S0 Diag(gamma_t) q_t + sum_{i<=t} (w_i * v_i) (q_t . (k_i * gamma_t / gamma_i)).
@pytest.mark.parametrize("gate", ["per_channel", "scalar"])
def test_zero_erase_is_gated_linear_attention(gate):
    rng = np.random.default_rng(13)
    q, k, v, g, b, w, S0 = rand_case(rng, T=17, dk=4, dv=3, gate=gate, g_lo=-7.0)
    b[:] = 0.0
    O, ST = oracle.forward_gdr2(q, k, v, g, b, w, S0, gate=gate)
    B, H, T, dk = q.shape
    for bb in range(B):
        for h in range(H):
            la = np.maximum(g[bb, h], -5.0) if gate == "per_channel" else np.repeat(g[bb, h][:, None], dk, 1)
            G = np.cumsum(la, axis=0)
            for t in range(T):
                exp = S0[bb, h] @ (np.exp(G[t]) * q[bb, h, t])
                for i in range(t + 1):
                    exp = exp + w[bb, h, i] * v[bb, h, i] * np.dot(q[bb, h, t], k[bb, h, i] * np.exp(G[t] - G[i]))
                assert rel(O[bb, h, t], exp) < RTOL


# The section's eq. (10) in its own orientation (state d_k x d_v, o = S^T q),
# with the transition written out as a matrix:
#   S_t = (I - k_t (b_t * k_t)^T) D_t S_{t-1} + k_t (w_t * v_t)^T.
# The oracle works in the transposed (d_v x d_k) orientation, so a swapped
# read and write direction (k vs b * k) fails here.
def test_product_form_in_the_sections_orientation():
    rng = np.random.default_rng(14)
    q, k, v, g, b, w, S0 = rand_case(rng, B=1, H=1, T=9, dk=4, dv=3, g_lo=-2.0)
    O, ST = oracle.forward_gdr2(q, k, v, g, b, w, S0)
    St = S0[0, 0].T.copy()                     # d_k x d_v
    for t in range(9):
        kt, bt, qt = k[0, 0, t], b[0, 0, t], q[0, 0, t]
        D = np.diag(np.exp(np.maximum(g[0, 0, t], -5.0)))
        P = np.eye(4) - np.outer(kt, bt * kt)
        St = P @ D @ St + np.outer(kt, w[0, 0, t] * v[0, 0, t])
        assert rel(O[0, 0, t], St.T @ qt) < RTOL
    assert rel(ST[0, 0], St.T) < RTOL


# A scalar decay is the per-channel decay broadcast over the key channels
# (whenever g >= -5, where the per-channel bound changes nothing).
def test_scalar_equals_broadcast():
    rng = np.random.default_rng(15)
    q, k, v, g, b, w, S0 = rand_case(rng, T=21, dk=5, dv=4, gate="scalar", g_lo=-4.0)
    gb = np.repeat(g[..., None], 5, -1)
    O1, S1 = oracle.forward_gdr2(q, k, v, g, b, w, S0, gate="scalar")
    O2, S2 = oracle.forward_gdr2(q, k, v, gb, b, w, S0, gate="per_channel")
    assert rel(O1, O2) < RTOL and rel(S1, S2) < RTOL


def test_decode_driver_matches_forward():
    rng = np.random.default_rng(16)
    q, k, v, g, b, w, S0 = rand_case(rng, B=2, H=2, T=6, dk=4, dv=3)
    mv = lambda x: np.moveaxis(x, 2, 0)
    o, S = oracle.decode_gdr2(mv(q), mv(k), mv(v), mv(g), mv(b), mv(w), S0)
    O, ST = oracle.forward_gdr2(q, k, v, g, b, w, S0)
    assert rel(np.moveaxis(o, 0, 2), O) < RTOL and rel(S, ST) < RTOL
