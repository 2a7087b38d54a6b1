"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test computes its expected value from a closed form, a special case or
a brute-force formulation that is independent of the oracle's token loop, so
that a dropped term, a wrong sign or index, a transposed operand or a wrong
update order in the oracle fails at least one of them.
"""
import os

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
    if gate == "per_channel":
        g = rng.uniform(g_lo, 0.0, (B, H, T, dk))
    else:
        g = rng.uniform(g_lo, 0.0, (B, H, T))
    beta = rng.uniform(0.0, 1.0, (B, H, T))
    S0 = 0.3 * rng.standard_normal((B, H, dv, dk))
    return q, k, v, g, beta, S0


# P1 -- "Token Mixer I", section "Mamba2: linear attention with decay":
# with no decay and a pure additive write, O = (Q K^T * M) V.
def test_p1_linear_attention():
    rng = np.random.default_rng(1)
    q, k, v, g, beta, _ = rand_case(rng, T=23, dk=6, dv=4)
    g[:] = 0.0
    zeros, ones = np.zeros_like(beta), np.ones_like(beta)
    O, ST = oracle.forward(q, k, v, g, beta, None, erase=zeros, write=ones)
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            Q, K, V = q[b, h], k[b, h], v[b, h]
            M = np.tril(np.ones((len(Q), len(Q))))
            assert rel(O[b, h], (Q @ K.T * M) @ V) < RTOL
            assert rel(ST[b, h], V.T @ K) < RTOL


# P2 -- same section: with decay, o_t = sum_{i<=t} v_i (q_t . (k_i * gamma_t/gamma_i)),
# plus the decayed initial state S0 Diag(gamma_t) q_t.
@pytest.mark.parametrize("gate", ["per_channel", "scalar"])
def test_p2_gated_linear_attention(gate):
    rng = np.random.default_rng(2)
    q, k, v, g, beta, S0 = rand_case(rng, T=19, dk=5, dv=3, gate=gate, g_lo=-7.0)
    zeros, ones = np.zeros_like(beta), np.ones_like(beta)
    O, ST = oracle.forward(q, k, v, g, beta, S0, gate=gate, erase=zeros, write=ones)
    B, H, T, dk = q.shape
    for b in range(B):
        for h in range(H):
            if gate == "per_channel":
                la = np.maximum(g[b, h], -5.0)          # the KDA lower bound
            else:
                la = np.repeat(g[b, h][:, None], dk, 1)  # scalar gate: no bound
            G = np.cumsum(la, axis=0)
            exp = np.zeros((T, v.shape[-1]))
            for t in range(T):
                exp[t] = S0[b, h] @ (np.exp(G[t]) * q[b, h, t])
                for i in range(t + 1):
                    exp[t] += v[b, h, i] * np.dot(q[b, h, t], k[b, h, i] * np.exp(G[t] - G[i]))
            assert rel(O[b, h], exp) < RTOL
            if gate == "scalar":
                # ((Q K^T) * Gamma) V with Gamma_ti = gamma_t / gamma_i, S0 = 0 part
                gs = np.cumsum(g[b, h])
                Gam = np.tril(np.exp(gs[:, None] - gs[None, :]))
                par = ((q[b, h] @ k[b, h].T) * Gam) @ v[b, h] + (S0[b, h] @ q[b, h].T).T * np.exp(gs)[:, None]
                assert rel(O[b, h], par) < RTOL


# P3 -- beta = 0 writes nothing: O_t = S0 Diag(gamma_t) q_t, S_T = S0 Diag(gamma_T).
def test_p3_beta_zero():
    rng = np.random.default_rng(3)
    q, k, v, g, beta, S0 = rand_case(rng, T=17, dk=4, dv=6, g_lo=-6.0)
    beta[:] = 0.0
    O, ST = oracle.forward(q, k, v, g, beta, S0)
    G = np.cumsum(np.maximum(g, -5.0), axis=2)
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            expO = np.stack([S0[b, h] @ (np.exp(G[b, h, t]) * q[b, h, t]) for t in range(q.shape[2])])
            assert rel(O[b, h], expO) < RTOL
            assert rel(ST[b, h], S0[b, h] * np.exp(G[b, h, -1])[None, :]) < RTOL


# P4 -- a scalar gate equals a per-channel gate holding the same value in every
# channel ("Token Mixer I", section "Gated DeltaNet-2": constraining the decay
# to a scalar recovers Gated DeltaNet); valid while g >= -5.
def test_p4_scalar_equals_broadcast():
    rng = np.random.default_rng(4)
    q, k, v, g, beta, S0 = rand_case(rng, T=40, dk=7, dv=5, gate="scalar", g_lo=-4.9)
    O1, S1 = oracle.forward(q, k, v, g, beta, S0, gate="scalar")
    gb = np.repeat(g[..., None], q.shape[-1], axis=-1)
    O2, S2 = oracle.forward(q, k, v, gb, beta, S0, gate="per_channel")
    assert rel(O1, O2) < RTOL and rel(S1, S2) < RTOL


# P5 -- orthonormal keys, beta = 1, no decay, S0 = 0: retrieval S k_i returns v_i
# exactly, and o_t = sum_{i<=t} (k_i . q_t) v_i ("Token Mixer I", section
# "Gated DeltaNet-2 / Preliminary": with a unit key and beta = 1 the delta rule
# overwrites the association of that key).  Overwrite: a key written twice
# returns the latest value.
def test_p5_orthonormal_retrieval_and_overwrite():
    rng = np.random.default_rng(5)
    dk, dv, T = 8, 5, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:, :T].T[None, None]                     # T orthonormal keys
    q = unit(rng.standard_normal((1, 1, T, dk)))
    v = rng.standard_normal((1, 1, T, dv))
    g = np.zeros((1, 1, T, dk))
    beta = np.ones((1, 1, T))
    O, ST = oracle.forward(q, k, v, g, beta, None)
    for i in range(T):
        assert np.max(np.abs(ST[0, 0] @ k[0, 0, i] - v[0, 0, i])) < 1e-12
    exp = np.stack([sum(np.dot(k[0, 0, i], q[0, 0, t]) * v[0, 0, i] for i in range(t + 1)) for t in range(T)])
    assert rel(O[0, 0], exp) < RTOL
    # overwrite: key 0 again with a new value
    k2 = np.concatenate([k, k[:, :, :1]], axis=2)
    v_new = rng.standard_normal((1, 1, 1, dv))
    v2 = np.concatenate([v, v_new], axis=2)
    q2 = np.concatenate([q, q[:, :, :1]], axis=2)
    _, ST2 = oracle.forward(q2, k2, v2, np.zeros((1, 1, T + 1, dk)), np.ones((1, 1, T + 1)), None)
    assert np.max(np.abs(ST2[0, 0] @ k[0, 0, 0] - v_new[0, 0, 0])) < 1e-12
    for i in range(1, T):
        assert np.max(np.abs(ST2[0, 0] @ k[0, 0, i] - v[0, 0, i])) < 1e-12


# P6 -- basis keys k_t = e_{c_t}: each state column follows a scalar recursion.
# A touched column becomes (1 - beta_t) alpha_{t,c} s + beta_t v_t (decay first,
# then the delta from the decayed state); an untouched column only decays.
# Also covers the -5 clamp of the per-channel gate.
def test_p6_basis_keys_closed_form():
    rng = np.random.default_rng(6)
    dk, dv, T = 6, 4, 30
    ch = rng.integers(0, dk, T)
    ch[:3] = [0, 1, 0]                               # a reused channel early on
    k = np.zeros((1, 1, T, dk))
    k[0, 0, np.arange(T), ch] = 1.0
    q = unit(rng.standard_normal((1, 1, T, dk)))
    v = rng.standard_normal((1, 1, T, dv))
    g = rng.uniform(-8.0, 0.0, (1, 1, T, dk))        # some entries below the -5 bound
    beta = rng.uniform(0.0, 1.0, (1, 1, T))
    S0 = rng.standard_normal((1, 1, dv, dk))
    O, ST = oracle.forward(q, k, v, g, beta, S0)
    S = S0[0, 0].copy()
    for t in range(T):
        a = np.exp(np.maximum(g[0, 0, t], -5.0))
        for c in range(dk):
            if c == ch[t]:
                S[:, c] = (1.0 - beta[0, 0, t]) * a[c] * S[:, c] + beta[0, 0, t] * v[0, 0, t]
            else:
                S[:, c] = a[c] * S[:, c]
        assert rel(O[0, 0, t], S @ q[0, 0, t]) < RTOL
    assert rel(ST[0, 0], S) < RTOL
    # distinct channels from S0 = 0: S_T[:, c_i] = beta_i v_i prod_{j>i} alpha_{j,c_i}
    Td = dk
    k = np.eye(dk)[None, None]
    v = rng.standard_normal((1, 1, Td, dv))
    g = rng.uniform(-3.0, 0.0, (1, 1, Td, dk))
    beta = rng.uniform(0.1, 1.0, (1, 1, Td))
    _, ST = oracle.forward(unit(rng.standard_normal((1, 1, Td, dk))), k, v, g, beta, None)
    for i in range(Td):
        decay = np.exp(np.sum(g[0, 0, i + 1:, i]))
        assert np.max(np.abs(ST[0, 0][:, i] - beta[0, 0, i] * v[0, 0, i] * decay)) < 1e-13


# P7 -- the chunkwise WY/UT form ("Reading notes: Kimi Delta Attention",
# section 4) equals the recurrence for every chunk size, partial last chunk
# included, and with the gate at its -5 bound everywhere.
@pytest.mark.parametrize("C", [1, 2, 3, 4, 8, 16, 32, 64])
@pytest.mark.parametrize("gate,glo", [("per_channel", -1.0), ("per_channel", -5.0), ("scalar", -2.0)])
def test_p7_chunk_form_equals_recurrence(C, gate, glo):
    rng = np.random.default_rng(7 + C)
    T = 130
    q, k, v, g, beta, S0 = rand_case(rng, B=1, H=1, T=T, dk=6, dv=5, gate=gate, g_lo=glo)
    if glo == -5.0:
        g[:] = -5.0
    O, ST = oracle.forward(q, k, v, g, beta, S0, gate=gate)
    Oc, Sc = chunk_form.chunk_forward(q[0, 0], k[0, 0], v[0, 0], g[0, 0], beta[0, 0], S0[0, 0], C=C, gate=gate)
    assert rel(Oc, O[0, 0]) < 1e-11
    assert rel(Sc, ST[0, 0]) < 1e-11


# P8 -- brute force over explicit d_k x d_k products ("Token Mixer I", section
# "Kimi Delta Attention as learnable position embeddings"):
# o_t = sum_i beta_i (q_t^T [prod_{j=i+1..t} (I - beta_j k_j k_j^T) Diag(alpha_j)] k_i) v_i,
# later factors on the left, S0 = 0.
def test_p8_bruteforce_product_form():
    rng = np.random.default_rng(8)
    T, dk, dv = 8, 4, 3
    q, k, v, g, beta, _ = rand_case(rng, B=1, H=1, T=T, dk=dk, dv=dv, g_lo=-2.0)
    O, _ = oracle.forward(q, k, v, g, beta, None)
    Q, K, V, A, b = q[0, 0], k[0, 0], v[0, 0], np.exp(g[0, 0]), beta[0, 0]
    for t in range(T):
        o = np.zeros(dv)
        for i in range(t + 1):
            P = np.eye(dk)
            for j in range(i + 1, t + 1):
                P = (np.eye(dk) - b[j] * np.outer(K[j], K[j])) @ np.diag(A[j]) @ P
            o += b[i] * (Q[t] @ P @ K[i]) * V[i]
        assert rel(O[0, 0, t], o) < RTOL


# P9 -- WY identity ("Reading notes: Kimi Delta Attention", section 4): with
# v = 0 the recurrence maps S0 to S0 P^r with
# P^r = prod Diag(alpha_i)(I - beta_i k_i k_i^T) = (I - sum_i w_i (k_i/gamma_i)^T) Diag(gamma_r),
# w_r = beta_r (I - sum_{i<r} w_i (k_i/gamma_i)^T) Diag(gamma_r) k_r.
def test_p9_wy_identity():
    rng = np.random.default_rng(9)
    T, dk, dv = 12, 5, 5
    q, k, v, g, beta, _ = rand_case(rng, B=1, H=1, T=T, dk=dk, dv=dv, g_lo=-1.0)
    v[:] = 0.0
    S0 = np.eye(dv, dk)[None, None]
    _, ST = oracle.forward(q, k, v, g, beta, S0)
    K, b = k[0, 0], beta[0, 0]
    G = np.cumsum(g[0, 0], axis=0)
    w = []
    for r in range(T):
        Pm = np.eye(dk) - sum((np.outer(w[i], K[i] / np.exp(G[i])) for i in range(r)), np.zeros((dk, dk)))
        w.append(b[r] * Pm @ (np.exp(G[r]) * K[r]))
    P = (np.eye(dk) - sum(np.outer(w[i], K[i] / np.exp(G[i])) for i in range(T))) @ np.diag(np.exp(G[-1]))
    assert rel(ST[0, 0], np.eye(dv, dk) @ P) < 1e-11


# P10 -- the final state is the whole resumable state ("Reading notes: Kimi
# Delta Attention", section 4, S_[t]^r = S_[t-1]^C P^r + H^r): one run equals
# two runs chained through S_T.
@pytest.mark.parametrize("T1", [1, 37, 64, 99])
def test_p10_split_resume(T1):
    rng = np.random.default_rng(10)
    q, k, v, g, beta, S0 = rand_case(rng, B=2, H=2, T=100, dk=6, dv=4)
    O, ST = oracle.forward(q, k, v, g, beta, S0)
    sl = lambda x, a, b: x[:, :, a:b]
    O1, S1 = oracle.forward(sl(q, 0, T1), sl(k, 0, T1), sl(v, 0, T1), sl(g, 0, T1), sl(beta, 0, T1), S0)
    O2, S2 = oracle.forward(sl(q, T1, 100), sl(k, T1, 100), sl(v, T1, 100), sl(g, T1, 100), sl(beta, T1, 100), S1)
    assert rel(np.concatenate([O1, O2], axis=2), O) < RTOL
    assert rel(S2, ST) < RTOL


# P11 -- the capacity table of "Lightweight LLM reproduction: Linear Attention"
# (aitujian), section 4.1.8 (tests/golden/capacity_table.txt).
def test_p11_capacity_table():
    path = os.path.join(os.path.dirname(__file__), "golden", "capacity_table.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    writes = np.array([float(r[0]) for r in rows])
    want = np.array([float(r[1]) for r in rows])
    T = len(writes)
    one = np.ones((1, 1, T, 1))
    O, _ = oracle.forward(one, one, writes.reshape(1, 1, T, 1), np.full((1, 1, T, 1), np.log(0.152)),
                          np.full((1, 1, T), 0.5), None)
    assert np.max(np.abs(O[0, 0, :, 0] - want)) <= 5e-4


# Bound: with |k| <= 1, beta in [0,1] and alpha in (0,1] every transition is a
# contraction, so |S_t|_F <= |S_{t-1}|_F + beta_t |v_t|.
def test_state_norm_bound():
    rng = np.random.default_rng(12)
    q, k, v, g, beta, S0 = rand_case(rng, B=1, H=1, T=200, dk=8, dv=8)
    S = S0
    for t in range(200):
        sl = lambda x: x[:, :, t:t + 1]
        _, Sn = oracle.forward(sl(q), sl(k), sl(v), sl(g), sl(beta), S)
        assert np.linalg.norm(Sn) <= np.linalg.norm(S) + beta[0, 0, t] * np.linalg.norm(v[0, 0, t]) + 1e-12
        S = Sn


# The decode driver is the same recurrence with steps as tokens.
def test_decode_driver_matches_forward():
    rng = np.random.default_rng(13)
    q, k, v, g, beta, S0 = rand_case(rng, B=2, H=3, T=9, dk=4, dv=4)
    O, ST = oracle.forward(q, k, v, g, beta, S0)
    mv = lambda x: np.moveaxis(x, 2, 0)
    o, S = oracle.decode(mv(q), mv(k), mv(v), mv(g), mv(beta), S0)
    assert rel(np.moveaxis(o, 0, 2), O) < 1e-15 and rel(S, ST) < 1e-15
