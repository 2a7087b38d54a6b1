"""The seeded input generator: exactness of the counter-based RNG, subset
consistency (a few heads of a big workload equal the same heads of the full
tensor) and the value recipes of the five workloads."""
import numpy as np
import torch

import gdr_workloads as W


def test_splitmix64_matches_python_ints():
    cnt = torch.tensor([0, 1, 2, 3, 12345, 2 ** 40 + 7, 2 ** 62, 2 ** 63 - 2], dtype=torch.int64)
    for seed, tid in [(0, 1), (3, 2), (2 ** 40, 7)]:
        got = W.raw_u64(seed, tid, cnt).tolist()
        base = W.stream_base(seed, tid)
        for c, x in zip(cnt.tolist(), got):
            e = W.mix64_int((base + (c + 1) * W._GOLDEN) & W._M64)
            assert (x & W._M64) == e


def test_uniform_and_normal_moments():
    idx = torch.arange(200000)
    u = W.uniform(5, 3, idx)
    assert float(u.min()) >= 0.0 and float(u.max()) < 1.0
    assert abs(float(u.mean()) - 0.5) < 5e-3
    n = W.normal(5, 3, idx)
    assert abs(float(n.mean())) < 1e-2 and abs(float(n.std()) - 1.0) < 1e-2


def test_subset_equals_full():
    w = W.small_chunk_case(2, 3, 50, 16, 8, "per_channel", torch.bfloat16)
    full = W.generate(w)
    sub = W.generate(w, heads=[4, 1])
    for key in ("q", "k", "v", "g", "beta", "S0"):
        f = full[key].reshape(6, *full[key].shape[2:])
        s = sub[key].reshape(2, *sub[key].shape[2:])
        assert torch.equal(s[0], f[4]) and torch.equal(s[1], f[1]), key


def test_recipes():
    w = W.WORKLOADS["kda_tiny_fp32"]
    x = W.generate(w)
    assert x["q"].dtype == torch.float32 and x["q"].shape == (1, 2, 256, 64)
    assert torch.allclose(x["k"].double().norm(dim=-1), torch.ones(1, 2, 256, dtype=torch.float64), atol=1e-6)
    assert float(x["g"].min()) >= -5.0 and float(x["g"].max()) < 0.0
    assert float(x["beta"].min()) > 0.0 and float(x["beta"].max()) < 1.0
    assert float(x["S0"].abs().max()) == 0.0
    w4 = W.WORKLOADS["kda_long_t65536"]
    s = W.generate(w4, heads=[3])
    g = s["g"][0, 0]
    fast = (g == -5.0).all(dim=0)
    assert int(fast.sum()) == W.LONG_FAST_CHANNELS
    slow = g[:, ~fast]
    assert float(slow.max()) <= -0.001 + 1e-7 and float(slow.min()) >= -0.05 - 1e-7
    assert s["q"].dtype == torch.bfloat16
    assert abs(float(s["S0"].std()) - 0.02) < 1e-3
    w2 = W.WORKLOADS["gdn_scalar_t4096"]
    s2 = W.generate(w2, heads=[0])
    assert s2["g"].shape == (1, 1, 4096)
    assert float(s2["g"].max()) < 0.0


def test_decode_layout():
    w = W.WORKLOADS["kda_decode_b256"]
    d = W.generate(w, heads=[0, 5], steps=4)
    assert d["q"].shape == (4, 2, 1, 128) and d["beta"].shape == (4, 2, 1)
    assert d["S0"].shape == (2, 1, 128, 128)
    d1 = W.generate(w, heads=[5], steps=2)
    assert torch.equal(d1["v"][1, 0, 0], d["v"][1, 1, 0])
