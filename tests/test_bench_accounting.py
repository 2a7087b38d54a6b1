"""The byte counts behind bench.py's roofline fractions, recomputed by hand
for every workload bench.py can run (CPU only)."""
import bench
import gdr_workloads as W

MB = 1e6


def bytes_of(name):
    return bench.algorithmic_bytes(W.WORKLOADS[name])


def test_headline_forward():
    # per head-token: q, k, v bf16 (3 x 256 B) + per-channel g fp32 (512) + beta (4) + O bf16 (256);
    # per head: S0 read and S_T written (2 x 64 KiB)
    heads, tokens = 2 * 32, 8192
    assert bytes_of("kda_d128_t8192") == heads * tokens * (768 + 512 + 4 + 256) + heads * 2 * 128 * 128 * 4
    assert abs(bytes_of("kda_d128_t8192") / MB - 815.8) < 0.1


def test_variants():
    heads, tokens, state = 64, 8192, 64 * 2 * 128 * 128 * 4
    # prologue: the gate pre-activation comes in bf16 (256 B instead of 512)
    assert bytes_of("kda_d128_t8192_prologue") == heads * tokens * (768 + 256 + 4 + 256) + state
    # gated output: the output gate pre-activation is read too (bf16, 256 B)
    assert bytes_of("kda_d128_t8192_gated") == heads * tokens * (768 + 512 + 4 + 256 + 256) + state
    # GDR-2: erase (d_k) and write (d_v) gates in bf16 replace beta
    assert bytes_of("gdr2_d128_t8192") == heads * tokens * (768 + 512 + 512 + 256) + state


def test_backward():
    # reads q, k, v, g, beta, dO; writes dq, dk, dv, dg, dbeta; S0 and dS_T read, dS0 written
    heads, tokens = 64, 8192
    per_token = (768 + 512 + 4 + 256) + (768 + 512 + 4)
    assert bytes_of("kda_d128_t8192_bwd") == heads * tokens * per_token + heads * 3 * 128 * 128 * 4


def test_decode_per_step():
    import dataclasses
    w = dataclasses.replace(W.WORKLOADS["kda_decode_b256"], T=1)
    heads = 256 * 32
    assert bench.algorithmic_bytes(w) == heads * (768 + 512 + 4 + 256 + 2 * 128 * 128 * 4)


def test_traffic_is_keyed_to_sources():
    # every recorded traffic figure belongs to a workload bench.py knows, with a source hash
    for name, ent in bench.TRAFFIC.items():
        assert name in W.WORKLOADS
        assert len(ent["src_sha"]) == 16 and ent["bytes_per_launch"] > 0


def test_traffic_only_for_the_sources_it_was_measured_on(tmp_path):
    # the stored DRAM figure is reported only while the path's sources hash to the
    # value recorded with it; other sources, or a batch-overridden workload (used
    # for small profiler captures), report none
    import dataclasses
    w = W.WORKLOADS["kda_d128_t8192"]
    peaks = {"hbm_gbs": 6453.4, "bf16_tflops": 1679.3, "source": "test"}
    other = tmp_path / "other.cu"
    other.write_text("// not a source of the path\n")
    assert bench.roofline(w, 1e-3, peaks, [str(other)])["traffic"] is None
    wb = dataclasses.replace(w, B=1, name=f"{w.name}_b1")
    assert bench.roofline(wb, 1e-3, peaks, bench.kernel_sources(w))["traffic"] is None
    # the fractions: against the measured copy peak and against the datasheet figure
    r = bench.roofline(w, 1e-3, peaks, [str(other)])
    assert abs(r["frac"] - bench.algorithmic_bytes(w) / 1e-3 / 1e9 / 6453.4) < 1e-4
    assert abs(r["frac_vs_spec"] - bench.algorithmic_bytes(w) / 1e-3 / 1e9 / bench.SPEC_HBM_GBS) < 1e-4
