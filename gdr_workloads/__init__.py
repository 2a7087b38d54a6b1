"""Seeded synthetic inputs for the gated delta rule workloads.

This module only draws random numbers and shapes them into the five
workloads; it holds none of the method's arithmetic (no gate cumsum, no
decay, no delta update).  Both the fp64 CPU oracle (through the tests) and
the CUDA library (through the tests and ``bench.py``) are fed from here, so
the two sides always see bit-identical inputs.

Generator
---------
Counter-based SplitMix64: element ``n`` of tensor ``tid`` under ``seed`` is
``mix64(base(seed, tid) + (n + 1) * 0x9E3779B97F4A7C15)`` (mod 2**64), where
``mix64`` is the published SplitMix64 output function (Steele, Lea & Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014).  The top 53
bits give a uniform double in [0, 1).  Normals use Box-Muller on the pair of
counters (2n, 2n+1).  Because every element is a pure function of
(seed, tid, flat index), any subset of a tensor (a few heads of a large
workload) can be generated without generating the rest, on CPU or GPU, with
identical results.

Value recipes follow the workload descriptions: q, k ~ N(0,1) L2-normalised
per token, v ~ N(0,1), beta = sigmoid(N(0,1)), per-channel or scalar
log-decay g, S0 zero or N(0, 0.02) (0.02 is the standard deviation).
Low-precision tensors are produced by rounding fp64 -> fp32 -> bf16, both
round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Sequence

import torch

_M64 = (1 << 64) - 1
_GOLDEN = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB
_STREAM = 0xD1B54A32D192ED03

# tensor ids: one independent stream per input tensor
TID_Q, TID_K, TID_V, TID_G, TID_BETA, TID_S0, TID_CHAN = 1, 2, 3, 4, 5, 6, 7
# raw inputs of the fused gate / normalisation prologue
TID_QRAW, TID_KRAW, TID_AGATE, TID_ALOG, TID_DTBIAS, TID_BLOGIT = 8, 9, 10, 11, 12, 13
TID_ERASE, TID_WRITE = 14, 15   # Gated Delta Rule-2 erase and write gates
TID_OGATE, TID_NORMW = 16, 17   # output gate pre-activation, RMSNorm weight
TID_DO, TID_DST = 18, 19         # gradients fed to the backward pass


def _s64(c: int) -> int:
    """Unsigned 64-bit constant -> the int64 with the same bits."""
    c &= _M64
    return c - (1 << 64) if c >= (1 << 63) else c


def mix64_int(z: int) -> int:
    """SplitMix64 output function on a Python int (exact, for reference)."""
    z &= _M64
    z = ((z ^ (z >> 30)) * _MIX1) & _M64
    z = ((z ^ (z >> 27)) * _MIX2) & _M64
    return z ^ (z >> 31)


def stream_base(seed: int, tid: int) -> int:
    return mix64_int(mix64_int(seed) ^ ((tid * _STREAM) & _M64))


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return torch.bitwise_and(torch.bitwise_right_shift(z, s), (1 << (64 - s)) - 1)


def _mix64_t(z: torch.Tensor) -> torch.Tensor:
    z = torch.bitwise_xor(z, _srl(z, 30)) * _s64(_MIX1)
    z = torch.bitwise_xor(z, _srl(z, 27)) * _s64(_MIX2)
    return torch.bitwise_xor(z, _srl(z, 31))


def raw_u64(seed: int, tid: int, counters: torch.Tensor) -> torch.Tensor:
    """int64 tensor holding the 64-bit outputs for the given counters."""
    base = _s64(stream_base(seed, tid))
    z = base + (counters.to(torch.int64) + 1) * _s64(_GOLDEN)
    return _mix64_t(z)


def uniform(seed: int, tid: int, counters: torch.Tensor) -> torch.Tensor:
    """fp64 uniforms in [0, 1) for the given counters."""
    u = _srl(raw_u64(seed, tid, counters), 11)
    return u.to(torch.float64) * (2.0 ** -53)


def normal(seed: int, tid: int, index: torch.Tensor) -> torch.Tensor:
    """fp64 standard normals for element indices (Box-Muller on 2n, 2n+1)."""
    index = index.to(torch.int64)
    u1 = uniform(seed, tid, 2 * index)
    u2 = uniform(seed, tid, 2 * index + 1)
    return torch.sqrt(-2.0 * torch.log1p(-u1)) * torch.cos((2.0 * math.pi) * u2)


def _softplus64(x: torch.Tensor) -> torch.Tensor:
    return torch.where(x > 30.0, x, torch.log1p(torch.exp(torch.clamp(x, max=30.0))))


def _sigmoid64(x: torch.Tensor) -> torch.Tensor:
    return 1.0 / (1.0 + torch.exp(-x))


def to_dtype(x64: torch.Tensor, dtype: torch.dtype) -> torch.Tensor:
    """fp64 -> fp32 (RNE) -> dtype (RNE)."""
    x32 = x64.to(torch.float32)
    return x32 if dtype == torch.float32 else x32.to(dtype)


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "chunk" or "decode"
    B: int
    H: int
    T: int               # tokens per sequence (chunk) or steps (decode)
    dk: int
    dv: int
    C: int
    gate: str            # "per_channel" or "scalar"
    dtype: torch.dtype   # dtype of q, k, v, O
    g_recipe: str
    s0: str              # "zero" or "normal002"
    seed: int
    description: str
    rule: str = "gdr"    # "gdr" (tied beta: KDA / Gated DeltaNet) or "gdr2" (erase and write gates)
    out: str = "plain"   # "plain" (o_t) or "gated" (Sigmoid(gate) * RMSNorm(o_t))
    direction: str = "fwd"   # "fwd" or "bwd" (the gradients of <dO, O> + <dS_T, S_T>)

    @property
    def tokens(self) -> int:
        """Tokens one pass processes: B*T for the forward, B per decode step."""
        return self.B * self.T


WORKLOADS: Dict[str, Workload] = {
    "kda_tiny_fp32": Workload(
        "kda_tiny_fp32", "chunk", 1, 2, 256, 64, 64, 64, "per_channel", torch.float32,
        "softplus_n01_plus1_clamp5", "zero", 0,
        "KDA forward, tiny, fp32: B1 H2 T256 d64 C64"),
    "gdn_scalar_t4096": Workload(
        "gdn_scalar_t4096", "chunk", 4, 16, 4096, 128, 128, 64, "scalar", torch.bfloat16,
        "scalar_softplus_n01_plus2", "zero", 1,
        "Gated DeltaNet (scalar gate) forward: B4 H16 T4096 d128 C64 bf16"),
    "kda_d128_t8192": Workload(
        "kda_d128_t8192", "chunk", 2, 32, 8192, 128, 128, 64, "per_channel", torch.bfloat16,
        "softplus_n02_clamp5", "normal002", 2,
        "KDA forward at head dim 128: B2 H32 T8192 d128 C64 bf16"),
    "kda_d128_t8192_prologue": Workload(
        "kda_d128_t8192_prologue", "chunk", 2, 32, 8192, 128, 128, 64, "per_channel", torch.bfloat16,
        "prologue", "normal002", 2,
        "KDA forward with the input prologue fused in (raw q, k; bf16 gate pre-activation; beta "
        "logits): B2 H32 T8192 d128 C64 bf16"),
    "gdr2_d128_t8192": Workload(
        "gdr2_d128_t8192", "chunk", 2, 32, 8192, 128, 128, 64, "per_channel", torch.bfloat16,
        "softplus_n02_clamp5", "normal002", 5,
        "Gated Delta Rule-2 forward (per-channel decay, erase and write gates): B2 H32 T8192 d128 C64 bf16",
        rule="gdr2"),
    "kda_d128_t8192_gated": Workload(
        "kda_d128_t8192_gated", "chunk", 2, 32, 8192, 128, 128, 64, "per_channel", torch.bfloat16,
        "softplus_n02_clamp5", "normal002", 2,
        "KDA forward with the output epilogue fused in (per-head RMSNorm times a sigmoid output gate): "
        "B2 H32 T8192 d128 C64 bf16", out="gated"),
    "kda_d128_t8192_bwd": Workload(
        "kda_d128_t8192_bwd", "chunk", 2, 32, 8192, 128, 128, 64, "per_channel", torch.bfloat16,
        "softplus_n02_clamp5", "normal002", 2,
        "KDA backward (gradients of q, k, v, g, beta, S0 from dO, dS_T): B2 H32 T8192 d128 C64 bf16",
        direction="bwd"),
    "gdr2_decode_b256": Workload(
        "gdr2_decode_b256", "decode", 256, 32, 1000, 128, 128, 1, "per_channel", torch.bfloat16,
        "softplus_n01_plus1_clamp5", "normal002", 6,
        "Gated Delta Rule-2 recurrent decode: B256 H32 d128, 1000 steps, fp32 state", rule="gdr2"),
    "kda_long_t65536": Workload(
        "kda_long_t65536", "chunk", 1, 32, 65536, 128, 128, 64, "per_channel", torch.bfloat16,
        "long_context_mix", "normal002", 3,
        "KDA long-context forward: B1 H32 T65536 d128 C64 bf16"),
    "kda_decode_b256": Workload(
        "kda_decode_b256", "decode", 256, 32, 1000, 128, 128, 1, "per_channel", torch.bfloat16,
        "softplus_n01_plus1_clamp5", "normal002", 4,
        "KDA recurrent decode: B256 H32 d128, 1000 steps, fp32 state"),
}

# the five workloads in the order the method's configurations list them
ORDER = ["kda_tiny_fp32", "gdn_scalar_t4096", "kda_d128_t8192", "kda_long_t65536", "kda_decode_b256"]

LONG_FAST_CHANNELS = 13  # round(0.1 * 128) channels per head pinned at g = -5


def _g_from_recipe(w: Workload, seed: int, idx: torch.Tensor, b: torch.Tensor, h: torch.Tensor,
                   c: Optional[torch.Tensor], fast: Optional[Dict]) -> torch.Tensor:
    r = w.g_recipe
    if r == "softplus_n01_plus1_clamp5":
        return torch.clamp(-_softplus64(normal(seed, TID_G, idx) + 1.0), min=-5.0)
    if r == "scalar_softplus_n01_plus2":
        return -_softplus64(normal(seed, TID_G, idx) + 2.0)
    if r == "softplus_n02_clamp5":
        return torch.clamp(-_softplus64(2.0 * normal(seed, TID_G, idx)), min=-5.0)
    if r == "slow_decay":               # parity cases only: the state carries across chunks
        return -(0.001 + 0.049 * uniform(seed, TID_G, idx))
    if r == "softplus_n02_unbounded":   # parity cases only: some values below -5
        return -_softplus64(2.0 * normal(seed, TID_G, idx) + 2.0)
    if r == "long_context_mix":
        u = uniform(seed, TID_G, idx)
        slow = -(0.001 + 0.049 * u)
        is_fast = fast["mask"][b * w.H + h, c]
        return torch.where(is_fast, torch.full_like(slow, -5.0), slow)
    raise ValueError(r)


def fast_channel_mask(w: Workload, device="cpu") -> torch.Tensor:
    """[B*H, dk] bool: the channels pinned at g=-5 in the long-context workload.

    Per head, the LONG_FAST_CHANNELS channels with the smallest draw from
    stream TID_CHAN are chosen.
    """
    n = w.B * w.H * w.dk
    u = uniform(w.seed, TID_CHAN, torch.arange(n, device=device)).view(w.B * w.H, w.dk)
    order = torch.argsort(u, dim=1)
    mask = torch.zeros(w.B * w.H, w.dk, dtype=torch.bool, device=device)
    mask.scatter_(1, order[:, :LONG_FAST_CHANNELS], True)
    return mask


def _chunked(n: int, block: int):
    s = 0
    while s < n:
        e = min(n, s + block)
        yield s, e
        s = e


def generate(w: Workload, device="cpu", heads: Optional[Sequence[int]] = None,
             steps: Optional[int] = None, step0: int = 0, block: int = 1 << 24) -> Dict[str, torch.Tensor]:
    """Inputs of workload ``w``.

    ``heads``: optional list of flat head ids (b*H + h); when given, tensors
    keep their full (B, H) extent only along the selected heads, returned as
    shape [len(heads), 1, ...] with the same values the full tensor holds
    there.  ``steps`` (decode only) limits the number of steps generated.

    Chunk workloads return q, k [B,H,T,dk], v [B,H,T,dv], g [B,H,T,dk] or
    [B,H,T], beta [B,H,T], S0 [B,H,dv,dk] (fp32).  Decode returns the same
    keys with a leading steps axis: q [S,B,H,dk] ... and S0 [B,H,dv,dk].
    Gated Delta Rule-2 workloads add the erase gate b (shape of k) and the
    write gate w (shape of v), sigmoid(N(0,1)) in the workload dtype.
    Gated-output workloads add the output gate pre-activation ogate (shape of
    v) ~ N(0,1) in the workload dtype and the RMSNorm weight norm_w [dv] ~
    1 + 0.1 N(0,1) fp32 (shared by the heads).
    """
    B, H, dk, dv = w.B, w.H, w.dk, w.dv
    if heads is None:
        head_ids = torch.arange(B * H, dtype=torch.int64, device=device)
        outB, outH = B, H
    else:
        head_ids = torch.as_tensor(list(heads), dtype=torch.int64, device=device)
        outB, outH = len(heads), 1
    nh = head_ids.numel()
    if w.g_recipe == "prologue":
        raise ValueError(f"{w.name} takes raw inputs: use generate_prologue")
    fast = {"mask": fast_channel_mask(w, device)} if w.g_recipe == "long_context_mix" else None
    seed = w.seed
    decode = w.kind == "decode"
    T = (steps if steps is not None else w.T)

    def field(tid, width, make, out_dtype):
        # flat index of element (t, head, j) in the full tensor
        if decode:
            shape = (T, nh, width) if width else (T, nh)
        else:
            shape = (nh, T, width) if width else (nh, T)
        out = torch.empty(shape, dtype=out_dtype, device=device)
        flat = out.view(-1)
        n = flat.numel()
        per_row = width if width else 1
        for s, e in _chunked(n, block):
            lin = torch.arange(s, e, dtype=torch.int64, device=device)
            j = lin % per_row
            rest = lin // per_row
            if decode:
                hsel = rest % nh
                t = rest // nh + step0
                hid = head_ids[hsel]
                full = (t * (B * H) + hid) * per_row + j
            else:
                t = rest % T
                hsel = rest // T
                hid = head_ids[hsel]
                full = (hid * w.T + t) * per_row + j
            flat[s:e] = make(tid, full, hid // H, hid % H, j if width else None, t)
        return out

    def qk_field(tid):
        raw = field(tid, dk, lambda tid_, full, b, h, c, t: normal(seed, tid_, full), torch.float64)
        nrm = torch.sqrt((raw * raw).sum(-1, keepdim=True))
        return to_dtype(raw / nrm, w.dtype)

    q = qk_field(TID_Q)
    k = qk_field(TID_K)
    v = to_dtype(field(TID_V, dv, lambda tid_, full, b, h, c, t: normal(seed, tid_, full), torch.float64), w.dtype)
    if w.gate == "per_channel":
        g = field(TID_G, dk, lambda tid_, full, b, h, c, t: _g_from_recipe(w, seed, full, b, h, c, fast),
                  torch.float64).to(torch.float32)
    else:
        g = field(TID_G, 0, lambda tid_, full, b, h, c, t: _g_from_recipe(w, seed, full, b, h, c, fast),
                  torch.float64).to(torch.float32)
    beta = field(TID_BETA, 0, lambda tid_, full, b, h, c, t: _sigmoid64(normal(seed, tid_, full)),
                 torch.float64).to(torch.float32)
    gates2 = {}
    if w.rule == "gdr2":
        sig = lambda tid_, full, b, h, c, t: _sigmoid64(normal(seed, tid_, full))
        gates2 = dict(b=(to_dtype(field(TID_ERASE, dk, sig, torch.float64), w.dtype), dk),
                      w=(to_dtype(field(TID_WRITE, dv, sig, torch.float64), w.dtype), dv))

    # initial state: [head, dv, dk], flat index over the full [B,H,dv,dk]
    if w.s0 == "zero":
        S0 = torch.zeros(nh, dv, dk, dtype=torch.float32, device=device)
    else:
        per = dv * dk
        S0 = torch.empty(nh, dv, dk, dtype=torch.float32, device=device)
        flat = S0.view(-1)
        for s, e in _chunked(flat.numel(), block):
            lin = torch.arange(s, e, dtype=torch.int64, device=device)
            full = head_ids[lin // per] * per + lin % per
            flat[s:e] = (0.02 * normal(seed, TID_S0, full)).to(torch.float32)

    if decode:
        shp = lambda x, *tail: x.view(T, outB, outH, *tail)
        out = dict(q=shp(q, dk), k=shp(k, dk), v=shp(v, dv),
                   g=shp(g, dk) if w.gate == "per_channel" else shp(g),
                   beta=shp(beta), S0=S0.view(outB, outH, dv, dk))
    else:
        shp = lambda x, *tail: x.view(outB, outH, T, *tail)
        out = dict(q=shp(q, dk), k=shp(k, dk), v=shp(v, dv),
                   g=shp(g, dk) if w.gate == "per_channel" else shp(g),
                   beta=shp(beta), S0=S0.view(outB, outH, dv, dk))
    for name, (x, width) in gates2.items():
        out[name] = shp(x, width)
    if w.out == "gated":
        out["ogate"] = shp(to_dtype(field(TID_OGATE, dv, lambda tid_, full, b, h, c, t: normal(seed, tid_, full),
                                          torch.float64), w.dtype), dv)
        out["norm_w"] = (1.0 + 0.1 * normal(seed, TID_NORMW, torch.arange(dv, device=device))).to(torch.float32)
    return out


def generate_prologue(w: Workload, device="cpu", heads: Optional[Sequence[int]] = None,
                      block: int = 1 << 24) -> Dict[str, torch.Tensor]:
    """Raw inputs of the forward with its gate / normalisation prologue.

    q_raw, k_raw [B,H,T,dk] ~ N(0,1) (not normalised), v [B,H,T,dv] ~ N(0,1)
    (the same values ``generate`` draws), gate pre-activation a [B,H,T,dk]
    (per-channel) or [B,H,T] (scalar) ~ N(0,1), A_log [H] ~ U(-1,1),
    dt_bias [H,dk] (per-channel) or [H] ~ N(0, 0.5^2), beta logits [B,H,T]
    ~ N(0,1) fp32, S0 as in ``generate``.  q_raw, k_raw, v and a are in the
    workload dtype; A_log, dt_bias and the logits are fp32.  ``heads`` selects
    flat head ids (b*H + h) as in ``generate``: tensors come back as
    [len(heads), 1, ...] with the values the full tensors hold there, and
    A_log, dt_bias as [len(heads)], [len(heads), ...] (the parameters of each
    selected head, so a sample can be laid out as B = 1, H = len(heads)).
    No prologue arithmetic here: the L2 normalisation,
    softplus gate and sigmoid belong to the oracle and the kernels.
    """
    assert w.kind == "chunk"
    B, H, T, dk, dv, seed = w.B, w.H, w.T, w.dk, w.dv, w.seed
    head_ids = torch.arange(B * H, dtype=torch.int64, device=device) if heads is None else \
        torch.as_tensor(list(heads), dtype=torch.int64, device=device)
    nh = head_ids.numel()
    outB, outH = (B, H) if heads is None else (nh, 1)

    def per_head(tid, width, make):
        # element (head, t, j) of the full [B*H, T, width] tensor
        per = T * width
        out = torch.empty(nh * per, dtype=torch.float64, device=device)
        for s, e in _chunked(nh * per, block):
            lin = torch.arange(s, e, dtype=torch.int64, device=device)
            out[s:e] = make(tid, head_ids[lin // per] * per + lin % per)
        return out

    def draw(tid, n, make):
        return make(tid, torch.arange(n, dtype=torch.int64, device=device))

    nrm = lambda tid, idx: normal(seed, tid, idx)
    q_raw = to_dtype(per_head(TID_QRAW, dk, nrm), w.dtype).view(outB, outH, T, dk)
    k_raw = to_dtype(per_head(TID_KRAW, dk, nrm), w.dtype).view(outB, outH, T, dk)
    v = to_dtype(per_head(TID_V, dv, nrm), w.dtype).view(outB, outH, T, dv)
    if w.gate == "per_channel":
        a = to_dtype(per_head(TID_AGATE, dk, nrm), w.dtype).view(outB, outH, T, dk)
        dt_bias = (0.5 * draw(TID_DTBIAS, H * dk, nrm)).to(torch.float32).view(H, dk)
    else:
        a = to_dtype(per_head(TID_AGATE, 1, nrm), w.dtype).view(outB, outH, T)
        dt_bias = (0.5 * draw(TID_DTBIAS, H, nrm)).to(torch.float32)
    A_log = (2.0 * draw(TID_ALOG, H, lambda tid, idx: uniform(seed, tid, idx)) - 1.0).to(torch.float32)
    b_logit = per_head(TID_BLOGIT, 1, nrm).to(torch.float32).view(outB, outH, T)
    if heads is not None:   # per-head parameters of the selected heads
        hsel = head_ids % H
        A_log, dt_bias = A_log[hsel], dt_bias[hsel]
    S0 = generate(dataclasses.replace(w, T=1, g_recipe="softplus_n01_plus1_clamp5"), device=device,
                  heads=heads)["S0"]
    return dict(q_raw=q_raw, k_raw=k_raw, v=v, a=a, A_log=A_log, dt_bias=dt_bias, b_logit=b_logit, S0=S0)


def generate_grads(w: Workload, device="cpu", heads: Optional[Sequence[int]] = None,
                   block: int = 1 << 24) -> Dict[str, torch.Tensor]:
    """Output-side gradients for the backward pass of chunk workload ``w``:
    dO [B,H,T,dv] ~ N(0,1) in the workload dtype and dS_T [B,H,dv,dk] ~ N(0,1)
    fp32, with the same head selection rule as ``generate``."""
    assert w.kind == "chunk"
    B, H, T, dk, dv, seed = w.B, w.H, w.T, w.dk, w.dv, w.seed
    head_ids = torch.arange(B * H, dtype=torch.int64, device=device) if heads is None else \
        torch.as_tensor(list(heads), dtype=torch.int64, device=device)
    nh = head_ids.numel()
    outB, outH = (B, H) if heads is None else (nh, 1)

    def per_head(tid, per):
        out = torch.empty(nh * per, dtype=torch.float64, device=device)
        for s, e in _chunked(nh * per, block):
            lin = torch.arange(s, e, dtype=torch.int64, device=device)
            out[s:e] = normal(seed, tid, head_ids[lin // per] * per + lin % per)
        return out

    dO = to_dtype(per_head(TID_DO, T * dv), w.dtype).view(outB, outH, T, dv)
    dST = per_head(TID_DST, dv * dk).to(torch.float32).view(outB, outH, dv, dk)
    return dict(dO=dO, dS_T=dST)


def small_chunk_case(B: int, H: int, T: int, dk: int, dv: int, gate: str, dtype: torch.dtype,
                     g_recipe: str = "softplus_n01_plus1_clamp5", s0: str = "normal002",
                     seed: int = 11, C: int = 64, rule: str = "gdr", out: str = "plain") -> Workload:
    """An ad-hoc chunk workload with the same value recipes (parity tests)."""
    return Workload(f"case_B{B}H{H}T{T}d{dk}x{dv}_{gate}_{rule}_{out}", "chunk", B, H, T, dk, dv, C, gate, dtype,
                    g_recipe, s0, seed, "parity case", rule=rule, out=out)
