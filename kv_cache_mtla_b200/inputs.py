"""Seeded synthetic inputs for the MTLA hot path.

This module only draws random numbers with the shapes and distributions of
the workloads; it holds none of the method's arithmetic. The tests, the
benchmark and the smoke check feed the same draws to the CUDA library and to
the CPU oracle.

Values are drawn in float32 from a seeded CPU ``torch.Generator``. For bf16
(and fp16) workloads every tensor the library receives in that type is rounded
to it (round-to-nearest-even) here, so that the conversion is exact and
both sides see identical numbers. Gate parameters, supplied gates and the
fp32 open-slot accumulator stay float32.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch

GATE_COMPUTED, GATE_SUPPLIED, GATE_UNIT = 0, 1, 2
GATE_CHANNEL_COMPUTED, GATE_CHANNEL_SUPPLIED = 3, 4


@dataclass(frozen=True)
class Workload:
    """Shape and distribution recipe of one workload."""
    name: str
    B: int
    H: int
    d_h: int
    d_c: int
    d_r: int
    s: int
    dtype: str               # "bf16", "fp16" or "fp32" (storage of activations, weights, cache)
    gate_mode: int = GATE_COMPUTED
    T: int = 0               # prefill length / prefix length
    steps: int = 0           # decode steps after the prefix
    weight_std: str = "fan_in"   # W_UK, W_UV ~ N(0,1)/sqrt(d_c)
    gate_w_std: float = 0.02     # std of the gate's linear layer (fan_in: 1/sqrt(d_c))
    gate_w_fan_in: bool = False
    seed: int = 0

    @property
    def D(self) -> int:
        return self.d_c + self.d_r

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads (sizes and distributions as stated for each).
TINY_FP32 = Workload("tiny_fp32", B=1, H=4, d_h=32, d_c=128, d_r=16, s=2, dtype="fp32",
                     T=64, steps=64, gate_w_fan_in=True, seed=0)
SPEECH_DECODE = Workload("speech_decode", B=16, H=8, d_h=64, d_c=256, d_r=32, s=2,
                         dtype="bf16", T=1024, steps=256, seed=2)
STRIDE_SWEEP = Workload("stride_sweep", B=64, H=8, d_h=64, d_c=256, d_r=32, s=2,
                        dtype="bf16", T=4096, steps=1, seed=3)
PREFILL = Workload("prefill", B=8, H=8, d_h=64, d_c=256, d_r=32, s=2, dtype="bf16",
                   T=8192, steps=0, seed=4)
LARGE_LATENT = Workload("large_latent", B=32, H=128, d_h=128, d_c=512, d_r=64, s=4,
                        dtype="bf16", gate_mode=GATE_SUPPLIED, T=65536, steps=1, seed=5)

WORKLOADS = {w.name: w for w in (TINY_FP32, SPEECH_DECODE, STRIDE_SWEEP, PREFILL, LARGE_LATENT)}


def _round(x: torch.Tensor, wl: Workload) -> torch.Tensor:
    if wl.dtype == "bf16":
        return x.to(torch.bfloat16).to(torch.float32)
    if wl.dtype == "fp16":
        return x.to(torch.float16).to(torch.float32)
    return x


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def weights(wl: Workload, seed_offset: int = 0) -> dict:
    """W_UK, W_UV [H,d_h,d_c] (storage dtype values), gate_w [s,d_c], gate_b [s]
    (fp32); with the per-channel computed gate gate_w [s,d_c,D], gate_b [s,D]."""
    g = _gen(wl.seed * 1000 + 17 + seed_offset)
    std = 1.0 / (wl.d_c ** 0.5)
    w_uk = _round(torch.randn(wl.H, wl.d_h, wl.d_c, generator=g) * std, wl)
    w_uv = _round(torch.randn(wl.H, wl.d_h, wl.d_c, generator=g) * std, wl)
    gstd = (1.0 / wl.d_c ** 0.5) if wl.gate_w_fan_in else wl.gate_w_std
    if wl.gate_mode == GATE_CHANNEL_COMPUTED:
        gate_w = torch.randn(wl.s, wl.d_c, wl.D, generator=g) * gstd
        gate_b = torch.zeros(wl.s, wl.D)
    else:
        gate_w = torch.randn(wl.s, wl.d_c, generator=g) * gstd
        gate_b = torch.zeros(wl.s)
    return dict(w_uk=w_uk, w_uv=w_uv, gate_w=gate_w, gate_b=gate_b)


def tokens(wl: Workload, T: int, stream: int = 0) -> dict:
    """Per-token inputs for T tokens of every sequence.

    c [B,T,d_c], kr [B,T,d_r] (pre-RoPE), qc [B,T,H,d_h], qr [B,T,H,d_r]
    (pre-RoPE), all N(0,1) in the storage dtype; gate_in [B,T] = sigmoid(N(0,1))
    (fp32) for supplied-gate workloads ([B,T,D] for per-channel ones), else None. ``stream`` selects an
    independent draw (e.g. the prefix vs the decode steps)."""
    g = _gen(wl.seed * 1000 + 101 + 7919 * stream)
    B, H = wl.B, wl.H
    c = _round(torch.randn(B, T, wl.d_c, generator=g), wl)
    kr = _round(torch.randn(B, T, wl.d_r, generator=g), wl)
    qc = _round(torch.randn(B, T, H, wl.d_h, generator=g), wl)
    qr = _round(torch.randn(B, T, H, wl.d_r, generator=g), wl)
    gate_in = None
    if wl.gate_mode == GATE_SUPPLIED:
        gate_in = torch.sigmoid(torch.randn(B, T, generator=g))
    elif wl.gate_mode == GATE_CHANNEL_SUPPLIED:
        gate_in = torch.sigmoid(torch.randn(B, T, wl.D, generator=g))
    return dict(c=c, kr=kr, qc=qc, qr=qr, gate_in=gate_in)


def grad_out(wl: Workload, T: int, stream: int = 0) -> torch.Tensor:
    """The gradient flowing into the path's output for the training backward:
    dout [B,T,H,d_h] ~ N(0,1) in the storage dtype."""
    g = _gen(wl.seed * 1000 + 433 + 7919 * stream)
    return _round(torch.randn(wl.B, T, wl.H, wl.d_h, generator=g), wl)


def layer_weights(wl: Workload, d_model: int) -> dict:
    """The layer's projections (storage dtype values): w_dkv [d_c, dm],
    w_kr [d_R, dm], w_q [H d_h, dm], w_qr [H d_R, dm] ~ N(0,1)/sqrt(dm),
    w_o [dm, H d_h] ~ N(0,1)/sqrt(H d_h); plus the path's W_UK, W_UV and
    gate parameters from weights()."""
    g = _gen(wl.seed * 1000 + 29)
    f = d_model ** -0.5
    w = dict(w_dkv=_round(torch.randn(wl.d_c, d_model, generator=g) * f, wl),
             w_kr=_round(torch.randn(wl.d_r, d_model, generator=g) * f, wl),
             w_q=_round(torch.randn(wl.H * wl.d_h, d_model, generator=g) * f, wl),
             w_qr=_round(torch.randn(wl.H * wl.d_r, d_model, generator=g) * f, wl),
             w_o=_round(torch.randn(d_model, wl.H * wl.d_h, generator=g) * (wl.H * wl.d_h) ** -0.5, wl))
    w.update(weights(wl))
    return w


def hidden(wl: Workload, d_model: int, T: int, stream: int = 0) -> torch.Tensor:
    """Layer inputs h [B, T, d_model] ~ N(0,1) in the storage dtype."""
    g = _gen(wl.seed * 1000 + 313 + 7919 * stream)
    return _round(torch.randn(wl.B, T, d_model, generator=g), wl)


def synthetic_cache(wl: Workload, n_tokens: int, max_slots: int, stream: int = 0) -> dict:
    """A cache state that holds ``n_tokens`` tokens, drawn directly instead of
    scanned: every slot value N(0,1) in the storage dtype, the fp32 open-slot
    accumulator N(0,1) with the last used slot equal to its rounding.
    cache [B,max_slots,D] (unused slots zero), acc [B,D]."""
    g = _gen(wl.seed * 1000 + 555 + 31 * stream)
    n_used = (n_tokens + wl.s - 1) // wl.s
    cache = torch.zeros(wl.B, max_slots, wl.D)
    if n_used > 0:
        cache[:, :n_used] = _round(torch.randn(wl.B, n_used, wl.D, generator=g), wl)
    acc = torch.randn(wl.B, wl.D, generator=g)
    if n_used > 0:
        cache[:, n_used - 1] = _round(acc, wl)
    return dict(cache=cache, acc=acc)


def one_hot_mask_probe(wl: Workload, T: int) -> dict:
    """Inputs whose outputs expose the attended slot set exactly.

    Zero queries give a uniform softmax; with unit gates, token t carries the
    one-hot latent e_{floor(t/s)} only at the first token of its block and
    zeros elsewhere, so slot j holds exactly e_j and the latent output of
    query i is the mean of e_j over the slots it attends."""
    assert T <= wl.s * wl.d_c, "one-hot probe needs d_c >= number of slots"
    c = torch.zeros(wl.B, T, wl.d_c)
    for t in range(0, T, wl.s):
        c[:, t, t // wl.s] = 1.0
    kr = torch.zeros(wl.B, T, wl.d_r)
    qc = torch.zeros(wl.B, T, wl.H, wl.d_h)
    qr = torch.zeros(wl.B, T, wl.H, wl.d_r)
    return dict(c=c, kr=kr, qc=qc, qr=qr, gate_in=None)
