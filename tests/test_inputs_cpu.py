"""CPU tests of the seeded input recipe (kv_cache_mtla_b200.inputs): the five
workloads' shapes and sizes, determinism and independence of the draws, the
storage rounding, and the stated distributions (within loose statistical
bounds: a wrong scale or a missing rounding fails them, sampling noise does
not)."""
import math

import torch

from kv_cache_mtla_b200 import inputs


def _bf16_exact(x):
    return torch.equal(x, x.to(torch.bfloat16).to(torch.float32))


def test_workload_sizes():
    w = inputs.WORKLOADS
    assert set(w) == {"tiny_fp32", "speech_decode", "stride_sweep", "prefill", "large_latent"}
    tiny, speech, sweep, pre, large = (w[k] for k in ("tiny_fp32", "speech_decode", "stride_sweep",
                                                       "prefill", "large_latent"))
    assert (tiny.B, tiny.H, tiny.d_h, tiny.d_c, tiny.d_r, tiny.s, tiny.T, tiny.dtype) == \
        (1, 4, 32, 128, 16, 2, 64, "fp32")
    assert (speech.B, speech.H, speech.d_h, speech.d_c, speech.d_r, speech.s, speech.T, speech.steps) == \
        (16, 8, 64, 256, 32, 2, 1024, 256)
    assert (sweep.B, sweep.T, sweep.D) == (64, 4096, 288)
    assert (pre.B, pre.T, pre.H, pre.d_h, pre.s) == (8, 8192, 8, 64, 2)
    assert (large.B, large.H, large.d_h, large.d_c, large.d_r, large.s, large.T, large.D) == \
        (32, 128, 128, 512, 64, 4, 65536, 576)
    assert large.gate_mode == inputs.GATE_SUPPLIED
    # seed = workload index (tiny 0, the others 2..5)
    assert [x.seed for x in (tiny, speech, sweep, pre, large)] == [0, 2, 3, 4, 5]


def test_draws_are_deterministic_and_streams_independent():
    wl = inputs.SPEECH_DECODE.with_(B=2)
    a, b = inputs.tokens(wl, 5, stream=0), inputs.tokens(wl, 5, stream=0)
    for k in ("c", "kr", "qc", "qr"):
        assert torch.equal(a[k], b[k])
    c = inputs.tokens(wl, 5, stream=1)
    assert not torch.equal(a["c"], c["c"])
    assert torch.equal(inputs.weights(wl)["w_uk"], inputs.weights(wl)["w_uk"])
    assert not torch.equal(inputs.weights(wl)["w_uk"], inputs.weights(wl.with_(seed=9))["w_uk"])


def test_storage_rounding():
    """bf16 workloads draw in fp32 and round to bf16 (RN); the fp32 workload
    keeps fp32 values (not all bf16-representable)."""
    wl = inputs.SPEECH_DECODE.with_(B=2)
    t = inputs.tokens(wl, 8)
    w = inputs.weights(wl)
    for x in (t["c"], t["kr"], t["qc"], t["qr"], w["w_uk"], w["w_uv"]):
        assert _bf16_exact(x)
    assert w["gate_w"].dtype == torch.float32 and not _bf16_exact(w["gate_w"])
    tiny = inputs.tokens(inputs.TINY_FP32, 64)
    assert not _bf16_exact(tiny["c"])


def test_distributions():
    wl = inputs.SPEECH_DECODE
    t = inputs.tokens(wl, 64)
    for k in ("c", "kr", "qc", "qr"):
        x = t[k].double()
        assert abs(x.mean().item()) < 0.02 and abs(x.std().item() - 1.0) < 0.02, k
    w = inputs.weights(wl)
    for k in ("w_uk", "w_uv"):
        sd = w[k].double().std().item()
        assert abs(sd * math.sqrt(wl.d_c) - 1.0) < 0.02, k          # N(0,1)/sqrt(d_c)
    assert abs(w["gate_w"].double().std().item() - 0.02) < 0.004    # N(0, 0.02)
    assert torch.count_nonzero(w["gate_b"]) == 0
    tw = inputs.weights(inputs.TINY_FP32)
    assert abs(tw["gate_w"].double().std().item() * math.sqrt(128) - 1.0) < 0.2   # fan-in for config 1
    big = inputs.tokens(inputs.LARGE_LATENT.with_(B=4), 256)
    g = big["gate_in"]
    assert g is not None and g.shape == (4, 256) and bool(((g > 0) & (g < 1)).all())
    z = torch.log(g / (1 - g)).double()                              # back to N(0,1)
    assert abs(z.mean().item()) < 0.1 and abs(z.std().item() - 1.0) < 0.1


def test_synthetic_cache_state():
    """A cache holding n tokens has ceil(n/s) slots, zeros after them, and its
    last slot equals the rounded open-slot accumulator."""
    wl = inputs.SPEECH_DECODE.with_(B=3, s=3)
    for n in (0, 1, 3, 4, 29):
        st = inputs.synthetic_cache(wl, n, 16)
        used = (n + wl.s - 1) // wl.s
        cache, acc = st["cache"], st["acc"]
        assert cache.shape == (3, 16, wl.D) and acc.shape == (3, wl.D)
        assert torch.count_nonzero(cache[:, used:]) == 0
        if used:
            assert torch.equal(cache[:, used - 1], acc.to(torch.bfloat16).to(torch.float32))
            assert torch.count_nonzero(cache[:, :used]) > 0
