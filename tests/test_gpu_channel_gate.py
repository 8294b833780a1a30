"""GPU parity of the per-channel merging gate (gate modes 3 and 4: one weight
per slot channel, the reading of W_t (.) x_t with W_t a vector; MTLA paper
summary page, Method (1), Sec. 4.1 Eq. 13) on every path: the CUDA-core
kernels (fp32 at 1e-5 and bf16), the small-head tensor-core decode and prefill,
the large-head cluster decode, and the chunked prefill. Reference: the float64
oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from gpu_harness import TOL, Problem, np64, oracle_cfg, rel_err
from kv_cache_mtla_b200 import inputs, mtla

pytestmark = pytest.mark.gpu
MODES = [inputs.GATE_CHANNEL_COMPUTED, inputs.GATE_CHANNEL_SUPPLIED]


@pytest.fixture(autouse=True)
def _clean_status():
    torch.cuda.synchronize()
    mtla.get_device_status()
    yield
    assert mtla.get_device_status() == mtla.OK


def _oracle_prefill(wl, w, toks):
    return oracle.prefill(oracle_cfg(wl), toks["c"], toks["kr"], toks["qc"], toks["qr"], w["w_uk"],
                          w["w_uv"], w["gate_w"], w["gate_b"], toks["gate_in"])


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("s", [2, 3])
def test_channel_gate_tiny(mode, dtype, s):
    """Tiny widths (CUDA-core kernels): prefill of 37 tokens and 37 decode steps
    against the oracle; cache and open slot too."""
    wl = inputs.TINY_FP32.with_(s=s, dtype=dtype, gate_mode=mode)
    T = 37
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    ref = _oracle_prefill(wl, w, toks)
    n = (T + s - 1) // s
    tol = TOL[dtype]
    pre = Problem(wl, max_slots=n + 1, max_tokens=T, weights=w)
    assert rel_err(np64(pre.prefill(toks, T)), ref["out"]) <= tol
    assert rel_err(np64(pre.buf.open_slot), ref["acc"]) <= 1e-5
    dec = Problem(wl, max_slots=n + 1, weights=w)
    out = np.stack([np64(dec.decode(toks, t, [t] * wl.B)) for t in range(T)], axis=1)
    assert rel_err(out, ref["out"]) <= tol
    assert rel_err(np64(dec.buf.cache[:, :n]), ref["cache"]) <= (tol if dtype == "fp32" else 4e-3)
    assert rel_err(np64(dec.buf.open_slot), ref["acc"]) <= 1e-5


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("s", [1, 2, 4])
def test_channel_gate_tensor_cores(mode, s):
    """Speech-decode widths (d_h=64, d_c=256, d_R=32; tensor-core prefill and
    small-head decode): a 200-token prompt as two chunks (the second starting
    inside a block), then 12 decode steps; every row against the oracle over
    all 212 tokens, and the open slot."""
    wl = inputs.SPEECH_DECODE.with_(B=3, H=8, s=s, gate_mode=mode)
    T0, S = 200, 12
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T0 + S)
    ref = _oracle_prefill(wl, w, toks)
    pb = Problem(wl, max_slots=(T0 + S) // s + 2, max_tokens=T0, weights=w)
    outs = [np64(pb.prefill_from(toks, 0, 77)), np64(pb.prefill_from(toks, 77, T0))]
    for k in range(S):
        outs.append(np64(pb.decode(toks, T0 + k, [T0 + k] * wl.B))[:, None])
    assert rel_err(np.concatenate(outs, axis=1), ref["out"]) <= TOL["bf16"]
    assert rel_err(np64(pb.buf.open_slot), ref["acc"]) <= 1e-5


@pytest.mark.parametrize("mode", MODES)
def test_channel_gate_large_heads(mode):
    """Large-latent widths (H=64, d_h=128, d_c=512, d_R=64, s=4; the two-CTA
    cluster decode): one step at mixed positions over a drawn cache, against
    the oracle's incremental step; the slot row written and the open slot."""
    wl = inputs.LARGE_LATENT.with_(B=6, H=64, gate_mode=mode)
    max_slots = 700
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, 1, stream=1)
    cache0 = inputs.synthetic_cache(wl, max_slots * wl.s - 1, max_slots)
    pos = np.array([0, 3, 4, 1001, 2047, max_slots * wl.s - 1])
    pb = Problem(wl, max_slots=max_slots, weights=w)
    pb.buf.cache.copy_(cache0["cache"].to(pb.dt))
    pb.buf.open_slot.copy_(cache0["acc"])
    out = np64(pb.decode(toks, 0, pos))
    cache_o = cache0["cache"].double().numpy().copy()
    acc_o = cache0["acc"].double().numpy().copy()
    gin = toks["gate_in"]
    ref = oracle.decode_step(oracle_cfg(wl), toks["c"][:, 0], toks["kr"][:, 0], toks["qc"][:, 0], toks["qr"][:, 0],
                             w["w_uk"], w["w_uv"], pos, cache_o, acc_o, w["gate_w"], w["gate_b"],
                             None if gin is None else gin[:, 0])
    assert rel_err(out, ref["out"]) <= TOL["bf16"]
    for b in range(wl.B):
        j = pos[b] // wl.s
        assert rel_err(np64(pb.buf.cache[b, j]), cache_o[b, j]) <= 4e-3
    assert rel_err(np64(pb.buf.open_slot), acc_o) <= 1e-5
