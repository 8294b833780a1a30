"""GPU parity with fp16 storage (MTLA_FP16: half-precision activations,
weights, cache and output, fp32 arithmetic on the CUDA cores; MTLA page, the
toolkit's attention backend taking fp16 or bf16): prefill, every decode step,
chunked prefill, the beam reorder and the training backward, against the
float64 oracle on the same fp16-valued inputs."""
import numpy as np
import pytest
import torch

import oracle
from gpu_harness import TOL, Problem, np64, oracle_cfg, rel_err
from kv_cache_mtla_b200 import inputs, mtla
from test_gpu_backward import BWD_TOL, oracle_backward, run_backward, check_all

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    torch.cuda.synchronize()
    mtla.get_device_status()
    yield
    assert mtla.get_device_status() == mtla.OK


def _oracle_prefill(wl, w, toks):
    return oracle.prefill(oracle_cfg(wl), toks["c"], toks["kr"], toks["qc"], toks["qr"], w["w_uk"],
                          w["w_uv"], w["gate_w"], w["gate_b"], toks["gate_in"])


@pytest.mark.parametrize("mode", [inputs.GATE_COMPUTED, inputs.GATE_SUPPLIED, inputs.GATE_CHANNEL_COMPUTED])
@pytest.mark.parametrize("s", [2, 3])
def test_fp16_tiny_prefill_and_decode(mode, s):
    """Tiny widths, T=37: the prefill's outputs, cache and open slot, and all 37
    decode steps, against the parallel-form oracle."""
    wl = inputs.TINY_FP32.with_(dtype="fp16", s=s, gate_mode=mode, B=2)
    T = 37
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    ref = _oracle_prefill(wl, w, toks)
    n = (T + s - 1) // s
    tol = TOL["fp16"]
    pre = Problem(wl, max_slots=n + 1, max_tokens=T, weights=w)
    assert pre.buf.cache.dtype == torch.float16
    assert rel_err(np64(pre.prefill(toks, T)), ref["out"]) <= tol
    assert rel_err(np64(pre.buf.cache[:, :n]), ref["cache"]) <= tol
    assert rel_err(np64(pre.buf.open_slot), ref["acc"]) <= 1e-5
    dec = Problem(wl, max_slots=n + 1, weights=w)
    out = np.stack([np64(dec.decode(toks, t, [t] * wl.B)) for t in range(T)], axis=1)
    assert rel_err(out, ref["out"]) <= tol
    assert rel_err(np64(dec.buf.cache[:, :n]), ref["cache"]) <= tol
    assert rel_err(np64(dec.buf.open_slot), ref["acc"]) <= 1e-5


def test_fp16_speech_widths_chunked_then_decode():
    """Speech widths (H=8, d_h=64, d_c=256, d_R=32, s=3): a 200-token prompt as
    two chunks (the second starting inside a block), then 8 decode steps; every
    row against the oracle."""
    wl = inputs.SPEECH_DECODE.with_(dtype="fp16", B=2, s=3)
    T, S = 200, 8
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T + S)
    ref = _oracle_prefill(wl, w, toks)
    pb = Problem(wl, max_slots=(T + S) // 3 + 2, max_tokens=T, weights=w)
    o1 = np64(pb.prefill_from(toks, 0, 121))
    o2 = np64(pb.prefill_from(toks, 121, T))
    dec = np.stack([np64(pb.decode(toks, T + k, [T + k] * wl.B)) for k in range(S)], axis=1)
    got = np.concatenate([o1, o2, dec], axis=1)
    assert rel_err(got, ref["out"]) <= TOL["fp16"]
    assert rel_err(np64(pb.buf.open_slot), ref["acc"]) <= 1e-5


def test_fp16_reorder_is_a_byte_copy():
    """The beam reorder on an fp16 cache copies 2-byte values exactly."""
    wl = inputs.TINY_FP32.with_(dtype="fp16", B=3, s=2)
    T = 20
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    pb = Problem(wl, max_slots=12, max_tokens=T, weights=w)
    pb.prefill(toks, T)
    cache_out = torch.zeros_like(pb.buf.cache)
    open_out = torch.zeros_like(pb.buf.open_slot)
    src = torch.tensor([2, 0, 2], dtype=torch.int32, device="cuda")
    n_tok = torch.tensor([T, T, T], dtype=torch.int32, device="cuda")
    mtla.reorder_cache(pb.cfg, src, n_tok, pb.buf.cache, pb.buf.open_slot, cache_out, open_out)
    torch.cuda.synchronize()
    for b, j in enumerate((2, 0, 2)):
        assert torch.equal(cache_out[b, :T // 2], pb.buf.cache[j, :T // 2])
        assert torch.equal(open_out[b], pb.buf.open_slot[j])


@pytest.mark.parametrize("mode", [inputs.GATE_COMPUTED, inputs.GATE_SUPPLIED])
def test_fp16_backward(mode):
    """The training backward from fp16 inputs (fp32 arithmetic, the CUDA-core
    path): every gradient within the fp32 bound of the oracle's backward."""
    wl = inputs.PREFILL.with_(dtype="fp16", B=2, s=3, gate_mode=mode)
    T = 130
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    dout = inputs.grad_out(wl, T)
    check_all(wl, run_backward(wl, T, w, toks, dout), oracle_backward(wl, w, toks, dout), tol=BWD_TOL)


@pytest.mark.parametrize("s", [1, 2, 4])
def test_fp16_tensor_cores_prefill_and_decode(s):
    """fp16 storage at the tensor-core widths (H=8, d_h=64, d_c=256, d_R=32):
    the tensor-core prefill over 300 tokens (three 128-position tiles and a
    ragged tail), then 12 decode steps on the small-head tensor-core decode;
    every row, the cache and the open slot against the oracle."""
    wl = inputs.SPEECH_DECODE.with_(dtype="fp16", B=3, s=s)
    T, S = 300, 12
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T + S)
    ref = _oracle_prefill(wl, w, toks)
    n = (T + S + s - 1) // s
    pb = Problem(wl, max_slots=n + 1, max_tokens=T, weights=w)
    assert pb.buf.cache.dtype == torch.float16
    o1 = np64(pb.prefill(toks, T))
    dec = np.stack([np64(pb.decode(toks, T + k, [T + k] * wl.B)) for k in range(S)], axis=1)
    assert rel_err(np.concatenate([o1, dec], axis=1), ref["out"]) <= TOL["fp16"]
    assert rel_err(np64(pb.buf.cache[:, :n]), ref["cache"]) <= TOL["fp16"]
    assert rel_err(np64(pb.buf.open_slot), ref["acc"]) <= 1e-5


def test_fp16_large_heads_cluster_decode():
    """fp16 storage at the large-latent widths (H=128, d_h=128, d_c=512,
    d_R=64, s=4, supplied gates): the 2-CTA cluster decode over a prompt of 90
    tokens (CUDA-core prefill at these widths) and 6 steps, against the
    oracle."""
    wl = inputs.LARGE_LATENT.with_(dtype="fp16", B=2)
    T, S = 90, 6
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T + S)
    ref = _oracle_prefill(wl, w, toks)
    n = (T + S + wl.s - 1) // wl.s
    pb = Problem(wl, max_slots=n + 2, max_tokens=T, weights=w)
    o1 = np64(pb.prefill(toks, T))
    dec = np.stack([np64(pb.decode(toks, T + k, [T + k] * wl.B)) for k in range(S)], axis=1)
    assert rel_err(np.concatenate([o1, dec], axis=1), ref["out"]) <= TOL["fp16"]
    assert rel_err(np64(pb.buf.open_slot), ref["acc"]) <= 1e-5
