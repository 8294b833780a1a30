"""GPU parity of the chunked prefill (``mtla_prefill_from``): a prompt processed
as several chunks, each continuing from the cache and open slot the previous
chunk left, gives the rows, the cache and the open slot of one parallel
forward over the whole prompt (MTLA Method (1): the slot being filled is
updated in place; Sec. 4.2: the stride-aware mask splits anywhere). The
reference is the float64 oracle over the whole prompt, on the same seeded
inputs; split points fall inside blocks and on block ends."""
import numpy as np
import pytest
import torch

import oracle
from gpu_harness import TOL, Problem, np64, oracle_cfg, oracle_rows, rel_err
from kv_cache_mtla_b200 import inputs, mtla

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    torch.cuda.synchronize()
    mtla.get_device_status()
    yield
    assert mtla.get_device_status() == mtla.OK


def _run_chunks(pb, toks, bounds):
    """Chunks [bounds[i], bounds[i+1]) through mtla_prefill_from; returns all rows."""
    outs = [np64(pb.prefill_from(toks, t0, t1)) for t0, t1 in zip(bounds[:-1], bounds[1:])]
    return np.concatenate(outs, axis=1)


@pytest.mark.parametrize("s", [1, 2, 3, 4])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_chunked_prefill_tiny(s, dtype):
    """Tiny widths (CUDA-core path): chunks of 7, 23 and 31 tokens (split at 7
    and 30: inside a block for s > 1, and on a block end for s = 3), every row,
    the cache and the open slot against one oracle prefill of 61 tokens."""
    wl = inputs.TINY_FP32.with_(s=s, dtype=dtype)
    T = 61
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    ref = oracle.prefill(oracle_cfg(wl), toks["c"], toks["kr"], toks["qc"], toks["qr"],
                         w["w_uk"], w["w_uv"], w["gate_w"], w["gate_b"], toks["gate_in"])
    n_slots = (T + s - 1) // s
    pb = Problem(wl, max_slots=n_slots + 2, max_tokens=T, weights=w)
    out = _run_chunks(pb, toks, [0, 7, 30, T])
    tol = TOL[dtype]
    assert rel_err(out, ref["out"]) <= tol
    assert rel_err(np64(pb.buf.cache[:, :n_slots]), ref["cache"]) <= (tol if dtype == "fp32" else 4e-3)
    assert rel_err(np64(pb.buf.open_slot), ref["acc"]) <= 1e-5


@pytest.mark.parametrize("s", [1, 2, 3, 4])
def test_chunked_prefill_tensor_cores(s):
    """Speech-decode widths (tensor-core path): chunks of 301, 254 and 145
    tokens, so a chunk spans several 128-position query tiles, its first query
    sits inside a block (301 mod s != 0 for s > 1) and the finished slots it
    attends come from earlier chunks and from itself. Every row, the cache and
    the open slot against one oracle prefill of 700 tokens."""
    wl = inputs.SPEECH_DECODE.with_(B=2, H=3, s=s)
    T = 700
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    ref = oracle.prefill(oracle_cfg(wl), toks["c"], toks["kr"], toks["qc"], toks["qr"], w["w_uk"],
                         w["w_uv"], w["gate_w"], w["gate_b"])
    n_slots = (T + s - 1) // s
    pb = Problem(wl, max_slots=n_slots + 5, max_tokens=T, weights=w)
    out = _run_chunks(pb, toks, [0, 301, 555, T])
    assert rel_err(out, ref["out"]) <= TOL["bf16"]
    assert rel_err(np64(pb.buf.cache[:, :n_slots]), ref["cache"]) <= 4e-3
    assert rel_err(np64(pb.buf.open_slot), ref["acc"]) <= 1e-5


def test_chunked_prefill_then_decode_steps():
    """A chunked prefill leaves the state decoding continues from: 40 tokens in
    two chunks, then 9 decode steps, against the oracle over all 49 tokens."""
    wl = inputs.SPEECH_DECODE.with_(B=3, H=4, s=3)
    T0, S = 40, 9
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T0 + S)
    ref = oracle.prefill(oracle_cfg(wl), toks["c"], toks["kr"], toks["qc"], toks["qr"], w["w_uk"],
                         w["w_uv"], w["gate_w"], w["gate_b"])
    pb = Problem(wl, max_slots=(T0 + S) // 3 + 2, max_tokens=T0, weights=w)
    out = [_run_chunks(pb, toks, [0, 17, T0])]
    for k in range(S):
        out.append(np64(pb.decode(toks, T0 + k, [T0 + k] * wl.B))[:, None])
    assert rel_err(np.concatenate(out, axis=1), ref["out"]) <= TOL["bf16"]
    assert rel_err(np64(pb.buf.open_slot), ref["acc"]) <= 1e-5


def test_chunked_prefill_full_size_sampled_rows():
    """The prefill workload (B=8, T=8192, H=8, d_h=64, d_c=256, d_R=32, s=2) as
    two chunks split inside a block (4001 + 4191 tokens): every row of
    sequence 0 and 512 random rows of every other sequence, including the rows
    around each 128-position tile edge and the split, against the oracle; every
    cache slot and the open slot too."""
    wl = inputs.PREFILL
    T = wl.T
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    n_slots = T // wl.s
    pb = Problem(wl, max_slots=n_slots, max_tokens=T, weights=w)
    out = _run_chunks(pb, toks, [0, 4001, T])
    rng = np.random.default_rng(11)
    edges = sorted({t for e in (4000, 4001, 4002) for t in (e,)} |
                   {t for q in range(0, T, 128) for t in (q, q + 127) if t < T})
    rows = [(0, t) for t in range(T)]
    for b in range(1, wl.B):
        ts = set(rng.choice(T, size=512, replace=False).tolist())
        ts |= set(rng.choice(edges, size=min(64, len(edges)), replace=False).tolist()) | {4000, 4001, 4002}
        rows += [(b, t) for t in sorted(ts)]
    ref, P = oracle_rows(wl, w, toks, rows)
    got = np.stack([out[b, t] for b, t in rows])
    assert rel_err(got, ref) <= TOL["bf16"]
    idx = [min(j * wl.s + wl.s - 1, T - 1) for j in range(n_slots)]
    assert rel_err(np64(pb.buf.cache), P[:, idx]) <= 4e-3
    assert rel_err(np64(pb.buf.open_slot), P[:, T - 1]) <= 1e-5
