"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
the same seeded inputs. Tolerances: max|gpu - ref| / max|ref| <= 2e-2 for bf16
storage with fp32 accumulation, <= 1e-5 for the fp32 path; slot contents and
the attended slot set exactly where the arithmetic is exact."""
import numpy as np
import pytest
import torch

import oracle
from gpu_harness import TOL, Problem, concat_tokens, elem_err, np64, oracle_cfg, oracle_rows, rel_err
from kv_cache_mtla_b200 import inputs, mtla

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    torch.cuda.synchronize()
    mtla.get_device_status()
    yield
    assert mtla.get_device_status() == mtla.OK


def _slots_from_P(P, T, s):
    n = (T + s - 1) // s
    idx = [min(j * s + s - 1, T - 1) for j in range(n)]
    return P[:, idx]


# ----------------------------------------------------------------- tiny fp32 (1e-5)

def test_tiny_fp32_workload_as_stated():
    """The tiny fp32 workload exactly as stated: B=1, H=4, d_h=32, d_c=128,
    d_R=16, s=2, T=64, inputs N(0,1), weights N(0,1)/sqrt(fan_in), sinusoidal
    PE, seed 0. All 64 decode steps, the parallel masked prefill and the oracle
    agree to 1e-5, and so do the cache and the open slot."""
    wl = inputs.TINY_FP32
    assert (wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, wl.T, wl.dtype, wl.seed) == (1, 4, 32, 128, 16, 2, 64, "fp32", 0)
    T = wl.T
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    ref = oracle.prefill(oracle_cfg(wl), toks["c"], toks["kr"], toks["qc"], toks["qr"],
                         w["w_uk"], w["w_uv"], w["gate_w"], w["gate_b"], toks["gate_in"])
    pre = Problem(wl, max_slots=T // 2, max_tokens=T, weights=w)
    out_p = np64(pre.prefill(toks, T))
    dec = Problem(wl, max_slots=T // 2, weights=w)
    out_d = np.stack([np64(dec.decode(toks, t, [t])) for t in range(T)], axis=1)
    for got in (out_p, out_d):
        assert rel_err(got, ref["out"]) <= 1e-5
        # elementwise, with the floor 1e-3 max|ref| for entries near zero
        assert elem_err(got, ref["out"]) <= 1e-3
    assert rel_err(out_d, out_p) <= 1e-5
    for pb in (pre, dec):
        assert rel_err(np64(pb.buf.cache), ref["cache"]) <= 1e-5
        assert rel_err(np64(pb.buf.open_slot), ref["acc"]) <= 1e-5


@pytest.mark.parametrize("s", [1, 2, 3, 4])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_tiny_prefill_and_decode(s, dtype):
    """Prefill of T tokens and T decode steps from an empty cache both match the
    oracle; decode equals prefill (the stride-aware mask reproduces incremental
    decoding); the cache and the open slot match. T = 61 leaves a ragged tail."""
    wl = inputs.TINY_FP32.with_(s=s, dtype=dtype)
    T = 61 if s > 1 else 64
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    ref = oracle.prefill(oracle_cfg(wl), toks["c"], toks["kr"], toks["qc"], toks["qr"],
                         w["w_uk"], w["w_uv"], w["gate_w"], w["gate_b"], toks["gate_in"])
    n_slots = (T + s - 1) // s
    tol = TOL[dtype]

    pre = Problem(wl, max_slots=n_slots + 1, max_tokens=T, weights=w)
    out_p = np64(pre.prefill(toks, T))
    assert rel_err(out_p, ref["out"]) <= tol
    assert rel_err(np64(pre.buf.cache[:, :n_slots]), ref["cache"]) <= (tol if dtype == "fp32" else 4e-3)
    assert rel_err(np64(pre.buf.open_slot), ref["acc"]) <= 1e-5

    dec = Problem(wl, max_slots=n_slots + 1, weights=w)
    outs = []
    for t in range(T):
        outs.append(np64(dec.decode(toks, t, [t] * wl.B)))
    out_d = np.stack(outs, axis=1)
    assert rel_err(out_d, ref["out"]) <= tol
    assert rel_err(out_d, out_p) <= tol
    assert rel_err(np64(dec.buf.cache[:, :n_slots]), ref["cache"]) <= (tol if dtype == "fp32" else 4e-3)
    assert rel_err(np64(dec.buf.open_slot), ref["acc"]) <= 1e-5


@pytest.mark.parametrize("s", [1, 2, 3, 4])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_mask_set_bit_exact(s, dtype):
    """One-hot probe: zero queries and unit gates, W_UV = [I | 0]. Output entry j
    of query t is nonzero exactly when slot j is attended, so the attended set
    must equal {0..floor(t/s)} bit for bit, with weight 1/(floor(t/s)+1)."""
    wl = inputs.TINY_FP32.with_(s=s, dtype=dtype, gate_mode=inputs.GATE_UNIT)
    T = min(wl.s * wl.d_h, 61)
    toks = inputs.one_hot_mask_probe(wl, T)
    w = inputs.weights(wl)
    eye = torch.zeros(wl.H, wl.d_h, wl.d_c)
    eye[:, torch.arange(wl.d_h), torch.arange(wl.d_h)] = 1.0
    w = dict(w, w_uv=eye, w_uk=torch.zeros_like(eye))
    n_slots = (T + s - 1) // s
    for mode in ("prefill", "decode"):
        pb = Problem(wl, max_slots=n_slots, max_tokens=T, weights=w)
        if mode == "prefill":
            out = np64(pb.prefill(toks, T))[0]
        else:
            out = np.stack([np64(pb.decode(toks, t, [t]))[0] for t in range(T)])
        for t in range(T):
            for h in range(wl.H):
                support = np.nonzero(out[t, h])[0].tolist()
                assert support == list(range(t // s + 1)), (mode, t, h)
                np.testing.assert_allclose(out[t, h, : t // s + 1], 1.0 / (t // s + 1),
                                           rtol=TOL[dtype] if dtype == "fp32" else 4e-3)


# ----------------------------------------------------------------- speech decode

def test_speech_decode_prefix_then_steps():
    """B=16, H=8, d_h=64, d_c=256, d_R=32, s=2: prefill a 1024-token prefix,
    then 256 decode steps; sampled prefill rows and every 16th decode step (all
    sequences) against the oracle's parallel form over the whole 1280-token
    stream."""
    wl = inputs.SPEECH_DECODE
    T, S = wl.T, wl.steps
    w = inputs.weights(wl)
    pre_t = inputs.tokens(wl, T, stream=0)
    dec_t = inputs.tokens(wl, S, stream=1)
    max_slots = (T + S + wl.s - 1) // wl.s
    pb = Problem(wl, max_slots=max_slots, max_tokens=T, weights=w)
    out_p = np64(pb.prefill(pre_t, T))
    outs = {}
    keep = set(range(0, S, 16)) | {1, 2, 3, 127, 254, 255}
    for k in range(S):
        o = pb.decode(dec_t, k, [T + k] * wl.B)
        if k in keep:
            outs[k] = np64(o)
    allt = concat_tokens(pre_t, dec_t)
    rows_p = [(b, t) for b in (0, 7, 15) for t in (0, 1, 2, 511, 512, 1022, 1023)]
    rows_d = [(b, T + k) for b in range(wl.B) for k in sorted(keep)]
    ref, P = oracle_rows(wl, w, allt, rows_p + rows_d)
    ref_p = ref[: len(rows_p)]
    got_p = np.stack([out_p[b, t] for b, t in rows_p])
    assert rel_err(got_p, ref_p) <= TOL["bf16"]
    ref_d = ref[len(rows_p):]
    got_d = np.stack([outs[t - T][b] for b, t in rows_d])
    assert rel_err(got_d, ref_d) <= TOL["bf16"]
    slots = _slots_from_P(P, T + S, wl.s)
    assert rel_err(np64(pb.buf.cache), slots) <= 4e-3
    assert rel_err(np64(pb.buf.open_slot), P[:, T + S - 1]) <= 1e-5


# ----------------------------------------------------------------- stride sweep

@pytest.mark.parametrize("s", [1, 2, 3, 4])
def test_stride_sweep_decode(s):
    """B=64, N=4096 tokens after the step (s=3 leaves a one-token last slot):
    synthetic cache of N-1 tokens, one decode step at pos = N-1, compared with
    the oracle's incremental step on sampled sequences; plus mixed positions."""
    wl = inputs.STRIDE_SWEEP.with_(s=s)
    N = wl.T
    max_slots = (N + s - 1) // s
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, 1, stream=1)
    cache0 = inputs.synthetic_cache(wl, N - 1, max_slots)
    for variant in ("uniform", "mixed"):
        if variant == "uniform":
            pos = np.full(wl.B, N - 1)
        else:
            pos = np.array([(N - 1 - 61 * b) % N for b in range(wl.B)])
            pos[5] = 0
            pos[6] = s - 1
        pb = Problem(wl, max_slots=max_slots, weights=w)
        pb.buf.cache.copy_(cache0["cache"].to(pb.dt))
        pb.buf.open_slot.copy_(cache0["acc"])
        out = np64(pb.decode(toks, 0, pos))
        sample = [0, 5, 6, 31, 63]
        sub = lambda x: None if x is None else x[sample]
        cfg = oracle_cfg(wl, B=len(sample))
        cache_o = cache0["cache"][sample].double().numpy().copy()
        acc_o = cache0["acc"][sample].double().numpy().copy()
        ref = oracle.decode_step(cfg, sub(toks["c"][:, 0]), sub(toks["kr"][:, 0]),
                                 sub(toks["qc"][:, 0]), sub(toks["qr"][:, 0]), w["w_uk"],
                                 w["w_uv"], pos[sample], cache_o, acc_o, w["gate_w"], w["gate_b"])
        assert rel_err(out[sample], ref["out"]) <= TOL["bf16"], variant
        for i, b in enumerate(sample):
            j = pos[b] // s
            assert rel_err(np64(pb.buf.cache[b, j]), cache_o[i, j]) <= 4e-3
        assert rel_err(np64(pb.buf.open_slot[sample]), acc_o) <= 1e-5


# ----------------------------------------------------------------- prefill

def test_prefill_full_size_sampled_rows():
    """B=8, T=8192, H=8, d_h=64, d_c=256, d_R=32, s=2: the whole prefill on the
    GPU; every row of sequence 0 and 512 random rows of every other sequence,
    plus, in each 128-position query tile, its first and last rows and a block
    start and end (t = 0 and s-1 mod s); all cache slots and the open slot
    against the oracle."""
    wl = inputs.PREFILL
    T = wl.T
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    n_slots = T // wl.s
    pb = Problem(wl, max_slots=n_slots, max_tokens=T, weights=w)
    out = np64(pb.prefill(toks, T))
    rng = np.random.default_rng(8)
    rows = [(0, t) for t in range(T)]
    for b in range(1, wl.B):
        ts = set(rng.choice(T, size=512, replace=False).tolist())
        for q in range(0, T, 128):
            ts |= {q, q + 127, q + 2 * int(rng.integers(0, 64)), q + 2 * int(rng.integers(0, 64)) + 1}
        rows += [(b, t) for t in sorted(ts)]
    ref, P = oracle_rows(wl, w, toks, rows)
    got = np.stack([out[b, t] for b, t in rows])
    assert rel_err(got, ref) <= TOL["bf16"]
    assert rel_err(np64(pb.buf.cache), _slots_from_P(P, T, wl.s)) <= 4e-3
    assert rel_err(np64(pb.buf.open_slot), P[:, T - 1]) <= 1e-5


# ----------------------------------------------------------------- large latent

def test_large_latent_decode():
    """B=32, H=128, d_c=512, d_R=64 (absorbed width 576), s=4, N=65536 tokens
    after the step (16384 slots per sequence), supplied gates sigmoid(N(0,1)):
    one decode step at pos = N-1 on a synthetic cache; every head of every
    sequence against the oracle's incremental step."""
    wl = inputs.LARGE_LATENT
    N = wl.T
    max_slots = N // wl.s
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, 1, stream=1)
    cache0 = inputs.synthetic_cache(wl, N - 1, max_slots)
    pb = Problem(wl, max_slots=max_slots, weights=w)
    pb.buf.cache.copy_(cache0["cache"].to(pb.dt))
    pb.buf.open_slot.copy_(cache0["acc"])
    pos = np.full(wl.B, N - 1)
    out = np64(pb.decode(toks, 0, pos))
    # every sequence, in groups of 8 (the oracle's float64 cache of a group is 600 MB)
    j = (N - 1) // wl.s
    for g0 in range(0, wl.B, 8):
        sample = list(range(g0, min(g0 + 8, wl.B)))
        sub = lambda x: x[sample]
        cfg = oracle_cfg(wl, B=len(sample))
        cache_o = cache0["cache"][sample].double().numpy().copy()
        acc_o = cache0["acc"][sample].double().numpy().copy()
        ref = oracle.decode_step(cfg, sub(toks["c"][:, 0]), sub(toks["kr"][:, 0]), sub(toks["qc"][:, 0]),
                                 sub(toks["qr"][:, 0]), w["w_uk"], w["w_uv"], pos[sample], cache_o, acc_o,
                                 gate_in=sub(toks["gate_in"][:, 0]))
        assert rel_err(out[sample], ref["out"]) <= TOL["bf16"], sample
        assert rel_err(np64(pb.buf.cache[sample, j]), cache_o[:, j]) <= 4e-3
        assert rel_err(np64(pb.buf.open_slot[sample]), acc_o) <= 1e-5
        del cache_o


# ----------------------------------------------------------------- device-side errors

def test_position_beyond_cache_latches_capacity():
    """pos >= max_slots*s skips that sequence (its output untouched) and latches
    CAPACITY; the other sequences are still computed correctly."""
    wl = inputs.TINY_FP32.with_(B=3)
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, 1)
    pb = Problem(wl, max_slots=4, weights=w)
    out = torch.full((wl.B, wl.H, wl.d_h), 7.0, device="cuda")
    pos = torch.tensor([0, 8, 0], dtype=torch.int32, device="cuda")  # 8 >= 4*2
    gw, gb = pb.gate_ptrs()
    from gpu_harness import dev
    mtla.decode_step(pb.cfg, dev(toks["c"][:, 0], pb.dt), dev(toks["kr"][:, 0], pb.dt),
                     dev(toks["qc"][:, 0], pb.dt), dev(toks["qr"][:, 0], pb.dt), pb.buf.w_uk,
                     pb.buf.w_uv, gw, gb, None, pos, pb.buf.cache, pb.buf.open_slot, out,
                     pb.buf.workspace)
    assert mtla.get_device_status() == mtla.ERR_CAPACITY
    assert torch.all(out[1] == 7.0)
    assert not torch.any(out[0] == 7.0)
    assert mtla.get_device_status() == mtla.OK   # cleared by the read


# ----------------------------------------------------------------- decode schedule / head widths

@pytest.mark.parametrize("H", [1, 8, 20, 32])
def test_decode_many_short_sequences(H):
    """Many sequences of 1 to ~5 slot tiles with mixed positions: the split
    plan crosses sequence boundaries inside one CTA's range. Head counts cover
    both padded head widths of the tensor-core kernel."""
    wl = inputs.SPEECH_DECODE.with_(B=150, H=H, s=3)
    max_slots = 700
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, 1, stream=1)
    cache0 = inputs.synthetic_cache(wl, max_slots * wl.s - 1, max_slots)
    rng = np.random.default_rng(H)
    pos = rng.integers(0, max_slots * wl.s, size=wl.B)
    pos[:3] = [0, 1, max_slots * wl.s - 1]
    pb = Problem(wl, max_slots=max_slots, weights=w)
    pb.buf.cache.copy_(cache0["cache"].to(pb.dt))
    pb.buf.open_slot.copy_(cache0["acc"])
    out = np64(pb.decode(toks, 0, pos))
    sample = [0, 1, 2, 17, 74, 75, 76, 148, 149]
    sub = lambda x: x[sample]
    cfg = oracle_cfg(wl, B=len(sample))
    cache_o = cache0["cache"][sample].double().numpy().copy()
    acc_o = cache0["acc"][sample].double().numpy().copy()
    ref = oracle.decode_step(cfg, sub(toks["c"][:, 0]), sub(toks["kr"][:, 0]), sub(toks["qc"][:, 0]),
                             sub(toks["qr"][:, 0]), w["w_uk"], w["w_uv"], pos[sample], cache_o,
                             acc_o, w["gate_w"], w["gate_b"])
    assert rel_err(out[sample], ref["out"]) <= TOL["bf16"]


@pytest.mark.parametrize("H,d_c,d_r,B", [(12, 256, 32, 24), (16, 128, 32, 30), (3, 256, 32, 40),
                                          (8, 256, 64, 20), (8, 128, 16, 20)])
def test_small_head_decode_ring_layouts(H, d_c, d_r, B):
    """Both slot-tile layouts of the small-head tensor-core kernel: the compact
    three-stage ring (32 RoPE columns in 64-byte rows, P^T over them; 8 and 16
    padded heads, d_c 128 and 256) and the padded two-stage ring (RoPE widths
    64 and 16). Up to 32 tiles per sequence, so CTAs take several tiles and
    their ranges cross sequences."""
    wl = inputs.SPEECH_DECODE.with_(B=B, H=H, d_c=d_c, d_r=d_r, s=2)
    max_slots = 4096
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, 1, stream=3)
    cache0 = inputs.synthetic_cache(wl, max_slots * wl.s - 1, max_slots)
    rng = np.random.default_rng(1000 + H + d_c + d_r)
    pos = rng.integers(0, max_slots * wl.s, size=wl.B)
    pos[:3] = [0, 255, max_slots * wl.s - 1]       # one slot; a whole tile (128 slots); full cache
    pb = Problem(wl, max_slots=max_slots, weights=w)
    pb.buf.cache.copy_(cache0["cache"].to(pb.dt))
    pb.buf.open_slot.copy_(cache0["acc"])
    out = np64(pb.decode(toks, 0, pos))
    cfg = oracle_cfg(wl)
    cache_o = cache0["cache"].double().numpy().copy()
    acc_o = cache0["acc"].double().numpy().copy()
    ref = oracle.decode_step(cfg, toks["c"][:, 0], toks["kr"][:, 0], toks["qc"][:, 0], toks["qr"][:, 0],
                             w["w_uk"], w["w_uv"], pos, cache_o, acc_o, w["gate_w"], w["gate_b"])
    assert rel_err(out, ref["out"]) <= TOL["bf16"]


def test_decode_skips_invalid_sequences_in_the_split_plan():
    """Sequences whose position is beyond the cache get no tiles; the others
    around them are still right, and CAPACITY is latched."""
    wl = inputs.SPEECH_DECODE.with_(B=40)
    max_slots = 300
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, 1, stream=1)
    cache0 = inputs.synthetic_cache(wl, 500, max_slots)
    pos = np.array([(37 * b) % 590 for b in range(wl.B)])
    bad = [3, 4, 20, 39]
    pos[bad] = max_slots * wl.s + 5
    pb = Problem(wl, max_slots=max_slots, weights=w)
    pb.buf.cache.copy_(cache0["cache"].to(pb.dt))
    pb.buf.open_slot.copy_(cache0["acc"])
    out = np64(pb.decode(toks, 0, pos))
    assert mtla.get_device_status() == mtla.ERR_CAPACITY
    good = [b for b in range(wl.B) if b not in bad]
    sub = lambda x: x[good]
    cfg = oracle_cfg(wl, B=len(good))
    cache_o = cache0["cache"][good].double().numpy().copy()
    acc_o = cache0["acc"][good].double().numpy().copy()
    ref = oracle.decode_step(cfg, sub(toks["c"][:, 0]), sub(toks["kr"][:, 0]), sub(toks["qc"][:, 0]),
                             sub(toks["qr"][:, 0]), w["w_uk"], w["w_uv"], pos[good], cache_o, acc_o,
                             w["gate_w"], w["gate_b"])
    assert rel_err(out[good], ref["out"]) <= TOL["bf16"]


# ----------------------------------------------------------------- tensor-core prefill edges

@pytest.mark.parametrize("s", [1, 2, 3, 4])
@pytest.mark.parametrize("T", [1, 63, 129, 300])
def test_prefill_ragged_lengths(s, T):
    """Speech-decode widths (d_h=64, d_c=256, d_R=32), lengths around the
    128-position query tiles and 128-slot key tiles, every row against the
    oracle; the cache and open slot too."""
    wl = inputs.SPEECH_DECODE.with_(B=2, H=3, s=s)
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    ref = oracle.prefill(oracle_cfg(wl), toks["c"], toks["kr"], toks["qc"], toks["qr"], w["w_uk"],
                         w["w_uv"], w["gate_w"], w["gate_b"])
    n_slots = (T + s - 1) // s
    pb = Problem(wl, max_slots=n_slots + 3, max_tokens=T, weights=w)
    out = np64(pb.prefill(toks, T))
    assert rel_err(out, ref["out"]) <= TOL["bf16"]
    assert rel_err(np64(pb.buf.cache[:, :n_slots]), ref["cache"]) <= 4e-3
    assert rel_err(np64(pb.buf.open_slot), ref["acc"]) <= 1e-5


@pytest.mark.parametrize("d_c, s, T, B, H", [(256, 2, 2500, 2, 8), (128, 2, 1100, 2, 10), (128, 3, 300, 1, 3)])
def test_prefill_many_items_per_cta(d_c, s, T, B, H):
    """More work items (128 positions x sequence x head) than SMs, so every
    persistent CTA walks several items and the ring, the query region and the
    TMEM columns pass from one item to the next; both compiled widths
    (d_c = 256 and 128, d_h = 64, d_R = 32). Every row against the oracle."""
    wl = inputs.SPEECH_DECODE.with_(B=B, H=H, s=s, d_c=d_c)
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    ref = oracle.prefill(oracle_cfg(wl), toks["c"], toks["kr"], toks["qc"], toks["qr"], w["w_uk"],
                         w["w_uv"], w["gate_w"], w["gate_b"])
    n_slots = (T + s - 1) // s
    pb = Problem(wl, max_slots=n_slots + 1, max_tokens=T, weights=w)
    out = np64(pb.prefill(toks, T))
    assert rel_err(out, ref["out"]) <= TOL["bf16"]
    assert rel_err(np64(pb.buf.cache[:, :n_slots]), ref["cache"]) <= 4e-3


@pytest.mark.parametrize("s", [1, 2, 3, 4])
def test_mask_set_bit_exact_speech_widths(s):
    """The one-hot mask probe at the speech-decode widths, where both the
    decode and the prefill run on the tensor-core kernels."""
    wl = inputs.SPEECH_DECODE.with_(B=1, H=2, s=s, gate_mode=inputs.GATE_UNIT)
    T = min(wl.s * wl.d_h, 150)
    toks = inputs.one_hot_mask_probe(wl, T)
    w = inputs.weights(wl)
    eye = torch.zeros(wl.H, wl.d_h, wl.d_c)
    eye[:, torch.arange(wl.d_h), torch.arange(wl.d_h)] = 1.0
    w = dict(w, w_uv=eye, w_uk=torch.zeros_like(eye))
    n_slots = (T + s - 1) // s
    for mode in ("prefill", "decode"):
        pb = Problem(wl, max_slots=n_slots, max_tokens=T, weights=w)
        if mode == "prefill":
            out = np64(pb.prefill(toks, T))[0]
        else:
            out = np.stack([np64(pb.decode(toks, t, [t]))[0] for t in range(T)])
        for t in range(T):
            for h in range(wl.H):
                support = np.nonzero(out[t, h])[0].tolist()
                assert support == list(range(t // s + 1)), (mode, t, h)
                np.testing.assert_allclose(out[t, h, : t // s + 1], 1.0 / (t // s + 1), rtol=4e-3)


# ----------------------------------------------------------------- many heads (cluster kernel)

@pytest.mark.parametrize("H,s", [(33, 4), (64, 1), (128, 4), (128, 3)])
def test_decode_many_heads(H, s):
    """Large-latent widths (d_h=128, d_c=512, d_R=64) with 32 < H <= 128: the
    decode runs on the two-CTA cluster kernel. Mixed positions put several
    sequences in one cluster's range and one sequence across clusters."""
    wl = inputs.LARGE_LATENT.with_(B=12, H=H, s=s)
    max_slots = 1500
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, 1, stream=1)
    cache0 = inputs.synthetic_cache(wl, max_slots * s - 1, max_slots)
    rng = np.random.default_rng(H + s)
    pos = rng.integers(0, max_slots * s, size=wl.B)
    pos[:4] = [0, s - 1, 63 * s, max_slots * s - 1]
    pb = Problem(wl, max_slots=max_slots, weights=w)
    pb.buf.cache.copy_(cache0["cache"].to(pb.dt))
    pb.buf.open_slot.copy_(cache0["acc"])
    out = np64(pb.decode(toks, 0, pos))
    cfg = oracle_cfg(wl)
    cache_o = cache0["cache"].double().numpy().copy()
    acc_o = cache0["acc"].double().numpy().copy()
    ref = oracle.decode_step(cfg, toks["c"][:, 0], toks["kr"][:, 0], toks["qc"][:, 0], toks["qr"][:, 0],
                             w["w_uk"], w["w_uv"], pos, cache_o, acc_o, gate_in=toks["gate_in"][:, 0])
    assert rel_err(out, ref["out"]) <= TOL["bf16"]
    for b in range(wl.B):
        j = pos[b] // s
        assert rel_err(np64(pb.buf.cache[b, j]), cache_o[b, j]) <= 4e-3
    assert rel_err(np64(pb.buf.open_slot), acc_o) <= 1e-5


@pytest.mark.gpu
@pytest.mark.parametrize("B,N", [(1, 65536), (40, 4096)])
def test_large_head_decode_split_extremes(B, N):
    """The large-head decode where one sequence is split over every cluster
    (B=1: more partials per sequence than a warp has lanes) and where the
    batch spans two 32-sequence groups of the prep and combine blocks (B=40)."""
    wl = inputs.LARGE_LATENT.with_(B=B)
    max_slots = N // wl.s
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, 1, stream=2)
    cache0 = inputs.synthetic_cache(wl, N - 1, max_slots)
    pb = Problem(wl, max_slots=max_slots, weights=w)
    pb.buf.cache.copy_(cache0["cache"].to(pb.dt))
    pb.buf.open_slot.copy_(cache0["acc"])
    rng = np.random.default_rng(B)
    pos = np.full(B, N - 1) if B == 1 else rng.integers(0, N, size=B)
    out = np64(pb.decode(toks, 0, pos))
    sample = [0] if B == 1 else [0, 31, 32, 39]
    sub = lambda x: x[sample]
    cfg = oracle_cfg(wl, B=len(sample))
    cache_o = cache0["cache"][sample].double().numpy().copy()
    acc_o = cache0["acc"][sample].double().numpy().copy()
    ref = oracle.decode_step(cfg, sub(toks["c"][:, 0]), sub(toks["kr"][:, 0]), sub(toks["qc"][:, 0]),
                             sub(toks["qr"][:, 0]), w["w_uk"], w["w_uv"], pos[sample], cache_o, acc_o,
                             gate_in=sub(toks["gate_in"][:, 0]))
    assert rel_err(out[sample], ref["out"]) <= TOL["bf16"]
    for i, b in enumerate(sample):
        j = pos[b] // wl.s
        assert rel_err(np64(pb.buf.cache[b, j]), cache_o[i, j]) <= 4e-3
    assert rel_err(np64(pb.buf.open_slot[sample]), acc_o) <= 1e-5


@pytest.mark.gpu
def test_small_head_decode_one_long_sequence():
    """Speech-decode widths with B=1 and 32768 slots: the one sequence is split
    over every CTA of the grid, and the combine merges all of their partials."""
    wl = inputs.SPEECH_DECODE.with_(B=1)
    N = 65536
    max_slots = N // wl.s
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, 1, stream=2)
    cache0 = inputs.synthetic_cache(wl, N - 1, max_slots)
    pb = Problem(wl, max_slots=max_slots, weights=w)
    pb.buf.cache.copy_(cache0["cache"].to(pb.dt))
    pb.buf.open_slot.copy_(cache0["acc"])
    pos = np.array([N - 1])
    out = np64(pb.decode(toks, 0, pos))
    cfg = oracle_cfg(wl)
    cache_o = cache0["cache"].double().numpy().copy()
    acc_o = cache0["acc"].double().numpy().copy()
    ref = oracle.decode_step(cfg, toks["c"][:, 0], toks["kr"][:, 0], toks["qc"][:, 0], toks["qr"][:, 0],
                             w["w_uk"], w["w_uv"], pos, cache_o, acc_o, G=w["gate_w"], g=w["gate_b"])
    assert rel_err(out, ref["out"]) <= TOL["bf16"]
    assert rel_err(np64(pb.buf.open_slot), acc_o) <= 1e-5


# ----------------------------------------------------------------- beam-search cache reorder


def _bits(t):
    """A tensor's bytes as a C-contiguous numpy array of its shape (bf16 as uint16)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _reorder_case(B, max_slots, s, dtype, src, n_tok, seed):
    cfg = mtla.make_config(B, 8, 64, 256, 32, s, max_slots, dtype=dtype)
    g = torch.Generator().manual_seed(seed)
    dt = torch.float32 if dtype == "fp32" else torch.bfloat16
    cache_in = torch.randn(B, max_slots, cfg.D, generator=g).to(dt)
    cache_out0 = torch.randn(B, max_slots, cfg.D, generator=g).to(dt)
    open_in = torch.randn(B, cfg.D, generator=g)
    open_out0 = torch.randn(B, cfg.D, generator=g)
    dev = lambda t: t.to("cuda").contiguous()
    co, oo = dev(cache_out0), dev(open_out0)
    mtla.reorder_cache(cfg, dev(src), dev(n_tok), dev(cache_in), dev(open_in), co, oo)
    status = mtla.get_device_status()
    want_c, want_o = _bits(cache_out0).copy(), open_out0.numpy().copy()
    want_status = oracle.reorder_cache(s, src.numpy(), n_tok.numpy(), _bits(cache_in), open_in.numpy(),
                                       want_c, want_o)
    return status, want_status, _bits(co), want_c, oo.cpu().numpy(), want_o


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_reorder_cache_matches_oracle(dtype):
    """Beam-search reorder against the oracle, byte for byte: parents with
    duplicates, token counts from 0 to a full cache (s = 3, so slot counts end
    inside a block), destination slots past the parent's count untouched."""
    B, max_slots, s = 37, 150, 3
    g = torch.Generator().manual_seed(5)
    src = torch.randint(0, B, (B,), generator=g, dtype=torch.int32)
    n_tok = torch.randint(0, max_slots * s + 1, (B,), generator=g, dtype=torch.int32)
    n_tok[:5] = torch.tensor([0, 1, s, s + 1, max_slots * s], dtype=torch.int32)
    src[:10] = torch.tensor([0, 1, 2, 3, 4, 4, 3, 2, 1, 0], dtype=torch.int32)
    st, want_st, c, want_c, o, want_o = _reorder_case(B, max_slots, s, dtype, src, n_tok, 11)
    assert st == mtla.OK and want_st == 0
    assert np.array_equal(c, want_c)
    assert np.array_equal(o, want_o)


def test_reorder_cache_full_size():
    """The benchmarked size: 64 sequences of 2048 filled slots (576 bytes),
    a random permutation of parents; byte for byte."""
    B, max_slots, s = 64, 2048, 2
    g = torch.Generator().manual_seed(6)
    src = torch.randperm(B, generator=g).to(torch.int32)
    n_tok = torch.full((B,), max_slots * s, dtype=torch.int32)
    st, want_st, c, want_c, o, want_o = _reorder_case(B, max_slots, s, "bf16", src, n_tok, 12)
    assert st == mtla.OK and want_st == 0
    assert np.array_equal(c, want_c)
    assert np.array_equal(o, want_o)


def test_reorder_cache_bad_parent_and_capacity():
    """A parent index outside [0, B) latches INVALID_ARG, a parent holding more
    tokens than the cache latches CAPACITY; the affected destinations keep
    their contents and every other destination is still copied."""
    B, max_slots, s = 8, 40, 2
    src = torch.tensor([1, 0, 3, B, 2, 5, 7, 6], dtype=torch.int32)
    n_tok = torch.tensor([80, 7, 1, 0, 33, 12, 79, 2], dtype=torch.int32)
    st, want_st, c, want_c, o, want_o = _reorder_case(B, max_slots, s, "bf16", src, n_tok, 13)
    assert want_st == 1 and st == mtla.ERR_INVALID_ARG
    assert np.array_equal(c, want_c) and np.array_equal(o, want_o)
    n_tok[2] = max_slots * s + 1                 # parent of destination 4
    src[3] = 4
    st, want_st, c, want_c, o, want_o = _reorder_case(B, max_slots, s, "bf16", src, n_tok, 14)
    assert want_st == 3 and st == mtla.ERR_CAPACITY
    assert np.array_equal(c, want_c) and np.array_equal(o, want_o)
