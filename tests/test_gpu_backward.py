"""GPU parity of the training backward (mtla_prefill_backward): the gradients
of sum(dout * out) of the parallel forward with respect to every input --
latents, decoupled keys, both query parts, W_UK, W_UV and the gate (computed:
G and g; supplied: the given weights) -- against the float64 oracle's
backward on the same seeded inputs ("Multi-head Temporal Latent Attention",
Results: trained from scratch; Key claims: the stride-aware mask in
training). The oracle's backward is itself pinned to central finite
differences of its forward on the CPU.

The kernels compute in fp32 for both storage types, from the same (bf16-
valued, for bf16 storage) inputs the oracle receives, so both are held to
the fp32 bound BWD_TOL: max |gpu - ref| / max |ref| per gradient."""
import numpy as np
import pytest
import torch

import oracle
from gpu_harness import TOL, dev, np64, oracle_cfg, rel_err
from kv_cache_mtla_b200 import inputs, mtla

pytestmark = pytest.mark.gpu

# the fp32 bound of the forward: measured errors are 1e-7 .. 5e-7 of each
# gradient's largest element (the gate's weight and bias taken together: the
# bias alone is one sum over all B*T tokens with heavy cancellation)
BWD_TOL = TOL["fp32"]


def tol_for(wl):
    """bf16 at the tensor-core widths (d_h=64, d_R=32, d_c 128 or 256) runs the
    tensor-core backward (bf16 operands: the bf16 bound); everything else the
    fp32 CUDA-core backward (the fp32 bound)."""
    tc = wl.dtype == "bf16" and wl.d_h == 64 and wl.d_r == 32 and wl.d_c in (128, 256)
    return TOL["bf16"] if tc else BWD_TOL


@pytest.fixture(autouse=True)
def _clean_status():
    torch.cuda.synchronize()
    mtla.get_device_status()
    yield
    assert mtla.get_device_status() == mtla.OK


def _grad_names(mode):
    names = ["dc", "dkr", "dq_c", "dq_r", "dw_uk", "dw_uv"]
    if mode == inputs.GATE_COMPUTED:
        names += ["dgate_w", "dgate_b"]
    if mode == inputs.GATE_SUPPLIED:
        names += ["dgate_in"]
    return names


ORACLE_NAME = {"dc": "dc", "dkr": "dkr", "dq_c": "dqc", "dq_r": "dqr", "dw_uk": "dw_uk", "dw_uv": "dw_uv",
               "dgate_w": "dG", "dgate_b": "dg", "dgate_in": "dgate_in"}


def run_backward(wl, T, w, toks, dout):
    """Device gradients of the path (dict of float32 tensors on the GPU)."""
    cfg = mtla.make_config(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, 1, dtype=wl.dtype, gate_mode=wl.gate_mode)
    dt = cfg.torch_dtype
    B, H = wl.B, wl.H
    shapes = dict(dc=(B, T, wl.d_c), dkr=(B, T, wl.d_r), dq_c=(B, T, H, wl.d_h), dq_r=(B, T, H, wl.d_r),
                  dw_uk=(H, wl.d_h, wl.d_c), dw_uv=(H, wl.d_h, wl.d_c), dgate_w=(wl.s, wl.d_c),
                  dgate_b=(wl.s,), dgate_in=(B, T))
    # poison the outputs: every element must be written
    grads = {k: torch.full(shapes[k], float("nan"), device="cuda") for k in _grad_names(wl.gate_mode)}
    ws = torch.empty(mtla.prefill_backward_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    computed = wl.gate_mode == inputs.GATE_COMPUTED
    mtla.prefill_backward(cfg, T, dev(toks["c"], dt), dev(toks["kr"], dt), dev(toks["qc"], dt),
                          dev(toks["qr"], dt), dev(w["w_uk"], dt), dev(w["w_uv"], dt),
                          dev(w["gate_w"], torch.float32) if computed else None,
                          dev(w["gate_b"], torch.float32) if computed else None,
                          dev(toks["gate_in"], torch.float32) if toks["gate_in"] is not None else None,
                          dev(dout, dt), grads, ws)
    torch.cuda.synchronize()
    return grads


def oracle_backward(wl, w, toks, dout, B=None):
    computed = wl.gate_mode == inputs.GATE_COMPUTED
    return oracle.prefill_backward(oracle_cfg(wl, B), toks["c"], toks["kr"], toks["qc"], toks["qr"], w["w_uk"],
                                   w["w_uv"], dout, w["gate_w"] if computed else None,
                                   w["gate_b"] if computed else None, toks["gate_in"])


def check_all(wl, grads, ref, tol=None):
    """Every gradient within tol; the computed gate's weight G and bias g are
    one linear layer and are compared as one parameter tensor."""
    got, want = {}, {}
    for k in _grad_names(wl.gate_mode):
        got[k] = np64(grads[k])
        want[k] = ref[ORACLE_NAME[k]]
        assert np.all(np.isfinite(got[k])), k
    if "dgate_b" in got:
        got["dgate"] = np.concatenate([got.pop("dgate_w").ravel(), got.pop("dgate_b")])
        want["dgate"] = np.concatenate([want.pop("dgate_w").ravel(), want.pop("dgate_b")])
    errs = {k: rel_err(got[k], want[k]) for k in got}
    tol = tol_for(wl) if tol is None else tol
    assert max(errs.values()) <= tol, errs


MODES = [inputs.GATE_COMPUTED, inputs.GATE_SUPPLIED, inputs.GATE_UNIT]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("s", [1, 2, 3])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_backward_tiny(mode, s, dtype):
    """The tiny workload's widths (H=4, d_h=32, d_c=128, d_R=16), T=61: a
    ragged last block for s=2 and s=3 (a slot that never finishes)."""
    wl = inputs.TINY_FP32.with_(s=s, gate_mode=mode, dtype=dtype, B=2)
    T = 61
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    dout = inputs.grad_out(wl, T)
    grads = run_backward(wl, T, w, toks, dout)
    check_all(wl, grads, oracle_backward(wl, w, toks, dout))


def test_backward_tiny_exact_config():
    """The tiny fp32 workload as stated: B=1, s=2, T=64, computed gate."""
    wl = inputs.TINY_FP32
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, wl.T)
    dout = inputs.grad_out(wl, wl.T)
    check_all(wl, run_backward(wl, wl.T, w, toks, dout), oracle_backward(wl, w, toks, dout))


@pytest.mark.parametrize("s,T", [(2, 300), (4, 257), (3, 130)])
def test_backward_speech_widths(s, T):
    """bf16 storage at the prefill workload's widths (H=8, d_h=64, d_c=256,
    d_R=32), several 128-row tiles and a ragged tail; gate weights N(0, 0.02)."""
    wl = inputs.PREFILL.with_(B=2, s=s)
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    dout = inputs.grad_out(wl, T)
    check_all(wl, run_backward(wl, T, w, toks, dout), oracle_backward(wl, w, toks, dout))


@pytest.mark.parametrize("d_c,s,T,mode", [(128, 2, 200, inputs.GATE_COMPUTED), (256, 1, 130, inputs.GATE_UNIT),
                                          (256, 3, 1, inputs.GATE_SUPPLIED), (256, 2, 2, inputs.GATE_COMPUTED),
                                          (128, 8, 333, inputs.GATE_SUPPLIED)])
def test_backward_tensor_core_shapes(d_c, s, T, mode):
    """The tensor-core backward's other cases: d_c=128, s=1 and s=8, every gate
    mode, T=1 and T=2 (no finished slot at all), T not a multiple of 4 (the
    statistics' padded pitch)."""
    wl = inputs.PREFILL.with_(B=2, d_c=d_c, s=s, gate_mode=mode)
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    dout = inputs.grad_out(wl, T)
    check_all(wl, run_backward(wl, T, w, toks, dout), oracle_backward(wl, w, toks, dout))


def test_backward_large_latent_widths():
    """The large-latent widths (H=128 > 8 warps per block, d_c=512, d_R=64:
    slot width 576, the widest), supplied gates, s=4, T=45."""
    wl = inputs.LARGE_LATENT.with_(B=1)
    T = 45
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    dout = inputs.grad_out(wl, T)
    check_all(wl, run_backward(wl, T, w, toks, dout), oracle_backward(wl, w, toks, dout))


@pytest.mark.parametrize("T", [1, 2])
def test_backward_degenerate_lengths(T):
    """T=1 (one token: its own partial is its only key, the softmax weight is
    1 and delta cancels the key term) and T=2 with s=2 (no finished slot)."""
    wl = inputs.TINY_FP32.with_(B=1)
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    dout = inputs.grad_out(wl, T)
    check_all(wl, run_backward(wl, T, w, toks, dout), oracle_backward(wl, w, toks, dout))


@pytest.mark.parametrize("wl,T", [(inputs.TINY_FP32.with_(B=2, s=3), 50), (inputs.PREFILL.with_(B=2, s=3), 300)],
                         ids=["cuda_cores", "tensor_cores"])
def test_backward_is_repeatable(wl, T):
    """Two calls on the same inputs: the heads' key gradients are summed in a
    fixed order, so the per-token gradients are the same bytes; the weight and
    gate gradients (atomic additions over token rows) agree to rounding."""
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    dout = inputs.grad_out(wl, T)
    g1 = run_backward(wl, T, w, toks, dout)
    g2 = run_backward(wl, T, w, toks, dout)
    for k in ("dc", "dkr", "dq_c", "dq_r"):
        assert torch.equal(g1[k], g2[k]), k
    for k in ("dw_uk", "dw_uv", "dgate_w", "dgate_b"):
        assert rel_err(np64(g1[k]), np64(g2[k])) <= 1e-6, k


@pytest.mark.parametrize("mode", [inputs.GATE_COMPUTED, inputs.GATE_SUPPLIED])
def test_training_pair_equals_backward(mode):
    """mtla_prefill_train + mtla_prefill_backward_saved: the forward's output is
    the bytes of mtla_prefill's, and the gradients are the bytes of
    mtla_prefill_backward's (the same kernels on the same kept rows; the gate
    gradients, sums of atomic additions, to rounding)."""
    wl = inputs.PREFILL.with_(B=2, s=3, gate_mode=mode)
    T = 300
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    dout = inputs.grad_out(wl, T)
    ref = run_backward(wl, T, w, toks, dout)
    cfg = mtla.make_config(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, (T + wl.s - 1) // wl.s, gate_mode=mode)
    dt = torch.bfloat16
    computed = mode == inputs.GATE_COMPUTED
    args = [dev(toks["c"], dt), dev(toks["kr"], dt), dev(toks["qc"], dt), dev(toks["qr"], dt),
            dev(w["w_uk"], dt), dev(w["w_uv"], dt),
            dev(w["gate_w"], torch.float32) if computed else None,
            dev(w["gate_b"], torch.float32) if computed else None,
            dev(toks["gate_in"], torch.float32) if toks["gate_in"] is not None else None]
    out_t = torch.empty(wl.B, T, wl.H, wl.d_h, device="cuda", dtype=dt)
    saved = torch.empty(mtla.prefill_train_saved_size(cfg, T), dtype=torch.uint8, device="cuda")
    mtla.prefill_train(cfg, T, *args, out_t, saved)
    out_p = torch.empty_like(out_t)
    cache = torch.zeros(wl.B, cfg.max_slots, wl.D, device="cuda", dtype=dt)
    op = torch.zeros(wl.B, wl.D, device="cuda")
    wsp = torch.empty(mtla.workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    mtla.prefill(cfg, T, *args, out_p, cache, op, wsp)
    torch.cuda.synchronize()
    assert torch.equal(out_t, out_p)
    grads = {k: torch.full_like(v, float("nan")) for k, v in ref.items()}
    ws = torch.empty(mtla.prefill_backward_saved_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    mtla.prefill_backward_saved(cfg, T, *args, saved, dev(dout, dt), grads, ws)
    torch.cuda.synchronize()
    for k in ref:
        if k in ("dgate_w", "dgate_b"):
            assert rel_err(np64(grads[k]), np64(ref[k])) <= 1e-6, k
        else:
            assert torch.equal(grads[k], ref[k]), k


def test_backward_many_slot_tiles():
    """Enough finished slots for the key-gradient kernel's banded order to run
    full bands of 8 slot tiles and a partial one (T=4096, s=2: 2048 slots, 16
    tiles of 128), and 32 query tiles; one head keeps the float64 oracle to
    seconds."""
    wl = inputs.PREFILL.with_(B=1, H=1, s=2)
    T = 4096
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    dout = inputs.grad_out(wl, T)
    check_all(wl, run_backward(wl, T, w, toks, dout), oracle_backward(wl, w, toks, dout))


def test_backward_weight_gradients_ragged_row_chunks():
    """dW_UK and dW_UV sum over all B*T token rows, sequences back to back, in
    chunks of 128-row tiles that are added in order: B=3, T=1500 gives 4500
    rows, so several chunks, a shorter last chunk and a last tile of 20 rows
    (the rest of its 128 rows read as zeros), checked against the oracle with
    every other gradient."""
    wl = inputs.PREFILL.with_(B=3, H=1, s=2)
    T = 1500
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    dout = inputs.grad_out(wl, T)
    check_all(wl, run_backward(wl, T, w, toks, dout), oracle_backward(wl, w, toks, dout))


def test_backward_full_size_sampled_rows():
    """The prefill workload exactly as bench.py times its backward (B=8,
    T=8192, H=8, d_c=256, s=2, computed gates, the same seed): the query
    gradients dqC and dqR of sampled rows -- the first and last rows, rows on
    both sides of query-tile (128) and slot-tile (128 slots = 256 positions)
    boundaries, and random rows, in three of the eight sequences -- against
    the oracle computing each row alone."""
    wl = inputs.PREFILL
    T = wl.T
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T)
    dout = inputs.grad_out(wl, T)
    grads = run_backward(wl, T, w, toks, dout)
    rng = np.random.default_rng(11)
    rows = []
    for b in (0, 3, wl.B - 1):
        fixed = [0, 1, 2, 127, 128, 129, 255, 256, 257, 4095, 4096, 8190, 8191]
        rows += [(b, i) for i in fixed + sorted(rng.integers(0, T, 10).tolist())]
    ref = oracle.backward_rows(oracle_cfg(wl), toks["c"], toks["kr"], toks["qc"], toks["qr"], w["w_uk"],
                               w["w_uv"], dout, rows, w["gate_w"], w["gate_b"])
    dqc = np.stack([np64(grads["dq_c"][b, i]) for b, i in rows])
    dqr = np.stack([np64(grads["dq_r"][b, i]) for b, i in rows])
    assert np.all(np.isfinite(dqc)) and np.all(np.isfinite(dqr))
    assert rel_err(dqc, ref["dqc"]) <= TOL["bf16"]
    assert rel_err(dqr, ref["dqr"]) <= TOL["bf16"]
