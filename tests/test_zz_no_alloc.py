"""The decode step without a workspace (mtla_decode_step_noalloc).

It is meant for callers that cannot allocate device memory themselves -- code
inside a framework whose pool allocator owns the GPU's memory, a serving loop
that cannot pay for a cudaMalloc in the middle of a step, a plug-in host that
passes only inputs and outputs -- and takes its scratch from the library's
built-in device array instead. Here it must give the same results as the
ordinary entry point (which gets a caller-allocated workspace) on two calls in
a row, through the C ABI, and refuse configs whose scratch would not fit.

This file is named so that pytest collects it last; it also passes when run
alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from gpu_harness import TOL, dev, np64, rel_err
from kv_cache_mtla_b200 import inputs, mtla

pytestmark = pytest.mark.gpu


def _state(wl, max_slots, n_tokens):
    cfg = mtla.make_config(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, max_slots, dtype=wl.dtype,
                           gate_mode=wl.gate_mode)
    buf = mtla.Buffers.allocate(cfg, inputs.weights(wl))
    c0 = inputs.synthetic_cache(wl, n_tokens, max_slots)
    buf.cache.copy_(c0["cache"].to(buf.cache.dtype))
    buf.open_slot.copy_(c0["acc"])
    return cfg, buf


def test_noalloc_matches_workspace_entry_on_two_calls():
    wl = inputs.SPEECH_DECODE.with_(B=4)
    max_slots, n0 = 64, 99
    cfg_a, a = _state(wl, max_slots, n0)          # ordinary entry point, own workspace
    cfg_b, b = _state(wl, max_slots, n0)          # no-allocation entry point
    assert mtla.workspace_size(cfg_b, 0) <= mtla.NOALLOC_SCRATCH_BYTES
    toks = inputs.tokens(wl, 2, stream=1)
    dt = a.cache.dtype
    torch.cuda.synchronize()
    mtla.get_device_status()
    for k, t in enumerate((n0, n0 + 1)):           # completes slot 49, then opens slot 50
        pos = torch.full((wl.B,), t, dtype=torch.int32, device="cuda")
        args = [dev(toks["c"][:, k], dt), dev(toks["kr"][:, k], dt), dev(toks["qc"][:, k], dt),
                dev(toks["qr"][:, k], dt)]
        out_a = torch.empty(wl.B, wl.H, wl.d_h, device="cuda", dtype=dt)
        out_b = torch.empty_like(out_a)
        mtla.decode_step(cfg_a, *args, a.w_uk, a.w_uv, a.gate_w, a.gate_b, None, pos, a.cache,
                         a.open_slot, out_a, a.workspace)
        mtla.decode_step_noalloc(cfg_b, *args, b.w_uk, b.w_uv, b.gate_w, b.gate_b, None, pos,
                                 b.cache, b.open_slot, out_b)
        torch.cuda.synchronize()
        assert rel_err(np64(out_b), np64(out_a)) <= TOL["bf16"], f"call {k}"
        assert rel_err(np64(b.cache), np64(a.cache)) <= TOL["bf16"], f"call {k}"
        assert rel_err(np64(b.open_slot), np64(a.open_slot)) <= TOL["bf16"], f"call {k}"
        assert np.isfinite(np64(out_b)).all()
    assert mtla.get_device_status() == mtla.OK


def test_noalloc_refuses_configs_beyond_its_scratch():
    wl = inputs.LARGE_LATENT.with_(B=64)
    cfg = mtla.make_config(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, 16384, dtype=wl.dtype,
                           gate_mode=wl.gate_mode)
    assert mtla.workspace_size(cfg, 0) > mtla.NOALLOC_SCRATCH_BYTES
    fake = 0x10000       # never dereferenced: the size check comes first, on the host
    st = mtla.decode_step_noalloc(cfg, fake, fake, fake, fake, fake, fake, None, None, fake,
                                  fake, fake, fake, fake, check=False)
    assert st == mtla.ERR_WORKSPACE
