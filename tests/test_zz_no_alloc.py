"""The decode step without a workspace (mtla_decode_step_noalloc).

It is meant for callers that cannot allocate device memory themselves -- code
inside a framework whose pool allocator owns the GPU's memory, a serving loop
that cannot pay for a cudaMalloc in the middle of a step, a plug-in host that
passes only inputs and outputs -- and takes its scratch from the library's
built-in device array instead. Here it must give the same bytes as the
ordinary entry point (which gets a caller-allocated workspace) on two calls in
a row, through the C ABI, after an earlier call has left other contents in the
shared array, and refuse configs whose scratch would not fit.

This file is named so that pytest collects it last; it also passes when run
alone in a fresh process.
"""
import pytest
import torch

from gpu_harness import dev
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


def _step(cfg, buf, toks, k, pos, out, noalloc):
    dt = buf.cache.dtype
    args = [dev(toks["c"][:, k], dt), dev(toks["kr"][:, k], dt), dev(toks["qc"][:, k], dt),
            dev(toks["qr"][:, k], dt), buf.w_uk, buf.w_uv, buf.gate_w, buf.gate_b, None, pos,
            buf.cache, buf.open_slot, out]
    if noalloc:
        mtla.decode_step_noalloc(cfg, *args)
    else:
        mtla.decode_step(cfg, *args, buf.workspace)


def test_noalloc_matches_workspace_entry_on_two_calls():
    """Both entry points run the same kernels on the same inputs, so the
    output, the cache and the open slot must agree byte for byte. Before the
    checked calls, a no-allocation call with another batch size, head count
    and cache length leaves the shared array holding a differently laid out
    query image and split partials: the checked calls must not read any of
    those leftovers."""
    dirty_wl = inputs.SPEECH_DECODE.with_(B=11, H=24)
    cfg_d, d = _state(dirty_wl, 200, 333)
    dirty_toks = inputs.tokens(dirty_wl, 1, stream=7)
    out_d = torch.empty(dirty_wl.B, dirty_wl.H, dirty_wl.d_h, device="cuda", dtype=d.cache.dtype)
    pos_d = torch.full((dirty_wl.B,), 333, dtype=torch.int32, device="cuda")
    _step(cfg_d, d, dirty_toks, 0, pos_d, out_d, noalloc=True)

    wl = inputs.SPEECH_DECODE.with_(B=4)
    max_slots, n0 = 64, 99
    cfg_a, a = _state(wl, max_slots, n0)          # ordinary entry point, own workspace
    cfg_b, b = _state(wl, max_slots, n0)          # no-allocation entry point
    assert mtla.workspace_size(cfg_b, 0) <= mtla.NOALLOC_SCRATCH_BYTES
    assert mtla.workspace_size(cfg_d, 0) <= mtla.NOALLOC_SCRATCH_BYTES
    toks = inputs.tokens(wl, 2, stream=1)
    torch.cuda.synchronize()
    assert mtla.get_device_status() == mtla.OK
    for k, t in enumerate((n0, n0 + 1)):           # completes slot 49, then opens slot 50
        pos = torch.full((wl.B,), t, dtype=torch.int32, device="cuda")
        out_a = torch.empty(wl.B, wl.H, wl.d_h, device="cuda", dtype=a.cache.dtype)
        out_b = torch.empty_like(out_a)
        _step(cfg_a, a, toks, k, pos, out_a, noalloc=False)
        _step(cfg_b, b, toks, k, pos, out_b, noalloc=True)
        torch.cuda.synchronize()
        assert torch.equal(out_b, out_a), f"call {k}: out differs"
        assert torch.equal(b.cache, a.cache), f"call {k}: cache differs"
        assert torch.equal(b.open_slot, a.open_slot), f"call {k}: open slot differs"
        assert torch.isfinite(out_b.float()).all()
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
