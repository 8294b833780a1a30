"""GPU parity of the dense projections around the MTLA path (``mtla_linear``,
the tcgen05 GEMM) and of the layer built from them, against the float64
oracle on the same seeded bf16 inputs."""
import numpy as np
import pytest
import torch

import oracle
from gpu_harness import np64, rel_err
from kv_cache_mtla_b200 import mtla

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    torch.cuda.synchronize()
    mtla.get_device_status()
    yield
    assert mtla.get_device_status() == mtla.OK


def _bf16_randn(g, *shape, scale=1.0):
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("M,N,K", [(300, 200, 520), (1, 64, 64), (4096, 512, 512), (128, 32, 512),
                                   (257, 1000, 8), (16, 288, 512), (1000, 129, 136)])
def test_linear_matches_oracle(M, N, K):
    """y = x W^T: partial row and column tiles (M, N not multiples of the
    128 x 64/128/256 output tiles), K below one 64-column box and not a multiple
    of it, every tile width. The result is bf16 (rounding <= 2^-8 relative), so
    the bound is 8e-3 of max|y|."""
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    x = _bf16_randn(g, M, K)
    w = _bf16_randn(g, N, K, scale=K ** -0.5)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    mtla.linear(x.cuda(), w.cuda(), y)
    ref = oracle.linear(x.float().numpy(), w.float().numpy())
    assert rel_err(np64(y), ref) <= 8e-3


def _layer_setup(wl, d_model, max_slots, max_tokens):
    from kv_cache_mtla_b200 import inputs
    cfg = mtla.make_config(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, max_slots, gate_mode=wl.gate_mode)
    W = inputs.layer_weights(wl, d_model)
    dW = {k: (v.to("cuda", torch.bfloat16 if k.startswith("w_") else torch.float32).contiguous()) for k, v in W.items()}
    ws = torch.empty(mtla.layer_workspace_size(cfg, d_model, max_tokens), dtype=torch.uint8, device="cuda")
    cache = torch.zeros(wl.B, max_slots, wl.D, dtype=torch.bfloat16, device="cuda")
    open_slot = torch.zeros(wl.B, wl.D, dtype=torch.float32, device="cuda")
    return cfg, W, dW, ws, cache, open_slot


def _oracle_layer(wl, W, h):
    from gpu_harness import oracle_cfg
    cfg = oracle_cfg(wl)
    B = wl.B
    return oracle.layer_forward(cfg, 0, np.zeros((B, 0, wl.D)), np.zeros((B, wl.D)), h, W,
                                W["gate_w"], W["gate_b"])


@pytest.mark.parametrize("s", [2, 3])
def test_layer_forward_chunks_then_decode(s):
    """Speech-model layer (d_model=512, H=8, d_h=64, d_c=256, d_R=32): 300
    tokens as two layer calls (the second from position 170, inside a block for
    s = 3), then 6 layer decode steps; y of every token against the oracle's
    layer over all 306 tokens, the open slot too. bf16 activations between the
    projections and the path add roundings of 2^-9 each."""
    from kv_cache_mtla_b200 import inputs
    wl = inputs.SPEECH_DECODE.with_(B=2, s=s)
    dm, T, S = 512, 300, 6
    cfg, W, dW, ws, cache, open_slot = _layer_setup(wl, dm, (T + S) // s + 2, T)
    lw = mtla.layer_weights(dW)
    h = inputs.hidden(wl, dm, T + S)
    hd = h.to("cuda", torch.bfloat16)
    ys = []
    for t0, t1 in ((0, 170), (170, T)):
        y = torch.empty(wl.B, t1 - t0, dm, dtype=torch.bfloat16, device="cuda")
        mtla.layer_forward(cfg, dm, t0, t1 - t0, hd[:, t0:t1].contiguous(), lw, dW["gate_w"], dW["gate_b"], None, y,
                           cache, open_slot, ws)
        ys.append(np64(y))
    for k in range(S):
        y = torch.empty(wl.B, dm, dtype=torch.bfloat16, device="cuda")
        pos = torch.full((wl.B,), T + k, dtype=torch.int32, device="cuda")
        mtla.layer_decode_step(cfg, dm, hd[:, T + k].contiguous(), lw, dW["gate_w"], dW["gate_b"], None, pos, cache,
                               open_slot, y, ws)
        ys.append(np64(y)[:, None])
    ref = _oracle_layer(wl, W, h.float().numpy())
    assert rel_err(np.concatenate(ys, axis=1), ref["y"]) <= 2e-2
    assert rel_err(np64(open_slot), ref["acc"]) <= 2e-2


def test_layer_large_heads():
    """Large-latent widths in the layer (d_model=1024, H=64, d_h=128, d_c=512,
    d_R=64, s=4, supplied gates off: computed gate): 40 tokens then 3 decode
    steps on the two-CTA cluster decode."""
    from kv_cache_mtla_b200 import inputs
    wl = inputs.LARGE_LATENT.with_(B=3, H=64, gate_mode=inputs.GATE_COMPUTED, gate_w_std=0.02)
    dm, T, S = 1024, 40, 3
    cfg, W, dW, ws, cache, open_slot = _layer_setup(wl, dm, 64, T)
    lw = mtla.layer_weights(dW)
    h = inputs.hidden(wl, dm, T + S)
    hd = h.to("cuda", torch.bfloat16)
    y0 = torch.empty(wl.B, T, dm, dtype=torch.bfloat16, device="cuda")
    mtla.layer_forward(cfg, dm, 0, T, hd[:, :T].contiguous(), lw, dW["gate_w"], dW["gate_b"], None, y0, cache,
                       open_slot, ws)
    ys = [np64(y0)]
    for k in range(S):
        y = torch.empty(wl.B, dm, dtype=torch.bfloat16, device="cuda")
        pos = torch.full((wl.B,), T + k, dtype=torch.int32, device="cuda")
        mtla.layer_decode_step(cfg, dm, hd[:, T + k].contiguous(), lw, dW["gate_w"], dW["gate_b"], None, pos, cache,
                               open_slot, y, ws)
        ys.append(np64(y)[:, None])
    ref = _oracle_layer(wl, W, h.float().numpy())
    assert rel_err(np.concatenate(ys, axis=1), ref["y"]) <= 2e-2
