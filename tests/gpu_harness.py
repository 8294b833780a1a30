"""Helpers shared by the GPU tests: upload seeded inputs, call the C ABI
through the binding, and compare with the oracle."""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle
from kv_cache_mtla_b200 import inputs, mtla

# max |gpu - ref| / max |ref|: the stated bounds for bf16 and fp32 storage; for
# fp16 storage (fp32 arithmetic, the output and the cached slots rounded to
# half precision, unit roundoff 2^-11 = 4.9e-4) ten unit roundoffs
TOL = {"bf16": 2e-2, "fp32": 1e-5, "fp16": 5e-3}


# (test, max-relative error, elementwise error) of every comparison, written
# out by conftest.py when MTLA_PARITY_LOG names a file
MARGINS = []


def rel_err(gpu, ref) -> float:
    """max |gpu - ref| / max |ref| over the whole tensor. Also records the
    elementwise relative error max |gpu - ref| / max(|ref|, 1e-3 max |ref|)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    denom = np.max(np.abs(ref))
    denom = denom if denom > 0 else 1.0
    diff = np.abs(gpu - ref)
    rel = float(np.max(diff) / denom)
    elem = float(np.max(diff / np.maximum(np.abs(ref), 1e-3 * denom)))
    MARGINS.append((os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], rel, elem))
    return rel


def elem_err(gpu, ref) -> float:
    """Elementwise relative error max |gpu - ref| / max(|ref|, 1e-3 max |ref|)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    denom = np.max(np.abs(ref))
    denom = denom if denom > 0 else 1.0
    return float(np.max(np.abs(gpu - ref) / np.maximum(np.abs(ref), 1e-3 * denom)))


def oracle_cfg(wl: inputs.Workload, B: int | None = None) -> oracle.Cfg:
    return oracle.Cfg(B if B is not None else wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s,
                      gate_mode=wl.gate_mode)


def config(wl: inputs.Workload, max_slots: int, B: int | None = None) -> mtla.Config:
    return mtla.make_config(B if B is not None else wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s,
                            max_slots, dtype=wl.dtype, gate_mode=wl.gate_mode)


def dev(t, dtype):
    return None if t is None else t.to("cuda", dtype).contiguous()


class Problem:
    """Device state of one workload: weights, cache, open slot, scratch."""

    def __init__(self, wl: inputs.Workload, max_slots: int, max_tokens: int = 0, weights=None,
                 B: int | None = None):
        self.wl = wl
        self.B = B if B is not None else wl.B
        self.cfg = config(wl, max_slots, self.B)
        self.dt = self.cfg.torch_dtype
        self.weights = weights if weights is not None else inputs.weights(wl)
        self.buf = mtla.Buffers.allocate(self.cfg, self.weights, max_tokens)

    def gate_ptrs(self):
        if self.wl.gate_mode in (inputs.GATE_COMPUTED, inputs.GATE_CHANNEL_COMPUTED):
            return self.buf.gate_w, self.buf.gate_b
        return None, None

    def prefill(self, toks: dict, T: int):
        B, wl = self.B, self.wl
        out = torch.empty(B, T, wl.H, wl.d_h, device="cuda", dtype=self.dt)
        gw, gb = self.gate_ptrs()
        mtla.prefill(self.cfg, T, dev(toks["c"][:, :T], self.dt), dev(toks["kr"][:, :T], self.dt),
                     dev(toks["qc"][:, :T], self.dt), dev(toks["qr"][:, :T], self.dt),
                     self.buf.w_uk, self.buf.w_uv, gw, gb,
                     dev(toks["gate_in"][:, :T], torch.float32) if toks["gate_in"] is not None else None,
                     out, self.buf.cache, self.buf.open_slot, self.buf.workspace)
        return out

    def prefill_from(self, toks: dict, t0: int, t1: int):
        """Chunked prefill of tokens t0 .. t1-1 (indices into toks) continuing from
        the current cache and open slot."""
        B, wl = self.B, self.wl
        T = t1 - t0
        out = torch.empty(B, T, wl.H, wl.d_h, device="cuda", dtype=self.dt)
        gw, gb = self.gate_ptrs()
        gin = toks["gate_in"]
        mtla.prefill_from(self.cfg, t0, T, dev(toks["c"][:, t0:t1], self.dt), dev(toks["kr"][:, t0:t1], self.dt),
                          dev(toks["qc"][:, t0:t1], self.dt), dev(toks["qr"][:, t0:t1], self.dt),
                          self.buf.w_uk, self.buf.w_uv, gw, gb,
                          dev(gin[:, t0:t1], torch.float32) if gin is not None else None,
                          out, self.buf.cache, self.buf.open_slot, self.buf.workspace)
        return out

    def decode(self, toks: dict, k: int, pos):
        """Decode step with the k-th token of every sequence at positions pos [B]."""
        B, wl = self.B, self.wl
        out = torch.empty(B, wl.H, wl.d_h, device="cuda", dtype=self.dt)
        gw, gb = self.gate_ptrs()
        pos_d = torch.as_tensor(pos, dtype=torch.int32).to("cuda").contiguous()
        gin = toks["gate_in"]
        mtla.decode_step(self.cfg, dev(toks["c"][:, k], self.dt), dev(toks["kr"][:, k], self.dt),
                         dev(toks["qc"][:, k], self.dt), dev(toks["qr"][:, k], self.dt),
                         self.buf.w_uk, self.buf.w_uv, gw, gb,
                         dev(gin[:, k], torch.float32) if gin is not None else None,
                         pos_d, self.buf.cache, self.buf.open_slot, out, self.buf.workspace)
        return out


def np64(t):
    return t.detach().float().cpu().double().numpy()


def concat_tokens(a: dict, b: dict) -> dict:
    out = {}
    for k in a:
        if a[k] is None:
            out[k] = None
        else:
            out[k] = torch.cat([a[k], b[k]], dim=1)
    return out


def oracle_rows(wl, weights, toks, rows, B=None):
    """Parallel-form oracle outputs for rows [(b, t)] over the given tokens."""
    cfg = oracle_cfg(wl, B)
    _, P = oracle.partials(cfg, toks["c"], toks["kr"], weights["gate_w"], weights["gate_b"],
                           toks["gate_in"])
    return oracle.attend_rows(cfg, toks["qc"], toks["qr"], weights["w_uk"], weights["w_uv"], P,
                              rows), P
