"""Python binding of libmtla.so (argument marshalling only).

Every function here forwards torch tensors' device pointers to the C ABI in
``include/mtla.h`` under the same name; all arithmetic runs in the library's
CUDA kernels. If the shared library is missing this module raises at import
of the first call -- there is no other implementation to fall back on.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmtla.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(7)
BF16, FP32, FP16 = 0, 1, 2
GATE_COMPUTED, GATE_SUPPLIED, GATE_UNIT = 0, 1, 2
GATE_CHANNEL_COMPUTED, GATE_CHANNEL_SUPPLIED = 3, 4


class MtlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = last_error_detail() if status == ERR_CUDA else ""
        super().__init__(f"{where}: {status_string(status)} (status {status})"
                         + (f" [{detail}]" if detail else ""))


class Config(ctypes.Structure):
    """Mirror of ``mtla_config``."""
    _fields_ = [
        ("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("d_h", ctypes.c_int32),
        ("d_c", ctypes.c_int32), ("d_r", ctypes.c_int32), ("stride", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("gate_mode", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float), ("rope_base", ctypes.c_float),
        ("max_slots", ctypes.c_int32),
    ]

    @property
    def D(self) -> int:
        return self.d_c + self.d_r

    @property
    def torch_dtype(self):
        return {FP32: torch.float32, FP16: torch.float16}.get(self.dtype, torch.bfloat16)


def make_config(B, H, d_h, d_c, d_r, s, max_slots, dtype="bf16", gate_mode=GATE_COMPUTED,
                softmax_scale=0.0, rope_base=10000.0) -> Config:
    dt = (FP32 if dtype in ("fp32", FP32, torch.float32) else
          FP16 if dtype in ("fp16", FP16, torch.float16) else BF16)
    return Config(B, H, d_h, d_c, d_r, s, dt, gate_mode, softmax_scale, rope_base, max_slots)


_lib = None
_vp = ctypes.c_void_p


class LayerWeights(ctypes.Structure):
    """Mirror of ``mtla_layer_weights`` (device pointers)."""
    _fields_ = [("w_dkv", _vp), ("w_kr", _vp), ("w_q", _vp), ("w_qr", _vp), ("w_uk", _vp), ("w_uv", _vp),
                ("w_o", _vp)]


def layer_weights(d: dict) -> LayerWeights:
    """LayerWeights from a dict of contiguous bf16 device tensors."""
    return LayerWeights(*[_ptr(d[k]) for k in ("w_dkv", "w_kr", "w_q", "w_qr", "w_uk", "w_uv", "w_o")])


def load() -> ctypes.CDLL:
    """Load libmtla.so (built by ``python -m kv_cache_mtla_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m kv_cache_mtla_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    cp = ctypes.POINTER(Config)
    lib.mtla_workspace_size.argtypes = [cp, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
    lib.mtla_workspace_size.restype = ctypes.c_int
    lib.mtla_decode_step.argtypes = [cp] + [_vp] * 13 + [_vp, ctypes.c_size_t, _vp]
    lib.mtla_decode_step.restype = ctypes.c_int
    lib.mtla_prefill.argtypes = [cp, ctypes.c_int32] + [_vp] * 12 + [_vp, ctypes.c_size_t, _vp]
    lib.mtla_prefill.restype = ctypes.c_int
    lib.mtla_prefill_from.argtypes = [cp, ctypes.c_int32, ctypes.c_int32] + [_vp] * 12 + [_vp, ctypes.c_size_t, _vp]
    lib.mtla_prefill_from.restype = ctypes.c_int
    lib.mtla_prefill_backward_workspace_size.argtypes = [cp, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
    lib.mtla_prefill_backward_workspace_size.restype = ctypes.c_int
    lib.mtla_prefill_backward.argtypes = [cp, ctypes.c_int32] + [_vp] * 19 + [_vp, ctypes.c_size_t, _vp]
    lib.mtla_prefill_backward.restype = ctypes.c_int
    lib.mtla_prefill_train_saved_size.argtypes = [cp, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
    lib.mtla_prefill_train_saved_size.restype = ctypes.c_int
    lib.mtla_prefill_backward_saved_workspace_size.argtypes = [cp, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
    lib.mtla_prefill_backward_saved_workspace_size.restype = ctypes.c_int
    lib.mtla_prefill_train.argtypes = [cp, ctypes.c_int32] + [_vp] * 11 + [ctypes.c_size_t, _vp]
    lib.mtla_prefill_train.restype = ctypes.c_int
    lib.mtla_prefill_backward_saved.argtypes = [cp, ctypes.c_int32] + [_vp] * 20 + [_vp, ctypes.c_size_t, _vp]
    lib.mtla_prefill_backward_saved.restype = ctypes.c_int
    lib.mtla_linear.argtypes = [_vp, _vp, _vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _vp]
    lib.mtla_linear.restype = ctypes.c_int
    lp = ctypes.POINTER(LayerWeights)
    lib.mtla_layer_workspace_size.argtypes = [cp, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
    lib.mtla_layer_workspace_size.restype = ctypes.c_int
    lib.mtla_layer_forward.argtypes = ([cp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _vp, lp]
                                       + [_vp] * 7 + [ctypes.c_size_t, _vp])
    lib.mtla_layer_forward.restype = ctypes.c_int
    lib.mtla_layer_decode_step.argtypes = [cp, ctypes.c_int32, _vp, lp] + [_vp] * 8 + [ctypes.c_size_t, _vp]
    lib.mtla_layer_decode_step.restype = ctypes.c_int
    lib.mtla_decode_step_noalloc.argtypes = [cp] + [_vp] * 13 + [_vp]
    lib.mtla_decode_step_noalloc.restype = ctypes.c_int
    lib.mtla_reorder_cache.argtypes = [cp] + [_vp] * 6 + [_vp]
    lib.mtla_reorder_cache.restype = ctypes.c_int
    lib.mtla_test_wait_timeout.argtypes = [ctypes.c_uint64, _vp, _vp]
    lib.mtla_test_wait_timeout.restype = ctypes.c_int
    lib.mtla_get_device_status.argtypes = [_vp]
    lib.mtla_get_device_status.restype = ctypes.c_int
    lib.mtla_status_string.argtypes = [ctypes.c_int]
    lib.mtla_status_string.restype = ctypes.c_char_p
    lib.mtla_last_error_detail.argtypes = []
    lib.mtla_last_error_detail.restype = ctypes.c_char_p
    lib.mtla_kernel_launches.argtypes = []
    lib.mtla_kernel_launches.restype = ctypes.c_uint64
    lib.mtla_set_profile_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]
    lib.mtla_set_profile_events.restype = None
    lib.mtla_profile_events_recorded.argtypes = []
    lib.mtla_profile_events_recorded.restype = ctypes.c_int32
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().mtla_status_string(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmtla must be contiguous")
    return t.data_ptr()


def _bf16(*tensors):
    """The bf16-only calls take raw pointers: a tensor of another dtype would be
    read as bf16 bytes, so refuse it here."""
    for t in tensors:
        if isinstance(t, torch.Tensor) and t.dtype != torch.bfloat16:
            raise TypeError(f"expected a bfloat16 tensor, got {t.dtype}")


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def workspace_size(cfg: Config, max_tokens: int = 0) -> int:
    n = ctypes.c_size_t(0)
    st = load().mtla_workspace_size(ctypes.byref(cfg), int(max_tokens), ctypes.byref(n))
    if st != OK:
        raise MtlaError(st, "mtla_workspace_size")
    return int(n.value)


def decode_step(cfg, c_new, kr_new, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in, pos, cache,
                open_slot, out, workspace, stream=None, check=True) -> int:
    """Forward to ``mtla_decode_step``; returns the status (raises if check)."""
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = load().mtla_decode_step(
        ctypes.byref(cfg), _ptr(c_new), _ptr(kr_new), _ptr(q_c), _ptr(q_r), _ptr(w_uk),
        _ptr(w_uv), _ptr(gate_w), _ptr(gate_b), _ptr(gate_in), _ptr(pos), _ptr(cache),
        _ptr(open_slot), _ptr(out), _ptr(workspace), ws, _stream(stream))
    if check and st != OK:
        raise MtlaError(st, "mtla_decode_step")
    return st


def decode_step_noalloc(cfg, c_new, kr_new, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in, pos,
                        cache, open_slot, out, stream=None, check=True) -> int:
    """Forward to ``mtla_decode_step_noalloc`` (no workspace: the library's
    built-in scratch array is used); returns the status (raises if check)."""
    st = load().mtla_decode_step_noalloc(
        ctypes.byref(cfg), _ptr(c_new), _ptr(kr_new), _ptr(q_c), _ptr(q_r), _ptr(w_uk),
        _ptr(w_uv), _ptr(gate_w), _ptr(gate_b), _ptr(gate_in), _ptr(pos), _ptr(cache),
        _ptr(open_slot), _ptr(out), _stream(stream))
    if check and st != OK:
        raise MtlaError(st, "mtla_decode_step_noalloc")
    return st


NOALLOC_SCRATCH_BYTES = 8 << 20


def prefill(cfg, T, c, kr, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in, out, cache_out,
            open_slot_out, workspace, stream=None, check=True) -> int:
    """Forward to ``mtla_prefill``; returns the status (raises if check)."""
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = load().mtla_prefill(
        ctypes.byref(cfg), int(T), _ptr(c), _ptr(kr), _ptr(q_c), _ptr(q_r), _ptr(w_uk),
        _ptr(w_uv), _ptr(gate_w), _ptr(gate_b), _ptr(gate_in), _ptr(out), _ptr(cache_out),
        _ptr(open_slot_out), _ptr(workspace), ws, _stream(stream))
    if check and st != OK:
        raise MtlaError(st, "mtla_prefill")
    return st


def prefill_from(cfg, t0, T, c, kr, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in, out, cache,
                 open_slot, workspace, stream=None, check=True) -> int:
    """Forward to ``mtla_prefill_from`` (chunked prefill of T tokens at
    positions t0.. continuing from ``cache`` / ``open_slot``, both in/out);
    returns the status (raises if check)."""
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = load().mtla_prefill_from(
        ctypes.byref(cfg), int(t0), int(T), _ptr(c), _ptr(kr), _ptr(q_c), _ptr(q_r), _ptr(w_uk),
        _ptr(w_uv), _ptr(gate_w), _ptr(gate_b), _ptr(gate_in), _ptr(out), _ptr(cache),
        _ptr(open_slot), _ptr(workspace), ws, _stream(stream))
    if check and st != OK:
        raise MtlaError(st, "mtla_prefill_from")
    return st


BACKWARD_GRADS = ("dc", "dkr", "dq_c", "dq_r", "dw_uk", "dw_uv", "dgate_w", "dgate_b", "dgate_in")


def prefill_backward_workspace_size(cfg: Config, T: int) -> int:
    n = ctypes.c_size_t(0)
    st = load().mtla_prefill_backward_workspace_size(ctypes.byref(cfg), int(T), ctypes.byref(n))
    if st != OK:
        raise MtlaError(st, "mtla_prefill_backward_workspace_size")
    return int(n.value)


def prefill_backward(cfg, T, c, kr, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in, dout, grads: dict,
                     workspace, stream=None, check=True) -> int:
    """Forward to ``mtla_prefill_backward``; ``grads`` maps the names in
    BACKWARD_GRADS to float32 device tensors (None where the gate mode has no
    such gradient). Returns the status (raises if check)."""
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = load().mtla_prefill_backward(
        ctypes.byref(cfg), int(T), _ptr(c), _ptr(kr), _ptr(q_c), _ptr(q_r), _ptr(w_uk), _ptr(w_uv),
        _ptr(gate_w), _ptr(gate_b), _ptr(gate_in), _ptr(dout), *[_ptr(grads.get(k)) for k in BACKWARD_GRADS],
        _ptr(workspace), ws, _stream(stream))
    if check and st != OK:
        raise MtlaError(st, "mtla_prefill_backward")
    return st


def prefill_train_saved_size(cfg: Config, T: int) -> int:
    n = ctypes.c_size_t(0)
    st = load().mtla_prefill_train_saved_size(ctypes.byref(cfg), int(T), ctypes.byref(n))
    if st != OK:
        raise MtlaError(st, "mtla_prefill_train_saved_size")
    return int(n.value)


def prefill_backward_saved_workspace_size(cfg: Config, T: int) -> int:
    n = ctypes.c_size_t(0)
    st = load().mtla_prefill_backward_saved_workspace_size(ctypes.byref(cfg), int(T), ctypes.byref(n))
    if st != OK:
        raise MtlaError(st, "mtla_prefill_backward_saved_workspace_size")
    return int(n.value)


def prefill_train(cfg, T, c, kr, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in, out, saved, stream=None,
                  check=True) -> int:
    """Forward to ``mtla_prefill_train`` (the forward keeping the backward's
    rows in ``saved``, a uint8 device tensor)."""
    st = load().mtla_prefill_train(
        ctypes.byref(cfg), int(T), _ptr(c), _ptr(kr), _ptr(q_c), _ptr(q_r), _ptr(w_uk), _ptr(w_uv), _ptr(gate_w),
        _ptr(gate_b), _ptr(gate_in), _ptr(out), _ptr(saved), saved.numel() * saved.element_size(), _stream(stream))
    if check and st != OK:
        raise MtlaError(st, "mtla_prefill_train")
    return st


def prefill_backward_saved(cfg, T, c, kr, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in, saved, dout,
                           grads: dict, workspace, stream=None, check=True) -> int:
    """Forward to ``mtla_prefill_backward_saved``; ``grads`` as for
    prefill_backward."""
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = load().mtla_prefill_backward_saved(
        ctypes.byref(cfg), int(T), _ptr(c), _ptr(kr), _ptr(q_c), _ptr(q_r), _ptr(w_uk), _ptr(w_uv),
        _ptr(gate_w), _ptr(gate_b), _ptr(gate_in), _ptr(saved), _ptr(dout),
        *[_ptr(grads.get(k)) for k in BACKWARD_GRADS], _ptr(workspace), ws, _stream(stream))
    if check and st != OK:
        raise MtlaError(st, "mtla_prefill_backward_saved")
    return st


def linear(x, w, y, stream=None, check=True) -> int:
    """Forward to ``mtla_linear``: y[M, N] = x[M, K] . w[N, K]^T (bf16)."""
    _bf16(x, w, y)
    M, K = x.shape[-2] if x.dim() > 1 else 1, x.shape[-1]
    M = x.numel() // K
    N = w.shape[0]
    st = load().mtla_linear(_ptr(x), _ptr(w), _ptr(y), int(M), int(N), int(K), _stream(stream))
    if check and st != OK:
        raise MtlaError(st, "mtla_linear")
    return st


def layer_workspace_size(cfg: Config, d_model: int, max_tokens: int = 0) -> int:
    n = ctypes.c_size_t(0)
    st = load().mtla_layer_workspace_size(ctypes.byref(cfg), int(d_model), int(max_tokens), ctypes.byref(n))
    if st != OK:
        raise MtlaError(st, "mtla_layer_workspace_size")
    return int(n.value)


def layer_forward(cfg, d_model, t0, T, h, lw: LayerWeights, gate_w, gate_b, gate_in, y, cache, open_slot,
                  workspace, stream=None, check=True) -> int:
    """Forward to ``mtla_layer_forward`` (the layer over T tokens at t0..)."""
    _bf16(h, y)
    ws = workspace.numel() * workspace.element_size()
    st = load().mtla_layer_forward(ctypes.byref(cfg), int(d_model), int(t0), int(T), _ptr(h), ctypes.byref(lw),
                                   _ptr(gate_w), _ptr(gate_b), _ptr(gate_in), _ptr(y), _ptr(cache),
                                   _ptr(open_slot), _ptr(workspace), ws, _stream(stream))
    if check and st != OK:
        raise MtlaError(st, "mtla_layer_forward")
    return st


def layer_decode_step(cfg, d_model, h, lw: LayerWeights, gate_w, gate_b, gate_in, pos, cache, open_slot, y,
                      workspace, stream=None, check=True) -> int:
    """Forward to ``mtla_layer_decode_step``."""
    _bf16(h, y)
    ws = workspace.numel() * workspace.element_size()
    st = load().mtla_layer_decode_step(ctypes.byref(cfg), int(d_model), _ptr(h), ctypes.byref(lw), _ptr(gate_w),
                                       _ptr(gate_b), _ptr(gate_in), _ptr(pos), _ptr(cache), _ptr(open_slot),
                                       _ptr(y), _ptr(workspace), ws, _stream(stream))
    if check and st != OK:
        raise MtlaError(st, "mtla_layer_decode_step")
    return st


def reorder_cache(cfg, src, n_tokens, cache_in, open_in, cache_out, open_out, stream=None,
                  check=True) -> int:
    """Forward to ``mtla_reorder_cache`` (beam-search reorder of the cache and
    open slots, out of place); returns the status (raises if check)."""
    st = load().mtla_reorder_cache(ctypes.byref(cfg), _ptr(src), _ptr(n_tokens), _ptr(cache_in),
                                   _ptr(open_in), _ptr(cache_out), _ptr(open_out), _stream(stream))
    if check and st != OK:
        raise MtlaError(st, "mtla_reorder_cache")
    return st


def test_wait_timeout(limit_ns: int, scratch, stream=None) -> int:
    """Forward to ``mtla_test_wait_timeout`` (the bounded-wait failure path)."""
    return int(load().mtla_test_wait_timeout(int(limit_ns), _ptr(scratch), _stream(stream)))


def last_error_detail() -> str:
    return load().mtla_last_error_detail().decode()


def get_device_status(stream=None) -> int:
    return int(load().mtla_get_device_status(_stream(stream)))


def kernel_launches() -> int:
    return int(load().mtla_kernel_launches())


class ProfileEvents:
    """Event pairs the library records around its main attention kernel
    (``mtla_set_profile_events``); ``durations_ms()`` after a synchronize."""

    def __init__(self, n_pairs: int):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n_pairs)]
        for e in self.events:          # torch creates the CUDA event at its first record
            e.record()
        torch.cuda.synchronize()
        self._arr = (ctypes.c_void_p * (2 * n_pairs))(*[e.cuda_event for e in self.events])
        self.n = n_pairs

    def __enter__(self):
        load().mtla_set_profile_events(self._arr, self.n)
        return self

    def __exit__(self, *exc):
        self.recorded = int(load().mtla_profile_events_recorded())
        load().mtla_set_profile_events(None, 0)

    def durations_ms(self):
        return [self.events[2 * i].elapsed_time(self.events[2 * i + 1]) for i in range(self.recorded)]


@dataclass
class Buffers:
    """Device buffers of one MTLA problem (weights, cache, open slot, scratch)."""
    cfg: Config
    w_uk: torch.Tensor
    w_uv: torch.Tensor
    gate_w: torch.Tensor
    gate_b: torch.Tensor
    cache: torch.Tensor
    open_slot: torch.Tensor
    workspace: torch.Tensor

    @staticmethod
    def allocate(cfg: Config, weights: dict, max_tokens: int = 0, device="cuda") -> "Buffers":
        dt = cfg.torch_dtype
        ws = workspace_size(cfg, max_tokens)
        return Buffers(
            cfg=cfg,
            w_uk=weights["w_uk"].to(device=device, dtype=dt).contiguous(),
            w_uv=weights["w_uv"].to(device=device, dtype=dt).contiguous(),
            gate_w=weights["gate_w"].to(device=device, dtype=torch.float32).contiguous(),
            gate_b=weights["gate_b"].to(device=device, dtype=torch.float32).contiguous(),
            cache=torch.zeros(cfg.batch, cfg.max_slots, cfg.D, device=device, dtype=dt),
            open_slot=torch.zeros(cfg.batch, cfg.D, device=device, dtype=torch.float32),
            workspace=torch.empty(max(ws, 256), device=device, dtype=torch.uint8),
        )
