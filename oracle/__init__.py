"""Float64 CPU oracle for the MTLA hot path -- TEST INFRASTRUCTURE.

This package is the yardstick the CUDA library is checked against. Only the
tests, the entry module's ``smoke()`` and the benchmark's CPU-baseline leg may
import it. The product path (``kv_cache_mtla_b200``) never imports, links or
calls anything here, and nothing here calls the product.

The arithmetic lives in ``mtla_oracle.c`` (plain C, float64, optional OpenMP
over independent rows); this module only compiles it with gcc and marshals
numpy arrays through ctypes. See the header of ``mtla_oracle.c`` for the
passages each function follows and the readings taken where the pages are
silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mtla_oracle.c")
_LIB = os.path.join(_HERE, "libmtla_oracle.so")

GATE_COMPUTED, GATE_SUPPLIED, GATE_UNIT = 0, 1, 2
GATE_CHANNEL_COMPUTED, GATE_CHANNEL_SUPPLIED = 3, 4

FAULT_NONE = 0
FAULT_DROP_OWN_PARTIAL = 1
FAULT_MASK_OFF_BY_ONE = 2
FAULT_TRANSPOSE_WUK = 3
FAULT_ROPE_SIGN = 4
FAULT_SCAN_NO_RESET = 5
FAULT_DROP_ROPE_KEY = 6
FAULT_GATE_WRONG_ROW = 7
FAULT_SCALE = 8
FAULT_FREQ_EXPONENT = 9
FAULT_PE_BASE = 10
FAULT_PAIR_ORDER = 11
FAULT_ROPE_HALF_SPLIT = 12
FAULT_PE_SWAP = 13
FAULT_CHUNK_NO_SEED = 14
FAULT_CHUNK_LOCAL_POS = 15
FAULT_CHANNEL_TRANSPOSE = 16
FAULT_BWD_NO_DELTA = 17
FAULT_BWD_PREFIX_SUM = 18
FAULT_BWD_NO_SIGMOID = 19


def build(force: bool = False) -> str:
    """Compile the oracle into ``libmtla_oracle.so`` beside its source."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("d_h", ctypes.c_int32),
        ("d_c", ctypes.c_int32), ("d_r", ctypes.c_int32), ("s", ctypes.c_int32),
        ("gate_mode", ctypes.c_int32), ("scale", ctypes.c_double),
        ("rope_base", ctypes.c_double), ("pe_base", ctypes.c_double),
    ]


@dataclass
class Cfg:
    B: int
    H: int
    d_h: int
    d_c: int
    d_r: int
    s: int
    gate_mode: int = GATE_COMPUTED
    scale: float = 0.0
    rope_base: float = 10000.0
    pe_base: float = 10000.0

    @property
    def D(self) -> int:
        return self.d_c + self.d_r

    def c(self) -> _Cfg:
        return _Cfg(self.B, self.H, self.d_h, self.d_c, self.d_r, self.s, self.gate_mode,
                    self.scale, self.rope_base, self.pe_base)


_lib = None
_P = ctypes.POINTER(ctypes.c_double)
_PI = ctypes.POINTER(ctypes.c_int64)


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.orc_pe.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_double, _P]
        _lib.orc_rope.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_double, _P, _P]
        _lib.orc_gate.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int64, _P, _P, _P, _P]
        _lib.orc_gate.restype = ctypes.c_double
        _lib.orc_gate_channels.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int64, _P, _P, _P, _P, _P]
        _lib.orc_partials.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int32] + [_P] * 7
        _lib.orc_attend_rows.argtypes = ([ctypes.POINTER(_Cfg), ctypes.c_int32] + [_P] * 5
                                         + [ctypes.c_int64, _PI, _P, _P])
        _lib.orc_prefill.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int32] + [_P] * 13
        _lib.orc_decode_step.argtypes = ([ctypes.POINTER(_Cfg), ctypes.c_int32] + [_P] * 9
                                         + [_PI] + [_P] * 5)
        _lib.orc_prefill_explicit.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int32] + [_P] * 10
        _lib.orc_prefill_from.argtypes = [ctypes.POINTER(_Cfg)] + [ctypes.c_int32] * 3 + [_P] * 15
        _lib.orc_set_fault.argtypes = [ctypes.c_int]
        _lib.orc_linear.argtypes = [ctypes.c_int64] * 3 + [_P] * 3
        _lib.orc_prefill_backward.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int32] + [_P] * 19
        _lib.orc_backward_rows.argtypes = ([ctypes.POINTER(_Cfg), ctypes.c_int32] + [_P] * 10 +
                                           [ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, _P, _P])
        _lib.orc_reorder_cache.argtypes = [ctypes.c_int32] * 5 + [ctypes.c_void_p] * 6
        _lib.orc_reorder_cache.restype = ctypes.c_int
    return _lib


def _d(a):
    """float64 C-contiguous copy (or view) of an array-like; None stays None."""
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data_as(_P)


def set_fault(f: int) -> None:
    """Plant one of the FAULT_* mistakes (tests of the pins only)."""
    _load().orc_set_fault(int(f))


def pe(t: int, d: int, base: float = 10000.0) -> np.ndarray:
    out = np.zeros(d)
    _load().orc_pe(t, d, base, _p(out))
    return out


def rope(t: int, x, base: float = 10000.0) -> np.ndarray:
    x = _d(x)
    y = np.zeros_like(x)
    _load().orc_rope(t, x.shape[-1], base, _p(x), _p(y))
    return y


def gate(cfg: Cfg, t: int, c_t, G=None, g=None, w_given=None) -> float:
    c_t = _d(c_t)
    wg = None if w_given is None else np.array([w_given], dtype=np.float64)
    return _load().orc_gate(ctypes.byref(cfg.c()), t, _p(c_t), _p(_d(G)), _p(_d(g)), _p(wg))


def gate_channels(cfg: Cfg, t: int, c_t, G=None, g=None, w_given=None) -> np.ndarray:
    """The D merging weights of token t (per-channel modes; the scalar modes
    repeat their one weight)."""
    c_t = _d(c_t)
    wv = np.zeros(cfg.D)
    wg = None if w_given is None else _d(np.atleast_1d(w_given))
    _load().orc_gate_channels(ctypes.byref(cfg.c()), t, _p(c_t), _p(_d(G)), _p(_d(g)), _p(wg), _p(wv))
    return wv


def partials(cfg: Cfg, c, kr, G=None, g=None, gate_in=None):
    """(w [B,T], P [B,T,D]) -- the block-prefix partial slots."""
    c, kr = _d(c), _d(kr)
    T = c.shape[1]
    w = np.zeros((cfg.B, T))
    P = np.zeros((cfg.B, T, cfg.D))
    G, g, gate_in = _d(G), _d(g), _d(gate_in)
    _load().orc_partials(ctypes.byref(cfg.c()), T, _p(c), _p(kr), _p(G), _p(g), _p(gate_in),
                         _p(w), _p(P))
    return w, P


def attend_rows(cfg: Cfg, qc, qr, w_uk, w_uv, P, rows, want_olat: bool = False):
    """Parallel-form outputs for selected (b, t) rows: out [n,H,d_h] (, olat [n,H,d_c])."""
    qc, qr, w_uk, w_uv, P = _d(qc), _d(qr), _d(w_uk), _d(w_uv), _d(P)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
    T = qc.shape[1]
    n = rows.shape[0]
    out = np.zeros((n, cfg.H, cfg.d_h))
    olat = np.zeros((n, cfg.H, cfg.d_c)) if want_olat else None
    _load().orc_attend_rows(ctypes.byref(cfg.c()), T, _p(qc), _p(qr), _p(w_uk), _p(w_uv), _p(P),
                            n, rows.ctypes.data_as(_PI), _p(out), _p(olat))
    return (out, olat) if want_olat else out


def prefill(cfg: Cfg, c, kr, qc, qr, w_uk, w_uv, G=None, g=None, gate_in=None):
    """Parallel forward from position 0: dict(out, w, cache, acc)."""
    c, kr, qc, qr, w_uk, w_uv = map(_d, (c, kr, qc, qr, w_uk, w_uv))
    G, g, gate_in = _d(G), _d(g), _d(gate_in)
    T = c.shape[1]
    n_slots = (T + cfg.s - 1) // cfg.s
    out = np.zeros((cfg.B, T, cfg.H, cfg.d_h))
    w = np.zeros((cfg.B, T))
    cache = np.zeros((cfg.B, n_slots, cfg.D))
    acc = np.zeros((cfg.B, cfg.D))
    _load().orc_prefill(ctypes.byref(cfg.c()), T, _p(c), _p(kr), _p(qc), _p(qr), _p(w_uk),
                        _p(w_uv), _p(G), _p(g), _p(gate_in), _p(out), _p(w), _p(cache), _p(acc))
    return dict(out=out, w=w, cache=cache, acc=acc)


def prefill_from(cfg: Cfg, t0: int, cache_in, acc_in, c, kr, qc, qr, w_uk, w_uv, G=None, g=None,
                 gate_in=None):
    """Chunked prefill: T new tokens at positions t0.. continuing from the state
    after t0 tokens (``cache_in`` [B, >= floor(t0/s), D], ``acc_in`` [B, D]).
    Returns dict(out [B,T,H,d_h], w [B,T], cache [B, ceil((t0+T)/s), D], acc [B,D])."""
    c, kr, qc, qr, w_uk, w_uv = map(_d, (c, kr, qc, qr, w_uk, w_uv))
    G, g, gate_in = _d(G), _d(g), _d(gate_in)
    cache_in, acc_in = _d(cache_in), _d(acc_in)
    T = c.shape[1]
    n_in = cache_in.shape[1]
    assert n_in >= t0 // cfg.s
    n_out = (t0 + T + cfg.s - 1) // cfg.s
    out = np.zeros((cfg.B, T, cfg.H, cfg.d_h))
    w = np.zeros((cfg.B, T))
    cache = np.zeros((cfg.B, n_out, cfg.D))
    acc = np.zeros((cfg.B, cfg.D))
    _load().orc_prefill_from(ctypes.byref(cfg.c()), int(t0), T, n_in, _p(cache_in), _p(acc_in), _p(c),
                             _p(kr), _p(qc), _p(qr), _p(w_uk), _p(w_uv), _p(G), _p(g), _p(gate_in),
                             _p(out), _p(w), _p(cache), _p(acc))
    return dict(out=out, w=w, cache=cache, acc=acc)


def decode_step(cfg: Cfg, c_new, kr_new, qc, qr, w_uk, w_uv, pos, cache, acc,
                G=None, g=None, gate_in=None, want_olat: bool = False):
    """One incremental step. ``cache`` [B,max_slots,D] and ``acc`` [B,D] are
    float64 numpy arrays updated in place. Returns dict(out, w[, olat])."""
    assert cache.dtype == np.float64 and cache.flags.c_contiguous
    assert acc.dtype == np.float64 and acc.flags.c_contiguous
    c_new, kr_new, qc, qr, w_uk, w_uv = map(_d, (c_new, kr_new, qc, qr, w_uk, w_uv))
    G, g, gate_in = _d(G), _d(g), _d(gate_in)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    out = np.zeros((cfg.B, cfg.H, cfg.d_h))
    w = np.zeros(cfg.B)
    olat = np.zeros((cfg.B, cfg.H, cfg.d_c)) if want_olat else None
    _load().orc_decode_step(ctypes.byref(cfg.c()), cache.shape[1], _p(c_new), _p(kr_new),
                            _p(qc), _p(qr), _p(w_uk), _p(w_uv), _p(G), _p(g), _p(gate_in),
                            pos.ctypes.data_as(_PI), _p(cache), _p(acc), _p(out), _p(w),
                            _p(olat))
    res = dict(out=out, w=w)
    if want_olat:
        res["olat"] = olat
    return res


def prefill_explicit(cfg: Cfg, c, kr, qc, qr, w_uk, w_uv, G=None, g=None, gate_in=None):
    """Non-absorbed parallel forward (explicit per-head k, v): out [B,T,H,d_h]."""
    c, kr, qc, qr, w_uk, w_uv = map(_d, (c, kr, qc, qr, w_uk, w_uv))
    G, g, gate_in = _d(G), _d(g), _d(gate_in)
    T = c.shape[1]
    out = np.zeros((cfg.B, T, cfg.H, cfg.d_h))
    _load().orc_prefill_explicit(ctypes.byref(cfg.c()), T, _p(c), _p(kr), _p(qc), _p(qr),
                                 _p(w_uk), _p(w_uv), _p(G), _p(g), _p(gate_in), _p(out))
    return out


def linear(x, w) -> np.ndarray:
    """y = x . w^T in float64 (x [..., K], w [N, K])."""
    x, w = _d(x), _d(w)
    K = x.shape[-1]
    M = x.size // K
    y = np.zeros(x.shape[:-1] + (w.shape[0],))
    _load().orc_linear(M, w.shape[0], K, _p(np.ascontiguousarray(x.reshape(M, K))), _p(w), _p(y))
    return y


def prefill_backward(cfg: Cfg, c, kr, qc, qr, w_uk, w_uv, dout, G=None, g=None, gate_in=None) -> dict:
    """Gradients of sum(dout * prefill(...)["out"]) with respect to every input
    of the parallel forward from position 0 (scalar gate modes): dict(dc, dkr,
    dqc, dqr, dw_uk, dw_uv, dG, dg, dgate_in) in float64 (``orc_prefill_backward``)."""
    c, kr, qc, qr, w_uk, w_uv, dout = map(_d, (c, kr, qc, qr, w_uk, w_uv, dout))
    G, g, gate_in = _d(G), _d(g), _d(gate_in)
    B, T = c.shape[:2]
    out = dict(dc=np.zeros_like(c), dkr=np.zeros_like(kr), dqc=np.zeros_like(qc), dqr=np.zeros_like(qr),
               dw_uk=np.zeros_like(w_uk), dw_uv=np.zeros_like(w_uv),
               dG=np.zeros((cfg.s, cfg.d_c)), dg=np.zeros(cfg.s), dgate_in=np.zeros((B, T)))
    _load().orc_prefill_backward(ctypes.byref(cfg.c()), T, _p(c), _p(kr), _p(qc), _p(qr), _p(w_uk), _p(w_uv),
                                 _p(G), _p(g), _p(gate_in), _p(dout),
                                 *[_p(out[k]) for k in ("dc", "dkr", "dqc", "dqr", "dw_uk", "dw_uv", "dG", "dg",
                                                        "dgate_in")])
    return out


def backward_rows(cfg: Cfg, c, kr, qc, qr, w_uk, w_uv, dout, rows, G=None, g=None, gate_in=None) -> dict:
    """Query-side gradients dqc [n, H, d_h] and dqr [n, H, d_R] of the rows
    [(b, i)] of the training backward, each computed alone
    (``orc_backward_rows``)."""
    c, kr, qc, qr, w_uk, w_uv, dout = map(_d, (c, kr, qc, qr, w_uk, w_uv, dout))
    G, g, gate_in = _d(G), _d(g), _d(gate_in)
    T = c.shape[1]
    rb = np.ascontiguousarray([r[0] for r in rows], dtype=np.int32)
    ri = np.ascontiguousarray([r[1] for r in rows], dtype=np.int32)
    n = len(rows)
    dqc = np.zeros((n, cfg.H, cfg.d_h))
    dqr = np.zeros((n, cfg.H, cfg.d_r))
    _load().orc_backward_rows(ctypes.byref(cfg.c()), T, _p(c), _p(kr), _p(qc), _p(qr), _p(w_uk), _p(w_uv),
                              _p(G), _p(g), _p(gate_in), _p(dout), n, rb.ctypes.data, ri.ctypes.data, _p(dqc),
                              _p(dqr))
    return dict(dqc=dqc, dqr=dqr)


def layer_forward(cfg: Cfg, t0: int, cache_in, acc_in, h, W: dict, G=None, g=None, gate_in=None):
    """The MTLA layer around the path, T tokens at positions t0.. continuing
    from the cache state after t0 tokens ("Multi-head Temporal Latent
    Attention", Method: MLA's low-rank compression kept -- h_t projected to the
    shared latent c_t and the decoupled key k_t, the queries projected per
    head; "Multi-Head Latent Attention and Sparse Indexers": the heads' outputs
    concatenated and projected back by W_O):
      c = h W_DKV^T [B,T,d_c]    k = h W_KR^T [B,T,d_R]
      qC = h W_Q^T [B,T,H,d_h]   qR = h W_QR^T [B,T,H,d_R]
      o = the path (prefill_from) [B,T,H,d_h]   y = o W_O^T [B,T,d_model]
    W holds w_dkv [d_c,dm], w_kr [d_R,dm], w_q [H*d_h,dm], w_qr [H*d_R,dm],
    w_uk, w_uv [H,d_h,d_c], w_o [dm, H*d_h]. Returns dict(y, cache, acc)."""
    h = _d(h)
    B, T, _ = h.shape
    c = linear(h, W["w_dkv"])
    kr = linear(h, W["w_kr"])
    qc = linear(h, W["w_q"]).reshape(B, T, cfg.H, cfg.d_h)
    qr = linear(h, W["w_qr"]).reshape(B, T, cfg.H, cfg.d_r)
    r = prefill_from(cfg, t0, cache_in, acc_in, c, kr, qc, qr, W["w_uk"], W["w_uv"], G, g, gate_in)
    y = linear(r["out"].reshape(B, T, cfg.H * cfg.d_h), W["w_o"])
    return dict(y=y, cache=r["cache"], acc=r["acc"])


def reorder_cache(s: int, src, n_tokens, cache_in, open_in, cache_out, open_out) -> int:
    """Beam-search reorder: destination b takes the filled slots and the open
    slot of parent src[b] (``orc_reorder_cache``). ``cache_in``/``cache_out``
    [B,max_slots,D] of any element type (copied as bytes; pass bf16 as its
    uint16 bits), ``open_in``/``open_out`` [B,D] float32; the outputs are
    numpy arrays updated in place. Returns the status (0, 1 or 3)."""
    for a in (cache_in, cache_out, open_in, open_out):
        assert isinstance(a, np.ndarray) and a.flags.c_contiguous
    assert cache_in.dtype == cache_out.dtype and cache_in.shape == cache_out.shape
    assert open_in.dtype == np.float32 and open_out.dtype == np.float32
    B, max_slots, D = cache_in.shape
    src = np.ascontiguousarray(src, dtype=np.int32)
    n_tokens = np.ascontiguousarray(n_tokens, dtype=np.int32)
    return int(_load().orc_reorder_cache(B, max_slots, D, int(s), cache_in.itemsize,
                                         src.ctypes.data, n_tokens.ctypes.data, cache_in.ctypes.data,
                                         open_in.ctypes.data, cache_out.ctypes.data, open_out.ctypes.data))
