"""CPU tests of the C ABI: the library builds, loads, exports every function
include/*.h declares, and rejects bad arguments on the host before any CUDA
call (no compute calls are made here)."""
import ctypes
import glob
import os
import re
import subprocess

import pytest
import torch

from kv_cache_mtla_b200 import build as kbuild
from kv_cache_mtla_b200 import mtla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return mtla.load()


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(mtla_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_entry_points():
    names = _declared_functions()
    for required in ("mtla_decode_step", "mtla_prefill", "mtla_workspace_size",
                     "mtla_get_device_status", "mtla_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", mtla.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in _declared_functions():
        assert name in exported, f"{name} declared in include/ but not exported"
        assert hasattr(lib, name)


def test_status_strings(lib):
    for code in range(7):
        assert mtla.status_string(code)
    assert mtla.status_string(99) == "unknown status"


def _cfg(**kw):
    base = dict(B=2, H=8, d_h=64, d_c=256, d_r=32, s=2, max_slots=16)
    base.update(kw)
    return mtla.make_config(base["B"], base["H"], base["d_h"], base["d_c"], base["d_r"],
                            base["s"], base["max_slots"])


def test_workspace_size_and_config_checks(lib):
    assert mtla.workspace_size(_cfg(), 0) > 0
    assert mtla.workspace_size(_cfg(), 32) >= mtla.workspace_size(_cfg(), 0)
    bad = {
        "d_c": (24, mtla.ERR_UNSUPPORTED),        # not a multiple of 16
        "d_r": (0, mtla.ERR_INVALID_ARG),
        "H": (129, mtla.ERR_UNSUPPORTED),
        "s": (9, mtla.ERR_UNSUPPORTED),
        "max_slots": (0, mtla.ERR_INVALID_ARG),
        "B": (-1, mtla.ERR_INVALID_ARG),
    }
    for k, (v, code) in bad.items():
        with pytest.raises(mtla.MtlaError) as e:
            mtla.workspace_size(_cfg(**{k: v}), 0)
        assert e.value.status == code, k
    big = _cfg(d_c=512, d_r=80)                    # d_c + d_r > 576
    with pytest.raises(mtla.MtlaError) as e:
        mtla.workspace_size(big, 0)
    assert e.value.status == mtla.ERR_UNSUPPORTED
    n = ctypes.c_size_t(0)
    assert lib.mtla_workspace_size(None, 0, ctypes.byref(n)) == mtla.ERR_INVALID_ARG
    # storage types: bf16, fp32, fp16 accepted; anything else refused
    for dt in (mtla.BF16, mtla.FP32, mtla.FP16):
        cfg = _cfg()
        cfg.dtype = dt
        assert mtla.workspace_size(cfg, 16) > 0
    cfg = _cfg()
    cfg.dtype = 3
    assert lib.mtla_workspace_size(ctypes.byref(cfg), 0, ctypes.byref(n)) == mtla.ERR_INVALID_ARG
    assert mtla.make_config(1, 4, 32, 128, 16, 2, 8, dtype="fp16").torch_dtype == torch.float16


FAKE = 0x10000  # aligned host-side placeholder: argument checks never dereference it


def _decode_args(**over):
    a = dict(c_new=FAKE, kr_new=FAKE, q_c=FAKE, q_r=FAKE, w_uk=FAKE, w_uv=FAKE, gate_w=FAKE,
             gate_b=FAKE, gate_in=None, pos=FAKE, cache=FAKE, open_slot=FAKE, out=FAKE,
             workspace=FAKE)
    a.update(over)
    return a


def _call_decode(lib, cfg, ws_bytes, **over):
    a = _decode_args(**over)
    return lib.mtla_decode_step(ctypes.byref(cfg), a["c_new"], a["kr_new"], a["q_c"], a["q_r"],
                                a["w_uk"], a["w_uv"], a["gate_w"], a["gate_b"], a["gate_in"],
                                a["pos"], a["cache"], a["open_slot"], a["out"], a["workspace"],
                                ws_bytes, None)


def test_decode_rejects_bad_pointers_before_launch(lib):
    cfg = _cfg()
    ws = mtla.workspace_size(cfg, 0)
    for name in ("c_new", "kr_new", "q_c", "q_r", "w_uk", "w_uv", "pos", "cache", "open_slot",
                 "out", "workspace", "gate_w", "gate_b"):
        assert _call_decode(lib, cfg, ws, **{name: None}) == mtla.ERR_INVALID_ARG, name
        assert _call_decode(lib, cfg, ws, **{name: FAKE + 8}) == mtla.ERR_INVALID_ARG, name
    assert _call_decode(lib, cfg, ws - 1) == mtla.ERR_WORKSPACE
    sup = _cfg()
    sup.gate_mode = mtla.GATE_SUPPLIED
    assert _call_decode(lib, sup, ws, gate_w=None, gate_b=None) == mtla.ERR_INVALID_ARG
    unit = _cfg()
    unit.gate_mode = mtla.GATE_UNIT
    # unit gates need no gate pointers; a too-small workspace is still caught on the host
    assert _call_decode(lib, unit, 0, gate_w=None, gate_b=None) == mtla.ERR_WORKSPACE


def _call_prefill(lib, cfg, T, ws_bytes, **over):
    a = dict(c=FAKE, kr=FAKE, q_c=FAKE, q_r=FAKE, w_uk=FAKE, w_uv=FAKE, gate_w=FAKE,
             gate_b=FAKE, gate_in=None, out=FAKE, cache_out=FAKE, open_slot_out=None,
             workspace=FAKE)
    a.update(over)
    return lib.mtla_prefill(ctypes.byref(cfg), T, a["c"], a["kr"], a["q_c"], a["q_r"],
                            a["w_uk"], a["w_uv"], a["gate_w"], a["gate_b"], a["gate_in"],
                            a["out"], a["cache_out"], a["open_slot_out"], a["workspace"],
                            ws_bytes, None)


def test_prefill_rejects_bad_arguments_before_launch(lib):
    cfg = _cfg(max_slots=16)
    ws = mtla.workspace_size(cfg, 32)
    assert _call_prefill(lib, cfg, 0, ws) == mtla.ERR_INVALID_ARG
    assert _call_prefill(lib, cfg, 33, ws) == mtla.ERR_CAPACITY      # ceil(33/2) > 16 slots
    assert _call_prefill(lib, cfg, 32, ws, cache_out=None) == mtla.ERR_INVALID_ARG
    assert _call_prefill(lib, cfg, 32, ws, open_slot_out=FAKE + 4) == mtla.ERR_INVALID_ARG
    assert _call_prefill(lib, cfg, 32, 16) == mtla.ERR_WORKSPACE
    assert _call_prefill(lib, cfg, 32, ws, q_c=None) == mtla.ERR_INVALID_ARG


def test_reorder_rejects_bad_arguments_before_launch(lib):
    """Null or unaligned pointers and overlapping input/output buffers are
    refused on the host, before any CUDA call."""
    cfg = _cfg(B=4, max_slots=16)
    cache_bytes = 4 * 16 * (256 + 32) * 2
    base = dict(src=FAKE, n_tokens=FAKE + 256, cache_in=FAKE + 0x100000, open_in=FAKE + 0x400000,
                cache_out=FAKE + 0x800000, open_out=FAKE + 0xC00000)

    def call(**over):
        a = dict(base)
        a.update(over)
        return lib.mtla_reorder_cache(ctypes.byref(cfg), a["src"], a["n_tokens"], a["cache_in"],
                                      a["open_in"], a["cache_out"], a["open_out"], None)
    for name in base:
        assert call(**{name: None}) == mtla.ERR_INVALID_ARG, name
        assert call(**{name: base[name] + 8}) == mtla.ERR_INVALID_ARG, name
    # the output cache starting inside the input cache, and the open slots in place
    assert call(cache_out=base["cache_in"] + cache_bytes - 16) == mtla.ERR_INVALID_ARG
    assert call(open_out=base["open_in"]) == mtla.ERR_INVALID_ARG
    bad = _cfg(B=4, max_slots=0)
    assert lib.mtla_reorder_cache(ctypes.byref(bad), *base.values(), None) == mtla.ERR_INVALID_ARG


def test_product_imports_nothing_from_the_oracle():
    """The product package must not import, link or call the oracle."""
    pkg = os.path.join(ROOT, "kv_cache_mtla_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*"), recursive=True):
        if not os.path.isfile(path) or path.endswith((".so", ".o", ".pyc")):
            continue
        text = open(path, errors="ignore").read()
        assert "import oracle" not in text and "from oracle" not in text, path
        assert "mtla_oracle" not in text and "orc_" not in text, path


def test_noalloc_limit_matches_header():
    """The binding's copy of MTLA_NOALLOC_SCRATCH_BYTES equals the macro in
    include/mtla.h, so the two cannot drift apart silently."""
    text = open(os.path.join(ROOT, "include", "mtla.h")).read()
    m = re.search(r"#define\s+MTLA_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m, "MTLA_NOALLOC_SCRATCH_BYTES not found in include/mtla.h"
    assert mtla.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_prefill_from_rejects_bad_arguments_on_the_host(lib):
    """mtla_prefill_from: a NULL open slot, a negative start and a chunk past
    the cache are refused before anything touches the device (the pointers
    below are never dereferenced)."""
    cfg = _cfg(max_slots=16)           # s = 2: 32 tokens fit
    fake = 0x10000
    args = [fake] * 4 + [fake, fake, None, None, None, fake, fake]
    ws = 1 << 30
    st = lambda t0, T, open_slot: lib.mtla_prefill_from(
        ctypes.byref(cfg), t0, T, *args, open_slot, fake, ws, None)
    cfg.gate_mode = mtla.GATE_UNIT
    assert st(3, 4, None) == mtla.ERR_INVALID_ARG
    assert st(-1, 4, fake) == mtla.ERR_INVALID_ARG
    assert st(30, 4, fake) == mtla.ERR_CAPACITY      # ceil(34 / 2) = 17 slots > 16


def test_backward_rejects_bad_arguments_on_the_host(lib):
    """mtla_prefill_backward: per-channel gates are refused, T <= 0, a missing
    gradient buffer for the gate mode and a short workspace too, all before
    the device is touched (the pointers below are never dereferenced)."""
    fake = 0x10000
    cfg = _cfg()
    n = mtla.prefill_backward_workspace_size(cfg, 100)
    assert n >= mtla.prefill_backward_workspace_size(cfg, 99) > 0
    cfg.gate_mode = mtla.GATE_CHANNEL_COMPUTED
    with pytest.raises(mtla.MtlaError) as e:
        mtla.prefill_backward_workspace_size(cfg, 100)
    assert e.value.status == mtla.ERR_UNSUPPORTED

    def call(cfg, T, gate, grads, ws_bytes):
        return lib.mtla_prefill_backward(ctypes.byref(cfg), T, *([fake] * 6), *gate, fake, *grads,
                                         fake, ws_bytes, None)

    plain = [fake] * 6
    cfg.gate_mode = mtla.GATE_COMPUTED
    assert call(cfg, 100, [fake, fake, None], plain + [None, None, None], n) == mtla.ERR_INVALID_ARG
    assert call(cfg, 0, [fake, fake, None], plain + [fake, fake, None], n) == mtla.ERR_INVALID_ARG
    assert call(cfg, 100, [fake, fake, None], plain + [fake, fake, None], n - 1) == mtla.ERR_WORKSPACE
    assert call(cfg, 100, [fake, fake, None], plain[:5] + [None] + [fake, fake, None], n) == mtla.ERR_INVALID_ARG
    cfg.gate_mode = mtla.GATE_SUPPLIED
    assert call(cfg, 100, [None, None, fake], plain + [None, None, None], n) == mtla.ERR_INVALID_ARG
    assert call(cfg, 100, [None, None, fake], plain + [None, None, fake + 4], n) == mtla.ERR_INVALID_ARG
    cfg.gate_mode = mtla.GATE_CHANNEL_SUPPLIED
    assert call(cfg, 100, [None, None, fake], plain + [None, None, fake], n) == mtla.ERR_UNSUPPORTED


def test_training_pair_sizes_and_refusals(lib):
    """The training pair exists where the backward runs on the tensor cores
    (bf16, d_h=64, d_R=32, d_c 128 or 256, scalar gates): sizes there,
    UNSUPPORTED elsewhere."""
    cfg = _cfg()
    assert mtla.prefill_train_saved_size(cfg, 300) > 0
    assert 0 < mtla.prefill_backward_saved_workspace_size(cfg, 300) < mtla.prefill_backward_workspace_size(cfg, 300)
    bad = [mtla.make_config(2, 8, 64, 256, 32, 2, 16, dtype="fp32"), _cfg(d_h=32), _cfg(d_c=512, d_r=64)]
    chan = _cfg()
    chan.gate_mode = mtla.GATE_CHANNEL_COMPUTED
    for c in bad + [chan]:
        with pytest.raises(mtla.MtlaError) as e:
            mtla.prefill_train_saved_size(c, 300)
        assert e.value.status == mtla.ERR_UNSUPPORTED


def test_layer_refuses_fp32_and_bad_widths_on_the_host(lib):
    """The layer is bf16 only; d_model must be a positive multiple of 8."""
    cfg = _cfg()
    assert mtla.layer_workspace_size(cfg, 512, 16) > mtla.workspace_size(cfg, 16)
    for dm in (0, 12):
        with pytest.raises(mtla.MtlaError) as e:
            mtla.layer_workspace_size(cfg, dm, 16)
        assert e.value.status == mtla.ERR_INVALID_ARG
    cfg32 = mtla.make_config(2, 8, 64, 256, 32, 2, 16, dtype="fp32")
    with pytest.raises(mtla.MtlaError) as e:
        mtla.layer_workspace_size(cfg32, 512, 16)
    assert e.value.status == mtla.ERR_UNSUPPORTED
