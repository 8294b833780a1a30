"""The bounded-wait failure path, on the GPU without a fault: a wait that
nothing completes runs out after a short host-chosen limit, the kernel latches
MTLA_ERR_TIMEOUT and returns, the host reads (and clears) the status, and the
next ordinary call still matches the oracle."""
import time

import numpy as np
import pytest
import torch

import oracle
from gpu_harness import TOL, Problem, np64, oracle_cfg, rel_err
from kv_cache_mtla_b200 import inputs, mtla

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_the_context_stays_usable():
    torch.cuda.synchronize()
    assert mtla.get_device_status() == mtla.OK
    scratch = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    t0 = time.perf_counter()
    assert mtla.test_wait_timeout(100_000, scratch) == mtla.OK         # 100 us
    assert mtla.get_device_status() == mtla.ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert mtla.get_device_status() == mtla.OK                         # cleared by the read
    # an ordinary call afterwards: a prefill and a decode step of the tiny fp32 workload
    wl = inputs.TINY_FP32.with_(s=3)
    T = 20
    w = inputs.weights(wl)
    toks = inputs.tokens(wl, T + 1)
    ref = oracle.prefill(oracle_cfg(wl), toks["c"], toks["kr"], toks["qc"], toks["qr"], w["w_uk"], w["w_uv"],
                         w["gate_w"], w["gate_b"])
    pb = Problem(wl, max_slots=8, max_tokens=T, weights=w)
    out = np64(pb.prefill(toks, T))
    dec = np64(pb.decode(toks, T, [T]))
    assert rel_err(out, ref["out"][:, :T]) <= TOL["fp32"]
    assert rel_err(dec, ref["out"][:, T]) <= TOL["fp32"]
    assert mtla.get_device_status() == mtla.OK


def test_wait_probe_rejects_bad_arguments():
    scratch = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    assert mtla.test_wait_timeout(0, scratch) == mtla.ERR_INVALID_ARG
    assert mtla.test_wait_timeout(2_000_000_000, scratch) == mtla.ERR_INVALID_ARG
    assert mtla.test_wait_timeout(1000, None) == mtla.ERR_INVALID_ARG
