#!/usr/bin/env python
"""Throughput of the MTLA hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mtla|reference]

Contract line (per rank; weak scaling, every rank runs an independent replica):
the large-latent decode -- B=32 sequences, H=128, d_h=128, d_c=512, d_R=64
(slot width 576, 1152 bytes), s=4, supplied gates sigmoid(N(0,1)). One step =
256 consecutive incremental decode steps of every sequence at positions
65280..65535, so each decode step attends 16321..16384 slots per sequence and
the cache ends holding N=65536 tokens: gate, RoPE of the new key, in-place
update of the slot being filled, query absorption through W_UK, stride-aware
masked attention over the slots (split over the SMs), merge of the splits and
output absorption through W_UV. The 604 MB cache is larger than the 126 MB L2,
and the L2 is also flushed before every step (outside the timed events).

`value` = latent-cache bytes read by the attention (slots attended x 1152 B)
per second over all ranks, from CUDA events around each step on the launching
stream; the 256 decode steps run as one CUDA graph captured through the public
API. `decode` gives the same run in tokens/s. `roofline` is the dominant kernel
(the decode attention) timed by event pairs the library records around each of
its launches in one profiled replay. `e2e` times the same steps through the
public API with every step's inputs (the 256 tokens' latents, keys, queries,
gates and positions) copied from pinned host memory and its outputs copied
back inside one timed region, pipelined on a copy stream.

Sub-objects measure the other workloads, each over its own clock-sampled timed
region: `prefill` (B=8, T=8192, s=2: TFLOP/s of the masked attention),
`layer` (the same sizes through the whole layer with d_model=512: the
projections, the path and W_O; and the largest projection GEMM alone),
`speech_decode` (B=16, H=8, a 1024-token prefix then 256 decode steps:
decode tokens/s separately from the prefix), `stride_sweep` (B=64, N=4096,
s=1..4: latent-cache GB/s of one decode step). `cpu_baseline` and
`--impl reference` time the float64 CPU oracle on a bounded sample of the
contract workload (a few of its sequences, one decode step each).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_mtla_b200 import inputs, mtla  # noqa: E402

METRIC = "decode latent-cache GB/s and tokens/s at N/s slots; prefill TFLOP/s; % roofline"
WL = inputs.LARGE_LATENT
GEN_STEPS = 256          # decode steps per sequence in one contract step


def _traffic(kernel, launch_scale=1.0):
    """DRAM bytes (read + write) of one launch of `kernel` from the committed ncu
    capture, scaled by `launch_scale` (units of the timed launch over units of
    the captured one), or None when the kernel's sources changed since the
    capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
        h = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["sources_sha256"]:
            return None
        return (rec["dram_bytes_read"] + rec["dram_bytes_write"]) * launch_scale
    except (OSError, KeyError, ValueError):
        return None


class L2Flush:
    """Evicts the 126 MB L2 between timed iterations: a 256 MiB write, then a
    256 MiB read of another buffer. The read leaves clean lines behind, so the
    timed kernels do not also pay for writing the flush's dirty lines back to
    HBM (up to a full L2 of them after the write alone)."""

    def __init__(self):
        n = 64 * 1024 * 1024                       # 256 MiB of fp32 each
        self.w = torch.empty(n, dtype=torch.float32, device="cuda")
        self.r = torch.ones(n, dtype=torch.float32, device="cuda")
        self.acc = torch.zeros(1, dtype=torch.float32, device="cuda")

    def __call__(self):
        self.w.zero_()
        self.acc += self.r.sum()

    desc = "flushed (256 MiB write, then 256 MiB read) before every timed"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return ws, rank


def _max_over_ranks(x: float, ws: int) -> float:
    """The largest of every rank's x (all ranks call it, in the same order)."""
    if ws == 1:
        return x
    dev = "cuda" if torch.cuda.is_available() else "cpu"   # cpu: gloo process groups
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def _barrier(ws: int):
    if ws > 1:
        torch.distributed.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def job_value(units_per_rank_step: float, ws: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's device time (weak scaling: every rank has the same per-step work)."""
    return units_per_rank_step * ws * steps / (max_ms / 1e3)


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region. The
    sampler is started before the region and the region begins only once the
    first sample has arrived (or after 3 s), so a region of T seconds holds
    about T / 50 ms samples."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index: int):
        self.dev = dev_index
        self.proc = None
        self.path = f"/tmp/mtla_clocks_{os.getpid()}_{id(self)}.csv"

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return self
        t0 = time.time()
        while time.time() - t0 < 3.0 and os.path.getsize(self.path) == 0:
            time.sleep(0.02)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        sms, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        return {"sm_mhz": statistics.median(sms) if sms else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sms)}


def _events(n, k=2):
    return [tuple(torch.cuda.Event(enable_timing=True) for _ in range(k)) for _ in range(n)]


# --------------------------------------------------------------------- contract


class LargeLatentReplica:
    """One rank's large-latent decode: weights, a cache holding 65280 tokens,
    and the inputs of 256 decode steps of every sequence, on the device."""

    def __init__(self, rank: int):
        wl = WL.with_(seed=WL.seed + 1000 * rank)
        self.wl = wl
        self.S = GEN_STEPS
        self.N0 = wl.T - self.S                           # tokens cached before the step
        self.max_slots = (wl.T + wl.s - 1) // wl.s        # 16384
        self.cfg = mtla.make_config(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, self.max_slots,
                                    dtype=wl.dtype, gate_mode=wl.gate_mode)
        self.buf = mtla.Buffers.allocate(self.cfg, inputs.weights(wl))
        c0 = inputs.synthetic_cache(wl, self.N0, self.max_slots)
        self.buf.cache.copy_(c0["cache"].to(torch.bfloat16))
        self.buf.open_slot.copy_(c0["acc"])
        del c0
        bf = torch.bfloat16
        tk = inputs.tokens(wl, self.S, stream=1)
        # host copies (pinned) of one step's inputs, step-major [S, B, ...]
        self.h = {k: tk[k].transpose(0, 1).to(bf).contiguous().pin_memory()
                  for k in ("c", "kr", "qc", "qr")}
        self.h["gate_in"] = tk["gate_in"].transpose(0, 1).contiguous().pin_memory()
        self.h["pos"] = (self.N0 + torch.arange(self.S, dtype=torch.int32)).repeat_interleave(
            wl.B).view(self.S, wl.B).contiguous().pin_memory()
        self.d = {k: v.to("cuda") for k, v in self.h.items()}
        self.out = torch.empty(self.S, wl.B, wl.H, wl.d_h, device="cuda", dtype=bf)
        self.h_out = torch.empty(self.out.shape, dtype=bf).pin_memory()
        self.h2d_bytes = sum(v.numel() * v.element_size() for v in self.h.values())
        self.d2h_bytes = self.out.numel() * 2
        self.tokens_per_step = wl.B * self.S
        self.slots = [(self.N0 + k) // wl.s + 1 for k in range(self.S)]
        self.slot_bytes = wl.D * 2
        self.bytes_per_step = wl.B * self.slot_bytes * sum(self.slots)
        self.sets = [(self.d, self.out)]

    def add_set(self):
        self.sets.append(({k: torch.empty_like(v) for k, v in self.d.items()},
                          torch.empty_like(self.out)))

    def use(self, j: int):
        self.d, self.out = self.sets[j]

    def decode(self, k: int):
        b, d = self.buf, self.d
        mtla.decode_step(self.cfg, d["c"][k], d["kr"][k], d["qc"][k], d["qr"][k], b.w_uk, b.w_uv,
                         None, None, d["gate_in"][k], d["pos"][k], b.cache, b.open_slot,
                         self.out[k], b.workspace)

    def step(self):
        for k in range(self.S):
            self.decode(k)


def _capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def measure_contract(args, ws, rank):
    """The large-latent decode: device-timed steps, the profiled attention
    launches, and the end-to-end pipeline with host buffers."""
    rep = LargeLatentReplica(rank)
    flush = L2Flush()
    st = torch.cuda.current_stream()
    rep.step()                                     # eager warm-up, sets up per-device state
    torch.cuda.synchronize()
    assert mtla.get_device_status() == mtla.OK

    cap = torch.cuda.Stream()
    cap.wait_stream(st)
    n0 = mtla.kernel_launches()
    g0 = _capture(rep.step, cap)
    kernels_per_step = mtla.kernel_launches() - n0
    prof = mtla.ProfileEvents(rep.S)
    with prof:
        g_prof = _capture(rep.step, cap)
    rep.add_set()
    rep.use(1)
    g1 = _capture(rep.step, cap)
    rep.use(0)
    st.wait_stream(cap)
    graphs = (g0, g1)

    for i in range(args.warmup):
        flush()
        graphs[i & 1].replay()
    flush()
    g_prof.replay()
    torch.cuda.synchronize()
    assert mtla.get_device_status() == mtla.OK

    # ---- device-timed steps
    evs = _events(args.steps)
    _barrier(ws)
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            flush()
            evs[i][0].record(st)
            g0.replay()
            evs[i][1].record(st)
        torch.cuda.synchronize()
    clocks = clk.summary()
    _barrier(ws)
    assert mtla.get_device_status() == mtla.OK
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = _max_over_ranks(sum(step_ms), ws)
    value = job_value(rep.bytes_per_step / 1e9, ws, args.steps, total_ms)
    tokens_s = job_value(rep.tokens_per_step, ws, args.steps, total_ms)

    # ---- dominant kernel: the decode attention, from the profiled replay
    attn_ms = statistics.mean(prof.durations_ms())
    hbm, _, peak_kind = _peaks()
    attn_bytes = rep.bytes_per_step / rep.S
    achieved = attn_bytes / (attn_ms / 1e3) / 1e9
    traffic = _traffic("k_lh_attn", launch_scale=statistics.mean(rep.slots) / rep.max_slots)

    # ---- end to end through the public API with host buffers
    e2e_ms = _e2e(rep, graphs, flush, args.steps, ws)
    e2e_value = job_value(rep.bytes_per_step / 1e9, ws, args.steps, e2e_ms)
    wl = rep.wl
    return {
        "value": value, "ms_per_step": total_ms / args.steps, "clocks": clocks,
        "gpu_launches": kernels_per_step * args.steps,
        "decode": {"tokens_per_s": tokens_s,
                   "ms_per_token_step": total_ms / args.steps / rep.S,
                   "latent_cache_GBps": value, "slots_per_seq": [rep.slots[0], rep.slots[-1]],
                   "kernels_per_token_step": kernels_per_step // rep.S},
        "roofline": {"kernel": "k_lh_attn (decode attention)", "bound": "hbm",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": traffic, "peak_source": f"{peak_kind} hbm_gbs (burst copy)",
                     "bytes_per_launch": attn_bytes, "avg_launch_us": attn_ms * 1e3,
                     "timing": f"CUDA event pairs recorded by the library around each of the "
                               f"{rep.S} attention launches of one profiled replay of the step "
                               f"(not counted in value)"},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": rep.h2d_bytes,
                "d2h_bytes_per_step": rep.d2h_bytes,
                "tokens_per_s": job_value(rep.tokens_per_step, ws, args.steps, e2e_ms),
                "pipeline": "one timed region over all steps: inputs of step i+1 copied in "
                            "(pinned, copy stream) while step i computes, outputs of step i "
                            "copied out while step i+1 computes; L2 flush before each step "
                            "inside the region"},
        "config": {"workload": f"large_latent decode: B={wl.B}/rank, H={wl.H}, d_h={wl.d_h}, "
                               f"d_c={wl.d_c}, d_R={wl.d_r}, s={wl.s}, supplied gates; "
                               f"{rep.S} decode steps per sequence at positions "
                               f"{rep.N0}..{wl.T - 1} ({rep.slots[0]}..{rep.slots[-1]} slots)",
                   "global_batch": wl.B * ws, "seq_len": wl.T, "decode_steps_per_step": rep.S,
                   "parallelism": f"replicas x{ws} (independent sequences)",
                   "l2": "cache (604 MB) larger than L2; also " + L2Flush.desc + " step"},
    }


def _e2e(rep, graphs, flush, K, ws):
    """One timed region over K steps: every step's inputs copied from pinned
    host memory into one of two device sets and its outputs copied back, on a
    copy stream, overlapping the neighbouring steps' compute."""
    st = torch.cuda.current_stream()
    cs = torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=False)
    e_beg, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    in_done, comp_done, out_done = [ev() for _ in range(K)], [ev() for _ in range(K)], [ev() for _ in range(K)]

    def copy_in(i):
        d = rep.sets[i & 1][0]
        for k, v in rep.h.items():
            d[k].copy_(v, non_blocking=True)
        in_done[i].record(cs)

    _barrier(ws)
    torch.cuda.synchronize()
    e_beg.record(st)
    cs.wait_event(e_beg)
    with torch.cuda.stream(cs):
        copy_in(0)
    for i in range(K):
        j = i & 1
        if i + 1 < K:
            with torch.cuda.stream(cs):
                if i >= 1:
                    cs.wait_event(comp_done[i - 1])     # step i-1 read the set step i+1 uses
                copy_in(i + 1)
        if i >= 2:
            st.wait_event(out_done[i - 2])               # outputs of step i-2 (same set) copied out
        st.wait_event(in_done[i])
        flush()
        graphs[j].replay()
        comp_done[i].record(st)
        with torch.cuda.stream(cs):
            cs.wait_event(comp_done[i])
            rep.h_out.copy_(rep.sets[j][1], non_blocking=True)
            out_done[i].record(cs)
    st.wait_event(out_done[K - 1])
    e_end.record(st)
    torch.cuda.synchronize()
    _barrier(ws)
    assert mtla.get_device_status() == mtla.OK
    return _max_over_ranks(e_beg.elapsed_time(e_end), ws)


# ------------------------------------------------------------- other workloads


def _timed_calls(call, n, flush, ws, profile=True):
    """n calls, each after an L2 flush, each between CUDA events; returns
    (median call ms, median attention-kernel ms or None, clocks), the
    medians taken as the max over ranks."""
    st = torch.cuda.current_stream()
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    evs = _events(n)
    prof = mtla.ProfileEvents(n) if profile else None
    _barrier(ws)
    with ClockSampler(torch.cuda.current_device()) as clk:
        if prof:
            prof.__enter__()
        for i in range(n):
            flush()
            evs[i][0].record(st)
            call()
            evs[i][1].record(st)
        torch.cuda.synchronize()
        if prof:
            prof.__exit__(None, None, None)
    assert mtla.get_device_status() == mtla.OK
    call_ms = _max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in evs), ws)
    kern_ms = _max_over_ranks(statistics.median(prof.durations_ms()), ws) if prof else None
    return call_ms, kern_ms, clk.summary()


def measure_prefill(n, flush, ws, rank):
    """Parallel prefill B=8, T=8192, s=2: the block-prefix scan and the
    stride-aware masked attention with absorption on both sides."""
    _, tflops_peak, peak_kind = _peaks()
    wl = inputs.PREFILL.with_(seed=inputs.PREFILL.seed + 1000 * rank)
    T = wl.T
    cfg = mtla.make_config(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, (T + wl.s - 1) // wl.s,
                           dtype=wl.dtype, gate_mode=wl.gate_mode)
    buf = mtla.Buffers.allocate(cfg, inputs.weights(wl), max_tokens=T)
    tk = inputs.tokens(wl, T)
    d = {k: tk[k].to("cuda", torch.bfloat16).contiguous() for k in ("c", "kr", "qc", "qr")}
    out = torch.empty(wl.B, T, wl.H, wl.d_h, device="cuda", dtype=torch.bfloat16)

    def call():
        mtla.prefill(cfg, T, d["c"], d["kr"], d["qc"], d["qr"], buf.w_uk, buf.w_uv, buf.gate_w,
                     buf.gate_b, None, out, buf.cache, buf.open_slot, buf.workspace)
    call_ms, kern_ms, clocks = _timed_calls(call, n, flush, ws)
    pairs = sum(t // wl.s + 1 for t in range(T))
    flops = 2 * pairs * (wl.D + wl.d_c) * wl.B * wl.H
    kern = flops / (kern_ms / 1e3) / 1e12
    return {"workload": f"prefill: B={wl.B}/rank, T={T}, H={wl.H}, d_h={wl.d_h}, d_c={wl.d_c}, "
                        f"d_R={wl.d_r}, s={wl.s}, computed gates",
            "TFLOPs": flops * ws / (call_ms / 1e3) / 1e12, "call_ms": call_ms,
            "attention_flops_per_call": flops, "calls": n,
            "roofline": {"kernel": "k_prefill_tc (masked attention with absorption)",
                         "bound": "tensor", "achieved": kern, "peak": tflops_peak,
                         "unit": "TFLOP/s", "frac": kern / tflops_peak,
                         "traffic": _traffic("k_prefill_tc"),
                         "peak_source": f"{peak_kind} bf16_tflops (burst)",
                         "avg_launch_us": kern_ms * 1e3},
            "clocks": clocks, "l2": L2Flush.desc + " call"}


def _backward_traffic():
    """DRAM bytes of the two tensor-core backward kernels of one call (their
    captures at this workload), or None when either's sources changed."""
    dq, dk = _traffic("k_bwd_dq_tc"), _traffic("k_bwd_dk_tc")
    return None if dq is None or dk is None else dq + dk


def measure_backward(n, flush, ws, rank):
    """Training backward at the prefill workload's sizes (B=8, T=8192, H=8,
    d_h=64, d_c=256, d_R=32, s=2, computed gates): every gradient of the path
    through mtla_prefill_backward; its masked-attention part (the two
    tensor-core kernels) against the bf16 peak."""
    _, tflops_peak, peak_kind = _peaks()
    wl = inputs.PREFILL.with_(seed=inputs.PREFILL.seed + 1000 * rank)
    T = wl.T
    cfg = mtla.make_config(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, 1, dtype=wl.dtype, gate_mode=wl.gate_mode)
    w = inputs.weights(wl)
    tk = inputs.tokens(wl, T)
    d = {k: tk[k].to("cuda", torch.bfloat16).contiguous() for k in ("c", "kr", "qc", "qr")}
    dw = {k: w[k].to("cuda", torch.bfloat16 if k.startswith("w_") else torch.float32).contiguous() for k in w}
    dout = inputs.grad_out(wl, T).to("cuda", torch.bfloat16)
    B, H = wl.B, wl.H
    g = dict(dc=(B, T, wl.d_c), dkr=(B, T, wl.d_r), dq_c=(B, T, H, wl.d_h), dq_r=(B, T, H, wl.d_r),
             dw_uk=(H, wl.d_h, wl.d_c), dw_uv=(H, wl.d_h, wl.d_c), dgate_w=(wl.s, wl.d_c), dgate_b=(wl.s,))
    grads = {k: torch.empty(v, device="cuda") for k, v in g.items()}
    wsb = torch.empty(mtla.prefill_backward_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")

    def call():
        mtla.prefill_backward(cfg, T, d["c"], d["kr"], d["qc"], d["qr"], dw["w_uk"], dw["w_uv"], dw["gate_w"],
                              dw["gate_b"], None, dout, grads, wsb)
    call_ms, kern_ms, clocks = _timed_calls(call, n, flush, ws)
    # the training pair: the forward keeping the backward's rows, and the
    # backward from them (no forward recompute)
    saved = torch.empty(mtla.prefill_train_saved_size(cfg, T), dtype=torch.uint8, device="cuda")
    out_t = torch.empty(B, T, H, wl.d_h, device="cuda", dtype=torch.bfloat16)
    ws_s = torch.empty(mtla.prefill_backward_saved_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    targs = (d["c"], d["kr"], d["qc"], d["qr"], dw["w_uk"], dw["w_uv"], dw["gate_w"], dw["gate_b"], None)
    fwd_ms, _, _ = _timed_calls(lambda: mtla.prefill_train(cfg, T, *targs, out_t, saved), n, flush, ws,
                                profile=False)
    bws_ms, _, _ = _timed_calls(lambda: mtla.prefill_backward_saved(cfg, T, *targs, saved, dout, grads, ws_s), n,
                                flush, ws, profile=False)
    pairs = sum(t // wl.s + 1 for t in range(T))
    # per (row, key) pair: the score and dobar.key dot products, dq, dkey and its
    # latent (value) part: 2 (3 D + 2 d_c) flops
    flops = 2 * pairs * (3 * wl.D + 2 * wl.d_c) * B * H
    kern = flops / (kern_ms / 1e3) / 1e12
    return {"workload": f"training backward: B={B}/rank, T={T}, H={H}, d_h={wl.d_h}, d_c={wl.d_c}, "
                        f"d_R={wl.d_r}, s={wl.s}, computed gates, bf16 inputs, fp32 gradients",
            "TFLOPs": flops * ws / (call_ms / 1e3) / 1e12, "call_ms": call_ms,
            "training_pair": {"forward_keeping_rows_ms": fwd_ms, "backward_from_kept_rows_ms": bws_ms,
                              "note": "mtla_prefill_train then mtla_prefill_backward_saved: no forward recompute"},
            "attention_flops_per_call": flops, "calls": n,
            "roofline": {"kernel": "k_bwd_dq_tc + k_bwd_dk_tc (masked attention backward, tensor cores)",
                         "bound": "tensor", "achieved": kern, "peak": tflops_peak, "unit": "TFLOP/s",
                         "frac": kern / tflops_peak, "traffic": _backward_traffic(),
                         "peak_source": f"{peak_kind} bf16_tflops (burst)",
                         "avg_launch_us": kern_ms * 1e3},
            "clocks": clocks, "l2": L2Flush.desc + " call"}


def measure_speech(n, flush, ws, rank, dtype="bf16"):
    """Speech-model-scale decode B=16, H=8, s=2: a 1024-token prefix by the
    prefill, then 256 decode steps (513..640 slots), as two CUDA graphs
    (bf16 storage, or fp16 with dtype="fp16")."""
    wl = inputs.SPEECH_DECODE.with_(seed=inputs.SPEECH_DECODE.seed + 1000 * rank, dtype=dtype)
    T, S = wl.T, wl.steps
    max_slots = (T + S + wl.s - 1) // wl.s
    cfg = mtla.make_config(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, max_slots, dtype=wl.dtype,
                           gate_mode=wl.gate_mode)
    buf = mtla.Buffers.allocate(cfg, inputs.weights(wl), max_tokens=T)
    bf = cfg.torch_dtype
    pre = inputs.tokens(wl, T, stream=0)
    dec = inputs.tokens(wl, S, stream=1)
    dp = {k: pre[k].to("cuda", bf).contiguous() for k in ("c", "kr", "qc", "qr")}
    dd = {k: dec[k].transpose(0, 1).to("cuda", bf).contiguous() for k in ("c", "kr", "qc", "qr")}
    pos = (T + torch.arange(S, dtype=torch.int32)).repeat_interleave(wl.B).view(S, wl.B).cuda()
    out_p = torch.empty(wl.B, T, wl.H, wl.d_h, device="cuda", dtype=bf)
    out_d = torch.empty(S, wl.B, wl.H, wl.d_h, device="cuda", dtype=bf)

    def prefill():
        mtla.prefill(cfg, T, dp["c"], dp["kr"], dp["qc"], dp["qr"], buf.w_uk, buf.w_uv,
                     buf.gate_w, buf.gate_b, None, out_p, buf.cache, buf.open_slot, buf.workspace)

    def decode():
        for k in range(S):
            mtla.decode_step(cfg, dd["c"][k], dd["kr"][k], dd["qc"][k], dd["qr"][k], buf.w_uk,
                             buf.w_uv, buf.gate_w, buf.gate_b, None, pos[k], buf.cache,
                             buf.open_slot, out_d[k], buf.workspace)
    st = torch.cuda.current_stream()
    prefill()
    decode()
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    cap.wait_stream(st)
    g_pre, g_dec = _capture(prefill, cap), _capture(decode, cap)
    prof = mtla.ProfileEvents(S)
    with prof:
        g_prof = _capture(decode, cap)
    st.wait_stream(cap)
    for _ in range(3):
        flush()
        g_pre.replay()
        g_dec.replay()
    flush()
    g_pre.replay()
    g_prof.replay()
    torch.cuda.synchronize()
    evs = _events(n, 3)
    _barrier(ws)
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(n):
            flush()
            evs[i][0].record(st)
            g_pre.replay()
            evs[i][1].record(st)
            g_dec.replay()
            evs[i][2].record(st)
        torch.cuda.synchronize()
    assert mtla.get_device_status() == mtla.OK
    pre_ms = _max_over_ranks(sum(a.elapsed_time(b) for a, b, c in evs), ws)
    dec_ms = _max_over_ranks(sum(b.elapsed_time(c) for a, b, c in evs), ws)
    slots = [(T + k) // wl.s + 1 for k in range(S)]
    hbm, _, peak_kind = _peaks()
    attn_ms = statistics.mean(prof.durations_ms())
    attn_bytes = wl.B * wl.D * 2 * statistics.mean(slots)
    return {"workload": f"speech_decode: B={wl.B}/rank, H={wl.H}, d_h={wl.d_h}, d_c={wl.d_c}, "
                        f"d_R={wl.d_r}, s={wl.s}, {wl.dtype} storage; prefill {T} tokens then {S} decode steps",
            "decode_tokens_per_s": wl.B * S * ws * n / (dec_ms / 1e3),
            "ms_per_token_step": dec_ms / n / S,
            "decode_latent_cache_GBps": wl.B * wl.D * 2 * sum(slots) * ws * n / (dec_ms / 1e3) / 1e9,
            "prefix_prefill_ms": pre_ms / n,
            "prefix_tokens_per_s": wl.B * T * ws * n / (pre_ms / 1e3),
            "steps": n, "slots_per_seq": [slots[0], slots[-1]],
            "roofline": {"kernel": "k_dec_attn_sh (decode attention)", "bound": "hbm",
                         "achieved": attn_bytes / (attn_ms / 1e3) / 1e9, "peak": hbm,
                         "unit": "GB/s", "frac": attn_bytes / (attn_ms / 1e3) / 1e9 / hbm,
                         "traffic": _traffic("k_dec_attn_sh") if wl.dtype == "bf16" else None,
                         "peak_source": f"{peak_kind} hbm_gbs", "avg_launch_us": attn_ms * 1e3},
            "clocks": clk.summary(), "cuda_graphs": "prefill graph + 256-step decode graph",
            "l2": L2Flush.desc + " step"}


def measure_layer(n, flush, ws, rank):
    """The MTLA layer around the path at the prefill workload's sizes (B=8,
    T=8192, d_model=512, H=8, d_h=64, d_c=256, d_R=32, s=2): the four input
    projections, the path, the output projection, all through
    mtla_layer_forward; and the largest projection GEMM alone (65536 x 512 x
    512) against the bf16 peak."""
    _, tflops_peak, peak_kind = _peaks()
    wl = inputs.PREFILL.with_(seed=inputs.PREFILL.seed + 1000 * rank)
    dm, T = 512, wl.T
    cfg = mtla.make_config(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, (T + wl.s - 1) // wl.s,
                           gate_mode=wl.gate_mode)
    W = inputs.layer_weights(wl, dm)
    dW = {k: v.to("cuda", torch.bfloat16 if k.startswith("w_") else torch.float32).contiguous()
          for k, v in W.items()}
    lw = mtla.layer_weights(dW)
    wsb = torch.empty(mtla.layer_workspace_size(cfg, dm, T), dtype=torch.uint8, device="cuda")
    cache = torch.empty(wl.B, cfg.max_slots, wl.D, dtype=torch.bfloat16, device="cuda")
    op = torch.zeros(wl.B, wl.D, dtype=torch.float32, device="cuda")
    h = inputs.hidden(wl, dm, T).to("cuda", torch.bfloat16)
    y = torch.empty(wl.B, T, dm, dtype=torch.bfloat16, device="cuda")

    def call():
        mtla.layer_forward(cfg, dm, 0, T, h, lw, dW["gate_w"], dW["gate_b"], None, y, cache, op, wsb)
    call_ms, attn_ms, clocks = _timed_calls(call, n, flush, ws)
    M = wl.B * T
    proj = 2 * M * dm * (wl.d_c + wl.d_r + wl.H * wl.d_h + wl.H * wl.d_r)
    outp = 2 * M * wl.H * wl.d_h * dm
    pairs = sum(t // wl.s + 1 for t in range(T))
    attn = 2 * pairs * (wl.D + wl.d_c) * wl.B * wl.H
    # the largest projection alone
    x = torch.randn(M, dm, device="cuda").to(torch.bfloat16)
    wq = dW["w_q"]
    yq = torch.empty(M, wq.shape[0], dtype=torch.bfloat16, device="cuda")
    g_ms, _, g_clocks = _timed_calls(lambda: mtla.linear(x, wq, yq), 4 * n, flush, ws, profile=False)
    g_flops = 2 * M * dm * wq.shape[0]
    g_tf = g_flops / (g_ms / 1e3) / 1e12
    return {"workload": f"layer: B={wl.B}/rank, T={T}, d_model={dm}, H={wl.H}, d_h={wl.d_h}, d_c={wl.d_c}, "
                        f"d_R={wl.d_r}, s={wl.s}: 4 input projections, the path, the output projection",
            "call_ms": call_ms, "attention_kernel_ms": attn_ms,
            "TFLOPs": (proj + outp + attn) * ws / (call_ms / 1e3) / 1e12,
            "flops_per_call": {"projections": proj, "output_projection": outp, "attention": attn},
            "clocks": clocks,
            "gemm": {"shape": f"{M} x {wq.shape[0]} x {dm} (M x N x K)", "ms": g_ms,
                     "roofline": {"kernel": "k_gemm", "bound": "tensor", "achieved": g_tf, "peak": tflops_peak,
                                  "unit": "TFLOP/s", "frac": g_tf / tflops_peak,
                                  "peak_source": f"{peak_kind} bf16_tflops (burst)"},
                     "clocks": g_clocks},
            "l2": L2Flush.desc + " call"}


def _decode_call(wl, N, max_slots=None):
    """A decode step at position N-1 over a cache drawn directly (N-1 tokens)."""
    max_slots = max_slots or (N + wl.s - 1) // wl.s
    cfg = mtla.make_config(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, max_slots, dtype=wl.dtype,
                           gate_mode=wl.gate_mode)
    buf = mtla.Buffers.allocate(cfg, inputs.weights(wl))
    c0 = inputs.synthetic_cache(wl, N - 1, max_slots)
    buf.cache.copy_(c0["cache"].to(torch.bfloat16))
    buf.open_slot.copy_(c0["acc"])
    del c0
    tk = inputs.tokens(wl, 1, stream=1)
    d = {k: (None if v is None else
             v[:, 0].to("cuda", torch.bfloat16 if k != "gate_in" else torch.float32).contiguous())
         for k, v in tk.items()}
    pos = torch.full((wl.B,), N - 1, dtype=torch.int32, device="cuda")
    out = torch.empty(wl.B, wl.H, wl.d_h, device="cuda", dtype=torch.bfloat16)
    gw, gb = (buf.gate_w, buf.gate_b) if wl.gate_mode == inputs.GATE_COMPUTED else (None, None)

    def call():
        mtla.decode_step(cfg, d["c"], d["kr"], d["qc"], d["qr"], buf.w_uk, buf.w_uv, gw, gb,
                         d["gate_in"], pos, buf.cache, buf.open_slot, out, buf.workspace)
    nbytes = wl.B * ((N - 1) // wl.s + 1) * wl.D * 2
    return call, nbytes


def measure_stride(n, flush, ws, rank):
    """Stride sweep B=64, H=8, N=4096, s=1..4: one decode step at position
    4095 over a cache of 4095 tokens (s=3: the last slot holds one token)."""
    hbm, _, peak_kind = _peaks()
    res = {"workload": "stride_sweep: B=64/rank, H=8, d_h=64, d_c=256, d_R=32, N=4096, "
                       "one decode step at position 4095", "per_s": {}}
    for s in (1, 2, 3, 4):
        wl = inputs.STRIDE_SWEEP.with_(s=s, seed=inputs.STRIDE_SWEEP.seed + 1000 * rank)
        call, nbytes = _decode_call(wl, wl.T)
        call_ms, kern_ms, clocks = _timed_calls(call, n, flush, ws)
        kern = nbytes / (kern_ms / 1e3) / 1e9
        res["per_s"][str(s)] = {
            "latent_cache_bytes": nbytes, "call_us": call_ms * 1e3,
            "call_GBps": nbytes * ws / (call_ms / 1e3) / 1e9,
            "roofline": {"kernel": "k_dec_attn_sh", "bound": "hbm", "achieved": kern, "peak": hbm,
                         "unit": "GB/s", "frac": kern / hbm, "avg_launch_us": kern_ms * 1e3,
                         "peak_source": f"{peak_kind} hbm_gbs"},
            "clocks": clocks}
        torch.cuda.empty_cache()
    res["l2"] = L2Flush.desc + " call"
    return res


# ------------------------------------------------------------------ CPU oracle


_CPU_DATA = {}


def _cpu_sample(n_seq: int, min_s: float = 0.0, max_reps: int = 1):
    """The float64 oracle on one decode step (position 65535, 16384 slots) of
    `n_seq` sequences of the contract workload, repeated until `min_s` seconds
    or `max_reps` calls. Returns (latent-cache bytes, seconds, threads, reps)."""
    import numpy as np

    import oracle
    wl = WL.with_(B=n_seq)
    N = wl.T
    max_slots = (N + wl.s - 1) // wl.s
    if n_seq not in _CPU_DATA:
        c0 = inputs.synthetic_cache(wl, N - 1, max_slots)
        _CPU_DATA[n_seq] = (inputs.weights(wl), inputs.tokens(wl, 1, stream=1),
                            c0["cache"].double().numpy(), c0["acc"].double().numpy())
        oracle.build()
    w, tk, cache0, acc0 = _CPU_DATA[n_seq]
    cfg = oracle.Cfg(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, wl.s, gate_mode=wl.gate_mode)
    reps, dt = 0, 0.0
    while reps < max_reps and (reps == 0 or dt < min_s):
        cache, acc = cache0.copy(), acc0.copy()
        t0 = time.perf_counter()
        oracle.decode_step(cfg, tk["c"][:, 0], tk["kr"][:, 0], tk["qc"][:, 0], tk["qr"][:, 0],
                           w["w_uk"], w["w_uv"], np.full(wl.B, N - 1), cache, acc,
                           gate_in=tk["gate_in"][:, 0])
        dt += time.perf_counter() - t0
        reps += 1
    threads = int(os.environ.get("OMP_NUM_THREADS", "0")) or len(os.sched_getaffinity(0))
    return wl.B * max_slots * wl.D * 2 * reps, dt, threads, reps


def run_reference(args, ws, rank):
    """The oracle arm: each step one oracle decode step of 2 of the 32
    sequences at full length, in the contract line's unit (latent-cache GB/s)."""
    if rank != 0:
        return
    n_seq = 2
    times, nbytes, threads = [], 0, 1
    for i in range(args.warmup + args.steps):
        b, dt, threads, _ = _cpu_sample(n_seq)
        if i >= args.warmup:
            times.append(dt)
            nbytes += b
    total = sum(times)
    value = nbytes / total / 1e9
    wl = WL
    sample = (f"one decode step (position {wl.T - 1}, {wl.T // wl.s} slots) of {n_seq} of the "
              f"{wl.B} sequences per step, float64 C oracle with OpenMP over (sequence, head)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"large_latent decode: B={wl.B}, H={wl.H}, d_h={wl.d_h}, "
                               f"d_c={wl.d_c}, d_R={wl.d_r}, s={wl.s}, supplied gates "
                               f"(oracle sample: {n_seq} sequences per step)"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------- kernel lines


def run_reorder_workload(args):
    """Beam-search reorder of the cache (``mtla_reorder_cache``): 64 sequences of
    4096 tokens at the stride-sweep widths with s = 2, i.e. 2048 filled slots of
    576 B each, parents a seeded random permutation. Algorithmic bytes = read +
    write of the filled slots and the fp32 open slots, against the measured
    HBM copy bandwidth (which counts read + write too). L2 flushed before every
    timed call; each call (one kernel) bracketed by CUDA events. The oracle's
    reorder of the same arrays is timed on the host beside it."""
    import numpy as np
    hbm, _, peak_kind = _peaks()
    wl = inputs.WORKLOADS["stride_sweep"].with_(s=2)
    B, N, s = wl.B, wl.T, wl.s
    max_slots = N // s
    cfg = mtla.make_config(B, wl.H, wl.d_h, wl.d_c, wl.d_r, s, max_slots)
    g = torch.Generator().manual_seed(0)
    h_cache = torch.randn(B, max_slots, cfg.D, generator=g).to(torch.bfloat16)
    h_open = torch.randn(B, cfg.D, generator=g)
    h_src = torch.randperm(B, generator=g).to(torch.int32)
    cache_in, open_in = h_cache.cuda(), h_open.cuda()
    cache_out, open_out = torch.empty_like(cache_in), torch.empty_like(open_in)
    src = h_src.cuda()
    n_tok = torch.full((B,), N, dtype=torch.int32, device="cuda")
    nbytes = 2 * (B * max_slots * cfg.D * 2 + B * cfg.D * 4)
    flush = L2Flush()

    def call():
        mtla.reorder_cache(cfg, src, n_tok, cache_in, open_in, cache_out, open_out)
    ms, _, clocks = _timed_calls(call, args.steps, flush, 1, profile=False)
    achieved = nbytes / (ms / 1e3) / 1e9
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        c_in = h_cache.view(torch.int16).numpy().view(np.uint16)
        c_out = np.empty_like(c_in)
        o_in, o_out = h_open.numpy(), np.empty_like(h_open.numpy())
        t0 = time.perf_counter()
        oracle.reorder_cache(s, h_src.numpy(), np.full(B, N, np.int32), c_in, o_in, c_out, o_out)
        dt = time.perf_counter() - t0
        cpu = {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"the whole reorder, once ({dt:.3f} s)"}
    line = {"workload": "beam_reorder",
            "config": {"B": B, "d_c": wl.d_c, "d_R": wl.d_r, "s": s, "tokens": N, "slots": max_slots,
                       "parents": "random permutation"},
            "kernel_ms": ms,
            "roofline": {"kernel": "k_reorder_cache", "bound": "hbm", "achieved": achieved, "peak": hbm,
                         "unit": "GB/s", "frac": achieved / hbm, "bytes_per_launch": nbytes,
                         "peak_source": f"{peak_kind} hbm_gbs"},
            "cpu_baseline": cpu, "clocks": clocks, "l2": L2Flush.desc + " call"}
    print(json.dumps(line), flush=True)


def run_kernel_workload(args):
    """Kernel-level line of one workload (not the contract line), for profiling
    runs: decode attention GB/s or prefill TFLOP/s against the measured peaks."""
    flush = L2Flush()
    name = args.workload
    if name.startswith("prefill"):
        print(json.dumps(measure_prefill(args.steps, flush, 1, 0)), flush=True)
        return
    if name.startswith("speech_decode"):
        dt = "fp16" if name.endswith("fp16") else "bf16"
        print(json.dumps(measure_speech(args.steps, flush, 1, 0, dtype=dt)), flush=True)
        return
    if name == "layer":
        print(json.dumps(measure_layer(args.steps, flush, 1, 0)), flush=True)
        return
    if name == "backward":
        print(json.dumps(measure_backward(args.steps, flush, 1, 0)), flush=True)
        return
    hbm, _, peak_kind = _peaks()
    if name == "large_latent_step":              # one decode step of the contract workload
        wl = inputs.LARGE_LATENT
    else:
        wl = inputs.WORKLOADS[name.split(":")[0]]
    if ":" in name:
        wl = wl.with_(s=int(name.split(":")[1]))
    call, nbytes = _decode_call(wl, wl.T)
    call_ms, kern_ms, clocks = _timed_calls(call, args.steps, flush, 1)
    kern = nbytes / (kern_ms / 1e3) / 1e9
    print(json.dumps({"workload": name, "config": {"B": wl.B, "H": wl.H, "d_h": wl.d_h,
                                                   "d_c": wl.d_c, "d_R": wl.d_r, "s": wl.s,
                                                   "N": wl.T},
                      "call_ms": call_ms, "attention_kernel_ms": kern_ms,
                      "call": {"value": nbytes / (call_ms / 1e3) / 1e9, "unit": "GB/s"},
                      "roofline": {"kernel": "decode attention", "bound": "hbm", "achieved": kern,
                                   "peak": hbm, "unit": "GB/s", "frac": kern / hbm,
                                   "peak_source": f"{peak_kind} hbm_gbs"},
                      "clocks": clocks, "l2": L2Flush.desc + " call"}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="mtla", choices=["mtla", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="contract line only (no prefill / speech / stride-sweep sub-objects)")
    ap.add_argument("--workload", default="large_latent",
                    help="large_latent (the contract line), or a kernel-level line of "
                         "large_latent_step, stride_sweep[:s], prefill, speech_decode, layer, backward or beam_reorder")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    ws, rank = _dist()
    try:
        if args.impl == "reference":
            run_reference(args, ws, rank)
        elif args.workload == "beam_reorder":
            if rank == 0:
                run_reorder_workload(args)
        elif args.workload != "large_latent":
            if rank == 0:
                run_kernel_workload(args)
        else:
            run_contract(args, ws, rank)
    finally:
        if ws > 1:
            torch.distributed.destroy_process_group()


def run_contract(args, ws, rank):
    res = measure_contract(args, ws, rank)
    torch.cuda.empty_cache()
    extras = {}
    if not args.no_extras:
        flush = L2Flush()
        extras["prefill"] = measure_prefill(900, flush, ws, rank)
        torch.cuda.empty_cache()
        extras["speech_decode"] = measure_speech(320, flush, ws, rank)
        torch.cuda.empty_cache()
        extras["speech_decode_fp16"] = measure_speech(320, flush, ws, rank, dtype="fp16")
        torch.cuda.empty_cache()
        extras["stride_sweep"] = measure_stride(6000, flush, ws, rank)
        torch.cuda.empty_cache()
        extras["layer"] = measure_layer(400, flush, ws, rank)
        torch.cuda.empty_cache()
        extras["backward"] = measure_backward(120, flush, ws, rank)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        n_seq = 8
        b, dt, threads, reps = _cpu_sample(n_seq, min_s=10.0, max_reps=4)
        cpu = {"value": b / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{reps} x one decode step (position {WL.T - 1}, {WL.T // WL.s} slots) "
                         f"of {n_seq} of the {WL.B} sequences, float64 C oracle with OpenMP "
                         f"over (sequence, head) ({dt:.1f} s)"}
    if rank == 0:
        line = {
            "metric": METRIC, "value": res["value"], "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) inputs and cache, random-init weights)",
            "config": res["config"], "decode": res["decode"], "roofline": res["roofline"],
            "cpu_baseline": cpu, "e2e": res["e2e"], "gpu_launches": res["gpu_launches"],
            "cuda_graphs": f"{GEN_STEPS} decode steps per graph, one replay per step",
            "clocks": res["clocks"],
        }
        line.update(extras)
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
