"""CPU pins for the float64 oracle: checks against what the pages and the
mathematics fix, none of which retypes the oracle's own formulas.

- printed values: the 9/(4s) cache footprint ("Multi-head Temporal Latent
  Attention", Key claims, Sec. 4.3) and the 1,152 B latent slot ("Multi-Head
  Latent Attention and Sparse Indexers", "Work the bytes with units and scope"),
  as fixtures in tests/golden/cache_footprint.txt;
- special case reducing to a library routine: s = 1 with unit gates is MLA,
  i.e. causal softmax attention on explicit keys/values (torch SDPA, float64);
- algebraic identity: absorbed form == explicit (non-absorbed) form (MLA
  absorption identities);
- invariant: incremental decoding == parallel masked forward (Sec. 4.2);
- brute force: dense enumerated mask over per-token partial slots (tests/brute_force.py);
- closed forms of the scan, the gate modes, PE and RoPE;
- exact values of the adopted PE / RoPE readings at width 8 (pair frequencies
  exactly 1, 0.1, 0.01, 0.001 at base 10000) and one gate worked by hand;
- chunked prefill: from position 0 it is the parallel forward; a prefix then a
  chunk equals one prefill (split points inside a block included); a chunk
  equals the same number of incremental decode steps;
- per-channel gate: equal channels reduce it to the scalar gate (computed and
  supplied); G = 0 gives a closed form; one value worked by hand; decoding
  equals the parallel form;
- the layer around the path: block-selecting projections make it the path
  itself; folding W_UK into W_Q and W_UV into W_O gives the same output;
- the training backward: every gradient against central finite differences.
Finally, each planted mistake in the oracle must trip at least one pin.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import brute_force as bf

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cache_footprint.txt")


def _golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split()
            vals[k] = float(v)
    return vals


def _rand_problem(B, H, d_h, d_c, d_r, s, T, seed, gate_mode=oracle.GATE_COMPUTED):
    rng = np.random.default_rng(seed)
    cfg = oracle.Cfg(B, H, d_h, d_c, d_r, s, gate_mode=gate_mode)
    p = dict(
        c=rng.standard_normal((B, T, d_c)),
        kr=rng.standard_normal((B, T, d_r)),
        qc=rng.standard_normal((B, T, H, d_h)),
        qr=rng.standard_normal((B, T, H, d_r)),
        w_uk=rng.standard_normal((H, d_h, d_c)) / math.sqrt(d_c),
        w_uv=rng.standard_normal((H, d_h, d_c)) / math.sqrt(d_c),
        G=rng.standard_normal((s, d_c)) / math.sqrt(d_c),
        g=rng.standard_normal(s) * 0.5,
        gate_in=1.0 / (1.0 + np.exp(-rng.standard_normal((B, T)))),
    )
    return cfg, p


# --------------------------------------------------------------------------- pins


def pin_cache_footprint():
    """Slot count * width per token equals the printed 9/(4s) (MQA units of 2 d_h),
    and the GLM latent slot equals the printed byte counts."""
    gold = _golden()
    d_h = 64
    for s in (1, 2, 3, 4):
        cfg = oracle.Cfg(1, 1, d_h, 4 * d_h, d_h // 2, s, gate_mode=oracle.GATE_UNIT)
        T = 12 * s
        rng = np.random.default_rng(s)
        res = oracle.prefill(cfg, rng.standard_normal((1, T, cfg.d_c)),
                             rng.standard_normal((1, T, cfg.d_r)),
                             rng.standard_normal((1, T, 1, d_h)),
                             rng.standard_normal((1, T, 1, cfg.d_r)),
                             rng.standard_normal((1, d_h, cfg.d_c)),
                             rng.standard_normal((1, d_h, cfg.d_c)))
        n_slots, width = res["cache"].shape[1:]
        per_token = n_slots * width / T / (2 * d_h)
        if abs(per_token - gold[f"mtla_elements_per_token_s{s}"]) > 1e-12:
            return False
    cfg = oracle.Cfg(1, 1, 128, 512, 64, 1, gate_mode=oracle.GATE_UNIT)
    rng = np.random.default_rng(0)
    T = 3
    res = oracle.prefill(cfg, rng.standard_normal((1, T, 512)), rng.standard_normal((1, T, 64)),
                         rng.standard_normal((1, T, 1, 128)), rng.standard_normal((1, T, 1, 64)),
                         rng.standard_normal((1, 128, 512)), rng.standard_normal((1, 128, 512)))
    bytes_per_pos = res["cache"].shape[2] * 2 * res["cache"].shape[1] // T   # bf16
    return (bytes_per_pos == gold["glm_bytes_per_layer_position"]
            and bytes_per_pos * 78 == gold["glm_bytes_per_position_78_layers"]
            and bytes_per_pos * 78 * 1048576 == gold["glm_bytes_1048576_positions_78_layers"])


def pin_s1_is_mla_sdpa():
    """s = 1, unit gates: MTLA == MLA == causal attention on explicit k, v."""
    B, H, d_h, d_c, d_r, T = 2, 3, 8, 16, 4, 9
    cfg, p = _rand_problem(B, H, d_h, d_c, d_r, 1, T, seed=11, gate_mode=oracle.GATE_UNIT)
    got = oracle.prefill(cfg, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"])["out"]
    # explicit keys/values, RoPE applied through the oracle's rotation
    kr_rot = np.stack([np.stack([oracle.rope(t, p["kr"][b, t]) for t in range(T)])
                       for b in range(B)])
    qr_rot = np.stack([np.stack([np.stack([oracle.rope(t, p["qr"][b, t, h]) for h in range(H)])
                                 for t in range(T)]) for b in range(B)])
    c = torch.tensor(p["c"])
    w_uk = torch.tensor(p["w_uk"])
    w_uv = torch.tensor(p["w_uv"])
    k = torch.cat([torch.einsum("btc,hdc->bhtd", c, w_uk),
                   torch.tensor(kr_rot)[:, None].expand(B, H, T, d_r)], dim=-1)
    v = torch.einsum("btc,hdc->bhtd", c, w_uv)
    q = torch.cat([torch.tensor(p["qc"]).permute(0, 2, 1, 3),
                   torch.tensor(qr_rot).permute(0, 2, 1, 3)], dim=-1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, is_causal=True, scale=1.0 / math.sqrt(d_h + d_r))
    ref = ref.permute(0, 2, 1, 3).numpy()
    return np.max(np.abs(got - ref)) < 1e-12


def pin_absorbed_equals_explicit():
    for s in (1, 2, 3, 4):
        cfg, p = _rand_problem(2, 2, 8, 24, 4, s, 11, seed=20 + s)
        a = oracle.prefill(cfg, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"],
                           p["G"], p["g"])["out"]
        e = oracle.prefill_explicit(cfg, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"],
                                    p["w_uv"], p["G"], p["g"])
        if not np.max(np.abs(a - e)) < 1e-12:
            return False
    return True


def pin_incremental_equals_parallel():
    for s in (1, 2, 3, 4):
        B, T = 2, 13
        cfg, p = _rand_problem(B, 2, 8, 16, 4, s, T, seed=40 + s)
        par = oracle.prefill(cfg, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"],
                             p["G"], p["g"])
        max_slots = (T + s - 1) // s + 1
        cache = np.zeros((B, max_slots, cfg.D))
        acc = np.zeros((B, cfg.D))
        outs = []
        for t in range(T):
            r = oracle.decode_step(cfg, p["c"][:, t], p["kr"][:, t], p["qc"][:, t], p["qr"][:, t],
                                   p["w_uk"], p["w_uv"], np.full(B, t), cache, acc,
                                   p["G"], p["g"])
            outs.append(r["out"])
        inc = np.stack(outs, axis=1)
        n = (T + s - 1) // s
        if not (np.max(np.abs(inc - par["out"])) < 1e-12
                and np.max(np.abs(cache[:, :n] - par["cache"])) < 1e-12
                and np.max(np.abs(acc - par["acc"])) < 1e-12):
            return False
    return True


def pin_brute_force():
    for s in (1, 2, 3, 4):
        for T in (1, s, 7, 16):
            B, H, d_h, d_c, d_r = 1, 2, 4, 8, 4
            cfg, p = _rand_problem(B, H, d_h, d_c, d_r, s, T, seed=60 + s * 17 + T,
                                   gate_mode=oracle.GATE_SUPPLIED)
            got = oracle.prefill(cfg, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"],
                                 gate_in=p["gate_in"])
            x = np.concatenate([p["c"][0], np.stack([oracle.rope(t, p["kr"][0, t])
                                                     for t in range(T)])], axis=1)
            P = bf.running_slots(x, p["gate_in"][0], s)
            q_full = np.concatenate(
                [p["qc"][0], np.stack([np.stack([oracle.rope(t, p["qr"][0, t, h])
                                                 for h in range(H)]) for t in range(T)])], axis=2)
            ref = bf.attention(q_full, P, p["w_uk"], p["w_uv"], s, d_c,
                               bf.softmax_scale(d_h, d_r))
            if not np.max(np.abs(got["out"][0] - ref)) < 1e-12:
                return False
            mask = bf.dense_mask(T, s)
            if any(mask[i].sum() != i // s + 1 for i in range(T)):
                return False
    return True


def pin_scan_closed_form():
    """Unit gates and all-ones latents: P_t = (t mod s + 1) * 1 on the latent
    part; finished slots hold s; the cache has ceil(T/s) slots."""
    for s in (1, 2, 3, 4):
        T, d_c, d_r = 10, 8, 4
        cfg = oracle.Cfg(1, 1, 4, d_c, d_r, s, gate_mode=oracle.GATE_UNIT)
        w, P = oracle.partials(cfg, np.ones((1, T, d_c)), np.zeros((1, T, d_r)))
        expect = np.array([(t % s) + 1 for t in range(T)], dtype=float)
        if not (np.all(w == 1.0) and np.allclose(P[0, :, :d_c], expect[:, None], atol=0)
                and np.all(P[0, :, d_c:] == 0.0)):
            return False
        res = oracle.prefill(cfg, np.ones((1, T, d_c)), np.zeros((1, T, d_r)),
                             np.zeros((1, T, 1, 4)), np.zeros((1, T, 1, d_r)),
                             np.zeros((1, 4, d_c)), np.zeros((1, 4, d_c)))
        n = math.ceil(T / s)
        if res["cache"].shape[1] != n:
            return False
        for j in range(n):
            full = min(s, T - j * s)
            if not np.all(res["cache"][0, j, :d_c] == full):
                return False
    return True


def pin_gate_modes():
    """UNIT -> 1; SUPPLIED passes through; COMPUTED with a zero row r gives
    sigmoid(g[r]) for tokens t = r mod s; at t = 0 the PE is (0,1,0,1,...) so
    only the odd latent entries reach the gate."""
    d_c, s = 8, 3
    rng = np.random.default_rng(5)
    c = rng.standard_normal(d_c)
    G = rng.standard_normal((s, d_c))
    g = np.array([0.3, -1.2, 2.0])
    sig = lambda z: 1.0 / (1.0 + math.exp(-z))
    if oracle.gate(oracle.Cfg(1, 1, 4, d_c, 4, s, gate_mode=oracle.GATE_UNIT), 5, c, G, g) != 1.0:
        return False
    if oracle.gate(oracle.Cfg(1, 1, 4, d_c, 4, s, gate_mode=oracle.GATE_SUPPLIED), 5, c, G, g,
                   w_given=0.37) != 0.37:
        return False
    cfg = oracle.Cfg(1, 1, 4, d_c, 4, s)
    for r in range(s):
        Gz = G.copy()
        Gz[r] = 0.0
        for t in (r, r + s, r + 5 * s):
            if abs(oracle.gate(cfg, t, c, Gz, g) - sig(g[r])) > 1e-15:
                return False
    z0 = g[0] + sum(G[0, i] * c[i] for i in range(1, d_c, 2))
    return abs(oracle.gate(cfg, 0, c, G, g) - sig(z0)) < 1e-14


def pin_rope():
    """Rotation of pairs: t = 0 is the identity, every pair keeps its norm,
    scores depend only on the position difference, and the rotation is
    counter-clockwise (RoFormer's matrix) -- the last is a convention."""
    rng = np.random.default_rng(9)
    d = 16
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    if not np.array_equal(oracle.rope(0, q), q):
        return False
    y = oracle.rope(37, q)
    if not np.allclose((y[0::2] ** 2 + y[1::2] ** 2), (q[0::2] ** 2 + q[1::2] ** 2), atol=1e-13):
        return False
    for m, n, dlt in ((3, 11, 5), (100, 7, 1000), (0, 64, 4095)):
        a = oracle.rope(m, q) @ oracle.rope(n, k)
        b = oracle.rope(m + dlt, q) @ oracle.rope(n + dlt, k)
        if abs(a - b) > 1e-9:
            return False
    e0 = np.zeros(d)
    e0[0] = 1.0
    y = oracle.rope(1, e0)
    return abs(y[0] - math.cos(1.0)) < 1e-15 and abs(y[1] - math.sin(1.0)) < 1e-15


def pin_pe():
    d = 32
    pe0 = oracle.pe(0, d)
    if not (np.all(pe0[0::2] == 0.0) and np.all(pe0[1::2] == 1.0)):
        return False
    for t in (1, 17, 5000):
        p = oracle.pe(t, d)
        if not np.allclose(p[0::2] ** 2 + p[1::2] ** 2, 1.0, atol=1e-14):
            return False
        if abs(p[0] - math.sin(t)) > 1e-12:      # the first pair turns at unit frequency
            return False
    return True


def pin_pe_values():
    """Exact values of the adopted PE reading: interleaved (sin, cos) pairs,
    pair k turning at base^(-2k/d) with base 10000. At width 8 the four pair
    frequencies are exactly 1, 0.1, 0.01 and 0.001; at width 4 they are 1 and
    0.01. Expected values are written from those literals, not from the
    oracle's formula."""
    t = 10
    want8 = [math.sin(10.0), math.cos(10.0), math.sin(1.0), math.cos(1.0),
             math.sin(0.1), math.cos(0.1), math.sin(0.01), math.cos(0.01)]
    if np.max(np.abs(oracle.pe(t, 8) - np.array(want8))) > 1e-14:
        return False
    want4 = [math.sin(3.0), math.cos(3.0), math.sin(0.03), math.cos(0.03)]
    return np.max(np.abs(oracle.pe(3, 4) - np.array(want4))) < 1e-14


def pin_rope_values():
    """Exact values of the adopted RoPE reading at width 8, t = 10: the unit
    vector e_2k comes out as (cos a_k, sin a_k) in pair k and e_2k+1 as
    (-sin a_k, cos a_k), with a_k = 10 * 10^-k (frequencies 1, 0.1, 0.01,
    0.001 of base 10000), and nothing leaks into the other pairs."""
    d, t = 8, 10
    for k in range(d // 2):
        a = t * 10.0 ** (-k)
        for which, pair in ((0, (math.cos(a), math.sin(a))), (1, (-math.sin(a), math.cos(a)))):
            e = np.zeros(d)
            e[2 * k + which] = 1.0
            want = np.zeros(d)
            want[2 * k], want[2 * k + 1] = pair
            if np.max(np.abs(oracle.rope(t, e) - want)) > 1e-14:
                return False
    return True


def pin_gate_value():
    """One gate worked by hand (Eq. 13 under the adopted reading): t = 3,
    s = 2, d_c = 4 takes row r = 3 mod 2 = 1; PE_3 at width 4 is
    (sin 3, cos 3, sin 0.03, cos 0.03); with c = (1, 2, 3, 4),
    G[1] = (0.5, -1, 0.25, 2), g[1] = 0.1:
      z = 0.1 + 0.5 sin 3 - 2 cos 3 + 0.75 sin 0.03 + 8 cos 0.03,
      w = 1 / (1 + e^-z)."""
    cfg = oracle.Cfg(1, 1, 4, 4, 4, 2)
    c = np.array([1.0, 2.0, 3.0, 4.0])
    G = np.array([[9.0, -7.0, 5.0, 3.0], [0.5, -1.0, 0.25, 2.0]])
    g = np.array([-4.0, 0.1])
    z = (0.1 + 0.5 * math.sin(3.0) - 2.0 * math.cos(3.0) + 0.75 * math.sin(0.03)
         + 8.0 * math.cos(0.03))
    return abs(oracle.gate(cfg, 3, c, G, g) - 1.0 / (1.0 + math.exp(-z))) < 1e-14


def _prefix_state(cfg, p, t0):
    """Cache and open slot after the first t0 tokens (parallel form)."""
    if t0 == 0:
        return np.zeros((cfg.B, 0, cfg.D)), np.zeros((cfg.B, cfg.D))
    r = oracle.prefill(cfg, p["c"][:, :t0], p["kr"][:, :t0], p["qc"][:, :t0], p["qr"][:, :t0],
                       p["w_uk"], p["w_uv"], p["G"], p["g"])
    return r["cache"], r["acc"]


def _chunk(p, t0):
    return {k: p[k][:, t0:] for k in ("c", "kr", "qc", "qr")}


def pin_prefill_from_start_is_prefill():
    """Chunked prefill from t0 = 0 is the parallel forward itself."""
    for s in (1, 3):
        cfg, p = _rand_problem(2, 2, 8, 16, 4, s, 10, seed=70 + s)
        ref = oracle.prefill(cfg, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"], p["G"], p["g"])
        cache0, acc0 = _prefix_state(cfg, p, 0)
        got = oracle.prefill_from(cfg, 0, cache0, acc0, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"],
                                  p["w_uv"], p["G"], p["g"])
        for k in ("out", "cache", "acc", "w"):
            if not np.max(np.abs(got[k] - ref[k])) < 1e-12:
                return False
    return True


def pin_prefill_chunks_compose():
    """Prefill of t0 tokens, then a chunk of T tokens from the resulting cache
    and open slot, equals one prefill of t0 + T tokens (its last T rows, its
    cache and open slot): the stride-aware mask makes the parallel form
    split anywhere, inside a block included (MTLA Sec. 4.2)."""
    for s in (1, 2, 3, 4):
        total = 17
        cfg, p = _rand_problem(2, 2, 8, 16, 4, s, total, seed=80 + s)
        full = oracle.prefill(cfg, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"], p["G"], p["g"])
        for t0 in sorted({1, s, 2 * s + 1, 7, 16}):
            cache0, acc0 = _prefix_state(cfg, p, t0)
            ch = _chunk(p, t0)
            got = oracle.prefill_from(cfg, t0, cache0, acc0, ch["c"], ch["kr"], ch["qc"], ch["qr"],
                                      p["w_uk"], p["w_uv"], p["G"], p["g"])
            if not (np.max(np.abs(got["out"] - full["out"][:, t0:])) < 1e-12
                    and np.max(np.abs(got["cache"] - full["cache"])) < 1e-12
                    and np.max(np.abs(got["acc"] - full["acc"])) < 1e-12):
                return False
    return True


def pin_prefill_from_equals_decode_steps():
    """A chunk of T tokens from a cache state equals T incremental decode steps
    from the same state (outputs, cache, open slot)."""
    for s in (2, 3):
        t0, T = 5, 8
        cfg, p = _rand_problem(2, 2, 8, 16, 4, s, t0 + T, seed=90 + s)
        cache0, acc0 = _prefix_state(cfg, p, t0)
        ch = _chunk(p, t0)
        got = oracle.prefill_from(cfg, t0, cache0, acc0, ch["c"], ch["kr"], ch["qc"], ch["qr"],
                                  p["w_uk"], p["w_uv"], p["G"], p["g"])
        max_slots = (t0 + T + s - 1) // s
        cache = np.zeros((cfg.B, max_slots, cfg.D))
        cache[:, :cache0.shape[1]] = cache0
        acc = acc0.copy()
        outs = []
        for k in range(T):
            r = oracle.decode_step(cfg, ch["c"][:, k], ch["kr"][:, k], ch["qc"][:, k], ch["qr"][:, k],
                                   p["w_uk"], p["w_uv"], np.full(cfg.B, t0 + k), cache, acc, p["G"], p["g"])
            outs.append(r["out"])
        if not (np.max(np.abs(np.stack(outs, axis=1) - got["out"])) < 1e-12
                and np.max(np.abs(cache - got["cache"])) < 1e-12
                and np.max(np.abs(acc - got["acc"])) < 1e-12):
            return False
    return True


def _channel_problem(s, T, seed, B=2, H=2, d_h=8, d_c=16, d_r=4):
    """A problem with per-channel gate parameters G [s, d_c, D], g [s, D] and
    supplied per-channel weights [B, T, D]."""
    cfg, p = _rand_problem(B, H, d_h, d_c, d_r, s, T, seed)
    rng = np.random.default_rng(seed + 1000)
    D = d_c + d_r
    p["Gc"] = rng.standard_normal((s, d_c, D)) / math.sqrt(d_c)
    p["gc"] = rng.standard_normal((s, D)) * 0.5
    p["gate_in_c"] = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, D))))
    return cfg, p


def pin_channel_gate_equal_columns_is_scalar():
    """Per-channel gate whose D columns are all the scalar gate's row (and
    biases equal) reproduces the scalar-gate forward; supplied per-channel
    weights equal across channels reproduce the scalar supplied gate."""
    for s in (1, 3):
        cfg, p = _channel_problem(s, 11, seed=100 + s)
        D = cfg.D
        ref = oracle.prefill(cfg, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"], p["G"], p["g"])
        cc = oracle.Cfg(cfg.B, cfg.H, cfg.d_h, cfg.d_c, cfg.d_r, s, gate_mode=oracle.GATE_CHANNEL_COMPUTED)
        Gc = np.repeat(p["G"][:, :, None], D, axis=2)
        gc = np.repeat(p["g"][:, None], D, axis=1)
        got = oracle.prefill(cc, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"], Gc, gc)
        if not (np.max(np.abs(got["out"] - ref["out"])) < 1e-12 and np.max(np.abs(got["cache"] - ref["cache"])) < 1e-12):
            return False
        cs = oracle.Cfg(cfg.B, cfg.H, cfg.d_h, cfg.d_c, cfg.d_r, s, gate_mode=oracle.GATE_SUPPLIED)
        ref = oracle.prefill(cs, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"], gate_in=p["gate_in"])
        cq = oracle.Cfg(cfg.B, cfg.H, cfg.d_h, cfg.d_c, cfg.d_r, s, gate_mode=oracle.GATE_CHANNEL_SUPPLIED)
        got = oracle.prefill(cq, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"],
                             gate_in=np.repeat(p["gate_in"][:, :, None], D, axis=2))
        if not np.max(np.abs(got["out"] - ref["out"])) < 1e-12:
            return False
    return True


def pin_channel_gate_closed_form():
    """G = 0: token t's weights are sigmoid(g[t mod s][k]) in channel k, so with
    all-ones latents and zero keys the partial slot of position t holds, in
    latent channel k, the sum of sigmoid(g[u mod s][k]) over its block's
    tokens u <= t, and zeros in the key channels."""
    s, T, d_c, d_r = 3, 10, 8, 4
    D = d_c + d_r
    cfg = oracle.Cfg(1, 1, 4, d_c, d_r, s, gate_mode=oracle.GATE_CHANNEL_COMPUTED)
    g = np.arange(s * D, dtype=float).reshape(s, D) * 0.1 - 1.0
    sig = 1.0 / (1.0 + np.exp(-g))
    _, P = oracle.partials(cfg, np.ones((1, T, d_c)), np.zeros((1, T, d_r)), np.zeros((s, d_c, D)), g)
    for t in range(T):
        want = sum(sig[u % s] for u in range(s * (t // s), t + 1))
        if not (np.max(np.abs(P[0, t, :d_c] - want[:d_c])) < 1e-14 and np.all(P[0, t, d_c:] == 0.0)):
            return False
    return True


def pin_channel_gate_value():
    """One per-channel gate worked by hand: t = 1, s = 2 (row 1), d_c = 2,
    D = 4; PE_1 at width 2 is (sin 1, cos 1); c = (1, 2);
    G[1] = [[1, 0, -1, 2], [0.5, 1, 0, -3]] (rows: latent inputs, columns:
    slot channels), g[1] = (0, 0.25, -0.5, 1):
      z = sin 1 * G[1][0] + 2 cos 1 * G[1][1] + g[1],  w = sigmoid(z)."""
    cfg = oracle.Cfg(1, 1, 4, 2, 2, 2, gate_mode=oracle.GATE_CHANNEL_COMPUTED)
    G = np.zeros((2, 2, 4))
    G[1] = [[1.0, 0.0, -1.0, 2.0], [0.5, 1.0, 0.0, -3.0]]
    g = np.array([[0.0, 0.0, 0.0, 0.0], [0.0, 0.25, -0.5, 1.0]])
    s1, c1 = math.sin(1.0), math.cos(1.0)
    z = [s1 * 1.0 + 2 * c1 * 0.5 + 0.0, 2 * c1 * 1.0 + 0.25, -s1 - 0.5, 2 * s1 - 6 * c1 + 1.0]
    want = np.array([1.0 / (1.0 + math.exp(-v)) for v in z])
    return np.max(np.abs(oracle.gate_channels(cfg, 1, np.array([1.0, 2.0]), G, g) - want)) < 1e-15


def pin_channel_incremental_equals_parallel():
    """Per-channel gates, computed and supplied: decoding step by step equals
    the parallel masked forward (outputs, cache, open slot)."""
    for mode in (oracle.GATE_CHANNEL_COMPUTED, oracle.GATE_CHANNEL_SUPPLIED):
        for s in (2, 3):
            B, T = 2, 11
            cfg, p = _channel_problem(s, T, seed=110 + s)
            cfg = oracle.Cfg(B, cfg.H, cfg.d_h, cfg.d_c, cfg.d_r, s, gate_mode=mode)
            gin = p["gate_in_c"] if mode == oracle.GATE_CHANNEL_SUPPLIED else None
            par = oracle.prefill(cfg, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"], p["Gc"], p["gc"], gin)
            max_slots = (T + s - 1) // s
            cache = np.zeros((B, max_slots, cfg.D))
            acc = np.zeros((B, cfg.D))
            outs = []
            for t in range(T):
                r = oracle.decode_step(cfg, p["c"][:, t], p["kr"][:, t], p["qc"][:, t], p["qr"][:, t], p["w_uk"],
                                       p["w_uv"], np.full(B, t), cache, acc, p["Gc"], p["gc"],
                                       None if gin is None else gin[:, t])
                outs.append(r["out"])
            if not (np.max(np.abs(np.stack(outs, axis=1) - par["out"])) < 1e-12
                    and np.max(np.abs(cache - par["cache"])) < 1e-12 and np.max(np.abs(acc - par["acc"])) < 1e-12):
                return False
    return True


def _layer_problem(B, H, d_h, d_c, d_r, s, T, dm, seed):
    cfg, p = _rand_problem(B, H, d_h, d_c, d_r, s, T, seed)
    rng = np.random.default_rng(seed + 500)
    W = dict(w_dkv=rng.standard_normal((d_c, dm)) / math.sqrt(dm),
             w_kr=rng.standard_normal((d_r, dm)) / math.sqrt(dm),
             w_q=rng.standard_normal((H * d_h, dm)) / math.sqrt(dm),
             w_qr=rng.standard_normal((H * d_r, dm)) / math.sqrt(dm),
             w_uk=p["w_uk"], w_uv=p["w_uv"],
             w_o=rng.standard_normal((dm, H * d_h)) / math.sqrt(H * d_h))
    h = rng.standard_normal((B, T, dm))
    return cfg, p, W, h


def pin_layer_selection_is_the_path():
    """Projections that select blocks of h (h = [c | k | qC | qR | 0]) and a W_O
    that copies o into the first columns make the layer the path itself: y's
    first H*d_h columns are the path's output, the rest zero. A transposed or
    misplaced projection breaks this."""
    B, H, d_h, d_c, d_r, s, T = 2, 2, 4, 8, 4, 3, 9
    cfg, p = _rand_problem(B, H, d_h, d_c, d_r, s, T, seed=130)
    widths = [d_c, d_r, H * d_h, H * d_r]
    dm = sum(widths) + 3
    eye = np.eye(dm)
    off = np.cumsum([0] + widths)
    W = dict(w_dkv=eye[off[0]:off[1]], w_kr=eye[off[1]:off[2]], w_q=eye[off[2]:off[3]], w_qr=eye[off[3]:off[4]],
             w_uk=p["w_uk"], w_uv=p["w_uv"], w_o=np.eye(dm, H * d_h))
    h = np.concatenate([p["c"], p["kr"], p["qc"].reshape(B, T, -1), p["qr"].reshape(B, T, -1),
                        np.zeros((B, T, 3))], axis=2)
    got = oracle.layer_forward(cfg, 0, np.zeros((B, 0, cfg.D)), np.zeros((B, cfg.D)), h, W, p["G"], p["g"])
    ref = oracle.prefill(cfg, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"], p["G"], p["g"])
    return (np.max(np.abs(got["y"][:, :, :H * d_h] - ref["out"].reshape(B, T, -1))) < 1e-12
            and np.all(got["y"][:, :, H * d_h:] == 0.0) and np.max(np.abs(got["cache"] - ref["cache"])) < 1e-12)


def pin_layer_absorption_fold():
    """W_UK folded into W_Q and W_UV folded into W_O ("Multi-Head Latent
    Attention and Sparse Indexers", "Latent attention changes the
    representation"): the layer with per-head query weights W_UK[h]^T W_Q[h]
    (so the path's qC is the absorbed latent query and its W_UK the identity) and
    output weights W_O[:, h] W_UV[h] (the path's W_UV the identity, d_h = d_c)
    gives the same y."""
    B, H, d_h, d_c, d_r, s, T, dm = 2, 3, 4, 8, 4, 2, 7, 12
    cfg, p, W, h = _layer_problem(B, H, d_h, d_c, d_r, s, T, dm, seed=140)
    ref = oracle.layer_forward(cfg, 0, np.zeros((B, 0, cfg.D)), np.zeros((B, cfg.D)), h, W, p["G"], p["g"])
    cf = oracle.Cfg(B, H, d_c, d_c, d_r, s, scale=1.0 / math.sqrt(d_h + d_r))
    eye = np.repeat(np.eye(d_c)[None], H, axis=0)
    wq = W["w_q"].reshape(H, d_h, dm)
    wo = W["w_o"].reshape(dm, H, d_h)
    Wf = dict(w_dkv=W["w_dkv"], w_kr=W["w_kr"], w_qr=W["w_qr"], w_uk=eye, w_uv=eye,
              w_q=np.einsum("hic,him->hcm", W["w_uk"], wq).reshape(H * d_c, dm),
              w_o=np.einsum("mhi,hic->mhc", wo, W["w_uv"]).reshape(dm, H * d_c))
    got = oracle.layer_forward(cf, 0, np.zeros((B, 0, cf.D)), np.zeros((B, cf.D)), h, Wf, p["G"], p["g"])
    return np.max(np.abs(got["y"] - ref["y"])) < 1e-12


def pin_backward_finite_differences():
    """Every gradient of the backward against central finite differences of
    L = sum(dout * out) (eps = 1e-6, float64), on sampled entries of every input
    tensor, for the computed, supplied and unit gates at s = 1, 2, 3."""
    rng = np.random.default_rng(150)
    for mode in (oracle.GATE_COMPUTED, oracle.GATE_SUPPLIED, oracle.GATE_UNIT):
        for s in (1, 2, 3):
            cfg, p = _rand_problem(2, 2, 4, 8, 4, s, 9, seed=160 + 10 * mode + s, gate_mode=mode)
            args = dict(c=p["c"], kr=p["kr"], qc=p["qc"], qr=p["qr"], w_uk=p["w_uk"], w_uv=p["w_uv"],
                        G=p["G"] if mode == oracle.GATE_COMPUTED else None,
                        g=p["g"] if mode == oracle.GATE_COMPUTED else None,
                        gate_in=p["gate_in"] if mode == oracle.GATE_SUPPLIED else None)
            dout = rng.standard_normal((2, 9, 2, 4))

            def loss(a):
                r = oracle.prefill(cfg, a["c"], a["kr"], a["qc"], a["qr"], a["w_uk"], a["w_uv"], a["G"], a["g"],
                                   a["gate_in"])
                return float(np.sum(dout * r["out"]))
            grads = oracle.prefill_backward(cfg, dout=dout, **args)
            names = {"c": "dc", "kr": "dkr", "qc": "dqc", "qr": "dqr", "w_uk": "dw_uk", "w_uv": "dw_uv",
                     "G": "dG", "g": "dg", "gate_in": "dgate_in"}
            for k, gk in names.items():
                if args[k] is None:
                    continue
                for _ in range(5):
                    idx = tuple(int(rng.integers(0, n)) for n in args[k].shape)
                    ap, am = {**args, k: args[k].copy()}, {**args, k: args[k].copy()}
                    ap[k][idx] += 1e-6
                    am[k][idx] -= 1e-6
                    fd = (loss(ap) - loss(am)) / 2e-6
                    if abs(fd - grads[gk][idx]) > 1e-6 * max(1.0, abs(fd)):
                        return False
    return True


PINS = {
    "cache_footprint": pin_cache_footprint,
    "s1_is_mla_sdpa": pin_s1_is_mla_sdpa,
    "absorbed_equals_explicit": pin_absorbed_equals_explicit,
    "incremental_equals_parallel": pin_incremental_equals_parallel,
    "brute_force": pin_brute_force,
    "scan_closed_form": pin_scan_closed_form,
    "gate_modes": pin_gate_modes,
    "rope": pin_rope,
    "pe": pin_pe,
    "pe_values": pin_pe_values,
    "rope_values": pin_rope_values,
    "gate_value": pin_gate_value,
    "prefill_from_start_is_prefill": pin_prefill_from_start_is_prefill,
    "prefill_chunks_compose": pin_prefill_chunks_compose,
    "prefill_from_equals_decode_steps": pin_prefill_from_equals_decode_steps,
    "channel_gate_equal_columns_is_scalar": pin_channel_gate_equal_columns_is_scalar,
    "channel_gate_closed_form": pin_channel_gate_closed_form,
    "channel_gate_value": pin_channel_gate_value,
    "channel_incremental_equals_parallel": pin_channel_incremental_equals_parallel,
    "layer_selection_is_the_path": pin_layer_selection_is_the_path,
    "layer_absorption_fold": pin_layer_absorption_fold,
    "backward_finite_differences": pin_backward_finite_differences,
}


@pytest.fixture(autouse=True)
def _no_fault():
    oracle.set_fault(oracle.FAULT_NONE)
    yield
    oracle.set_fault(oracle.FAULT_NONE)


@pytest.mark.parametrize("name", sorted(PINS))
def test_pin(name):
    assert PINS[name](), f"oracle pin {name} failed"


FAULTS = {
    "drop_own_partial": oracle.FAULT_DROP_OWN_PARTIAL,
    "mask_off_by_one": oracle.FAULT_MASK_OFF_BY_ONE,
    "transpose_wuk": oracle.FAULT_TRANSPOSE_WUK,
    "rope_sign": oracle.FAULT_ROPE_SIGN,
    "scan_no_reset": oracle.FAULT_SCAN_NO_RESET,
    "drop_rope_key": oracle.FAULT_DROP_ROPE_KEY,
    "gate_wrong_row": oracle.FAULT_GATE_WRONG_ROW,
    "scale": oracle.FAULT_SCALE,
    "freq_exponent": oracle.FAULT_FREQ_EXPONENT,
    "pe_base": oracle.FAULT_PE_BASE,
    "pair_order": oracle.FAULT_PAIR_ORDER,
    "rope_half_split": oracle.FAULT_ROPE_HALF_SPLIT,
    "pe_swap": oracle.FAULT_PE_SWAP,
    "chunk_no_seed": oracle.FAULT_CHUNK_NO_SEED,
    "chunk_local_pos": oracle.FAULT_CHUNK_LOCAL_POS,
    "channel_transpose": oracle.FAULT_CHANNEL_TRANSPOSE,
    "bwd_no_delta": oracle.FAULT_BWD_NO_DELTA,
    "bwd_prefix_sum": oracle.FAULT_BWD_PREFIX_SUM,
    "bwd_no_sigmoid": oracle.FAULT_BWD_NO_SIGMOID,
}


@pytest.mark.parametrize("fault", sorted(FAULTS))
def test_planted_mistake_is_caught(fault):
    oracle.set_fault(FAULTS[fault])
    failed = [name for name, pin in PINS.items() if not pin()]
    assert failed, f"planted mistake {fault} passed every pin"


def test_mask_probe_support():
    """The one-hot probe used for the GPU mask test: zero queries and unit gates
    give o_lat = mean of e_j over the slots query i attends, i.e. support
    {0..floor(i/s)} (oracle side of the bit-exact mask test)."""
    from kv_cache_mtla_b200 import inputs
    for s in (1, 2, 3, 4):
        wl = inputs.TINY_FP32.with_(s=s, gate_mode=inputs.GATE_UNIT)
        T = 23
        p = inputs.one_hot_mask_probe(wl, T)
        cfg = oracle.Cfg(wl.B, wl.H, wl.d_h, wl.d_c, wl.d_r, s, gate_mode=oracle.GATE_UNIT)
        _, P = oracle.partials(cfg, p["c"], p["kr"])
        rows = np.array([[0, t] for t in range(T)])
        w = np.zeros((wl.H, wl.d_h, wl.d_c))
        _, olat = oracle.attend_rows(cfg, p["qc"], p["qr"], w, w, P, rows, want_olat=True)
        for t in range(T):
            support = np.nonzero(olat[t, 0])[0]
            assert list(support) == list(range(t // s + 1))
            assert np.allclose(olat[t, 0, support], 1.0 / (t // s + 1), atol=1e-15)


# ----------------------------------------------------------------- beam-search reorder


def test_reorder_worked_example():
    """Hand-worked case: 3 sequences, 3 slots of width 2, s = 2. Parents
    src = [2, 2, 0] (a duplicate, a cycle-free gather); n_tokens indexed by
    parent = [1, 4, 3]. Destination 0 and 1 take parent 2's ceil(3/2) = 2
    slots, destination 2 takes parent 0's ceil(1/2) = 1 slot; the rest of
    each destination keeps its old value (999). A scatter instead of a gather,
    a token count read at the destination, or floor instead of ceil each
    change this result."""
    ci = np.arange(18, dtype=np.uint16).reshape(3, 3, 2)
    co = np.full_like(ci, 999)
    oi = np.arange(6, dtype=np.float32).reshape(3, 2)
    oo = np.zeros_like(oi)
    assert oracle.reorder_cache(2, [2, 2, 0], [1, 4, 3], ci, oi, co, oo) == 0
    want = np.array([[[12, 13], [14, 15], [999, 999]],
                     [[12, 13], [14, 15], [999, 999]],
                     [[0, 1], [999, 999], [999, 999]]], dtype=np.uint16)
    assert np.array_equal(co, want)
    assert np.array_equal(oo, np.array([[4, 5], [4, 5], [0, 1]], dtype=np.float32))


def test_reorder_slot_count_is_ceil():
    """n tokens fill ceil(n/s) slots: 0, 1, s, s+1 and a full cache."""
    s, max_slots = 3, 4
    for n, slots in ((0, 0), (1, 1), (3, 1), (4, 2), (12, 4)):
        ci = np.arange(max_slots * 2, dtype=np.float32).reshape(1, max_slots, 2) + 1
        co = np.zeros_like(ci)
        oo = np.zeros((1, 2), np.float32)
        assert oracle.reorder_cache(s, [0], [n], ci, np.ones((1, 2), np.float32), co, oo) == 0
        copied = int((co[0] != 0).any(axis=1).sum())
        assert copied == slots, (n, copied)


def test_reorder_composes_like_a_gather():
    """Reordering by p and then by q (token counts follow the first reorder)
    equals one reorder by p[q]; a permutation followed by its inverse restores
    every filled slot."""
    rng = np.random.default_rng(7)
    B, max_slots, D, s = 9, 11, 4, 2
    ci = rng.standard_normal((B, max_slots, D)).astype(np.float32)
    oi = rng.standard_normal((B, D)).astype(np.float32)
    n = rng.integers(0, max_slots * s + 1, size=B).astype(np.int32)
    p = rng.integers(0, B, size=B)
    q = rng.integers(0, B, size=B)
    c1, o1 = np.zeros_like(ci), np.zeros_like(oi)
    oracle.reorder_cache(s, p, n, ci, oi, c1, o1)
    c2, o2 = np.zeros_like(ci), np.zeros_like(oi)
    oracle.reorder_cache(s, q, n[p], c1, o1, c2, o2)
    c3, o3 = np.zeros_like(ci), np.zeros_like(oi)
    oracle.reorder_cache(s, p[q], n, ci, oi, c3, o3)
    assert np.array_equal(c2, c3) and np.array_equal(o2, o3)
    perm = rng.permutation(B)
    back = np.argsort(perm)
    c4, o4 = np.zeros_like(ci), np.zeros_like(oi)
    oracle.reorder_cache(s, perm, n, ci, oi, c4, o4)
    c5, o5 = np.zeros_like(ci), np.zeros_like(oi)
    oracle.reorder_cache(s, back, n[perm], c4, o4, c5, o5)
    for b in range(B):
        k = (n[b] + s - 1) // s
        assert np.array_equal(c5[b, :k], ci[b, :k])
    assert np.array_equal(o5, oi)


def test_reorder_bad_parent_and_capacity():
    """A parent outside [0, B) gives status 1 and leaves its destination
    alone; a parent holding more tokens than the cache gives status 3."""
    ci = np.ones((2, 2, 2), np.float32)
    oi = np.ones((2, 2), np.float32)
    co, oo = np.zeros_like(ci), np.zeros_like(oi)
    assert oracle.reorder_cache(2, [0, 2], [4, 4], ci, oi, co, oo) == 1
    assert co[1].sum() == 0 and oo[1].sum() == 0 and co[0].sum() == 4
    co, oo = np.zeros_like(ci), np.zeros_like(oi)
    assert oracle.reorder_cache(2, [1, 0], [4, 5], ci, oi, co, oo) == 3
    assert co[0].sum() == 0 and co[1].sum() == 4


def test_backward_rows_are_the_backward_s_rows():
    """orc_backward_rows (one row's query gradients, computed alone) gives the
    rows of the whole backward's dqc and dqr, whose every entry the
    finite-difference pin holds; rows in any order, repeated, every gate mode."""
    rng = np.random.default_rng(170)
    for mode in (oracle.GATE_COMPUTED, oracle.GATE_SUPPLIED, oracle.GATE_UNIT):
        for s in (1, 3):
            B, T = 2, 11
            cfg, p = _rand_problem(B, 2, 4, 8, 4, s, T, seed=180 + 10 * mode + s, gate_mode=mode)
            G = p["G"] if mode == oracle.GATE_COMPUTED else None
            g = p["g"] if mode == oracle.GATE_COMPUTED else None
            gin = p["gate_in"] if mode == oracle.GATE_SUPPLIED else None
            dout = rng.standard_normal((B, T, 2, 4))
            full = oracle.prefill_backward(cfg, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"], dout,
                                           G, g, gin)
            rows = [(b, i) for b in range(B) for i in range(T)][::-1] + [(1, 5)]
            got = oracle.backward_rows(cfg, p["c"], p["kr"], p["qc"], p["qr"], p["w_uk"], p["w_uv"], dout, rows,
                                       G, g, gin)
            for r, (b, i) in enumerate(rows):
                assert np.max(np.abs(got["dqc"][r] - full["dqc"][b, i])) < 1e-12
                assert np.max(np.abs(got["dqr"][r] - full["dqr"][b, i])) < 1e-12


def test_linear_is_the_library_matmul():
    """orc_linear, the projections' reference, equals numpy's matmul (a library
    routine) on ragged shapes, and a transposed or offset read would not."""
    rng = np.random.default_rng(3)
    for M, N, K in ((1, 1, 1), (7, 5, 3), (33, 17, 70)):
        x, w = rng.standard_normal((M, K)), rng.standard_normal((N, K))
        assert np.max(np.abs(oracle.linear(x, w) - x @ w.T)) < 1e-12
