"""Benchmark of the LTE sparse-attention hot path on B200.

Default (one GPU): the prefill workload -- B=32, T=4096, 16 query heads over
4 KV heads, head dim 128, bf16, sink 4, window 512, cap 512, retention mask
Bernoulli(0.1) fed directly -- one step = lte_evict_compact (compaction and
column-segment copy) + lte_sparse_attn_prefill.  `value` = B*T tokens per
second of device time (max over ranks; every rank runs its own batch, so the
scaling is weak and no collective touches the data path).

Also reported on the same JSON line:
  roofline     the attention kernel's attended FLOPs / its CUDA-event time
               against the measured bf16 peak;
  e2e          the same step from pinned host buffers (H2D of q, k, v, mask
               and D2H of o inside the timed region);
  decode       the decode workload (4096-token prompt, B=32, CNN scored live,
               deferred batch 64): its 512 generated tokens, each fed once
               to each of 4 layer caches (> L2), in one CUDA graph;
  cpu_baseline the CPU oracle on a bounded sample of the same workload.
`--impl reference` times the CPU oracle alone (the reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import lte_inputs as LI  # noqa: E402
from learnable_kv_token_b200 import dist as DI  # noqa: E402

METRIC = "LTE sparse-attn prefill & decode tokens/s at 1 B200; % tensor/HBM roofline"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def attended_pairs(mask: np.ndarray, sink: int, window: int, cap: int) -> np.ndarray:
    """|S_t| per (b, h, t) from a fed mask [B,Hkv,T]: window + out-of-window
    sinks + min(C, retained tokens that left the window).  Work count only."""
    B, H, T = mask.shape
    m = mask.astype(np.int64).copy()
    m[..., :sink] = 0
    cnt = np.cumsum(m, axis=-1)
    t = np.arange(T)
    win = np.minimum(t + 1, window)
    sinks = np.clip(t - window + 1, 0, sink)
    n = np.zeros_like(cnt)
    if window < T:                       # retained tokens that have left the window
        n[..., window:] = cnt[..., :T - window]
    return win[None, None] + sinks[None, None] + np.minimum(n, cap)


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons while timing."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[1])); mx.append(float(f[2]))
            except ValueError:
                continue
            for n, val in zip(names, f[4:8]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_id(device):
    """nvidia-smi -i identifier of a torch device (UUID, so that
    CUDA_VISIBLE_DEVICES remapping does not matter)."""
    try:
        u = str(torch.cuda.get_device_properties(device).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return device.index if device.index is not None else 0


def source_hash(*files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_from_profiles(kernel_file, launch_units):
    """DRAM bytes per launch from the committed ncu summary, scaled to this
    launch by units processed, or None when the kernel changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        tr = json.load(f)
    ent = tr.get(kernel_file)
    if not ent or ent.get("source_hash") != source_hash(*ent.get("sources", [kernel_file])):
        return None
    return ent["dram_bytes_per_unit"] * launch_units


# ------------------------------------------------------------------------- oracle timing
def oracle_sample(wl, seconds_min, seconds_max, rows_per_unit=None):
    """Run the CPU oracle on (b, h) units of the workload until seconds_min
    have elapsed; returns (tokens_equivalent, seconds, description)."""
    from threadpoolctl import threadpool_limits

    from oracle import lte_oracle as O
    g = LI.generator(wl.seed)
    B = 1
    q, k, v = LI.qkv(B, wl.T, wl.Hq, wl.Hkv, wl.D, wl.dtype, g)
    mask = LI.bernoulli_mask(B, wl.Hkv, wl.T, wl.mask_rate, g)
    G = wl.G
    rows = list(range(wl.T)) if rows_per_unit is None else \
        list(range(wl.T - 1, -1, -max(1, wl.T // rows_per_unit)))
    qn = q.double().numpy(); kn = k.double().numpy(); vn = v.double().numpy()
    done_rows, t0 = 0, time.perf_counter()
    units = 0
    with threadpool_limits(1):
        for h in range(wl.Hkv):
            m = O.fed_mask(mask[0, h].numpy(), wl.sink)
            O.prefill_unit(qn[0, :, h * G:(h + 1) * G], kn[0, :, h], vn[0, :, h], m, wl.sink,
                           wl.window, wl.cap, wl.scale, rows=rows)
            done_rows += len(rows)
            units += 1
            el = time.perf_counter() - t0
            if el >= seconds_min or el >= seconds_max:
                break
    el = time.perf_counter() - t0
    desc = f"{units} (batch, KV-head) unit(s) x {len(rows)} rows of the {wl.name} workload"
    return done_rows / wl.Hkv, el, desc


_POOL_INPUTS = {}


def _oracle_inputs():
    """Sequence 0 of the prefill workload as float64 arrays, in this process's
    globals (forked oracle workers inherit them)."""
    from oracle import lte_oracle as O
    wl = LI.WORKLOADS["prefill"]
    g = LI.generator(wl.seed)
    q, k, v = LI.qkv(1, wl.T, wl.Hq, wl.Hkv, wl.D, wl.dtype, g)
    mask = LI.bernoulli_mask(1, wl.Hkv, wl.T, wl.mask_rate, g)
    _POOL_INPUTS.update(wl=wl, q=q.double().numpy(), k=k.double().numpy(), v=v.double().numpy(),
                        m=[O.fed_mask(mask[0, h].numpy(), wl.sink) for h in range(wl.Hkv)])


def _oracle_pool_task(task):
    """Oracle rows `rows` of KV head h of sequence 0 on one core."""
    from threadpoolctl import threadpool_limits

    from oracle import lte_oracle as O
    h, rows = task
    d = _POOL_INPUTS
    wl, G = d["wl"], d["wl"].G
    with threadpool_limits(1):
        O.prefill_unit(d["q"][0, :, h * G:(h + 1) * G], d["k"][0, :, h], d["v"][0, :, h], d["m"][h],
                       wl.sink, wl.window, wl.cap, wl.scale, rows=rows)
    return len(rows)


def start_oracle_pool():
    """A process pool for the all-core oracle leg, forked now, before this
    process makes its first GPU call (its workers run numpy only).  One worker
    per host core, at most 128."""
    import multiprocessing as mp
    _oracle_inputs()
    cores = max(1, min(os.cpu_count() or 1, 128))
    return mp.get_context("fork").Pool(cores), cores


def oracle_sample_all_cores(pool, cores, seconds, one_core_rate):
    """The oracle on every host core: `cores` single-threaded workers compute
    rows of sequence 0's four units of the prefill workload, the whole sequence
    repeated until about `seconds` of wall time; returns (tokens_equivalent,
    seconds, description)."""
    wl = LI.WORKLOADS["prefill"]
    chunk = 128
    per_seq = [(h, list(range(r0, min(r0 + chunk, wl.T)))) for h in range(wl.Hkv)
               for r0 in range(0, wl.T, chunk)]
    reps = max(1, int(round(seconds * one_core_rate * cores / wl.T)))
    limit = 20 * seconds + 120                                  # a failed worker ends the leg
    pool.map_async(_oracle_pool_task, per_seq[:cores]).get(limit)      # workers warm
    t0 = time.perf_counter()
    rows = sum(pool.map_async(_oracle_pool_task, per_seq * reps, chunksize=1).get(limit))
    el = time.perf_counter() - t0
    desc = (f"{cores} single-threaded processes, sequence 0 of the {wl.name} workload "
            f"(4 units x {wl.T} rows) computed {reps} time(s)")
    return rows / wl.Hkv, el, desc


def run_reference(args, rank, world):
    if rank != 0:
        return
    wl = LI.WORKLOADS["prefill"]
    for _ in range(args.warmup):
        oracle_sample(wl, 0.0, 1e9, rows_per_unit=128)
    tok, sec = 0.0, 0.0
    for _ in range(args.steps):
        a, b, desc = oracle_sample(wl, 0.0, 1e9, rows_per_unit=128)
        tok += a; sec += b
    value = tok / sec
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sec / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "prefill B=32 T=4096 Hq=16 Hkv=4 D=128 s=4 w=512 C=512 mask~Bern(0.1)",
                       "global_batch": wl.B, "seq_len": wl.T, "parallelism": "replicas"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"per step: {desc} (128 strided rows of KV head 0)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------- GPU arm
def prefill_bench(args, rank, world, device):
    from learnable_kv_token_b200 import layer, lte as L
    wl = LI.WORKLOADS["prefill"]
    if args.batch:                                  # smaller case for profiler captures
        wl = wl.with_(B=args.batch)
    inp = LI.lte_inputs(wl.with_(seed=DI.shard_seed(wl.seed, rank)), T=wl.T)
    q, k, v, mask = inp["q"], inp["k"], inp["v"], inp["mask"]
    B, T, Hq, Hkv, D = wl.B, wl.T, wl.Hq, wl.Hkv, wl.D
    pairs = attended_pairs(mask.numpy(), wl.sink, wl.window, wl.cap)
    flops = 4.0 * D * wl.G * float(pairs.sum())         # QK^T + PV per (row, head, key)
    p = layer.LayerParams(sink=wl.sink, window=wl.window, cap=wl.cap, tau=wl.tau)
    dims = p.dims(B, T, Hq, Hkv, D, torch.bfloat16)
    qd, kd, vd, md = (x.to(device) for x in (q, k, v, mask))
    bufs = layer.PrefillBuffers(B, T, Hq, Hkv, D, torch.bfloat16, wl.sink, dims, device,
                                want_r=False)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        L.lte_evict_compact(dims, None, md, T, bufs.idx, bufs.nret, bufs.cnt, kd, vd, bufs.k_col,
                            bufs.v_col, stream)
        if ev is not None:
            ev[0].record(stream)
        L.lte_sparse_attn_prefill(dims, qd, kd, vd, bufs.cnt, bufs.k_col, bufs.v_col, bufs.o,
                                  bufs.lse, bufs.ws, stream)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    DI.barrier(world)
    torch.cuda.synchronize()
    with Clocks(gpu_id(device)) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
    DI.barrier(world)
    ms_total = t_start.elapsed_time(t_end)
    attn_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    ms_total = DI.max_over_ranks(ms_total, world, device)
    attn_ms = DI.max_over_ranks(attn_ms, world, device)
    ms_step = ms_total / args.steps
    assert L.lte_read_device_error(bufs.ws) == (0, 0)

    # e2e: pinned host buffers, H2D of the inputs and D2H of o inside the timed
    # region, through layer.HostPrefill (sub-batches of 4 sequences: the copies
    # in and out overlap each other and the compute)
    hq, hk, hv, hm = (x.pin_memory() for x in (q, k, v, mask))
    ho = torch.empty(bufs.o.shape, dtype=bufs.o.dtype).pin_memory()
    n_e2e = max(3, min(args.steps, 10))
    hp = layer.HostPrefill(B, T, Hq, Hkv, D, torch.bfloat16, p, chunk=4 if B % 4 == 0 else B,
                           device=device)
    hp.run(hq, hk, hv, hm, ho, stream)
    torch.cuda.synchronize()
    DI.barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_e2e):
        hp.run(hq, hk, hv, hm, ho, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = DI.max_over_ranks(e0.elapsed_time(e1) / n_e2e, world, device)
    assert all(e == (0, 0) for e in hp.device_errors())
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hm))
    d2h = ho.numel() * ho.element_size()

    return {
        "B": B, "T": T, "flops": flops, "pairs": float(pairs.sum()), "ms_step": ms_step,
        "attn_ms": attn_ms, "clocks": clk.summary(), "e2e_ms": e2e_ms, "h2d": h2d, "d2h": d2h,
        "launches": 2 * args.steps, "units": B * Hkv * ((T + 32 - 1) // 32),
        "e2e_ok": bool((ho.view(torch.int16) == bufs.o.cpu().view(torch.int16)).all()),
        "full_causal_pairs": B * Hkv * T * (T + 1) / 2,
    }


def decode_bench(args, rank, world, device, n_layers=4):
    """Decode after the 4096-token prompt: each of `n_layers` layer caches (together
    larger than L2) is initialised from the prompt's prefill, then fed the
    workload's generated tokens, one per step, rotating over the layers, in one
    CUDA graph.  The graph is replayed once to warm up; the caches are then put
    back to their post-prompt state and the timed replay feeds every generated
    token exactly once per layer cache, at positions T0 .. T0 + S - 1."""
    from learnable_kv_token_b200 import layer
    wl = LI.WORKLOADS["decode"]
    inp = LI.lte_inputs(wl.with_(seed=DI.shard_seed(wl.seed, rank)))
    q, k, v, cnn = inp["q"], inp["k"], inp["v"], inp["cnn"]
    B, T0, Hq, Hkv, D = wl.B, wl.T, wl.Hq, wl.Hkv, wl.D
    S = wl.decode_steps
    p = layer.LayerParams(sink=wl.sink, window=wl.window, cap=wl.cap, tau=wl.tau)
    qd, kd, vd = (x.to(device) for x in (q, k, v))
    cd = tuple(x.to(device) for x in cnn)
    kp, vp, qp = kd[:, :T0].contiguous(), vd[:, :T0].contiguous(), qd[:, :T0].contiguous()
    dims = p.dims(B, T0, Hq, Hkv, D, torch.bfloat16)
    torch.cuda.synchronize()
    tp0 = time.perf_counter()
    out = layer.prefill(qp, kp, vp, p, cnn=cd)
    torch.cuda.synchronize()
    prefill_cnn_ms = 1e3 * (time.perf_counter() - tp0)
    decs = []
    for _ in range(n_layers):
        cache = layer.DecodeCache(B, Hkv, D, torch.bfloat16, wl.sink, wl.window, wl.cap, device)
        cache.init_from_prefill(dims, kp, vp, out, T0)
        decs.append(layer.Decoder(dims, cd, p.past1, p.past2, cache, wl.score_batch, device))
    del out, qp, kp, vp
    torch.cuda.synchronize()
    snaps = [d.cache.snapshot() for d in decs]

    def rewind():
        torch.cuda.synchronize()
        for d, sn in zip(decs, snaps):
            d.cache.restore(sn)
        torch.cuda.synchronize()

    qs = qd[:, T0:].permute(1, 0, 2, 3).contiguous()
    ks = kd[:, T0:].permute(1, 0, 2, 3).contiguous()
    vs = vd[:, T0:].permute(1, 0, 2, 3).contiguous()
    del qd, kd, vd
    assert qs.shape[0] == S
    stream = torch.cuda.Stream(device)
    # warm-up: a few eager steps per layer
    with torch.cuda.stream(stream):
        for i in range(3):
            for d in decs:
                d.step(qs[i], ks[i], vs[i], stream=stream)
    rewind()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            for t in range(S):
                for d in decs:
                    d.step(qs[t], ks[t], vs[t], stream=stream)
    with torch.cuda.stream(stream):    # replay() launches on the current stream
        graph.replay()                 # warm replay
    rewind()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    DI.barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    n_steps = S * n_layers
    ms_step = DI.max_over_ranks(e0.elapsed_time(e1) / n_steps, world, device)
    assert all(d_.device_error() == (0, 0) for d_ in decs)
    ret = decs[0].cache.ret_total.clone()
    t_meta = int(decs[0].cache.meta[0])
    assert t_meta == T0 + S
    del graph
    # the laLTE pair step: one gated linear-attention layer step (16 heads,
    # dk = dv = 128, its own fp32 state per layer) followed by the LTE layer
    # step, over the same 4 layers, in one CUDA graph, for the hybrid
    # workload's generated tokens (each fed once per layer in the timed
    # replay, the caches rewound to the prompt and the states zeroed before it).
    # The GLA step is launched with programmatic dependent launch, so each
    # kernel's CTAs are resident and through their prologue when its
    # predecessor ends.
    from learnable_kv_token_b200 import lte as L
    S_pair = LI.WORKLOADS["hybrid"].decode_steps
    H_g, dk_g = 16, 128
    gq, gk, gv, ga = (x.transpose(0, 1).contiguous().to(device) for x in
                      LI.gla_inputs(B, S_pair, H_g, dk_g, dk_g, LI.generator(wl.seed + 2000)))
    go = torch.empty_like(gv[0])
    states = [torch.zeros(B, H_g, dk_g, dk_g, dtype=torch.float32, device=device)
              for _ in range(n_layers)]

    def rewind_pair():
        rewind()
        for st_ in states:
            st_.zero_()
        torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for d_, st_ in zip(decs, states):
            L.lte_gla_decode_step(gq[0], gk[0], gv[0], ga[0], go, st_, stream)
            d_.step(qs[0], ks[0], vs[0], stream=stream)
    rewind_pair()
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(pgraph, stream=stream):
            for t in range(S_pair):
                for d_, st_ in zip(decs, states):
                    L.lte_gla_decode_step(gq[t], gk[t], gv[t], ga[t], go, st_, stream)
                    d_.step(qs[t], ks[t], vs[t], stream=stream)
    with torch.cuda.stream(stream):
        pgraph.replay()
    rewind_pair()
    DI.barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        pgraph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    pair_ms = DI.max_over_ranks(e0.elapsed_time(e1) / (S_pair * n_layers), world, device)
    assert all(d_.device_error() == (0, 0) for d_ in decs)
    del pgraph, states, snaps
    gla_bytes = 2 * B * H_g * dk_g * dk_g * 4 + B * H_g * dk_g * (4 * 2 + 4)
    # algorithmic bytes of one layer step (steady state)
    n_keys = (min(wl.window, t_meta) + wl.sink + torch.clamp(ret, max=wl.cap)).sum().item()
    units = B * Hkv
    row = 2 * D * 2                                   # K + V bf16
    bytes_step = (n_keys * row                        # attended K/V
                  + 2 * B * Hq * D * 2                # q in, o out
                  + units * row * 2                   # new token write + leaving-token move
                  + units * row * (wl.score_batch + 6) / wl.score_batch)   # deferred scoring reads
    # the library fuses the whole step into one kernel when every (batch, KV head)
    # unit gets its own CTA (units <= SMs) and the CNN fits its tensor-core scoring
    # tile (c_hid * k1 <= 160); otherwise a step is an update kernel + an attention kernel
    n_sm = torch.cuda.get_device_properties(device).multi_processor_count
    fused = units <= n_sm and wl.c_hid * wl.k1 <= 160
    return {"ms_step": ms_step, "bytes": bytes_step, "n_keys": n_keys, "B": B, "units": units,
            "prefill_with_cnn_ms": prefill_cnn_ms, "fused": fused,
            "launches": (1 if fused else 2) * n_steps,
            "pair_ms": pair_ms, "pair_bytes": bytes_step + gla_bytes}


def sweep_bench(args, rank, world, device, only=None, reps=5):
    """The long-context sparsity sweep: B=4, T=16384, Hq=16 / Hkv=4, D=128, bf16,
    s=4, w=1024, C in {0, 1024, 4096, 16384} x retention rate in {0, 5, 25,
    100} %, per-KV-head rates ~ U[0, 2 rate] clipped (rate 100 % retains every
    token, so C = 16384 is full causal attention).  Per point: compaction once,
    then `reps` attention launches timed with CUDA events after 2 warm-ups;
    the attended FLOPs are counted exactly from the drawn mask.  Inputs are
    larger than L2 (q 256 MiB).  `only` = (cap, rate) restricts it to one point
    (profiler captures)."""
    from learnable_kv_token_b200 import layer, lte as L
    wl = LI.WORKLOADS["sweep"]
    B = args.batch or wl.B
    T, Hq, Hkv, D = wl.T, wl.Hq, wl.Hkv, wl.D
    seed = DI.shard_seed(wl.seed, rank)
    g = LI.generator(seed)
    q, k, v = (x.to(device) for x in LI.qkv(B, T, Hq, Hkv, D, wl.dtype, g))
    stream = torch.cuda.current_stream(device)
    pk = peaks()
    points = []
    bufs = None
    for cap in LI.SWEEP_CAPS:
        for rate in LI.SWEEP_RATES:
            if only is not None and (cap, rate) != only:
                continue
            mask = LI.rate_mask(B, Hkv, T, rate, LI.generator(seed + 1000 + cap + int(rate * 100)))
            pairs = attended_pairs(mask.numpy(), wl.sink, wl.window, cap)
            flops = 4.0 * D * wl.G * float(pairs.sum())
            p = layer.LayerParams(sink=wl.sink, window=wl.window, cap=cap, tau=wl.tau)
            dims = p.dims(B, T, Hq, Hkv, D, torch.bfloat16)
            if bufs is None:
                bufs = layer.PrefillBuffers(B, T, Hq, Hkv, D, torch.bfloat16, wl.sink, dims, device,
                                            want_r=False)
            md = mask.to(device)

            def compact():
                L.lte_evict_compact(dims, None, md, T, bufs.idx, bufs.nret, bufs.cnt, k, v,
                                    bufs.k_col, bufs.v_col, stream)

            def attn():
                L.lte_sparse_attn_prefill(dims, q, k, v, bufs.cnt, bufs.k_col, bufs.v_col, bufs.o,
                                          bufs.lse, bufs.ws, stream)

            def timed(fn, n):
                for _ in range(2):
                    fn()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(n):
                    fn()
                e1.record(stream)
                torch.cuda.synchronize()
                return DI.max_over_ranks(e0.elapsed_time(e1) / n, world, device)

            t_c = timed(compact, 3)
            compact()
            t_a = timed(attn, reps)
            assert L.lte_read_device_error(bufs.ws) == (0, 0)
            tf = flops / (t_a / 1e3) / 1e12
            rates = mask[..., wl.sink:].float().mean(dim=-1)
            points.append({
                "cap": cap, "rate": rate, "attended_flops": flops,
                "frac_of_full_causal": float(pairs.sum()) / (B * Hkv * T * (T + 1) / 2),
                "head_rate_min": float(rates.min()), "head_rate_max": float(rates.max()),
                "attn_ms": t_a, "compact_ms": t_c,
                "tokens_per_s": DI.job_throughput(B * T, world, (t_a + t_c) / 1e3),
                "achieved_tflops": tf, "frac": tf / pk["bf16_tflops"],
                "frac_of_sustained": tf / pk["bf16_tflops_sustained"]})
            del md
    del q, k, v, bufs
    worst = min(points, key=lambda x: x["frac"]) if points else None
    return {"workload": f"sweep B={B} T={T} Hq=16 Hkv=4 D=128 bf16 s=4 w=1024, C x per-head "
                        "rate ~ U[0, 2 rate] clipped; step = evict_compact + sparse_attn_prefill; "
                        "inputs larger than L2",
            "peak": pk["bf16_tflops"], "peak_source": pk["source"], "points": points,
            "worst": None if worst is None else {"cap": worst["cap"], "rate": worst["rate"],
                                                 "frac": worst["frac"]},
            "launches": len(points) * (5 + reps + 2 + 1)}


def rows_bench(args, rank, world, device, dec):
    """The hot-path rows outside the two headline steps, each launch timed alone
    with CUDA events after warm-up, on the hybrid workload (B=32, 4096-token
    prompts, Hq=16 / Hkv=4, D=128, the CNN scored live, tau 0.5): retention
    scoring (a1), compaction with the column copy (a2), sparse-attention prefill
    over the scored mask (a3 at the scored retention rate), gated linear
    attention prefill and decode step (a7); and the laLTE pair -- one gated
    linear-attention layer followed by one LTE layer -- as tokens/s."""
    from learnable_kv_token_b200 import layer
    from learnable_kv_token_b200 import lte as L
    wl = LI.WORKLOADS["hybrid"]
    if args.batch:                                  # smaller case for profiler captures
        wl = wl.with_(B=args.batch)
    B, T, Hq, Hkv, D = wl.B, wl.T, wl.Hq, wl.Hkv, wl.D
    seed = DI.shard_seed(wl.seed, rank)
    inp = LI.lte_inputs(wl.with_(seed=seed), T=T)
    q, k, v = (inp[x].to(device) for x in ("q", "k", "v"))
    cnn = tuple(x.to(device) for x in inp["cnn"])
    p = layer.LayerParams(sink=wl.sink, window=wl.window, cap=wl.cap, tau=wl.tau)
    dims = p.dims(B, T, Hq, Hkv, D, torch.bfloat16)
    bufs = layer.PrefillBuffers(B, T, Hq, Hkv, D, torch.bfloat16, wl.sink, dims, device, want_r=True)
    c, _keep = L.make_cnn(*cnn, p.past1, p.past2)
    n_scored = T - layer.cnn_future(cnn[0], cnn[2], p.past1, p.past2)
    stream = torch.cuda.current_stream(device)

    def timed(fn, reps=5):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return DI.max_over_ranks(e0.elapsed_time(e1) / reps, world, device)

    t_score = timed(lambda: L.lte_score(dims, c, k, v, 0, n_scored, bufs.r, bufs.mask, stream))
    t_compact = timed(lambda: L.lte_evict_compact(dims, None, bufs.mask, n_scored, bufs.idx,
                                                  bufs.nret, bufs.cnt, k, v, bufs.k_col,
                                                  bufs.v_col, stream))
    t_attn = timed(lambda: L.lte_sparse_attn_prefill(dims, q, k, v, bufs.cnt, bufs.k_col,
                                                     bufs.v_col, bufs.o, bufs.lse, bufs.ws, stream))
    assert L.lte_read_device_error(bufs.ws) == (0, 0)
    # backward of the attention (fixed attended sets); dO = q stands in for the
    # incoming gradient (any [B,T,Hq,D] tensor: the work does not depend on it)
    dq = torch.empty(B, T, Hq, D, dtype=torch.float32, device=device)
    dk = torch.empty(B, T, Hkv, D, dtype=torch.float32, device=device)
    dv = torch.empty_like(dk)
    ws_b = torch.zeros(L.lte_workspace_bytes(dims, L.LTE_WS_BACKWARD) + 16, dtype=torch.uint8,
                       device=device)
    t_bwd = timed(lambda: L.lte_sparse_attn_backward(dims, q, k, v, bufs.cnt, None, bufs.idx,
                                                     bufs.nret, bufs.k_col, bufs.v_col, bufs.o,
                                                     bufs.lse, q, dq, dk, dv, ws_b, stream))
    assert L.lte_read_device_error(ws_b) == (0, 0)
    # backward through the scoring CNN (dL/dr = the scores themselves stand in
    # for an incoming gradient: the work does not depend on its values)
    dw1 = torch.empty_like(cnn[0]); db1 = torch.empty_like(cnn[1])
    dw2 = torch.empty_like(cnn[2]); db2 = torch.empty_like(cnn[3])
    ws_s = torch.zeros(L.lte_score_backward_workspace_bytes(dims, c) + 16, dtype=torch.uint8,
                       device=device)
    t_sbwd = timed(lambda: L.lte_score_backward(dims, c, k, v, n_scored, bufs.r, dk, dv, dw1, db1,
                                                dw2, db2, ws_s, stream))
    assert L.lte_read_device_error(ws_s) == (0, 0)
    del dq, dk, dv, ws_b, ws_s, dw1, db1, dw2, db2
    mask = bufs.mask.cpu().numpy()
    nret = int(bufs.nret.sum())
    pairs = attended_pairs(mask, wl.sink, wl.window, wl.cap).sum()
    attn_flops = 4.0 * D * wl.G * float(pairs)
    bwd_flops = 2.5 * attn_flops           # S, dP, dQ, dK, dV over the attended pairs
    # CNN backward: layer 1 recomputed, dx and dw1 (each 2 c_hid 2D k1 flops per
    # position), layer 2 terms (small)
    sbwd_flops = 3.0 * 2 * B * Hkv * T * wl.c_hid * 2 * D * wl.k1
    score_flops = 2.0 * B * Hkv * n_scored * (wl.c_hid * 2 * D * wl.k1 + wl.c_hid * wl.k2)
    score_bytes = B * T * Hkv * D * 2 * 2 + B * Hkv * n_scored * 5
    compact_bytes = (B * Hkv * T * (1 + 8) + B * Hkv * 4
                     + 2 * (wl.sink * B * Hkv + nret) * 2 * D * 2)
    del bufs, q, k, v

    H, dk = 16, 128
    gq, gk, gv, ga = (x.to(device) for x in LI.gla_inputs(B, T, H, dk, dk, LI.generator(seed + 1000)))
    go = torch.empty_like(gv)
    state = torch.zeros(B, H, dk, dk, dtype=torch.float32, device=device)
    t_gla = timed(lambda: L.lte_gla_prefill(gq, gk, gv, ga, go, state, stream))
    q1, k1_, v1, a1, o1 = (x[:, 0].contiguous() for x in (gq, gk, gv, ga, go))
    # decode steps rotate over 6 layer states (6 x 32 MiB > L2), as a layer stack would
    states = [state.clone() for _ in range(6)]
    it_st = iter(range(1 << 30))
    t_gla_dec = timed(lambda: L.lte_gla_decode_step(q1, k1_, v1, a1, o1, states[next(it_st) % 6],
                                                    stream), reps=60)
    gla_bytes = B * T * H * dk * (4 * 2 + 4) + B * H * dk * dk * 4
    gla_dec_bytes = 2 * B * H * dk * dk * 4 + B * H * dk * (4 * 2 + 4)
    pk = peaks()

    def hbm(nbytes, ms):
        gbs = nbytes / (ms / 1e3) / 1e9
        return {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / pk["hbm_gbs"], "bytes": nbytes}

    def tensor(flops, ms):
        tf = flops / (ms / 1e3) / 1e12
        return {"bound": "tensor", "achieved": tf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": tf / pk["bf16_tflops"], "flops": flops}

    lte_prefill_ms = t_score + t_compact + t_attn
    return {
        "workload": f"hybrid B={B} T=4096 (prompt) Hq=16 Hkv=4 D=128 bf16 s=4 w=512 C=512, CNN "
                    "32ch k5/k3 scored live, tau 0.5; GLA 16 heads dk=dv=128, chunk 64",
        "a1_score_ms": t_score, "a1_roofline": tensor(score_flops, t_score),
        "a1_bytes_rate": dict(hbm(score_bytes, t_score), traffic=traffic_from_profiles(
            "learnable_kv_token_b200/csrc/score_tcgen05.cu", B * Hkv * n_scored)),
        "a2_compact_ms": t_compact, "a2_roofline": hbm(compact_bytes, t_compact),
        "a3_attn_ms": t_attn, "a3_roofline": tensor(attn_flops, t_attn),
        "a3_retention_rate": float(mask[..., wl.sink:n_scored].mean()),
        "a3b_backward_ms": t_bwd, "a3b_roofline": tensor(bwd_flops, t_bwd),
        "a1b_score_backward_ms": t_sbwd,
        "a1b_roofline": dict(tensor(sbwd_flops, t_sbwd),
                             note="lte_score_backward: layer-1 recompute, dx and dw1 on tcgen05 "
                                  "(hi/lo bf16 operands: 2-3x the MMA work of these algorithmic "
                                  "flops), the elementwise pass on CUDA cores; FLOPs = 3 x 2 x "
                                  "c_hid x 2D x k1 per (b, KV head, position)"),
        "a3b_note": "lte_sparse_attn_backward (dQ with D_t, column work list, dK/dV window, "
                    "dK/dV column: 4 launches, tcgen05) on the same scored mask; FLOPs = 2.5 x "
                    "the forward's",
        "a7_gla_prefill_ms": t_gla, "a7_prefill_roofline": hbm(gla_bytes, t_gla),
        "a7_gla_decode_us": 1e3 * t_gla_dec, "a7_decode_roofline": hbm(gla_dec_bytes, t_gla_dec),
        "pair_prefill": {"value": DI.job_throughput(B * T, world, (t_gla + lte_prefill_ms) / 1e3),
                         "unit": "tokens/s", "ms": t_gla + lte_prefill_ms},
        "pair_decode": (None if dec is None else
                        {"value": DI.job_throughput(dec["B"], world, dec["pair_ms"] / 1e3),
                         "unit": "tokens/s", "us": 1e3 * dec["pair_ms"],
                         "roofline": hbm(dec["pair_bytes"], dec["pair_ms"]),
                         "sum_of_separate_steps_us": 1e3 * (t_gla_dec + dec["ms_step"]),
                         "note": "GLA step then LTE step per layer, 4 layers rotated, one CUDA "
                                 "graph of 256 generated tokens x 4 layers, each token fed once, "
                                 "programmatic dependent launch"}),
        "launches": 2 + 5 * 3 + 5 + 50 + 4 * 7 + 4 * 7,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="lte", choices=["lte", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-rows", action="store_true",
                    help="skip the per-row measurements (scoring, compaction, GLA, hybrid pair)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="oracle CPU sample length (0 skips the cpu_baseline leg)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the long-context sparsity sweep (16 points)")
    ap.add_argument("--sweep-only", default=None, metavar="CAP,RATE",
                    help="run only this sweep point (e.g. 16384,0.05), for profiler captures")
    ap.add_argument("--batch", type=int, default=0,
                    help="batch override of the prefill and per-row workloads, for profiler "
                         "captures (default: the workloads')")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    rank, world, local = DI.env_ranks()

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    pool = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        pool, pool_cores = start_oracle_pool()        # forked before the first GPU call
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    DI.init(world, "nccl", device, timeout_s=120)
    from learnable_kv_token_b200 import build as _b  # noqa: F401  (library is prebuilt in-tree)

    pk = peaks()
    if args.sweep_only:
        c_, r_ = args.sweep_only.split(",")
        sw = sweep_bench(args, rank, world, device, only=(int(c_), float(r_)))
        if rank == 0:
            print(json.dumps({"sweep": sw}), flush=True)
        DI.shutdown(world)
        return
    pf = prefill_bench(args, rank, world, device)
    dec = None if args.no_decode else decode_bench(args, rank, world, device)
    rows = None if args.no_rows else rows_bench(args, rank, world, device, dec)
    sweep = None if args.no_sweep else sweep_bench(args, rank, world, device)

    if rank == 0:
        value = DI.job_throughput(pf["B"] * pf["T"], world, pf["ms_step"] / 1e3)
        attn_tflops = pf["flops"] / (pf["attn_ms"] / 1e3) / 1e12
        traffic = traffic_from_profiles("learnable_kv_token_b200/csrc/attn_prefill_tc.cu",
                                        pf["units"])
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": pf["ms_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"prefill B={pf['B']} T=4096 Hq=16 Hkv=4 D=128 bf16 s=4 w=512 C=512 "
                                   "mask~Bern(0.1) fed; step = evict_compact + sparse_attn_prefill",
                       "global_batch": pf["B"] * world, "seq_len": pf["T"],
                       "parallelism": f"dp{world} (independent sequences per GPU)",
                       "l2": f"inputs larger than L2 (q {pf['B'] * pf['T'] * 16 * 128 * 2 >> 20} MiB, "
                             f"k/v {pf['B'] * pf['T'] * 4 * 128 * 2 >> 20} MiB each)"},
            "roofline": {"kernel": "attn_prefill_tc_kernel", "bound": "tensor",
                         "achieved": attn_tflops, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": attn_tflops / pk["bf16_tflops"],
                         "frac_of_sustained": attn_tflops / pk["bf16_tflops_sustained"],
                         "peak_source": pk["source"], "traffic": traffic,
                         "attended_flops_per_launch": pf["flops"],
                         "kernel_ms": pf["attn_ms"],
                         "sparsity_vs_full_causal": pf["pairs"] / pf["full_causal_pairs"]},
            "clocks": pf["clocks"],
            "e2e": {"value": DI.job_throughput(pf["B"] * pf["T"], world, pf["e2e_ms"] / 1e3),
                    "unit": "tokens/s",
                    "h2d_bytes_per_step": pf["h2d"], "d2h_bytes_per_step": pf["d2h"],
                    "path": "layer.HostPrefill: sub-batches of 4 sequences, copies in/out "
                            "overlapping the compute", "o_equals_device_step": pf["e2e_ok"]},
            "gpu_launches": pf["launches"] + (dec["launches"] if dec else 0),
        }
        if dec is not None:
            gbs = dec["bytes"] / (dec["ms_step"] / 1e3) / 1e9
            line["decode"] = {
                "workload": "decode B=32, 4096-token prompt, Hq=16 Hkv=4 D=128 bf16 s=4 w=512 "
                            "C=512, CNN scored live (tau 0.5, deferred batch 64); the 512 "
                            "generated tokens, each fed once to each of 4 layer caches (> L2), "
                            "2048 steps in one CUDA graph",
                "value": DI.job_throughput(dec["B"], world, dec["ms_step"] / 1e3), "unit": "tokens/s",
                "us_per_layer_step": 1e3 * dec["ms_step"],
                "roofline": {"bound": "hbm",
                             "scope": "whole decode step (" + ("one fused kernel" if dec["fused"]
                                                               else "2 kernels") + ")",
                             "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": gbs / pk["hbm_gbs"], "bytes_per_step": dec["bytes"],
                             "traffic": (traffic_from_profiles("learnable_kv_token_b200/csrc/decode.cu",
                                                               dec["units"])
                                         if dec["fused"] else None)},
                "prompt_prefill_with_cnn_ms": dec["prefill_with_cnn_ms"],
            }
        if rows is not None:
            line["rows"] = {k: v for k, v in rows.items() if k != "launches"}
        if sweep is not None:
            line.setdefault("rows", {})["sweep"] = {k: v for k, v in sweep.items()
                                                    if k != "launches"}
        if world == 1 and args.cpu_seconds > 0:
            tok, sec, desc = oracle_sample(LI.WORKLOADS["prefill"], args.cpu_seconds / 2,
                                           1.25 * args.cpu_seconds)
            one = tok / sec
            tok_n, sec_n, desc_n = oracle_sample_all_cores(pool, pool_cores, args.cpu_seconds / 2, one)
            line["cpu_baseline"] = {"value": tok_n / sec_n, "unit": "tokens/s", "cores": pool_cores,
                                    "kind": "oracle", "sample": desc_n,
                                    "one_core": {"value": one, "unit": "tokens/s", "cores": 1,
                                                 "sample": desc}}
        print(json.dumps(line), flush=True)
    if pool is not None:
        pool.terminate()
    DI.shutdown(world)


if __name__ == "__main__":
    main()
