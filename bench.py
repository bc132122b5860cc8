"""Benchmark of the routed top-k MoE layer (one JSON line on rank 0).

Headline workload: the Qwen3-Next-shaped decode layer with IQ2_XS-style
experts (hidden 2048, 512 experts of width 512, top-10, one token per call).
All selected experts are resident; the calls cycle through 48 pairwise-disjoint
top-10 sets (480 experts, 436 MB of packed weights, far above the 126 MB L2), so
every call streams its experts from HBM.  Calls are issued as CUDA-graph
replays of the C-ABI call.

A step is a fixed number of graph replays (`calls_per_step` layer calls:
50 passes over the 48 decode sets, 50 batched-decode calls, 10 prefill calls),
so `--steps K` times exactly K steps.  On one GPU the line also carries a
`workloads` map with the other workloads (IQ1_M-style cold decode, batched
decode, prefill), each measured the same way.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2..5] [--workloads 3,4,5|none]
  python bench.py --impl reference ...   # the fp64 CPU oracle, timed on host cores

Multi-GPU (torchrun): every rank runs an independent replica (the layer has no
exchange step); value = all ranks' tokens / the slowest rank's device time.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import fixtures  # noqa: E402

METRIC = "routed-MoE-layer tokens/sec on 1 B200; achieved HBM GB/s vs ~8 TB/s peak"
N_SETS = 48
# calls captured in one CUDA graph, and graph replays per step
GRAPH_CALLS = {2: 240, 3: 240, 4: 10, 5: 10}
REPLAYS_PER_STEP = {2: 10, 3: 10, 4: 5, 5: 1}
DTYPE = {2: "f32", 3: "f32", 4: "f32", 5: "bf16"}


def calls_per_step(cfg: int) -> int:
    return GRAPH_CALLS[cfg] * REPLAYS_PER_STEP[cfg]


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


class ClockSampler:
    """nvidia-smi samples every 100 ms; only samples taken inside the timed
    window (host timestamps) are summarised, unless the window saw none."""

    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.window = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    @staticmethod
    def summarise(rows, window=None):
        def ts(r):
            try:
                return datetime.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                return None

        inside = [r for r in rows if window and ts(r) is not None and window[0] <= ts(r) <= window[1]]
        use = inside if inside else rows

        def num(v):
            v = v.strip()
            return float(v) if v.replace(".", "", 1).isdigit() else None

        sm = [num(r[2]) for r in use if num(r[2]) is not None]
        mx = [num(r[3]) for r in use if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i in range(4) if "Active" in r[6 + i] and "Not" not in r[6 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(use), "samples_in_window": len(inside)}

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 9]
        return self.summarise(rows, self.window)


# The source files of each measured kernel: counters taken for a kernel stay
# valid while these files are unchanged.
_HDRS = ("internal.cuh", "layout.cuh")
_SRC_OF = {k: ("decode_fused.cu",) + _HDRS for k in ("decode", "decode_iq1", "batched")}
_SRC_OF["prefill"] = ("grouped_tc.cu", "route.cu", "ptx.cuh") + _HDRS


def max_over_ranks(ms, world, device=None):
    """The slowest rank's time; every rank calls this at the same points."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world, steps, tokens_per_step, ms):
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time (ms)."""
    return world * steps * tokens_per_step / (ms / 1e3)


def pack_inputs(x, ids, weights):
    """One call's inputs (x fp32 [T, H], ids int32 [T, k], weights fp32 [T, k])
    as one byte array, in that order, so that a step moves them host -> device
    with a single copy; x starts the array (16-byte aligned with the buffer)
    and each part's size is a multiple of 4 bytes."""
    parts = [np.ascontiguousarray(a).view(np.uint8).reshape(-1) for a in (x, ids, weights)]
    return np.concatenate(parts)


def input_views(buf, T, H, k):
    """Typed views (x, ids, weights) of a torch uint8 tensor made by pack_inputs."""
    import torch

    nx, ni = 4 * T * H, 4 * T * k
    return (buf[:nx].view(torch.float32).view(T, H), buf[nx:nx + ni].view(torch.int32).view(T, k),
            buf[nx + ni:nx + 2 * ni].view(torch.float32).view(T, k))


def _source_sha(files):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "routed_expert_ffn_iq2_b200", "csrc")
    for fn in sorted(files):
        h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


def _traffic(kernel_key: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel
    sources have not changed since it was taken (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel_key)
    if not d or d.get("source_sha") != _source_sha(_SRC_OF[kernel_key]):
        return None
    return d.get("dram_bytes_per_launch")


# end-to-end leg: pipelines (stream, workspace, staging buffers) that take the
# calls in turn; three keep the copy engines and the SMs busy for the
# prefill call (copy in, layer and copy out of ~0.6 + 0.8 + 0.6 ms)
E2E_PIPES = 3


def layer_for_workload(w, experts=None, max_tokens=None, extra_pool: int = 0, device: str = "cuda"):
    """A MoeLayer holding the experts of a fixtures.Workload (by default the
    selected ones) and its shared expert, uploaded through the C ABI."""
    import routed_expert_ffn_iq2_b200 as R

    ids = w.selected() if experts is None else list(experts)
    per = max(fixtures.expert_bytes(q, w.hidden, w.ffn) for q in (1, 2)) + 64
    sh = w.shared()
    pool = per * len(ids) + (sh.nbytes + 64 if sh is not None else 0) + extra_pool
    max_ffn = max(w.ffn, w.shared_ffn if sh is not None else 0)
    L = R.MoeLayer(w.hidden, w.n_experts, max_ffn, max_tokens or w.n_tokens, w.top_k, w.grid_iq2, w.grid_iq1, pool,
                   device=device)
    for i in range(0, len(ids), 32):
        chunk = ids[i:i + 32]
        R._native._check(L.upload(chunk, [w.expert(e) for e in chunk]), "upload")
    if sh is not None:
        R._native._check(L.set_shared(sh), "set_shared")
    return L


# ------------------------------------------------------------------ workloads


class Problem:
    """Per-config inputs: `sets` of (x [T,H], ids [T,k], weights [T,k]) cycled by the calls."""

    def __init__(self, cfg: int):
        self.cfg = cfg
        seed = fixtures.SEED_BASE + cfg
        if cfg in (2, 3):
            self.w = fixtures.workload(cfg)
            ids = fixtures.decode_id_sets(seed, N_SETS, self.w.top_k, self.w.n_experts)
            st = fixtures.Stream(seed, 6)
            wts = [fixtures.normalised_positive_weights(st, self.w.top_k)[None, :] for _ in range(N_SETS)]
            xs = fixtures.make_x(seed, N_SETS, self.w.hidden, tag=7)
            self.sets = [(xs[i:i + 1], ids[i:i + 1], wts[i]) for i in range(N_SETS)]
            self.resident = sorted(set(ids.reshape(-1).tolist()))
        elif cfg in (4, 5):
            self.w = fixtures.workload(cfg)
            self.sets = [(self.w.x, self.w.ids, self.w.weights)]
            self.resident = self.w.selected()
        else:
            raise SystemExit("bench supports --config 2..5 (config 1 is a parity case)")
        w = self.w
        self.tokens_per_call = self.sets[0][0].shape[0]
        self.call_bytes = []
        self.call_flops = []
        sh = w.shared()
        for x, ids, _ in self.sets:
            uniq = sorted(set(ids.reshape(-1).tolist()))
            b = sum(fixtures.expert_bytes(int(w.qtypes[e]), w.hidden, w.ffn) for e in uniq)
            if sh is not None:
                b += sh.nbytes
            b += x.nbytes * 2 + ids.nbytes * 2  # x in, out back, ids and weights in
            self.call_bytes.append(b)
            pairs = ids.size + (x.shape[0] if sh is not None else 0)
            self.call_flops.append(2.0 * 3 * w.hidden * w.ffn * pairs)

    def name(self):
        return self.w.name


def _oracle_step(oracle, P: Problem, i: int, cache):
    w = P.w
    x, ids, wt = P.sets[i % len(P.sets)]
    experts = [None] * w.n_experts
    for e in set(ids.reshape(-1).tolist()):
        experts[e] = w.expert(e)
    if "grids" not in cache:
        cache["grids"] = (oracle.expand_grid(1, w.grid_iq2), oracle.expand_grid(2, w.grid_iq1))
    g2, g1 = cache["grids"]
    return oracle.moe_layer(x, ids, wt, experts, w.shared(), g2, g1)


def cpu_oracle_rate(P: Problem, budget_s: float, max_steps: int):
    """Time the fp64 oracle as it stands on the host cores: layer calls/s as tokens/s."""
    import oracle

    cores = oracle.set_threads(0)
    cache = {}
    if P.cfg == 5:
        # bounded sample: the first 32 tokens of the prefill batch
        sub = Problem.__new__(Problem)
        sub.__dict__.update(P.__dict__)
        x, ids, wt = P.sets[0]
        sub.sets = [(x[:32], ids[:32], wt[:32])]
        P = sub
    _oracle_step(oracle, P, 0, cache)  # warm (grid expansion, expert bytes)
    t0 = time.perf_counter()
    n = 0
    while n < max_steps:
        _oracle_step(oracle, P, n, cache)
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    toks = n * P.sets[0][0].shape[0]
    sample = f"{n} layer calls x {P.sets[0][0].shape[0]} token(s) of {P.name()}, fp64 oracle, {dt:.1f} s"
    return toks / dt, cores, sample


def roofline(P: Problem, per_call_s: float, peaks):
    """Achieved rate of one call against the measured peak (bytes or FLOPs per call / call time)."""
    n = len(P.sets)
    G = GRAPH_CALLS[P.cfg]
    mean_bytes = float(np.mean([P.call_bytes[i % n] for i in range(G)]))
    mean_flops = float(np.mean([P.call_flops[i % n] for i in range(G)]))
    if P.cfg == 5:
        ach = mean_flops / per_call_s / 1e12
        peak = peaks["bf16_tflops_sustained"]
        return {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                "traffic": _traffic("prefill"), "peak_kind": f"{peaks['src']} bf16 sustained",
                "flops_per_call": mean_flops}, mean_bytes
    ach = mean_bytes / per_call_s / 1e9
    peak = peaks["hbm_gbs"]
    return {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
            "traffic": _traffic({2: "decode", 3: "decode_iq1"}.get(P.cfg, "batched")),
            "peak_kind": f"{peaks['src']} HBM copy", "bytes_per_call": mean_bytes}, mean_bytes


# ------------------------------------------------------------------ one workload on the GPU


def measure(cfg: int, steps: int, warmup: int, world: int, rank: int, local: int, dev, e2e_on: bool,
            cpu_budget: float = 0.0):
    """Time `steps` steps of workload `cfg` (max over ranks) and its end-to-end leg."""
    import torch

    import routed_expert_ffn_iq2_b200 as R

    P = Problem(cfg)
    w = P.w
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)
    per = max(fixtures.expert_bytes(q, w.hidden, w.ffn) for q in (1, 2)) + 64
    sh = w.shared()
    pool = per * len(P.resident) + (sh.nbytes + 64 if sh is not None else 0)
    L = R.MoeLayer(w.hidden, w.n_experts, max(w.ffn, w.shared_ffn), P.tokens_per_call, w.top_k, w.grid_iq2,
                   w.grid_iq1, pool, device=str(dev), stream=stream)
    for i in range(0, len(P.resident), 32):
        chunk = P.resident[i:i + 32]
        R._native._check(L.upload(chunk, [w.expert(e) for e in chunk]), "upload")
        for e in chunk:  # host copies are no longer needed
            w._experts.pop(e, None)
    if sh is not None:
        R._native._check(L.set_shared(sh), "set_shared")

    # each set's inputs live in one device buffer (x, ids, weights), so the
    # end-to-end leg below copies them host -> device in one transfer
    packed = [pack_inputs(*s[:3]) for s in P.sets]
    dbuf = [torch.from_numpy(pk).to(dev) for pk in packed]
    views = [input_views(b, s[0].shape[0], w.hidden, w.top_k) for b, s in zip(dbuf, P.sets)]
    dx, di, dw = [v[0] for v in views], [v[1] for v in views], [v[2] for v in views]
    do = [torch.empty((s[0].shape[0], w.hidden), dtype=torch.float32, device=dev) for s in P.sets]
    nsets = len(P.sets)

    def call(i):
        j = i % nsets
        rc = R.redlite_moe_layer(dx[j], dx[j].shape[0], di[j], dw[j], w.top_k, L.table, L.shared, do[j])
        if rc != 0:
            raise RuntimeError(f"redlite_moe_layer rc={rc}")

    G, reps = GRAPH_CALLS[cfg], REPLAYS_PER_STEP[cfg]
    for i in range(3):
        call(i)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(G):
            call(i)
    for _ in range(max(warmup, 3) * reps):
        graph.replay()
    stream.synchronize()
    if L.read_status() != 0:
        raise RuntimeError(f"device status {L.read_status()}")

    def barrier():
        if world > 1:
            import torch.distributed as dist

            dist.barrier()

    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.25)  # nvidia-smi is up before the timed window opens
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    ev0.record(stream)
    for _ in range(steps * reps):
        graph.replay()
    ev1.record(stream)
    ev1.synchronize()
    t1 = time.time()
    torch.cuda.synchronize()
    barrier()
    time.sleep(0.15)
    clk.mark(t0, t1)
    clocks = clk.stop()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    cps = calls_per_step(cfg)
    launches_per_call = R.launches_per_call(dx[0].shape[0], w.top_k, sh is not None)
    del graph

    # end-to-end through the public call with host buffers (pinned), per call
    # (redlite_moe_layer_host): H2D of the call's x, ids and weights (one
    # packed transfer); the layer; D2H of out.  E2E_PIPES pipelines -- each
    # its own stream, workspace and staging buffers over the same resident
    # experts -- take the calls in turn, so calls' transfers run on the copy
    # engines while other calls' kernels compute (a pipeline's own copy in,
    # layer and copy out stay in order on its stream).
    e2e = None
    if e2e_on:
        NP = E2E_PIPES
        streams = [stream] + [torch.cuda.Stream(dev) for _ in range(NP - 1)]
        tables, extra_ws = [L.table], []
        for p in range(1, NP):
            t = R._native.redlite_moe_table.from_buffer_copy(bytes(L.table))
            ws = torch.zeros(L.workspace.numel(), dtype=torch.uint8, device=dev)
            t.workspace, t.stream = ws.data_ptr(), streams[p].cuda_stream
            R._native._check(R._native.redlite_moe_workspace_reset(t), "redlite_moe_workspace_reset")
            tables.append(t)
            extra_ws.append(ws)
        hbuf = [[torch.from_numpy(pk).pin_memory() for pk in packed] for _ in range(NP)]
        ho = [[torch.empty((s[0].shape[0], w.hidden), dtype=torch.float32).pin_memory() for s in P.sets]
              for _ in range(NP)]
        db2 = [dbuf] + [[torch.empty_like(b) for b in dbuf] for _ in range(NP - 1)]
        do2 = [do] + [[torch.empty_like(o) for o in do] for _ in range(NP - 1)]
        e_calls = min(steps * cps, 2400 if nsets > 1 else steps * cps)
        e_calls = max(NP, e_calls - e_calls % NP)  # whole rounds of the pipelines

        def e2e_call(i):
            p, j = i % NP, (i // NP) % nsets
            rc = R.redlite_moe_layer_host(hbuf[p][j], db2[p][j], dx[j].shape[0], w.top_k, tables[p], L.shared,
                                          do2[p][j], ho[p][j])
            if rc != 0:
                raise RuntimeError(f"redlite_moe_layer_host rc={rc}")

        for i in range(2 * NP):
            e2e_call(i)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start_ev = torch.cuda.Event()
        e0.record(streams[0])
        start_ev.record(streams[0])
        for st in streams[1:]:
            st.wait_event(start_ev)
        for i in range(e_calls):
            e2e_call(i)
        for st in streams[1:]:
            ev = torch.cuda.Event()
            ev.record(st)
            streams[0].wait_event(ev)
        e1.record(streams[0])
        e1.synchronize()
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": job_rate(world, e_calls, P.tokens_per_call, ems), "unit": "tokens/s",
               "h2d_bytes_per_step": int(hbuf[0][0].nbytes) * cps, "d2h_bytes_per_step": int(ho[0][0].nbytes) * cps,
               "calls": e_calls, "pipelines": NP}
        del extra_ws, db2, do2

    status = L.read_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    del L, dbuf, do
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and cpu_budget > 0:
        rate, cores, sample = cpu_oracle_rate(P, cpu_budget, max_steps=10 ** 6)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}

    peaks = _peaks()
    per_call_s = ms / 1e3 / (steps * cps)
    roof, mean_bytes = roofline(P, per_call_s, peaks)
    tokens_per_step = cps * P.tokens_per_call
    return {
        "workload": P.name(),
        "value": job_rate(world, steps, tokens_per_step, ms), "unit": "tokens/s",
        "ms_per_step": ms / steps, "steps": steps, "calls_per_step": cps, "tokens_per_step": tokens_per_step,
        "us_per_call": per_call_s * 1e6, "dtype": DTYPE[cfg],
        "weight_gbs": mean_bytes / per_call_s / 1e9,
        "roofline": roof, "e2e": e2e, "clocks": clocks, "cpu_baseline": cpu,
        "gpu_launches": launches_per_call * steps * cps,
        "l2": ("inputs larger than L2: calls cycle 48 disjoint top-10 sets over 480 resident experts (436 MB)"
               if nsets > 1 else f"inputs larger than L2 (expert bytes per call {mean_bytes / 1e6:.0f} MB)"),
        "issue": f"CUDA graph of {G} layer calls, {reps} replays per step",
    }


# ------------------------------------------------------------------ the other rows of the path


def _graph_time(fn, n_calls, reps, stream):
    """Device time per call (us) of `fn` captured n_calls times in a CUDA graph."""
    import torch

    for _ in range(3):
        fn(0)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n_calls):
            fn(i)
    g.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) * 1e3 / (reps * n_calls)


def measure_components(dev):
    """Router, block, slot pool and projection GEMVs on their own (one GPU):
    device time per call and the rate each is bound by."""
    import ctypes

    import torch

    import routed_expert_ffn_iq2_b200 as R

    peaks = _peaks()
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)
    res = {}
    # router: 64 tokens x 512 logits -> top-10
    st = fixtures.Stream(0x5EED0004, 4)
    lg = torch.from_numpy(st.normal(64 * 512).reshape(64, 512).astype(np.float32)).to(dev)
    ids = torch.empty((64, 10), dtype=torch.int32, device=dev)
    wts = torch.empty((64, 10), dtype=torch.float32, device=dev)
    us = _graph_time(lambda i: R.redlite_moe_route_topk(lg, 64, 512, 10, ids, wts, stream), 100, 20, stream)
    res["router"] = {"workload": "route-top10-t64-e512", "us_per_call": us, "tokens_per_s": 64 / (us * 1e-6)}
    # projection GEMVs, one token: the recurrent layer's ssm_ba (Q8_0, 2048 -> 64) and ssm_out (Q4_K,
    # 4096 -> 2048), the attention layer's attn_k (Q4_K, 2048 -> 512)
    for name, qt, rows, k in (("ssm_ba-q8_0-2048x64", 3, 64, 2048), ("ssm_out-q4_k-4096x2048", 4, 2048, 4096),
                              ("attn_k-q4_k-2048x512", 4, 512, 2048)):
        nmat = max(1, (256 << 20) // R.redlite_proj_matrix_bytes(qt, rows, k))  # cycle > L2 of copies
        mats = [torch.from_numpy(fixtures.make_proj_matrix(800, qt, rows, k)).to(dev)]
        big = mats[0].repeat(min(nmat, 64))
        mb = R.redlite_proj_matrix_bytes(qt, rows, k)
        nm = big.numel() // mb
        xv = torch.from_numpy(fixtures.make_x(801, 1, k)).to(dev)
        yv = torch.empty((1, rows), dtype=torch.float32, device=dev)
        us = _graph_time(lambda i: R.redlite_proj_gemv(qt, big[(i % nm) * mb:(i % nm + 1) * mb], rows, k, xv, 1, yv,
                                                        stream), nm, 10, stream)
        gbs = (mb + 4 * (k + rows)) / (us * 1e-6) / 1e9
        res["proj_" + name] = {"us_per_call": us, "roofline": {"bound": "hbm", "achieved": gbs,
                                                               "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                                               "frac": gbs / peaks["hbm_gbs"]},
                               "copies_cycled": nm, "l2": "matrix copies cycled" if nm * mb > (126 << 20) else
                               "matrix copies cycled (inside L2)"}
    # block and pool: 64 IQ2_XS-style experts of width 512, hidden 2048, top-10, one token per call
    H, E, F, k = 2048, 64, 512, 10
    seed = 0x5EED00B0
    g2, g1 = fixtures.make_grid(seed, 1), fixtures.make_grid(seed, 2)
    experts = [fixtures.make_expert(seed, 1, H, F, e) for e in range(E)]
    L = R.MoeLayer(H, E, F, 1, k, g2, g1, pool_bytes=(E + 1) * (fixtures.expert_bytes(1, H, F) + 64), device=str(dev),
                   stream=stream)
    for i in range(0, E, 16):
        R._native._check(L.upload(list(range(i, i + 16)), experts[i:i + 16]), "upload")
    hs = torch.from_numpy(fixtures.make_x(seed, 48, H)).to(dev)
    gam = torch.from_numpy((1.0 + 0.1 * fixtures.Stream(seed, 2).normal(H)).astype(np.float32)).to(dev)
    rw = torch.from_numpy((0.05 * fixtures.Stream(seed, 3).normal(E * H)).reshape(E, H).astype(np.float32)).to(dev)
    scratch = torch.zeros(R.redlite_moe_block_scratch_bytes(H, E, 1, k), dtype=torch.uint8, device=dev)
    out = torch.empty((1, H), dtype=torch.float32, device=dev)
    us = _graph_time(lambda i: R.redlite_moe_block(hs[i % 48:i % 48 + 1], 1, gam, 1e-6, rw, k, L.table, None, out,
                                                   scratch), 96, 20, stream)
    if L.read_status() != 0:
        raise RuntimeError(f"block: device status {L.read_status()}")
    res["block"] = {"workload": "block-rmsnorm-router-iq2xs-h2048-e64-f512-top10-t1", "us_per_call": us,
                    "tokens_per_s": 1 / (us * 1e-6)}
    # slot pool: capacity 24, every call a fresh top-10 (cycling through 6 disjoint sets of the 64
    # experts), misses filled host -> device on a copy stream while the previous layer call runs
    pool = R.SlotPool(E, 24)
    gb = fixtures.matrix_bytes(1, F, H)
    slot_bytes = 2 * ((gb + 15) // 16 * 16) + fixtures.matrix_bytes(1, H, F)
    slots = torch.zeros(24 * slot_bytes, dtype=torch.uint8, device=dev)
    host = (R.redlite_moe_expert * E)()
    keep = []
    for e, ex in enumerate(experts):
        mats = []
        for m, (r, c) in zip((ex.gate, ex.up, ex.down), ((F, H), (F, H), (H, F))):
            t = torch.from_numpy(R.redlite_moe_pack_matrix(1, r, c, m)).pin_memory()
            mats.append(t)
        keep += mats
        host[e] = R.redlite_moe_expert(1, F, *[t.data_ptr() for t in mats])
    PL = R.MoeLayer(H, E, F, 1, k, g2, g1, pool_bytes=16, device=str(dev), stream=stream)
    PL.table.min_ffn = F
    sets = [list(range(10 * j, 10 * j + 10)) for j in range(6)]
    copy_s = torch.cuda.Stream(dev)
    xin = torch.from_numpy(fixtures.make_x(seed, 1, H)).to(dev)
    wt = torch.full((1, k), 0.1, dtype=torch.float32, device=dev)
    idt = [torch.tensor([s], dtype=torch.int32, device=dev) for s in sets]
    pend = []
    n_calls = 60
    for warm in (True, False):
        stream.synchronize()
        t0 = time.perf_counter()
        c0 = (pool.counters.loads, pool.counters.bytes)
        for i in range(n_calls if not warm else 6):
            rc, tok = pool.acquire(sets[i % 6], host, H, slots, slot_bytes, PL.table_dev, copy_s, stream)
            while rc == R.REDLITE_EAGAIN:  # every slot in flight: retire the oldest call
                torch.cuda.current_stream().synchronize()
                stream.synchronize()
                rc, tok = pool.acquire(sets[i % 6], host, H, slots, slot_bytes, PL.table_dev, copy_s, stream)
            R._native._check(rc, "pool acquire")
            R._native._check(R.redlite_moe_layer(xin, 1, idt[i % 6], wt, k, PL.table, None, out), "layer")
            pool.release(tok, stream)
        stream.synchronize()
        dt = time.perf_counter() - t0
    loads = pool.counters.loads - c0[0]
    nbytes = pool.counters.bytes - c0[1]
    if PL.read_status() != 0:
        raise RuntimeError(f"pool: device status {PL.read_status()}")
    # the link's own rate for reference: one 64 MB copy from pinned host memory, device-timed
    hbig = torch.empty(64 << 20, dtype=torch.uint8).pin_memory()
    dbig = torch.empty(64 << 20, dtype=torch.uint8, device=dev)
    for _ in range(2):
        dbig.copy_(hbig, non_blocking=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(4):
        dbig.copy_(hbig, non_blocking=True)
    e1.record()
    e1.synchronize()
    peak = 4 * (64 << 20) / (e0.elapsed_time(e1) * 1e-3) / 1e9
    del hbig, dbig
    res["pool"] = {"workload": "pool-cap24-e64-iq2xs-top10-t1, a fresh selection per call", "calls": n_calls,
                   "us_per_call": dt * 1e6 / n_calls, "loads": int(loads), "h2d_gbs": nbytes / dt / 1e9,
                   "roofline": {"bound": "h2d", "achieved": nbytes / dt / 1e9, "peak": peak, "unit": "GB/s",
                                "frac": nbytes / dt / 1e9 / peak,
                                "peak_kind": "measured: one 64 MB pinned host-to-device copy"},
                   "note": "host wall time of acquire + layer per call (fills from pinned host memory on the "
                           "pool's copy streams)"}
    pool.close()
    del keep, L, PL
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--workloads", default="3,4,5", help="other workloads on one GPU, or 'none'")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-components", action="store_true", help="skip router/block/pool/projection timings")
    args = ap.parse_args()
    steps = max(1, args.steps)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        P = Problem(args.config)
        rate, cores, sample = cpu_oracle_rate(P, args.cpu_budget, max_steps=max(args.steps, 1) * 48)
        peaks = _peaks()
        line = {
            "impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * P.tokens_per_call / rate,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": P.name(), "tokens_per_step": P.tokens_per_call},
            "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "peaks_src": peaks["src"],
        }
        print(json.dumps(line), flush=True)
        return

    import torch

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from routed_expert_ffn_iq2_b200 import build as B

    B.build()

    head = measure(args.config, steps, args.warmup, world, rank, local, dev, not args.no_e2e,
                   cpu_budget=0.0 if args.no_cpu_baseline else args.cpu_budget)
    others = {}
    if world == 1 and args.workloads != "none":
        for c in [int(v) for v in args.workloads.split(",") if v.strip()]:
            if c != args.config:
                r = measure(c, steps, args.warmup, world, rank, local, dev, not args.no_e2e)
                r.pop("cpu_baseline", None)
                others[str(c)] = r

    comps = measure_components(dev) if world == 1 and not args.no_components else None
    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": head["dtype"], "data": "synthetic",
            "config": {"workload": head["workload"], "tokens_per_step": head["tokens_per_step"],
                       "calls_per_step": head["calls_per_step"],
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": head["l2"], "issue": head["issue"]},
            "us_per_call": head["us_per_call"],
            "weight_gbs": head["weight_gbs"],
            "roofline": head["roofline"],
            "cpu_baseline": head["cpu_baseline"],
            "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"],
            "clocks": head["clocks"],
        }
        if others:
            line["workloads"] = others
        if comps:
            line["components"] = comps
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
