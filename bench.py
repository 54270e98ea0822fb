#!/usr/bin/env python
"""Throughput of the hashed n-gram embedding lookup on B200 (one JSON line on rank 0).

A step is one pass of the whole path -- remap + hash, gather, projections, gate + conv +
residual -- over one batch of the workload (default: prefill on the 20M-row tables,
32 x 8192 tokens, 2 tables of 9,999,991 rows x 2560 bf16 = 95.4 GiB in HBM).  Inputs are
resident in HBM when the timed region starts; the e2e figure repeats the measurement
through the same public call with the inputs copied from pinned host memory and the output
copied back every step.

Multi-GPU (torchrun): every rank runs its own replica on its own batch (the lookup has no
cross-token exchange), so scaling is weak; time is the max over ranks.

--impl reference times the CPU oracle (the only reference this method has) on a bounded
sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

L2_BYTES = 126 * 2 ** 20


def kernel_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu summary
    (profiles/traffic.json), or None when that summary was taken on a different version of
    the kernel's source files than the ones built here."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    entry = json.load(open(p)).get(kernel, {}).get(workload)
    if not entry:
        return None
    for rel, digest in entry["sources"].items():
        src = os.path.join(ROOT, rel)
        if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != digest:
            return None
    return entry["dram_bytes_per_launch"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    sm_max=d.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, sm_max=1965.0, source="fallback")


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled through NVML every 20 ms
    while the timed region runs (read-only queries)."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int, period_s: float = 0.02):
        self.cuda_index = cuda_index
        self.period = period_s
        self.rows = []
        self.handle = None
        self.error = None
        self._stop = threading.Event()

    def _open(self):
        import pynvml
        pynvml.nvmlInit()
        bus = None
        try:
            props = torch.cuda.get_device_properties(self.cuda_index)
            bus = getattr(props, "pci_bus_id", None)
            dom = getattr(props, "pci_domain_id", 0)
            dev = getattr(props, "pci_device_id", 0)
            if bus is not None:
                bus = f"{dom:08x}:{bus:02x}:{dev:02x}.0"
        except Exception:
            bus = None
        if bus:
            try:
                return pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = self.cuda_index
        if vis:
            ids = [v.strip() for v in vis.split(",")]
            if idx < len(ids) and ids[idx].isdigit():
                idx = int(ids[idx])
        return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        import pynvml
        while not self._stop.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
                reasons = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
                power = pynvml.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                self.rows.append((time.perf_counter(), sm, reasons, power))
            except Exception as e:  # keep the benchmark running; report the failure
                self.error = str(e)
                return
            time.sleep(self.period)

    def __enter__(self):
        try:
            import pynvml
            self.handle = self._open()
            self.max_sm = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
            time.sleep(3 * self.period)
        except Exception as e:
            self.error = str(e)
            self.handle = None
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.handle is not None:
            self.thread.join(timeout=2)

    def summary(self, t0=None, t1=None):
        rows = [r for r in self.rows if (t0 is None or r[0] >= t0) and (t1 is None or r[0] <= t1)]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": getattr(self, "max_sm", None), "reasons": ["unsampled"],
                    "samples": 0, "error": self.error}
        reasons = sorted({name for r in rows for bit, name in self.REASONS.items() if r[2] & bit})
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": self.max_sm, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(r[3] for r in rows), "source": "nvml"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "engram":
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's time (device-measured on each rank) -- the job's time."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------------------
# CPU oracle on a bounded sample (the reference arm and the cpu_baseline object)
def host_cpu() -> str:
    """CPU model and logical core count of this host (for the CPU-baseline record)."""
    model = "unknown CPU"
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return f"{model}, {os.cpu_count()} logical cores"


_WEIGHTS = {}


def oracle_sample(wl, n_tok_sample: int, seq: int = 0):
    """Time the oracle's steps (remap, hash, gather, gate + conv + residual) on the first
    n_tok_sample tokens of sequence `seq`.  Table rows are regenerated from the seeded
    generator before the clock starts (the tables are never materialised on the host)."""
    import oracle
    b = seq % wl.B
    T = min(wl.T, n_tok_sample)
    ids = wl.ids()[b:b + 1, :T]
    remap = wl.remap()
    t_gen0 = time.perf_counter()
    idx_probe = oracle.hash_ids(remap[ids], wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id)
    if wl.table_dtype == "fp8":
        tables = [synth.fill_rows_fp8(wl.table_spec(h), wl.d_e, idx_probe[:, h]) for h in range(wl.H)]
        scales = [wl.table_scale(h) for h in range(wl.H)]
    else:
        tables = [synth.fill_rows_bf16(wl.table_spec(h), wl.d_e, idx_probe[:, h]) for h in range(wl.H)]
        scales = None
    local_idx = np.tile(np.arange(T, dtype=np.uint32)[:, None], (1, wl.H))
    M = wl.branches
    hrows = ((b * wl.T + np.arange(T))[:, None] * M + np.arange(M)[None, :]).reshape(-1)
    h = synth.fill_rows_bf16(wl.h_spec(0), wl.d_h, hrows).reshape(T, M, wl.d_h)
    key = (wl.index, wl.seeds()["weights"], M, wl.d_h, wl.d_m, wl.conv_kernel)
    if key not in _WEIGHTS:   # regenerated once per process
        _WEIGHTS[key] = (synth.fill_bf16(wl.wk_spec(), (M * wl.d_h, wl.d_m)),
                         synth.fill_bf16(wl.wv_spec(), (wl.d_h, wl.d_m)),
                         synth.fill_bf16(wl.conv_spec(), (wl.d_h, wl.conv_kernel)))
    Wk, Wv, cw = _WEIGHTS[key]
    one = np.full(wl.d_h, 0x3F80, dtype=np.uint16)
    t_gen = time.perf_counter() - t_gen0
    t0 = time.perf_counter()
    xr = oracle.remap(ids, remap)
    idx = oracle.hash_ids(xr, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id)
    m = oracle.gather(local_idx, tables, scales)   # compact tables hold exactly the rows idx names
    for br in range(M):      # the branches share m and W_v; each has its own h row and W_k
        oracle.gate_conv(h[:, br], m, Wk[br * wl.d_h:(br + 1) * wl.d_h], Wv, one, one, one, cw, 1, T,
                         dil=wl.conv_dilation, eps=wl.eps)
    dt = time.perf_counter() - t0
    assert np.array_equal(idx, idx_probe)
    return T, dt, t_gen


def _oracle_job(job):
    """One oracle sample in a worker process: returns (tokens, compute seconds)."""
    wl, n_tok, seq = job
    T, dt, _ = oracle_sample(wl, n_tok, seq)
    return T, dt


class OraclePool:
    """The unmodified oracle on several host cores: independent samples (one sequence each) in
    spawned worker processes.  A round's time is its longest worker's compute time (each
    worker times only the oracle's steps, after regenerating its table rows), so the round
    throughput is all tokens over that time.  Spawned, not forked: the parent has a CUDA
    context."""

    def __init__(self, procs: int, wl):
        import multiprocessing as mp
        self.procs = max(1, procs)
        self.pool = mp.get_context("spawn").Pool(self.procs) if self.procs > 1 else None
        if self.pool is not None:   # import, build check and library load in every worker, untimed
            self.pool.map(_oracle_job, [(wl, 4, k) for k in range(self.procs)])

    def round(self, wl, n_tok: int, seq0: int = 0):
        """One sample per worker; returns (tokens, seconds of the longest worker)."""
        jobs = [(wl, n_tok, seq0 + k) for k in range(self.procs)]
        res = self.pool.map(_oracle_job, jobs) if self.pool is not None else [_oracle_job(jobs[0])]
        return sum(r[0] for r in res), max(r[1] for r in res)

    def close(self):
        if self.pool is not None:
            self.pool.close()
            self.pool.join()


def oracle_procs(args, wl) -> int:
    """Host processes for the oracle: --oracle-procs, else every core up to 32."""
    cores = os.cpu_count() or 1
    n = args.oracle_procs if args.oracle_procs > 0 else min(cores, 32)
    return max(1, min(n, cores))


def run_reference(args, wl, world, rank):
    """Reference arm: the CPU oracle on the host cores, rank 0 only, one bounded round of
    samples per step (one sequence per core)."""
    if rank != 0:
        return
    procs = oracle_procs(args, wl)
    pool = OraclePool(procs, wl)
    per_tok = []
    for k in range(args.warmup):
        Tw, dtw, _ = oracle_sample(wl, 8, seq=k)
        per_tok.append(dtw / Tw)
    # size each step's sample so that all timed steps take about --reference-seconds
    est = min(per_tok) if per_tok else 0.01
    n_sample = int(max(4, min(args.oracle_tokens, args.reference_seconds / max(1e-9, est * args.steps))))
    times, toks = [], 0
    for k in range(args.steps):
        tk, dt = pool.round(wl, n_sample, seq0=k * procs)
        times.append(dt)
        toks += tk
    pool.close()
    T = toks // (args.steps * procs)
    tps = toks / sum(times)
    sample = (f"{args.steps} rounds of {procs} samples (1 sequence x {T} tokens of {wl.name} each, one per "
              f"process; a round timed by its longest worker); fp64 scalar C, {procs} processes on "
              f"{host_cpu()}; table-row regeneration not timed")
    line = {
        "impl": "reference", "metric": "engram_tokens_per_s", "value": tps, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        # a step of this arm is one measured round of samples (procs x T tokens), not the
        # workload's whole batch; the time one whole batch would take is extrapolated apart
        "ms_per_step": 1e3 * sum(times) / args.steps, "tokens_per_step": procs * T,
        "ms_per_workload_batch_extrapolated": wl.n_tok / tps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, world),
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": procs, "kind": "oracle", "sample": sample},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl, world, ids_kind=None):
    """The workload's description, identical in both arms' lines."""
    c = {"workload": wl.name, "tokens_per_step_per_gpu": wl.n_tok, "B": wl.B, "T": wl.T,
         "orders": list(wl.orders), "K": wl.K, "H": wl.H, "table_rows": wl.primes[0], "d_e": wl.d_e,
         "d_m": wl.d_m, "d_h": wl.d_h, "branches": wl.branches, "table_dtype": wl.table_dtype,
         "table_GiB": round(wl.table_bytes / 2 ** 30, 2),
         "parallelism": f"replicas x{world}",
         "l2": "inputs larger than L2 (hidden states and tables each exceed 126 MB)"
         if l2_exceeded(wl) else "L2 flushed between timed steps (252 MiB write, outside the per-step events)"}
    if wl.host_tables:
        c.update(tables="pinned mapped host memory", ids=ids_kind or wl.ids_kind)
    return c


def l2_exceeded(wl) -> bool:
    """True when one step's hidden states alone exceed L2, so no input survives in L2 from
    one step to the next."""
    return wl.n_tok * wl.d_h * 2 > L2_BYTES


# ---------------------------------------------------------------------------------------
def measure_decode_steps(E, fill_gpu, plan, weights, tables, wl_dec, steps, warmup, stream, dev):
    """One-token decode steps (wl_dec's batch, hash history and conv state carried from step to
    step) through engram_forward on already-resident tables; L2 flushed between steps (outside
    each step's events).  Returns per-step time, the CUDA-event stage breakdown and launches."""
    B = wl_dec.B
    hist = torch.from_numpy(wl_dec.history()).to(dev)
    state = fill_gpu.filled((B, wl_dec.state_len, wl_dec.d_h), wl_dec.state_spec(), dev)
    ids_all = torch.from_numpy(synth.zipf_ids(wl_dec.vocab_in, wl_dec.zipf_s, (warmup + steps, B, 1),
                                              wl_dec.seeds()["ids"])).to(dev)
    h = fill_gpu.filled((B, wl_dec.d_h), wl_dec.h_spec(0), dev)
    out = torch.empty((B, wl_dec.d_h), dtype=torch.bfloat16, device=dev)
    ws = E.alloc_workspace(plan, B, dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    nst = E.ENGRAM_FORWARD_STAGES + 1

    def step(k, evs=None):
        E.engram_forward(plan, weights, tables, ids_all[k], h, out, ws, history=hist, conv_state=state,
                         stream=stream, stage_events=evs)

    for k in range(warmup):
        step(k)
    torch.cuda.synchronize()
    n0 = E.kernel_launches()
    step(0)
    torch.cuda.synchronize()
    launches = E.kernel_launches() - n0
    # the K steps as one CUDA graph, as the main measurement does (no host launch gaps); a
    # second graph of the same steps carries the per-stage events
    se = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
          for _ in range(steps)]
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(nst)] for _ in range(steps)]
    for row in evs:
        for e in row:
            e.record(stream)
    for a, b in se:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()

    def capture(with_events):
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
            cs = torch.cuda.current_stream()
            for k in range(steps):
                flush.fill_(k)
                if not with_events:
                    se[k][0].record(cs)
                E.engram_forward(plan, weights, tables, ids_all[warmup + k], h, out, ws, history=hist,
                                 conv_state=state, stream=cs, stage_events=evs[k] if with_events else None)
                if not with_events:
                    se[k][1].record(cs)
        stream.wait_stream(cap)
        torch.cuda.synchronize()
        return g

    g_time, g_ev = capture(False), capture(True)
    g_time.replay()   # upload
    torch.cuda.synchronize()
    g_time.replay()
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in se)
    g_ev.replay()
    torch.cuda.synchronize()
    names = ["hash", "gather", "proj", "gate_conv"]
    stages = {n: statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(steps))
              for i, n in enumerate(names)}
    if E.engram_device_status(clear=True):
        raise SystemExit("device status raised during the decode steps")
    return {"ms_per_step": ms, "us_per_step": ms * 1e3, "tokens_per_s": B / (ms / 1e3), "stages_ms": stages,
            "gpu_launches_per_step": launches, "path_bits": E.engram_forward_path(plan, B, 1)}


def run_engram(args, wl, world, rank, local):
    import hashed_gram_embedding_remap_b200 as E
    from synth import fill_gpu

    dev = f"cuda:{local}"
    torch.cuda.set_device(local)
    fill_gpu.build()
    stream = torch.cuda.current_stream()
    free, _ = torch.cuda.mem_get_info()
    M = wl.branches
    need = wl.table_bytes + 4 * wl.n_tok * (wl.d_h * 8 * M + wl.d_m * 2)
    if need > free:
        raise SystemExit(f"not enough device memory: need ~{need / 2**30:.1f} GiB, free {free / 2**30:.1f} GiB")
    # per-rank input: each rank draws its own batch (seed offset by rank)
    fill = fill_gpu.filled_fp8 if wl.table_dtype == "fp8" else fill_gpu.filled
    tables = [fill((wl.primes[h], wl.d_e), wl.table_spec(h), dev) for h in range(wl.H)]
    ids_np = wl.ids(step=rank)
    ids = torch.from_numpy(ids_np).to(dev)
    remap = None if wl.identity_remap else torch.from_numpy(wl.remap()).to(dev)
    h = fill_gpu.filled((wl.h_rows, wl.d_h), wl.h_spec(rank), dev)       # [n_tok * M, d_h]
    wk = fill_gpu.filled((M * wl.d_h, wl.d_m), wl.wk_spec(), dev)
    wv = fill_gpu.filled((wl.d_h, wl.d_m), wl.wv_spec(), dev)
    one = torch.full((wl.d_h,), 0x3F80, dtype=torch.int16, device=dev).view(torch.bfloat16)
    cw = fill_gpu.filled((wl.d_h, wl.conv_kernel), wl.conv_spec(), dev)
    history = torch.from_numpy(wl.history()).to(dev) if wl.decode else None
    state = fill_gpu.filled((wl.B * M, wl.state_len, wl.d_h), wl.state_spec(), dev) if wl.decode else None
    flags = (E.ENGRAM_FLAG_SINGLE_CTA_MMA if args.single_cta_mma else 0) | (
        E.ENGRAM_FLAG_ROW_ORDER_GATHER if args.row_order_gather else 0) | (
        E.ENGRAM_FLAG_BULK_GATHER if args.bulk_gather else 0)
    plan = E.Plan.from_workload(wl, flags=flags)
    path = E.engram_forward_path(plan, wl.B, wl.T)
    packed = E.pack_weights(plan, wk, wv) if args.packed and E.engram_packed_weights_size(plan) else None
    weights = E.Weights(wk, wv, one, one, one, cw, packed=packed)
    out = torch.empty((wl.h_rows, wl.d_h), dtype=torch.bfloat16, device=dev)
    ws = E.alloc_workspace(plan, wl.n_tok, dev)
    nstage = E.ENGRAM_FORWARD_STAGES + 1

    # Row ids of the batch (the library's own remap + hash, untimed): distinct rows per
    # table for the byte count of the HBM roofline
    xr = ids
    if remap is not None:
        xr = torch.empty_like(ids)
        E.engram_remap(plan, ids, remap, xr)
    idx = torch.empty((wl.n_tok, wl.H), dtype=torch.int32, device=dev)
    E.engram_hash(plan, xr, idx, history=history)
    distinct_rows = sum(int(torch.unique(idx[:, t]).numel()) for t in range(wl.H))

    def step(evs=None):
        E.engram_forward(plan, weights, tables, ids, h, out, ws, remap=remap, history=history,
                         conv_state=state, stream=stream, stage_events=evs)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    n_launch0 = E.kernel_launches()   # the library's own count of the kernels one step launches
    step()
    torch.cuda.synchronize()
    launches_per_step = E.kernel_launches() - n_launch0
    E.engram_device_status(clear=True)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nstage)] for _ in range(args.steps)]
    bounds = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
              for _ in range(args.steps)]
    for row, (b0, b1) in zip(evs, bounds):   # create the events before the timed region (and before capture)
        for e in row:
            e.record(stream)
        b0.record(stream)
        b1.record(stream)
    # Workloads whose per-step inputs fit in L2 (decode steps): L2 is flushed between timed
    # steps by a 2 x L2 write outside each step's start / end events, and the run's time is the
    # sum of the per-step intervals (the whole call, history update included).  The per-stage
    # events go in a separate replay: an event between two kernels stops the second from
    # starting early (programmatic dependent launch).
    flush_l2 = not l2_exceeded(wl)
    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev) if flush_l2 else None

    def timed_step(k, cs, with_events):
        if flush_buf is not None:
            flush_buf.fill_(k)
        if flush_l2 and not with_events:
            bounds[k][0].record(cs)
        E.engram_forward(plan, weights, tables, ids, h, out, ws, remap=remap, history=history,
                         conv_state=state, stream=cs, stage_events=evs[k] if with_events else None)
        if flush_l2 and not with_events:
            bounds[k][1].record(cs)

    graph = graph_ev = None
    if not args.eager:
        # The whole timed region (K steps) as one CUDA graph: no host launch overhead between
        # kernels, which decode-sized steps would otherwise see.  A second graph of the same K
        # steps carries the per-stage events and is replayed right after the timed one.
        def capture(with_events):
            g = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream()
            cap.wait_stream(stream)
            with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
                cs = torch.cuda.current_stream()
                for k in range(args.steps):
                    timed_step(k, cs, with_events)
            stream.wait_stream(cap)
            torch.cuda.synchronize()
            g.replay()            # one untimed replay: uploads the graph
            torch.cuda.synchronize()
            return g
        graph = capture(False)
        graph_ev = capture(True)
    barrier(world)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        t_host0 = time.perf_counter()
        start.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for k in range(args.steps):
                timed_step(k, stream, False)
        stop.record(stream)
        torch.cuda.synchronize()
        t_host1 = time.perf_counter()
    barrier(world)
    elapsed_ms = start.elapsed_time(stop)
    if flush_l2:
        elapsed_ms = sum(b0.elapsed_time(b1) for b0, b1 in bounds)
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    if graph_ev is not None:
        graph_ev.replay()
    else:
        for k in range(args.steps):
            timed_step(k, stream, True)
    torch.cuda.synchronize()
    stage_names = ["hash", "gather", "proj", "gate_conv"]
    stage_ms = {n: statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(args.steps))
                for i, n in enumerate(stage_names)}
    status = E.engram_device_status(clear=True)
    if status:
        raise SystemExit(f"device status {status:#x} after the timed region")

    # ---- e2e: inputs from pinned host memory, result back to pinned host memory.
    # Every step copies its ids and hidden states host->device and its output device->host.
    # The copies run on their own streams with two device buffer sets, so that the H2D of
    # step k+1, the compute of step k and the D2H of step k-1 overlap (the host link is
    # full duplex); events order each buffer's reuse.
    e2e = None
    if not args.no_e2e:
        nbuf = 2
        ids_host = torch.from_numpy(ids_np).pin_memory()
        h_host = torch.empty((wl.h_rows, wl.d_h), dtype=torch.bfloat16).pin_memory()
        h_host.copy_(h.cpu())
        out_host = torch.empty((wl.h_rows, wl.d_h), dtype=torch.bfloat16).pin_memory()
        ids_d = [torch.empty_like(ids) for _ in range(nbuf)]
        h_d = [torch.empty_like(h) for _ in range(nbuf)]
        out_d = [torch.empty_like(out) for _ in range(nbuf)]
        s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_steps(n_steps, comp):
            """Issue n_steps pipelined steps; comp is the compute stream (the capture stream
            while capturing)."""
            ev_h2d = [torch.cuda.Event() for _ in range(nbuf)]
            ev_comp = [torch.cuda.Event() for _ in range(nbuf)]
            ev_d2h = [torch.cuda.Event() for _ in range(nbuf)]
            s_h2d.wait_stream(comp)
            s_d2h.wait_stream(comp)
            for k in range(n_steps):
                b = k % nbuf
                with torch.cuda.stream(s_h2d):
                    if k >= nbuf:
                        s_h2d.wait_event(ev_comp[b])        # compute of step k-2 done reading buffer b
                    ids_d[b].copy_(ids_host, non_blocking=True)
                    h_d[b].copy_(h_host, non_blocking=True)
                    ev_h2d[b].record(s_h2d)
                comp.wait_event(ev_h2d[b])
                if k >= nbuf:
                    comp.wait_event(ev_d2h[b])              # out buffer b copied out (step k-2)
                E.engram_forward(plan, weights, tables, ids_d[b], h_d[b], out_d[b], ws, remap=remap,
                                 history=history, conv_state=state, stream=comp)
                ev_comp[b].record(comp)
                with torch.cuda.stream(s_d2h):
                    s_d2h.wait_event(ev_comp[b])
                    out_host.copy_(out_d[b], non_blocking=True)
                    ev_d2h[b].record(s_d2h)
            comp.wait_stream(s_h2d)
            comp.wait_stream(s_d2h)

        e2e_steps(max(1, args.warmup), stream)
        torch.cuda.synchronize()
        g2 = None
        if not args.eager:
            g2 = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream()
            cap.wait_stream(stream)
            with torch.cuda.graph(g2, stream=cap, capture_error_mode="thread_local"):
                e2e_steps(args.steps, torch.cuda.current_stream())
            stream.wait_stream(cap)
            torch.cuda.synchronize()
            g2.replay()
            torch.cuda.synchronize()
        barrier(world)
        s2, t2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        if g2 is not None:
            g2.replay()
        else:
            e2e_steps(args.steps, stream)
        t2.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(s2.elapsed_time(t2), world)
        h2d = ids_host.numel() * 4 + h_host.numel() * 2
        d2h = out_host.numel() * 2
        # host-link reference: the same bytes copied alone, H2D and D2H at once (full duplex)
        lk0, lk1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        best_link = 1e9
        for _ in range(3):
            lk0.record(stream)
            with torch.cuda.stream(s_h2d):
                s_h2d.wait_stream(stream)
                h_d[0].copy_(h_host, non_blocking=True)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_stream(stream)
                out_host.copy_(out_d[1], non_blocking=True)
            stream.wait_stream(s_h2d)
            stream.wait_stream(s_d2h)
            lk1.record(stream)
            torch.cuda.synchronize()
            best_link = min(best_link, lk0.elapsed_time(lk1))
        e2e_step_ms = e2e_ms / args.steps
        e2e = {"value": wl.n_tok * world * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "mode": ("eager" if args.eager else "one CUDA graph of the K steps")
                       + "; H2D, engram_forward and D2H on three streams with two buffer sets",
               "link_copy_ms": best_link, "link_frac": best_link / e2e_step_ms}

    peaks = load_peaks()
    n_tok = wl.n_tok
    flops = 2.0 * n_tok * wl.d_m * (M + 1) * wl.d_h     # M key projections + the value projection
    proj_s = stage_ms["proj"] / 1e3
    tflops = flops / proj_s / 1e12
    # A timed region of at most a second is a burst for the tensor pipe (clocks have not yet
    # settled under the power cap): the denominator is the measured burst bf16 rate; longer
    # regions use the sustained one.
    timed_s = elapsed_ms / 1e3
    burst = timed_s <= 1.0
    peak_tf = peaks["bf16"] if burst else peaks["bf16_sus"]
    pair = bool(path & E.ENGRAM_PATH_PAIR_MMA)
    roofline = {"bound": "tensor",
                "kernel": ("proj_pair_kernel (cta_group::2 " if pair else "proj_kernel (")
                          + "tcgen05 k/v projections + gate partials)",
                "achieved": tflops, "peak": peak_tf, "unit": "TFLOP/s", "frac": tflops / peak_tf,
                "frac_of_sustained": tflops / peaks["bf16_sus"],
                "traffic": kernel_traffic("proj_pair_kernel" if pair else "proj_kernel", wl.name),
                "peak_source": f"{peaks['source']} bf16 {'burst' if burst else 'sustained'} "
                               f"(timed region {timed_s:.2f} s)",
                "algorithmic_per_launch": flops}
    # HBM view of the memory-bound part of the path.  Algorithmic bytes per step (the
    # method's own, no intermediates): each distinct table row once, hidden states read,
    # outputs written, token ids read; beside them the same with every token's rows.
    row_b = wl.d_e * wl.table_elem_bytes
    hout = n_tok * M * wl.d_h * 2 * 2
    alg_distinct = distinct_rows * row_b + hout + n_tok * 4
    alg_tokrows = n_tok * wl.H * row_b + hout + n_tok * 4
    gate_bytes = n_tok * (wl.d_h * 2 + M * (wl.d_h * 2 * 2 + 8))   # v (fp16) once; h read, out written, scalars
    hbm = {"peak_GBps": peaks["hbm"], "nominal_GBps": 8000.0,
           "distinct_rows_per_step": distinct_rows, "token_rows_per_step": n_tok * wl.H,
           "algorithmic_bytes_distinct_rows": alg_distinct, "algorithmic_bytes_token_rows": alg_tokrows,
           "gate_conv_GBps": gate_bytes / (stage_ms["gate_conv"] / 1e3) / 1e9}
    hbm["gate_conv_frac"] = hbm["gate_conv_GBps"] / peaks["hbm"]
    gather_bytes = n_tok * (wl.H * row_b + wl.d_m * 2 + wl.H * 4)   # rows read + m written + row ids
    hbm["gather_GBps"] = gather_bytes / (max(1e-6, stage_ms["gather"]) / 1e3) / 1e9
    hbm["gather_frac"] = hbm["gather_GBps"] / peaks["hbm"]
    # the path outside the projection: hash + gather + gate/conv, over the method's bytes (every
    # distinct row once, h, out, ids), and beside that with every token's rows
    path_ms = stage_ms["hash"] + stage_ms["gather"] + stage_ms["gate_conv"]
    hbm["path_ms"] = path_ms
    hbm["path_frac"] = alg_distinct / (path_ms / 1e3) / 1e9 / peaks["hbm"]
    hbm["path_frac_token_rows"] = alg_tokrows / (path_ms / 1e3) / 1e9 / peaks["hbm"]
    hbm["path_frac_nominal"] = alg_distinct / (path_ms / 1e3) / 1e9 / hbm["nominal_GBps"]
    # bytes these kernels move, their intermediates included (m written by the gather and read
    # back by the projection, v written by the projection and read by the gate kernel)
    hbm["incl_intermediates_GBps"] = (gather_bytes + gate_bytes) / (path_ms / 1e3) / 1e9
    hbm["incl_intermediates_frac"] = hbm["incl_intermediates_GBps"] / peaks["hbm"]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # tokens per worker scaled to the per-token work (about 20 s of CPU time per worker)
        cpu_tok = max(32, int(args.cpu_baseline_tokens * (2 * 2560 * 2560) / (wl.d_m * wl.d_h * (M + 1))))
        T1, dt1, _ = oracle_sample(wl, max(8, cpu_tok // 4))    # one core, for the record
        procs = oracle_procs(args, wl)
        pool = OraclePool(procs, wl)
        toks, dt = pool.round(wl, cpu_tok)
        pool.close()
        cpu = {"value": toks / dt, "unit": "tokens/s", "cores": procs, "kind": "oracle",
               "sample": f"{procs} samples of 1 sequence x {toks // procs} tokens of {wl.name}, one per process, "
                         f"fp64 scalar C on {host_cpu()}; one process alone: {T1 / dt1:.1f} tokens/s; "
                         f"table-row regeneration not timed"}

    value = n_tok * world * args.steps / (elapsed_ms / 1e3)
    line = {
        "metric": "engram_tokens_per_s", "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Zipf ids, counter-based bf16 tables/weights)",
        "config": workload_config(wl, world),
        "weights_layout": "packed" if packed is not None else "row-major",
        "path": {"pair_mma": bool(path & E.ENGRAM_PATH_PAIR_MMA), "row_order_gather": bool(path & E.ENGRAM_PATH_ROW_ORDER),
                 "bulk_gather": bool(path & E.ENGRAM_PATH_BULK_GATHER), "path_bits": path},
        "stages_ms": stage_ms, "hbm": hbm, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": args.steps * launches_per_step,
        "launch_mode": "eager" if args.eager else "one CUDA graph of the K timed steps (stage times from a "
                                                  "second replay of the same steps with event nodes)",
        "clocks": clocks.summary(t_host0, t_host1),
    }
    # The decode workload's steps on the same resident tables (decode20m and prefill20m share
    # the table geometry, the hash and the weights' shapes; only the seeded contents differ),
    # so that one bench run also reports the decode step time.
    if wl.name == "prefill20m" and not args.no_decode_steps:
        wl_dec = synth.get_workload("decode20m")
        dec = measure_decode_steps(E, fill_gpu, plan, weights, tables, wl_dec, max(args.steps, 20),
                                   max(args.warmup, 3), stream, dev)
        dec["workload"] = "decode20m shapes (256 sequences x 1 token, history and conv state) on the prefill20m tables"
        line["decode_steps"] = dec
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_hostpinned(args, wl, world, rank, local):
    """Tables in pinned, mapped host memory.  Per decode step: the row ids are hashed and the
    distinct rows staged into HBM on a side stream, overlapped with a stand-in for the layers
    that precede the lookup (a 2560x2560 bf16 GEMM on the compute stream); the streams join
    before the gather and gate/conv.  Timed as one CUDA graph of K steps; the serial order
    (everything on one stream) is timed the same way for the overlap figure."""
    import hashed_gram_embedding_remap_b200 as E
    from synth import fill_gpu

    dev = f"cuda:{local}"
    torch.cuda.set_device(local)
    fill_gpu.build()
    comp = torch.cuda.current_stream()
    pref = torch.cuda.Stream(priority=-1)   # prefetch kernels get SMs ahead of the stand-in GEMM
    t0 = time.perf_counter()
    eb = wl.table_elem_bytes
    bufs = [fill_gpu.HostMapped(wl.primes[h], wl.d_e, elem_bytes=eb) for h in range(wl.H)]
    for h, b in enumerate(bufs):
        (fill_gpu.fill_fp8_ if eb == 1 else fill_gpu.fill_)(b.tensor, wl.table_spec(h))
    torch.cuda.synchronize()
    t_alloc = time.perf_counter() - t0
    tables = [b.tensor for b in bufs]
    plan = E.Plan.from_workload(wl, host_tables=True)
    B = wl.B
    K = args.steps
    kind = args.ids or wl.ids_kind
    ids_all = (synth.uniform_ids(wl.vocab_in, (K + args.warmup, B, 1), wl.seeds()["ids"]) if kind == "uniform"
               else synth.zipf_ids(wl.vocab_in, wl.zipf_s, (K + args.warmup, B, 1), wl.seeds()["ids"]))
    ids_dev = torch.from_numpy(ids_all).to(dev)
    history = torch.from_numpy(wl.history()).to(dev)
    state = fill_gpu.filled((B, wl.state_len, wl.d_h), wl.state_spec(), dev)
    h = fill_gpu.filled((B, wl.d_h), wl.h_spec(0), dev)
    wk = fill_gpu.filled((wl.d_h, wl.d_m), wl.wk_spec(), dev)
    wv = fill_gpu.filled((wl.d_h, wl.d_m), wl.wv_spec(), dev)
    one = torch.full((wl.d_h,), 0x3F80, dtype=torch.int16, device=dev).view(torch.bfloat16)
    cw = fill_gpu.filled((wl.d_h, wl.conv_kernel), wl.conv_spec(), dev)
    packed = E.pack_weights(plan, wk, wv) if args.packed and E.engram_packed_weights_size(plan) else None
    weights = E.Weights(wk, wv, one, one, one, cw, packed=packed)
    out = torch.empty((B, wl.d_h), dtype=torch.bfloat16, device=dev)
    ws = E.alloc_workspace(plan, B, dev)
    idx = torch.empty((B, wl.H), dtype=torch.int32, device=dev)
    tdt = torch.uint8 if eb == 1 else torch.bfloat16
    staging = [torch.empty((B, wl.d_e), dtype=tdt, device=dev) for _ in range(wl.H)]
    sidx = torch.empty((B, wl.H), dtype=torch.int32, device=dev)
    uniq = torch.empty((wl.H, B), dtype=torch.int32, device=dev)
    nu = torch.empty((wl.H,), dtype=torch.int32, device=dev)
    m = torch.empty((B, wl.d_m), dtype=torch.bfloat16, device=dev)
    # optional HBM row cache in front of the host tables
    cache = E.RowCache(plan, args.cache_slots, dev) if args.cache_slots else None
    row_flags = torch.empty((wl.H, B), dtype=torch.int32, device=dev)
    n_hits = torch.zeros((wl.H,), dtype=torch.int32, device=dev)
    ga = torch.randn(2560, 2560, device=dev, dtype=torch.bfloat16)
    gb = torch.randn(2560, 2560, device=dev, dtype=torch.bfloat16)
    gc_ = torch.empty(2560, 2560, device=dev, dtype=torch.bfloat16)
    nstage = 4
    # external=True: recorded as event nodes when captured, so they can be timed after a replay
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(nstage)] for _ in range(K)]
    for row in ev:
        for e in row:
            e.record(comp)
    torch.cuda.synchronize()

    # L2 is flushed between timed steps (a 2 x L2 write outside each step's start/end events);
    # a step's time is its own event interval, and the run's time the sum over steps.
    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    se = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
          for _ in range(K)]
    for a, b in se:
        a.record(comp)
        b.record(comp)

    def one_step(k, overlap, evs=None, bounds=None):
        x = ids_dev[k]
        cs = torch.cuda.current_stream()           # the capture stream while capturing
        side = pref if overlap else cs
        if bounds is not None:
            flush_buf.fill_(k)
            bounds[0].record(cs)
        if overlap:
            pref.wait_stream(cs)
        with torch.cuda.stream(side):
            if evs is not None:
                evs[0].record(side)
            if cache is not None:
                E.engram_hash(plan, x, idx, history=history, stream=side)
                E.engram_stage_rows_cached(plan, idx, tables, cache, staging, sidx, uniq, nu, row_flags, n_hits,
                                           stream=side)
            else:   # hash + in-batch dedup + host-link copy (one kernel for a decode step)
                E.engram_stage_rows_from_ids(plan, x, tables, staging, idx, sidx, uniq, nu, history=history,
                                             stream=side)
            if evs is not None:
                evs[1].record(side)
        torch.matmul(ga, gb, out=gc_)              # stand-in for the layers before the lookup
        if overlap:
            cs.wait_stream(pref)
        if evs is not None:
            evs[2].record(cs)
        E.engram_gather(plan, sidx, staging, m, stream=cs, rows_bound=B)
        E.engram_gate_conv(plan, weights, h, m, B, 1, out, ws, conv_state=state, stream=cs)
        E.engram_advance_history(plan, x, history, stream=cs)
        if evs is not None:
            evs[3].record(cs)
        if bounds is not None:
            bounds[1].record(cs)

    def capture(overlap, with_events):
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(comp)
        with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
            for k in range(K):
                one_step(args.warmup + k, overlap, ev[k] if with_events else None, se[k])
        comp.wait_stream(cap)
        torch.cuda.synchronize()
        return g

    for k in range(args.warmup - 1):
        one_step(k, True)
    n_launch0 = E.kernel_launches()   # the library's own count of the kernels one step launches
    one_step(args.warmup - 1, True)
    torch.cuda.synchronize()
    launches_per_step = E.kernel_launches() - n_launch0
    results = {}
    for name, overlap in (("overlapped", True), ("serial", False)):
        g = capture(overlap, name == "overlapped")
        g.replay()
        torch.cuda.synchronize()
        if cache is not None:
            # the upload replay above ran the timed steps' own ids: empty the cache and warm it
            # on the warm-up steps only, so that the timed steps meet no row they inserted
            cache.reset(comp)
            for k in range(args.warmup):
                one_step(k, False)
            torch.cuda.synchronize()
        st, sp = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local) as clocks:
            c0 = time.perf_counter()
            st.record(comp)
            g.replay()
            sp.record(comp)
            torch.cuda.synchronize()
            c1 = time.perf_counter()
        results[name] = (sum(a.elapsed_time(b) for a, b in se) / K, clocks.summary(c0, c1))
        del g
    prefetch_ms = statistics.mean(ev[k][0].elapsed_time(ev[k][1]) for k in range(K))
    tail_ms = statistics.mean(ev[k][2].elapsed_time(ev[k][3]) for k in range(K))
    row_cache = None
    if cache is not None:
        # hit rate of the timed id stream under the timed protocol (cache emptied, warmed on the
        # warm-up steps), stepped one by one with the distinct-row counts read back
        cache.reset(comp)
        for k in range(args.warmup):
            one_step(k, False)
        hits = distinct = 0
        for k in range(K):
            n_hits.zero_()
            one_step(args.warmup + k, False)
            torch.cuda.synchronize()
            hits += int(n_hits.sum().item())
            distinct += int(nu.sum().item())
        row_cache = {"slots_per_table": args.cache_slots,
                     "GB": round(wl.H * args.cache_slots * wl.d_e * eb / 1e9, 2),
                     "hit_rate": hits / max(1, distinct),
                     "distinct_rows_per_step": distinct / K,
                     "host_bytes_per_step": (distinct - hits) / K * wl.d_e * eb}
    # GEMM alone, for the overlap figure
    gs, ge = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(5):
        torch.matmul(ga, gb, out=gc_)
    gs.record(comp)
    for _ in range(50):
        torch.matmul(ga, gb, out=gc_)
    ge.record(comp)
    torch.cuda.synchronize()
    gemm_ms = gs.elapsed_time(ge) / 50
    nu_h = nu.cpu().numpy()
    uniq_bytes = int(nu_h.sum()) * wl.d_e * eb
    # host-link reference: pinned host -> device cudaMemcpyAsync, 1 GiB, best of 5
    hsrc = torch.empty(1 << 29, dtype=torch.int16).pin_memory()
    ddst = torch.empty(1 << 29, dtype=torch.int16, device=dev)
    best = 1e9
    for _ in range(5):
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(comp)
        ddst.copy_(hsrc, non_blocking=True)
        a1.record(comp)
        torch.cuda.synchronize()
        best = min(best, a0.elapsed_time(a1))
    h2d_gbps = (1 << 30) / (best / 1e3) / 1e9
    # zero-copy staging throughput on a large batch (8192 tokens x H rows)
    big_n = 8192
    big_idx = torch.randint(0, min(wl.primes), (big_n, wl.H), dtype=torch.int32, device=dev)
    big_stage = [torch.empty((big_n, wl.d_e), dtype=tdt, device=dev) for _ in range(wl.H)]
    big_sidx = torch.empty((big_n, wl.H), dtype=torch.int32, device=dev)
    big_uniq = torch.empty((wl.H, big_n), dtype=torch.int32, device=dev)
    big_nu = torch.empty((wl.H,), dtype=torch.int32, device=dev)
    for _ in range(2):
        E.engram_stage_rows(plan, big_idx, tables, big_stage, big_sidx, big_uniq, big_nu, stream=comp)
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(comp)
    for _ in range(5):
        E.engram_stage_rows(plan, big_idx, tables, big_stage, big_sidx, big_uniq, big_nu, stream=comp)
    b1.record(comp)
    torch.cuda.synchronize()
    big_bytes = int(big_nu.cpu().numpy().sum()) * wl.d_e * eb
    big_gbps = big_bytes / (b0.elapsed_time(b1) / 5 / 1e3) / 1e9
    ovl_ms, ovl_clk = results["overlapped"]
    ser_ms, _ = results["serial"]
    saved = ser_ms - ovl_ms
    line = {
        "metric": "engram_tokens_per_s", "value": B / (ovl_ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ovl_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": f"synthetic; ids {kind}",
        "config": workload_config(wl, world, ids_kind=kind),
        "step_includes": "hash + distinct-row staging from host (side stream; one kernel without a row cache) "
                         "|| 2560^3 bf16 GEMM stand-in; "
                         "then gather + projections + gate/conv + history update",
        "host_link": {"bound": "host-link", "staged_rows_per_step": int(nu_h.sum()),
                      "staged_bytes_per_step": uniq_bytes, "prefetch_ms": prefetch_ms,
                      "prefetch_GBps": uniq_bytes / (prefetch_ms / 1e3) / 1e9,
                      "bulk_stage_GBps": big_gbps, "h2d_memcpy_peak_GBps": h2d_gbps,
                      "bulk_frac_of_h2d": big_gbps / h2d_gbps},
        "overlap": {"serial_ms_per_step": ser_ms, "overlapped_ms_per_step": ovl_ms, "gemm_ms": gemm_ms,
                    "prefetch_ms": prefetch_ms, "hidden_fraction": max(0.0, min(1.0, saved / max(1e-9, min(gemm_ms, prefetch_ms))))},
        "tail_ms": tail_ms, "table_setup_s": t_alloc, "clocks": ovl_clk,
        "launch_mode": "one CUDA graph of the K timed steps", "gpu_launches": K * launches_per_step,
        "row_cache": row_cache,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    for b in bufs:
        b.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["engram", "reference"], default="engram")
    ap.add_argument("--workload", default="prefill20m", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--no-decode-steps", action="store_true",
                    help="prefill20m: skip timing decode20m's steps on the same tables after the main line")
    ap.add_argument("--single-cta-mma", action="store_true",
                    help="never pair CTAs for the projection's MMAs (ENGRAM_FLAG_SINGLE_CTA_MMA)")
    ap.add_argument("--row-order-gather", action="store_true",
                    help="gather the rows grouped by row id: in-batch dedup of the HBM reads "
                         "(ENGRAM_FLAG_ROW_ORDER_GATHER)")
    ap.add_argument("--bulk-gather", action="store_true",
                    help="gather bf16 rows with bulk copies staged in shared memory (ENGRAM_FLAG_BULK_GATHER)")
    ap.add_argument("--oracle-tokens", type=int, default=128)
    ap.add_argument("--cpu-baseline-tokens", type=int, default=768)
    ap.add_argument("--oracle-procs", type=int, default=0,
                    help="host processes for the oracle (0 = all cores, at most 32)")
    ap.add_argument("--reference-seconds", type=float, default=90.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch every step from the host (no CUDA graph)")
    ap.add_argument("--ids", choices=["uniform", "zipf"], default=None, help="id distribution (host-pinned workload)")
    ap.add_argument("--table-rows", type=int, default=0, help="override the table size (largest prime <= N)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's sequences per step")
    ap.add_argument("--no-packed", dest="packed", action="store_false",
                    help="stream the row-major projection weights instead of their packed copy "
                         "(engram_pack_weights, made once before timing; used when d_h % 256 == 0)")
    ap.add_argument("--cache-slots", type=int, default=0,
                    help="host-resident tables: HBM row cache of this many slots per table (power of two; 0 = none)")
    ap.add_argument("--table-dtype", choices=["bf16", "fp8"], default="bf16",
                    help="table element type: bf16 rows, or e4m3 codes with one scale per table")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = synth.get_workload(args.workload)
    if args.table_rows:
        # same kernels and shapes with smaller tables (for profiling captures that must stay small)
        p = synth.largest_prime_below(args.table_rows + 1) if synth.workloads.is_prime(args.table_rows) is False \
            else args.table_rows
        wl = wl.with_(primes=(p,) * wl.H, name=f"{wl.name}[rows={p}]")
    if args.ids:
        wl = wl.with_(ids_kind=args.ids)
    if args.table_dtype == "fp8":
        wl = wl.with_(table_dtype="fp8", name=f"{wl.name}-fp8")
    if args.batch:
        wl = wl.with_(B=args.batch, name=f"{wl.name}[B={args.batch}]")
    if args.cache_slots:
        wl = wl.with_(name=f"{wl.name}[cache={args.cache_slots}]")
    if not args.packed:
        wl = wl.with_(name=f"{wl.name}[row-major weights]")
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, wl, world, rank)
        elif wl.host_tables:
            run_hostpinned(args, wl, world, rank, local)
        else:
            run_engram(args, wl, world, rank, local)
    finally:
        if world > 1 and args.impl == "engram":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
