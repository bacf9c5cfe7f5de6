"""Throughput of block-causal linear attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl blin|reference]
                    [--config all|720p|480p|wide|decode|denoise]

Headline (default ``--config all``): one step = one blin_prefill of the
720p-like latent video (B=1, H=70, d=32, 21 x 45 x 80 tokens, blocks of 3
frames, bf16 storage, lognormal Q/K channel scales) on inputs already resident
in HBM.  The inputs (1355 MB moved per step) are larger than L2, so no flush is
needed between steps.  The line also reports the per-kernel roofline, an
end-to-end figure with host copies inside the timed region, the float64
oracle's CPU rate and the SM clocks seen while timing, plus sub-records:

  480p, wide   the same prefill measurement on the 480p-like and the
               wide-head (B=4, H=32, d=64, one-frame blocks) workloads;
  decode       80 blin_block_step calls (one 3-frame 30 x 52 block each,
               commit=1): per-block latency percentiles, the same calls
               replayed as one CUDA graph, device memory after every block;
  denoise      16 blocks, each denoised by 4 read-only block steps (fresh
               Q/K/V, commit=0) and then committed once, replayed as a graph;
  tconv        the Mix-FFN's causal block temporal convolution over the same
               latent video (C = 2240 channels), bytes against the HBM peak;
  nvfp4_720p   the 720p prefill on NVFP4 Q/K/V (4-bit codes with block
               scales): 118 instead of 256 bytes per token-head.

With N > 1 GPUs every rank runs its own independent copy of the workload (weak
scaling; heads and videos never exchange data) and each time is the max over
ranks.  ``--impl reference`` times the float64 CPU oracle (the only reference
this method has) on a bounded sample of the same workload and prints the same
line with ``"impl": "reference"``.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "block-causal linear-attn tokens·heads/s and % of B200 HBM peak, 1 GPU"
UNIT = "tokens*heads/s"
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------- helpers
def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _strip_comments(src: str) -> str:
    """C/C++ source without comments or blank lines (string literals kept as they are)."""
    out, i, n = [], 0, len(src)
    while i < n:
        if src.startswith("//", i):
            i = src.find("\n", i)
            i = n if i < 0 else i
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif src[i] == '"':
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(src[i])
            i += 1
    return "\n".join(line.rstrip() for line in "".join(out).splitlines() if line.strip())


def kernel_source_hash() -> str:
    """Hash of the CUDA sources' code (comments excluded): recorded ncu counters stay valid across
    comment edits and are dropped as soon as any code changes."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_causal_linear_rope_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                h.update(name.encode() + _strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches these sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            doc = json.load(f)
    except Exception:
        return None
    if doc.get("source_hash") != kernel_source_hash():
        return None
    return doc.get("per_launch_bytes", {}).get(workload, {}).get(kernel)


class ClockSampler:
    """nvidia-smi samples (every 200 ms) while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []     # (host arrival time, csv line)
        self.windows = []   # [start, end) host times of the timed regions

    def timed(self, start: float, end: float):
        self.windows.append((start, end))

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        # samples taken while a timed region ran (a sample reaches us up to one period late)
        inside = [ln for t, ln in self.lines if any(a <= t <= b + 0.2 for a, b in self.windows)]
        for line in inside or [ln for _, ln in self.lines]:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(ngpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's time (device clocks are per rank; the job is as slow as its slowest)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_workload(w: workloads.Workload, rank: int) -> workloads.Workload:
    """Rank r's independent copy of the workload (its own seed; heads never exchange data)."""
    return w.with_(seed=w.seed + rank)


def job_throughput(units_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job tokens*heads/s: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (ms_max * 1e-3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- oracle timing
def oracle_sample(w: workloads.Workload, q, k, v, rows_total: int, seed: int = 0, heads: int = 0):
    """Time the explicit pair-sum oracle on `rows_total` seeded query rows of `heads` seeded heads
    (0: all heads); returns (token*heads per second, seconds)."""
    import oracle
    pos, blk = oracle.grid(w.T, w.Hg, w.Wg, w.F)
    rng = np.random.default_rng([seed, 5])
    rows = np.sort(rng.choice(w.N, size=rows_total, replace=False))
    qs = q.reshape(-1, w.N, w.d)
    ks = k.reshape(-1, w.N, w.d)
    vs = v.reshape(-1, w.N, w.d)
    if 0 < heads < qs.shape[0]:
        hsel = np.sort(rng.choice(qs.shape[0], size=heads, replace=False))
        qs, ks, vs = qs[hsel], ks[hsel], vs[hsel]
    t0 = time.perf_counter()
    oracle.attention_rows(qs, ks, vs, pos, blk, rows, w.split, w.theta, w.eps)
    dt = time.perf_counter() - t0
    return rows_total * qs.shape[0] / dt, dt


def oracle_recurrence_rate(w: workloads.Workload, q, k, v):
    """Time the float64 state-form oracle (O(N d^2)) on the whole workload: token*heads per second."""
    import oracle
    pos, blk = oracle.grid(w.T, w.Hg, w.Wg, w.F)
    t0 = time.perf_counter()
    oracle.recurrence(q, k, v, pos, blk, w.split, w.theta, w.eps)
    dt = time.perf_counter() - t0
    return w.B * w.H * w.N / dt, dt


def omp_threads() -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else (os.cpu_count() or 1)


def run_reference(args, w):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1 and rank != 0:
        return
    q, k, v = workloads.call_tensors(w)
    # A bounded sample per step: one seeded query row per core (the oracle parallelises over
    # rows) of a seeded subset of heads, sized so the whole run stays near a minute whatever K is.
    rows = args.ref_rows or omp_threads()
    heads = max(1, min(w.B * w.H, 7000 // max(1, args.steps + args.warmup)))
    for i in range(args.warmup):
        oracle_sample(w, q, k, v, rows, seed=1 + i, heads=heads)
    times = []
    for i in range(args.steps):
        _, dt = oracle_sample(w, q, k, v, rows, seed=100 + i, heads=heads)
        times.append(dt)
    per_step = sum(times) / len(times)
    value = rows * heads / per_step
    sample = (f"{rows} seeded query rows x {heads} seeded heads of the {w.name} workload per step, "
              f"explicit O(N^2) float64 pair sum (all keys each row may see)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 0,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": omp_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(w, world):
    return {"workload": f"{w.name} prefill: B={w.B} H={w.H} d={w.d} {w.dtype}, latent {w.T}x{w.Hg}x{w.Wg} "
                        f"(N={w.N}), blocks of {w.F} frames, RoPE split {w.split}, theta {w.theta:g}, eps {w.eps:g}",
            "tokens_per_head": w.N, "heads_per_gpu": w.B * w.H, "head_dim": w.d, "block_frames": w.F,
            "l2": "inputs larger than L2 (no flush)", "parallelism": f"independent replica per GPU x{world}"}


# ----------------------------------------------------------------------------- GPU arm
def _load_blin(args):
    import torch

    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    import block_causal_linear_rope_b200 as blin
    return torch, blin, world, rank, local


def _prefill_args(blin, w, qd, kd, vd, od, ws, stream_ptr):
    """Pre-marshalled C-ABI arguments of one blin_prefill call (no state)."""
    geom = blin._geom(w.T, w.Hg, w.Wg, w.F, w.split, w.theta, w.eps)
    return (ctypes.c_void_p(qd.data_ptr()), ctypes.c_void_p(kd.data_ptr()), ctypes.c_void_p(vd.data_ptr()),
            ctypes.c_void_p(od.data_ptr()), blin.BF16 if w.dtype == "bf16" else blin.F32, w.B, w.H, w.d,
            ctypes.byref(geom), None, ctypes.c_void_p(ws.data_ptr()), ws.numel(), ctypes.c_void_p(stream_ptr)), geom


def measure_prefill(args, w, torch, blin, world, rank, clk, full: bool):
    """Device-resident prefill steps of workload w: the headline numbers, per-kernel event times and
    the roofline; with `full`, also the end-to-end figure (host copies inside the timed region) and
    the CPU baseline.  Returns the record (a dict)."""
    dt_t = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    wr = replica_workload(w, rank)
    q, k, v = workloads.call_tensors(wr)
    qh, kh, vh = (torch.from_numpy(x).to(dt_t).pin_memory() for x in (q, k, v))
    qd, kd, vd = (x.to("cuda") for x in (qh, kh, vh))
    od = torch.empty_like(qd)
    grid = (w.T, w.Hg, w.Wg)
    ws = torch.empty(blin.workspace_size(w.B, w.H, w.d, grid, w.F, w.split, w.theta, w.eps),
                     dtype=torch.uint8, device="cuda")
    cargs, geom = _prefill_args(blin, w, qd, kd, vd, od, ws, torch.cuda.current_stream().cuda_stream)
    prefill_c = blin.lib.blin_prefill

    def step():
        rc = prefill_c(*cargs)
        if rc != 0:
            raise RuntimeError(blin.lib.blin_last_error().decode())

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    path = blin.last_path()
    barrier(world)
    torch.cuda.synchronize()
    timer = blin.LaunchTimer()
    sets = [timer.new_set() for _ in range(args.steps)]
    arm = blin.LaunchTimer.arm_set
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # (1) the headline: K steps back to back, timed by two events on the launching stream;
    # nothing is recorded between the kernels
    n0 = blin.launch_count()
    t_wall = time.time()
    start.record()
    for _ in range(args.steps):
        step()
    end.record()
    torch.cuda.synchronize()
    clk.timed(t_wall, time.time())
    launches = blin.launch_count() - n0
    barrier(world)
    torch.cuda.synchronize()
    # (2) the same K steps again with an event pair around every launch, for the per-kernel
    # durations behind the roofline (events between kernels also keep the next kernel from
    # starting early, so this pass is slower)
    t_wall = time.time()
    for i in range(args.steps):
        arm(sets[i])
        step()
    torch.cuda.synchronize()
    clk.timed(t_wall, time.time())
    blin.lib.blin_set_timing_events(None, 0)
    barrier(world)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(end) / args.steps, world)
    per_kernel = timer.elapsed_ms()
    avg = {kname: sum(d[kname] for d in per_kernel) / len(per_kernel) for kname in blin.KERNELS}
    status = blin.device_status()
    if status != 0:
        raise SystemExit(f"kernel watchdog fired (code {status})")

    units = w.B * w.H * w.N  # token*heads per GPU per step
    elem = 2 if w.dtype == "bf16" else 4
    launched = {kname: avg[kname] for kname in blin.KERNELS if blin.KERNEL_BYTES_PER_UNIT.get(kname) is not None
                and avg[kname] > 0.0005}
    alg = {kname: blin.KERNEL_BYTES_PER_UNIT[kname] * w.d * elem * units for kname in launched}
    dom = max(launched, key=lambda k_: launched[k_])
    peak, peak_kind = hbm_peak()
    achieved = alg[dom] / (launched[dom] * 1e-3) / 1e9
    whole = 4 * units * w.d * elem / (ms * 1e-3) / 1e9
    rec = {
        "value": job_throughput(units, world, ms), "unit": UNIT, "ms_per_step": ms, "path": path,
        "workload": config_dict(w, world)["workload"],
        "hbm_gbs_whole_step": whole, "hbm_frac_whole_step": whole / peak,
        "kernel_ms": launched,
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"{peak_kind} hbm_gbs",
                     "traffic": recorded_traffic(dom, w.name),
                     "algorithmic_bytes_per_launch": alg[dom]},
        "gpu_launches": launches,
    }
    if not full:
        return rec

    # ---- end to end through the C ABI: pinned host inputs in, host output back.  Heads are
    # independent and contiguous ([B*H][N][d]), so the step is cut into head chunks that flow
    # through three streams (copy in, compute, copy out): one blin_prefill per chunk, and the
    # host-to-device and device-to-host copies overlap each other and the kernels.
    oh = torch.empty_like(qh).pin_memory()
    h2d = 3 * qh.numel() * qh.element_size()
    d2h = oh.numel() * oh.element_size()
    od_ref = od.clone()  # the device-resident steps' output
    BH = w.B * w.H
    nchunk = min(BH, args.e2e_chunks)
    bounds = [BH * i // nchunk for i in range(nchunk + 1)]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    rows = lambda x: x.view(BH, w.N, w.d)
    qh3, kh3, vh3, oh3 = rows(qh), rows(kh), rows(vh), rows(oh)
    qd3, kd3, vd3, od3 = rows(qd), rows(kd), rows(vd), rows(od)
    ws_chunk = torch.empty(max(blin.workspace_size(1, bounds[i + 1] - bounds[i], w.d, grid, w.F, w.split, w.theta,
                                                   w.eps) for i in range(nchunk)), dtype=torch.uint8, device="cuda")
    chunk_args = []
    for i in range(nchunk):
        h0, h1 = bounds[i], bounds[i + 1]
        chunk_args.append((ctypes.c_void_p(qd3[h0].data_ptr()), ctypes.c_void_p(kd3[h0].data_ptr()),
                           ctypes.c_void_p(vd3[h0].data_ptr()), ctypes.c_void_p(od3[h0].data_ptr()),
                           blin.BF16 if w.dtype == "bf16" else blin.F32, 1, h1 - h0, w.d, ctypes.byref(geom), None,
                           ctypes.c_void_p(ws_chunk.data_ptr()), ws_chunk.numel(),
                           ctypes.c_void_p(s_cmp.cuda_stream)))
    ev_in = [torch.cuda.Event() for _ in range(nchunk)]
    ev_cmp = [torch.cuda.Event() for _ in range(nchunk)]
    ev_out = torch.cuda.Event()

    def e2e_step():
        cur = torch.cuda.current_stream()
        for s_ in (s_in, s_cmp, s_out):
            s_.wait_stream(cur)
        for i in range(nchunk):
            h0, h1 = bounds[i], bounds[i + 1]
            with torch.cuda.stream(s_in):
                qd3[h0:h1].copy_(qh3[h0:h1], non_blocking=True)
                kd3[h0:h1].copy_(kh3[h0:h1], non_blocking=True)
                vd3[h0:h1].copy_(vh3[h0:h1], non_blocking=True)
                ev_in[i].record(s_in)
            s_cmp.wait_event(ev_in[i])
            rc = prefill_c(*chunk_args[i])
            if rc != 0:
                raise RuntimeError(blin.lib.blin_last_error().decode())
            ev_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[i])
                oh3[h0:h1].copy_(od3[h0:h1], non_blocking=True)
        ev_out.record(s_out)
        cur.wait_event(ev_out)
        cur.wait_stream(s_in)
        cur.wait_stream(s_cmp)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(3, min(args.steps // 4, 200))
    e_start.record()
    for _ in range(e_steps):
        e2e_step()
    e_end.record()
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e_start.elapsed_time(e_end) / e_steps, world)
    # the chunked output must equal the one-call output (same kernels, same inputs, heads independent)
    if not torch.equal(oh.to("cuda"), od_ref):
        raise SystemExit("end-to-end output differs from the device-resident step")
    rec["e2e"] = {"value": job_throughput(units, world, e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                  "d2h_bytes_per_step": d2h, "ms_per_step": e_ms, "head_chunks": nchunk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # a bounded sample of about 10-20 s: rows scaled by the keys each row sees
        cpu_rows = args.cpu_rows or max(64, int(2000 * 32760 / w.N))
        rate, secs = oracle_sample(w, q, k, v, cpu_rows)
        rec_rate, rec_secs = oracle_recurrence_rate(w, q, k, v)
        rec["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": omp_threads(), "kind": "oracle",
                               "sample": f"{cpu_rows} seeded query rows x {w.B * w.H} heads of {w.name}, "
                                         f"explicit O(N^2) float64 pair sum, {secs:.1f} s",
                               "recurrence": {"value": rec_rate, "unit": UNIT,
                                              "sample": f"the whole {w.name} workload through the float64 "
                                                        f"state-form oracle (O(N d^2)), {rec_secs:.1f} s"}}
    return rec


def measure_decode(args, w, torch, blin, world, rank, clk, denoise_steps: int = 0):
    """Minute-long autoregressive decode: w.steps blin_block_step calls (one block of w.F frames each)
    against the constant-size (S, z) cache.  With denoise_steps = K > 0, every block is first run K
    times read-only (commit=0, fresh Q/K/V each: denoising steps) and then committed once.
    Per-block latency from events around each block, the same sequence replayed as one CUDA graph,
    device memory after every block, and the state's size."""
    wr = replica_workload(w, rank)
    dt_t = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    nb, F = w.steps, w.F
    calls_per_block = denoise_steps + 1
    # inputs resident on the device before timing: a few distinct seeded blocks, cycled over the
    # calls (drawing all 80 blocks' 2.5e9 normals would take the host about a minute)
    ndist = min(nb * calls_per_block, 8)
    distinct = [tuple(torch.from_numpy(workloads.block_tensor(wr.with_(seed=wr.seed + 1000 * j), tid, 0, F))
                      .to("cuda", dt_t) for tid in (0, 1, 2)) for j in range(ndist)]
    out = torch.empty_like(distinct[0][0])
    st = blin.BlockState(w.B, w.H, w.d)
    st.reserve(F * w.HW)
    geom = blin._geom(F, w.Hg, w.Wg, F, w.split, w.theta, w.eps)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    dt_c = blin.BF16 if w.dtype == "bf16" else blin.F32
    step_c = blin.lib.blin_block_step
    cargs = []
    for b in range(nb):
        for s_ in range(calls_per_block):
            q, k, v = distinct[(b * calls_per_block + s_) % ndist]
            commit = 1 if s_ == denoise_steps else 0
            cargs.append((ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
                          ctypes.c_void_p(out.data_ptr()), dt_c, w.B, w.H, w.d, ctypes.byref(geom), st.handle,
                          commit, stream))

    def sequence(events=None):
        st.reset()
        for b in range(nb):
            if events is not None:
                events[b][0].record()
            for a in cargs[b * calls_per_block:(b + 1) * calls_per_block]:
                rc = step_c(*a)
                if rc != 0:
                    raise RuntimeError(blin.lib.blin_last_error().decode())
            if events is not None:
                events[b][1].record()

    for _ in range(max(1, args.warmup // 5)):
        sequence()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nb)]
    lat, mem_flat = [], True
    reps = max(1, min(args.steps // 100, 10))
    barrier(world)
    t_wall = time.time()
    for _ in range(reps):
        sequence(evs)
        torch.cuda.synchronize()
        lat += [a.elapsed_time(b) * 1e3 for a, b in evs]
        mem_flat &= torch.cuda.mem_get_info()[0] == free0
    clk.timed(t_wall, time.time())
    # host time to enqueue one block (plan, tensor maps, launches)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    sequence()
    host_us = (time.perf_counter() - t0) / nb * 1e6
    torch.cuda.synchronize()
    # the same calls captured once in a CUDA graph and replayed: per-block device time without
    # host launch overhead
    graph_us, graph_err = None, None
    try:
        cg = torch.cuda.CUDAGraph()
        st.reset()
        torch.cuda.synchronize()
        with torch.cuda.graph(cg):
            cs = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
            for a in cargs:
                rc = step_c(*(a[:-1] + (cs,)))
                if rc != 0:
                    raise RuntimeError(blin.lib.blin_last_error().decode())
        for _ in range(2):
            cg.replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        for _ in range(reps):
            cg.replay()
        g1.record()
        torch.cuda.synchronize()
        graph_us = max_over_ranks(g0.elapsed_time(g1) * 1e3 / (reps * nb), world)
        del cg
    except Exception as exc:  # capture unsupported: report why, keep the stream numbers
        graph_err = str(exc).splitlines()[0][:200]
    status = blin.device_status()
    if status != 0:
        raise SystemExit(f"kernel watchdog fired (code {status})")
    lat = np.array(lat)
    units = w.B * w.H * F * w.HW
    p50 = max_over_ranks(float(np.percentile(lat, 50)), world)
    p99 = max_over_ranks(float(np.percentile(lat, 99)), world)
    elem = 2 if w.dtype == "bf16" else 4
    # per call: Q, K, V read, O written; state read (and written by the commit)
    alg_call = 4 * units * w.d * elem + st.nbytes
    alg_block = calls_per_block * alg_call + st.nbytes
    peak, peak_kind = hbm_peak()
    per_block_us = graph_us if graph_us is not None else p50
    rec = {
        "workload": f"{w.name}: {nb} blocks of {F}x{w.Hg}x{w.Wg} tokens, B={w.B} H={w.H} d={w.d} {w.dtype}, "
                    + (f"each block {denoise_steps} read-only block steps (commit=0, fresh Q/K/V) then one commit"
                       if denoise_steps else "one block_step (commit=1) per block")
                    + f"; {ndist} distinct seeded inputs cycled",
        "calls_per_block": calls_per_block,
        "latency_us_per_block": {"p50": p50, "p99": p99, "min": float(lat.min()), "max": float(lat.max()),
                                 "graph_replay": graph_us, "graph_error": graph_err,
                                 "host_enqueue": host_us},
        "latency_us_per_call_graph": None if graph_us is None else graph_us / calls_per_block,
        "value": job_throughput(units * calls_per_block, world, per_block_us * 1e-3), "unit": UNIT,
        "roofline": {"bound": "hbm", "kernel": "block step (all launches)", "achieved": alg_block / (per_block_us * 1e-6) / 1e9,
                     "peak": peak, "unit": "GB/s", "frac": alg_block / (per_block_us * 1e-6) / 1e9 / peak,
                     "peak_source": f"{peak_kind} hbm_gbs", "timing": "graph replay" if graph_us is not None else "p50",
                     "algorithmic_bytes_per_block": alg_block},
        "state_bytes": st.nbytes, "device_memory_flat": bool(mem_flat),
    }
    st.free()
    return rec


def measure_tconv(args, w, torch, blin, world, rank, clk):
    """Causal block temporal convolution over a whole latent video (one call): time per call,
    and algorithmic bytes (x read, y written) against the HBM peak."""
    wr = w.with_(seed=w.seed + rank)
    x, taps, bias = workloads.conv_tensors(wr)
    dt_t = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    xd = torch.from_numpy(x.reshape(w.B, -1, w.C)).to("cuda", dt_t)
    td, bd = torch.from_numpy(taps).cuda(), torch.from_numpy(bias).cuda()
    yd = torch.empty_like(xd)
    geom = blin._geom(w.T, w.Hg, w.Wg, w.F, (0, 0, 0), 1e4, 0.0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cargs = (ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(td.data_ptr()), ctypes.c_void_p(bd.data_ptr()),
             ctypes.c_void_p(yd.data_ptr()), blin.BF16 if w.dtype == "bf16" else blin.F32, w.B, w.C,
             ctypes.byref(geom), None, 0, stream)
    call = blin.lib.blin_tconv

    def step():
        rc = call(*cargs)
        if rc != 0:
            raise RuntimeError(blin.lib.blin_last_error().decode())

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall = time.time()
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clk.timed(t_wall, time.time())
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    elem = 2 if w.dtype == "bf16" else 4
    alg = 2 * w.B * w.N * w.C * elem
    peak, peak_kind = hbm_peak()
    return {"workload": f"{w.name}: causal block temporal convolution, B={w.B} C={w.C} {w.dtype}, latent "
                        f"{w.T}x{w.Hg}x{w.Wg}, blocks of {w.F} frames, taps (previous, current, next) + bias",
            "ms_per_step": ms, "value": w.B * w.N * w.C / (ms * 1e-3), "unit": "token*channels/s",
            "roofline": {"bound": "hbm", "kernel": "tconv", "achieved": alg / (ms * 1e-3) / 1e9, "peak": peak,
                         "unit": "GB/s", "frac": alg / (ms * 1e-3) / 1e9 / peak, "peak_source": f"{peak_kind} hbm_gbs",
                         "algorithmic_bytes_per_launch": alg}}


def measure_nvfp4(args, w, torch, blin, world, rank, clk):
    """The prefill on NVFP4 Q/K/V (packed E2M1 codes, one E4M3 scale per 16 elements, a global
    scale per tensor; bf16 output): time per step and algorithmic bytes against the HBM peak."""
    wr = replica_workload(w, rank)
    ops = [blin.Nvfp4Tensor(torch.from_numpy(dt), torch.from_numpy(sc), gs)
           for dt, sc, gs in workloads.nvfp4_call_tensors(wr)]
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device="cuda")
    grid = (w.T, w.Hg, w.Wg)
    ws = torch.empty(blin.workspace_size(w.B, w.H, w.d, grid, w.F, w.split, w.theta, w.eps), dtype=torch.uint8,
                     device="cuda")
    geom = blin._geom(w.T, w.Hg, w.Wg, w.F, w.split, w.theta, w.eps)
    cs = [o.c() for o in ops]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cargs = (ctypes.byref(cs[0]), ctypes.byref(cs[1]), ctypes.byref(cs[2]), ctypes.c_void_p(out.data_ptr()), w.B,
             w.H, w.d, ctypes.byref(geom), None, ctypes.c_void_p(ws.data_ptr()), ws.numel(), stream)
    call = blin.lib.blin_prefill_nvfp4

    def step():
        rc = call(*cargs)
        if rc != 0:
            raise RuntimeError(blin.lib.blin_last_error().decode())

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall = time.time()
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clk.timed(t_wall, time.time())
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    units = w.B * w.H * w.N
    per_unit = 3 * (w.d // 2 + w.d // 16) + 2 * w.d  # q, k, v packed codes and scales read; bf16 o written
    alg = units * per_unit
    peak, peak_kind = hbm_peak()
    return {"workload": f"{w.name} prefill with NVFP4 q, k, v (E2M1 + E4M3 per 16 elements + global scale), "
                        f"bf16 o: B={w.B} H={w.H} d={w.d}, latent {w.T}x{w.Hg}x{w.Wg}, blocks of {w.F} frames",
            "ms_per_step": ms, "value": job_throughput(units, world, ms), "unit": UNIT,
            "bytes_per_token_head": per_unit,
            "roofline": {"bound": "hbm", "kernel": "whole step (3 launches)", "achieved": alg / (ms * 1e-3) / 1e9,
                         "peak": peak, "unit": "GB/s", "frac": alg / (ms * 1e-3) / 1e9 / peak,
                         "peak_source": f"{peak_kind} hbm_gbs", "algorithmic_bytes_per_step": alg}}


def run_blin(args):
    torch, blin, world, rank, local = _load_blin(args)
    main_name = "720p" if args.config == "all" else args.config
    with ClockSampler(local) as clk:
        time.sleep(0.25)  # let the sampler start
        if main_name in ("decode", "denoise"):
            w = workloads.CONFIGS["decode"]
            rec = measure_decode(args, w, torch, blin, world, rank, clk, 4 if main_name == "denoise" else 0)
            main = {"metric": "decode block_step tokens*heads/s (graph-replayed blocks)", "value": rec["value"],
                    "ms_per_step": rec["latency_us_per_block"]["p50"] * 1e-3, "roofline": rec["roofline"],
                    "config": {"workload": rec["workload"], "parallelism": f"independent replica per GPU x{world}",
                               "l2": "per-block inputs live in HBM; no flush"}, "decode": rec}
        else:
            w = workloads.CONFIGS[main_name]
            rec = measure_prefill(args, w, torch, blin, world, rank, clk, full=True)
            main = {"metric": METRIC, "value": rec["value"], "ms_per_step": rec["ms_per_step"],
                    "config": config_dict(w, world)}
            for key in ("path", "hbm_gbs_whole_step", "hbm_frac_whole_step", "kernel_ms", "roofline", "e2e",
                        "gpu_launches", "cpu_baseline"):
                if key in rec:
                    main[key] = rec[key]
        subs = {}
        if args.config == "all" and not args.no_sub_records:
            for name in ("480p", "wide"):
                subs[name] = measure_prefill(args, workloads.CONFIGS[name], torch, blin, world, rank, clk, full=False)
            subs["decode"] = measure_decode(args, workloads.CONFIGS["decode"], torch, blin, world, rank, clk, 0)
            subs["denoise"] = measure_decode(args, workloads.CONFIGS["decode"].with_(steps=16), torch, blin, world,
                                             rank, clk, 4)
            subs["tconv"] = measure_tconv(args, workloads.CONV_CONFIGS["conv-480p"], torch, blin, world, rank, clk)
            subs["nvfp4_720p"] = measure_nvfp4(args, workloads.CONFIGS["720p"], torch, blin, world, rank, clk)
        time.sleep(0.25)
    line = {"metric": main.pop("metric"), "value": main.pop("value"), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": main.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": workloads.CONFIGS[
                "decode" if main_name in ("decode", "denoise") else main_name].dtype, "data": "synthetic"}
    line.update(main)
    line["clocks"] = clk.summary()
    if subs:
        line["sub_records"] = subs
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="blin", choices=["blin", "reference"])
    ap.add_argument("--config", default="all", choices=["all", "480p", "720p", "wide", "decode", "denoise"],
                    help="all: the 720p headline plus 480p, wide, decode and denoise sub-records")
    ap.add_argument("--cpu-rows", type=int, default=None,
                    help="oracle rows for the CPU baseline (default: scaled to about 10-20 s)")
    ap.add_argument("--ref-rows", type=int, default=None,
                    help="oracle rows per reference-arm step (default: sized so the whole run stays near a minute)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub-records", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=7, help="head chunks pipelined through the e2e step")
    args = ap.parse_args()
    if args.impl == "reference":
        name = "720p" if args.config == "all" else args.config
        run_reference(args, workloads.CONFIGS["decode" if name == "denoise" else name])
    else:
        run_blin(args)


if __name__ == "__main__":
    main()
