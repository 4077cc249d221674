#!/usr/bin/env python
"""Benchmark of the B200 RAM-Net layer core.

One step = one ``ramnet_scan_forward`` call (address decode of keys and queries, CAPE,
Gated Sparse Update, sparse read, RMSNorm, gate), made as its two launches.  The headline
workload is the 1.3B-like Top-16 long-context prefill: B=4 sequences x T=16384 tokens x
H=16 heads, d_p=4, U=5 (M=1024 slots), K=16, d_v=128, CAPE on, bf16 inputs and output,
fp32 slot state, zero initial state.  The 340M-like Top-8 and Top-32 prefills are timed
the same way and reported under "prefill".  Inputs are resident in HBM when timing starts;
L2 is flushed (256 MiB write) between timed steps.

The JSON line also carries:
  roofline     algorithmic bytes of the recurrence launch / its device time, against the
               measured HBM copy bandwidth (MEASURED_PEAKS.json);
  onchip       the slot-state bytes the recurrence moves through tensor memory (12*K*d_v per
               token-head) / its device time, against the measured tensor-memory bandwidth;
  e2e          the same metric through the public API with pinned host buffers (H2D of the
               step's inputs and D2H of y inside the timed region);
  decode       the batched decode step (B=256, H=16, M=4096, K=16, d_v=128, state resident
               in HBM), 1024 consecutive steps replayed from one CUDA graph;
  cpu_baseline the CPU oracle on a bounded sample of the same workload (rank 0, N=1 only).

``--impl reference`` times the CPU oracle itself (the reference arm: there is no
reference implementation to install; the pages ship no code).

Multi-GPU (torchrun): every (b,h) head is independent, so each rank runs its own full
batch with no data-path collective (weak scaling); NCCL is used only for the barrier and
the max-over-ranks of the step time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from sparse_slot_recurrent_b200.workloads import WORKLOADS, generate  # noqa: E402

METRIC = "RAM-Net layer tokens/s (prefill scan, decode step) and % of HBM roofline"
# the largest prefill configuration is the headline; the other two are timed beside it
PREFILL = "prefill_1p3b_top16"
E2E_PIECES = 16  # runs along T of the end-to-end call (copies of one run overlap another's kernels)
PREFILL_ALL = ("prefill_340m_top8", "prefill_340m_top32", "prefill_1p3b_top16")
LAUNCHES_PER_STEP = 2  # route (k_route) and recurrence (k_scan)
SM_COUNT = 148
# tensor-memory bytes per clock per SM (32x32b.x4 load and store, many warps, batched waits),
# measured with a tcgen05.ld/st probe on B200; the on-chip roofline denominator
TMEM_BYTES_PER_CLK_SM = 120.0
DECODE = "decode_b256"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # HBM3e nominal (DGX B200 figure), for context beside the measured peak
L2_FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------------ accounting

def prefill_algorithmic_bytes(w, in_bytes=2, out_bytes=2, state_in=False) -> int:
    """Bytes a step must move at least: per token-head the two address logit vectors, v,
    g, z and y; per head the final state (S fp32 [M,d_v] + m fp32 [M]); the zero initial
    state is not read."""
    per_th = 2 * w.L * in_bytes + w.d_v * in_bytes + in_bytes + w.d_v * in_bytes + w.d_v * out_bytes
    per_head = w.M * w.d_v * 4 + w.M * 4
    n_th = w.B * w.T * w.H
    return n_th * per_th + w.B * w.H * per_head * (2 if state_in else 1)


def recur_algorithmic_bytes(w, in_bytes=2, out_bytes=2) -> int:
    """The recurrence launch alone: v and z in, y out per token-head, final state per head."""
    return w.B * w.T * w.H * w.d_v * (2 * in_bytes + out_bytes) + w.B * w.H * (w.M * w.d_v * 4 + w.M * 4)


def route_algorithmic_bytes(w, in_bytes=2) -> int:
    """The address launch alone: key and query logits and the write gate per token-head."""
    return w.B * w.T * w.H * (2 * w.L * in_bytes + in_bytes)


def decode_algorithmic_bytes(w, in_bytes=2, out_bytes=2) -> int:
    """Per (b,h) per step: inputs and y, the K write rows read and written, the K read rows
    read, and the K masses read and written (fp32)."""
    per_unit = 2 * w.L * in_bytes + w.d_v * in_bytes + in_bytes + w.d_v * in_bytes + w.d_v * out_bytes
    per_unit += w.K * w.d_v * 4 * 3 + w.K * 4 * 2
    return w.B * w.H * per_unit


def state_elements_per_step(K: int, d_v: int, heads: int) -> int:
    """State elements a decode step touches: K read rows + K write rows per head."""
    return heads * 2 * K * d_v


# ------------------------------------------------------------------ environment helpers

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# host-only sources of the library: they launch the kernels but hold no device code
HOST_ONLY_SOURCES = ("ramnet_api.cu", "scan_noalloc.cu")


def kernel_source_hash() -> str:
    """Hash of the device-code sources (a profile's counters apply while it is unchanged)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_slot_recurrent_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")) and name not in HOST_ONLY_SOURCES:
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode())
                h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu capture, only if the kernel sources are
    unchanged since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) == 3 and parts[0] == kernel and parts[1] == kernel_source_hash():
                    return {"dram_bytes_per_launch": int(parts[2]), "source_hash": parts[1]}
    except OSError:
        pass
    return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while active."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ distributed plumbing

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def dist_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def dist_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda") if torch.cuda.is_available() else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(tokens_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank processed tokens_per_rank in at most max_ms."""
    return world * tokens_per_rank / (max_ms / 1e3)


# ------------------------------------------------------------------ oracle (CPU) timing

def oracle_sample(w, n_heads: int, threads: int, T: int | None = None):
    """Run the CPU oracle on the first n_heads (b,h) heads of the workload, over the first
    T tokens (whole sequences by default); returns (seconds, token-heads processed)."""
    import oracle
    oracle.build()
    nb = max(1, (n_heads + w.H - 1) // w.H)
    sub = w.with_(B=nb, T=T or w.T)
    inp = generate(sub, seed=0)
    ocfg = oracle.OracleConfig(d_p=w.d_p, U=w.U, K=w.K, d_v=w.d_v)
    t0 = time.perf_counter()
    oracle.scan_forward(ocfg, inp["k_logits"], inp["q_logits"], inp["v"], inp["g"], inp["z"],
                        cape_mask=inp["cape_mask"], pos0=inp["pos0"], nthreads=threads)
    return time.perf_counter() - t0, nb * w.H * sub.T


def cpu_baseline(w, cores: int):
    n_heads = w.B * w.H  # the whole workload: a few seconds on 16 cores
    secs, th = oracle_sample(w, n_heads, cores)
    heads = ((n_heads + w.H - 1) // w.H) * w.H
    return {"value": th / w.H / secs, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{heads} (b,h) heads x T={w.T} tokens of {w.name} (tokens/s = token-heads/s / H)",
            "seconds": round(secs, 3)}


def decode_cpu_baseline(w, cores: int, max_seconds: float = 10.0):
    """The CPU oracle's decode step on a bounded sample of the decode workload: 8 sequences
    x H heads, steps until about max_seconds; units split over the host cores (the oracle
    call releases the interpreter lock)."""
    import concurrent.futures
    import numpy as np
    import oracle
    oracle.build()
    sub = w.with_(B=min(w.B, 8))
    inp = generate(sub, seed=0)
    gen = torch.Generator().manual_seed(1)
    S = torch.randn((sub.B, sub.H, sub.M, sub.d_v), generator=gen).double().numpy()
    m = (torch.rand((sub.B, sub.H, sub.M), generator=gen) * 1.5 + 0.5).double().numpy()
    ocfg = oracle.OracleConfig(d_p=w.d_p, U=w.U, K=w.K, d_v=w.d_v)
    units = sub.B * sub.H
    parts = [(units * i // cores, units * (i + 1) // cores) for i in range(cores)]
    parts = [pr for pr in parts if pr[1] > pr[0]]
    steps = 0
    t0 = time.perf_counter()
    with concurrent.futures.ThreadPoolExecutor(len(parts)) as ex:
        while steps < sub.T and (time.perf_counter() - t0) < max_seconds:
            r = steps % sub.ring
            args = [inp[k][:, r].contiguous() for k in ("k_logits", "q_logits", "v", "g", "z")]
            pos = torch.full((sub.B,), steps, dtype=torch.int32)
            list(ex.map(lambda pr: oracle.decode_step(ocfg, *args, S, m, pos=pos, cape_mask=inp["cape_mask"],
                                                      units=pr), parts))
            steps += 1
    secs = time.perf_counter() - t0
    return {"value": sub.B * steps / secs, "unit": "tokens/s", "cores": len(parts), "kind": "oracle",
            "sample": f"{sub.B} sequences x {sub.H} heads x {steps} consecutive steps of {w.name}",
            "seconds": round(secs, 3)}


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, timed on the host cores, rank 0 only."""
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    cores = os.cpu_count() or 1
    n_heads = min(w.B * w.H, cores)
    # keep the timed steps to about two minutes: shorten the sequences of each step's sample
    # when whole sequences would take longer
    t_step = None
    for _ in range(args.warmup):
        t_step, _ = oracle_sample(w, n_heads, cores)
    T = w.T
    if t_step is not None and t_step * args.steps > 120.0:
        T = max(64, int(w.T * 120.0 / (t_step * args.steps)))
    secs = []
    th = 0
    for _ in range(args.steps):
        s, th = oracle_sample(w, n_heads, cores, T=T)
        secs.append(s)
    ms = 1e3 * statistics.mean(secs)
    value = th / w.H / (ms / 1e3)
    heads = ((n_heads + w.H - 1) // w.H) * w.H
    sample = f"{heads} (b,h) heads x the first {T} of T={w.T} tokens of {w.name} per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w, world):
    io = "bf16" if w.in_dtype == torch.bfloat16 else "fp32"
    return {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "d_p": w.d_p, "U": w.U, "M": w.M, "K": w.K,
            "d_v": w.d_v, "in_dtype": io, "out_dtype": io, "state": "fp32", "cape": w.cape,
            "l2": "flushed between timed steps (256 MiB write)",
            "parallelism": f"dp{world} (independent heads per rank, no collective)"}


# ------------------------------------------------------------------ GPU arm

def onchip_state_bytes(w) -> int:
    """State bytes the recurrence moves on chip per launch: per token-head K write rows read
    and written and K read rows read (fp32, 12*K*d_v bytes)."""
    return w.B * w.T * w.H * 12 * w.K * w.d_v


def time_prefill(args, world, rank, local, w, with_e2e: bool):
    """Time the prefill step (route + recurrence, the two launches ramnet_scan_forward makes)
    on workload w; returns the per-workload object of the JSON line."""
    from sparse_slot_recurrent_b200 import ramnet
    cfg = ramnet.Config(d_p=w.d_p, U=w.U, K=w.K, d_v=w.d_v)
    dev = torch.device("cuda", local)
    inp = generate(w, seed=rank)
    host = {k: v.pin_memory() for k, v in inp.items() if torch.is_tensor(v)}
    d = {k: v.to(dev) for k, v in host.items()}
    out_dtype = torch.bfloat16 if w.in_dtype == torch.bfloat16 else torch.float32
    y = torch.empty((w.B, w.T, w.H, w.d_v), dtype=out_dtype, device=dev)
    S = torch.empty((w.B, w.H, w.M, w.d_v), dtype=torch.float32, device=dev)
    m = torch.empty((w.B, w.H, w.M), dtype=torch.float32, device=dev)
    ws = torch.empty(ramnet.scan_workspace_bytes(cfg, w.B, w.T, w.H), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    lay = ramnet.scan_layout(cfg, w.in_dtype)

    def route():
        ramnet.scan_route(cfg, d["k_logits"], d["q_logits"], d["g"], ws, cape_mask=d["cape_mask"], pos0=d["pos0"],
                          stream=stream)

    def recur():
        ramnet.scan_recur(cfg, d["v"], d["z"], y, S, m, ws, stream=stream)

    def step():  # the same two launches scan_forward makes
        route()
        recur()

    for _ in range(args.warmup):
        step()
    ramnet.sync_status(stream)
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    dist_barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        route()
        ev[i][1].record(stream)
        recur()
        ev[i][2].record(stream)
    torch.cuda.synchronize(dev)
    dist_barrier(world)
    clk = clocks.stop()
    ramnet.sync_status(stream)
    ms = statistics.mean(a.elapsed_time(c) for a, _, c in ev)
    route_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
    recur_ms = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
    ms_max = dist_max(ms, world)
    tokens = w.B * w.T
    value = weak_scaling_value(tokens, world, ms_max)

    # roofline of the dominant kernel (the recurrence) against measured HBM bandwidth, plus
    # the same figures for the address launch and the whole step
    peak, peak_kind = measured_peaks()
    nb = 2 if w.in_dtype == torch.bfloat16 else 4
    alg_recur = recur_algorithmic_bytes(w, in_bytes=nb, out_bytes=nb)
    alg_route = route_algorithmic_bytes(w, in_bytes=nb)
    alg = prefill_algorithmic_bytes(w, in_bytes=nb, out_bytes=nb)
    achieved = alg_recur / (recur_ms / 1e3) / 1e9
    traffic = recorded_traffic(f"recur:{w.name}")
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": traffic["dram_bytes_per_launch"] if traffic else None,
                "kernel": "k_scan (ramnet_scan_recur)", "algorithmic_bytes": alg_recur,
                "ms_per_launch": recur_ms, "peak_kind": f"{peak_kind} hbm_gbs (burst copy)",
                "frac_of_nominal": achieved / NOMINAL_HBM_GBS}
    # on-chip: the slot state the recurrence reads and writes (tensor memory), against the
    # tensor-memory bandwidth of a tcgen05.ld/st probe (TMEM_BYTES_PER_CLK_SM) at the sampled SM clock
    sm_mhz = clk["sm_mhz"] if clk else 1965.0
    ctas = w.B * w.H * lay.ncta
    onchip_peak = TMEM_BYTES_PER_CLK_SM * min(ctas, SM_COUNT) * sm_mhz * 1e6 / 1e9
    onchip_ach = onchip_state_bytes(w) / (recur_ms / 1e3) / 1e9
    onchip = {"bytes_per_token_head": 12 * w.K * w.d_v, "achieved": onchip_ach, "peak": onchip_peak, "unit": "GB/s",
              "frac": onchip_ach / onchip_peak, "sm_mhz": sm_mhz, "sms_used": min(ctas, SM_COUNT),
              "peak_basis": f"{TMEM_BYTES_PER_CLK_SM} B/clk/SM tensor-memory load+store probe x SMs x SM clock"}
    kernels = {
        "route (k_route)": {"ms": route_ms, "algorithmic_bytes": alg_route,
                            "achieved_gbs": alg_route / (route_ms / 1e3) / 1e9},
        "recur (k_scan)": {"ms": recur_ms, "algorithmic_bytes": alg_recur, "achieved_gbs": achieved},
        "step": {"ms": ms, "algorithmic_bytes": alg, "achieved_gbs": alg / (ms / 1e3) / 1e9,
                 "frac": alg / (ms / 1e3) / 1e9 / peak},
    }

    # end to end through the public API from pinned host memory: ramnet_scan_forward_host reads
    # the step's per-token inputs from the host and writes y back to the host, in E2E_PIECES runs
    # along T whose copies overlap the kernels
    e2e = None
    if with_e2e:
        keys = ("k_logits", "q_logits", "v", "g", "z")
        yh = torch.empty(y.shape, dtype=y.dtype).pin_memory()
        h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
        d2h = yh.numel() * yh.element_size()
        scratch = torch.empty(ramnet.scan_forward_host_scratch_bytes(cfg, w.B, w.T, w.H, w.in_dtype, out_dtype,
                                                                     E2E_PIECES), dtype=torch.uint8, device=dev)

        def e2e_step():
            ramnet.scan_forward_host(cfg, host["k_logits"], host["q_logits"], host["v"], host["g"], host["z"], yh, S, m,
                                     scratch, pieces=E2E_PIECES, cape_mask=d["cape_mask"], pos0=d["pos0"],
                                     stream=stream)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        n_e2e = max(3, min(args.steps, 20))
        ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_e2e)]
        dist_barrier(world)
        for i in range(n_e2e):
            flush.zero_()
            ee[i][0].record(stream)
            e2e_step()
            ee[i][1].record(stream)
        torch.cuda.synchronize(dev)
        ramnet.sync_status(stream)
        e_ms = dist_max(statistics.mean(a.elapsed_time(b) for a, b in ee), world)
        e2e = {"value": weak_scaling_value(tokens, world, e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms, "steps": n_e2e, "pieces": E2E_PIECES,
               "call": "ramnet_scan_forward_host"}
        del scratch
    del flush, ws, y, S, m, d
    torch.cuda.empty_cache()
    return {"workload": w.name, "config": config_of(w, world), "value": value, "unit": "tokens/s",
            "ms_per_step": ms_max, "steps": args.steps, "roofline": roofline, "onchip": onchip, "kernels": kernels,
            "e2e": e2e, "clocks": clk, "gpu_launches": LAUNCHES_PER_STEP * args.steps,
            "plan": {"chunk": lay.chunk, "ctas_per_head": lay.ncta, "scan_warps": lay.scan_warps}}


def run_gpu(args, world, rank, local):
    from sparse_slot_recurrent_b200 import ramnet
    ramnet.load()
    if args.no_prefill:  # decode only (profiler captures of the decode step)
        decode = run_decode(args, world, local)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            decode["cpu_baseline"] = decode_cpu_baseline(WORKLOADS[DECODE], os.cpu_count() or 1)
        if rank == 0:
            print(json.dumps({"metric": METRIC, "decode": decode}), flush=True)
        return
    head = WORKLOADS[args.workload]
    if args.prefill_batch:  # fewer sequences of the same layer (profiler captures); headline only
        head = head.with_(B=args.prefill_batch, name=f"{head.name}_b{args.prefill_batch}")
    others = [] if (args.only_headline or args.prefill_batch) else [n for n in PREFILL_ALL if n != head.name]
    main = time_prefill(args, world, rank, local, head, with_e2e=not args.no_e2e)
    prefill = {head.name: {k: v for k, v in main.items() if k != "e2e"}}
    for name in others:
        prefill[name] = time_prefill(args, world, rank, local, WORKLOADS[name], with_e2e=False)
    decode = None if args.no_decode else run_decode(args, world, local)

    if rank == 0:
        line = {"metric": METRIC, "value": main["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": main["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded; shapes of the 340M / 1.3B layers)", "config": main["config"],
                "roofline": main["roofline"], "onchip": main["onchip"], "kernels": main["kernels"], "e2e": main["e2e"],
                "gpu_launches": main["gpu_launches"], "clocks": main["clocks"], "prefill": prefill, "decode": decode}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(head, os.cpu_count() or 1)
            if decode is not None:
                decode["cpu_baseline"] = decode_cpu_baseline(WORKLOADS[DECODE], os.cpu_count() or 1)
        print(json.dumps(line), flush=True)


def run_decode(args, world, local):
    """1024 consecutive decode steps of the batched workload, one CUDA graph."""
    from sparse_slot_recurrent_b200 import ramnet
    w = WORKLOADS[DECODE]
    if args.decode_batch:
        w = w.with_(B=args.decode_batch)
    cfg = ramnet.Config(d_p=w.d_p, U=w.U, K=w.K, d_v=w.d_v)
    dev = torch.device("cuda", local)
    inp = generate(w, seed=0)
    ring = [{k: inp[k][:, r].contiguous().to(dev) for k in ("k_logits", "q_logits", "v", "g", "z")}
            for r in range(w.ring)]
    mask = inp["cape_mask"].to(dev)
    gen = torch.Generator(device=dev).manual_seed(1)
    S = torch.randn((w.B, w.H, w.M, w.d_v), device=dev, generator=gen)
    m = torch.rand((w.B, w.H, w.M), device=dev, generator=gen) * 1.5 + 0.5
    pos = torch.arange(w.T, dtype=torch.int32, device=dev).view(w.T, 1).expand(w.T, w.B).contiguous()
    y = torch.empty((w.B, w.H, w.d_v), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.Stream(dev)

    def steps():
        for t in range(w.T):
            r = ring[t % w.ring]
            ramnet.decode_step(cfg, r["k_logits"], r["q_logits"], r["v"], r["g"], r["z"], S, m, pos=pos[t],
                               cape_mask=mask, y=y, stream=stream)

    with torch.cuda.stream(stream):
        steps()  # warm-up outside the graph
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        steps()
    reps = max(1, min(args.steps, 5))
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            graph.replay()
    stream.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    dist_barrier(world)
    with torch.cuda.stream(stream):
        for i in range(reps):
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
    stream.synchronize()
    ramnet.sync_status(stream)
    ms = dist_max(statistics.mean(a.elapsed_time(b) for a, b in ev), world)
    del graph
    peak, peak_kind = measured_peaks()
    alg = decode_algorithmic_bytes(w)
    step_ms = ms / w.T
    achieved = alg / (step_ms / 1e3) / 1e9
    return {"workload": w.name, "steps_per_replay": w.T, "replays": reps, "B": w.B, "H": w.H, "M": w.M, "K": w.K,
            "d_v": w.d_v, "value": weak_scaling_value(w.B * w.T, world, ms), "unit": "tokens/s",
            "ms_per_step": step_ms, "gpu_launches_per_replay": w.T,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None, "kernel": "k_step_warp",
                         "algorithmic_bytes_per_step": alg, "peak_kind": f"{peak_kind} hbm_gbs",
                         "frac_of_nominal": achieved / NOMINAL_HBM_GBS},
            "l2": "state (8 GiB) larger than L2",
            "state_elements_per_step": state_elements_per_step(w.K, w.d_v, w.B * w.H)}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ramnet", "reference"], default="ramnet")
    ap.add_argument("--workload", default=PREFILL, choices=[k for k, v in WORKLOADS.items() if not v.decode],
                    help="headline prefill workload (default: the 1.3B-like Top-16 long-context layer)")
    ap.add_argument("--only-headline", action="store_true", help="time only the headline prefill workload")
    ap.add_argument("--prefill-batch", type=int, default=0,
                    help="sequences of the headline prefill workload (default: the workload's; smaller for profiler "
                         "captures, timed as that workload only)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="sequences of the decode workload (default 256; smaller for profiler captures)")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill workloads (decode only)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup()
    if world != args.gpus and rank == 0:
        print(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using {world}", file=sys.stderr)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            if not torch.cuda.is_available():
                raise SystemExit("the ramnet arm needs a CUDA device")
            run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
