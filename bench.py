"""Benchmark of SparSTAR's per-scale block-sparse attention forward.

One step = the whole path for one scale of the 72,000-token workload
(H = 16, D = 128, bf16, density 0.09375): pool Q, pool K, score, select,
attention, each a launch of libsparstar through its C ABI on one stream,
with the inputs resident in HBM.  The metric is effective TFLOP/s over the
selected tiles (algorithmic attention FLOPs = 4 * D * sum over selected
(query block, key block) pairs of valid queries x valid keys) per step time.

Multi-GPU: the path has no exchange step; ``--gpus N`` runs N independent
replicas (one process per GPU, launched by torch.distributed.run), timing is
the max over ranks, and the value is the work of all ranks over that time.

``--impl reference`` times the CPU oracle instead (the comparison arm): each
step is a bounded sample of the same workload (one head's selection and a
set of its query rows in fp64), projected to the full step.
"""
import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from datetime import timedelta

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_attention_18_b200 import synth  # noqa: E402

METRIC = "sparse-attn fwd ms + TFLOP/s at 72k-token scale; % of bf16 TC peak"
UNIT = "TFLOP/s"
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic of one attention launch on the benchmark workload, from an
# ncu capture (dram__bytes_read.sum + dram__bytes_write.sum), keyed by the
# SHA-256 of the kernel source it was taken on; reported only while the
# source is unchanged.
ATTN_TRAFFIC = {
    "source_sha256": "e0af731107adf0fe4e9531a4dc2aaa9a1c32fdc93728c7cd175d924d95dc16d1",
    "bytes_per_launch": 3580000000 + 290000000,  # largest workload, one launch (3.58 GB + 290 MB)
}


def attn_source_sha256() -> str:
    path = os.path.join(ROOT, "block_sparse_attention_18_b200", "csrc", "attn_sm100.cu")
    with open(path, "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attention_flops(kv_idx: np.ndarray, kv_cnt: np.ndarray, Lq: int, Lk: int, D: int) -> float:
    """4 * D * sum over the listed tiles of valid query rows x valid keys."""
    B, H, nQB, max_sel = kv_idx.shape
    nKB = (Lk + 127) // 128
    vq = np.minimum(128, Lq - 128 * np.arange(nQB)).astype(np.float64)
    vk = np.minimum(128, Lk - 128 * np.arange(nKB)).astype(np.float64)
    slot = np.arange(max_sel)[None, None, None, :] < kv_cnt[..., None]
    ok = slot & (kv_idx >= 0) & (kv_idx < nKB)
    keys = np.where(ok, vk[np.clip(kv_idx, 0, nKB - 1)], 0.0).sum(axis=-1)  # [B,H,nQB]
    return float(4.0 * D * (keys * vq[None, None, :]).sum())


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons every 20 ms while
    running.  Each sample keeps its host arrival time, so that summary()
    can keep only the samples taken inside a given window (the timed
    region); started ahead of the region, it is already sampling when the
    region begins."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []  # (host arrival time, csv line)
        self.window = None

    def _gpu_id(self):
        try:
            uuid = torch.cuda.get_device_properties(self.dev).uuid
            return "GPU-%s" % uuid
        except Exception:
            return str(self.dev)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self._gpu_id(), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def wait_first(self, timeout_s=3.0):
        """Block (bounded) until the sampler has produced a line."""
        t_end = time.monotonic() + timeout_s
        while self.proc is not None and not self.lines and time.monotonic() < t_end:
            time.sleep(0.01)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for t, line in self.lines:
            if self.window is not None and not (self.window[0] <= t <= self.window[1]):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, val in zip(names, parts[3:]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [s for s in sm if s > 0.5 * (mx or max(sm))] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (n_gpus, world))
    if world > 1:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=timedelta(seconds=120))
    return world, rank, local


def barrier(world: int, device):
    if world > 1:
        if torch.distributed.get_backend() == "nccl":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


def job_throughput(flops_per_rank: float, ms_per_step: float, world: int) -> float:
    """Whole-job TFLOP/s: every rank (replica) does flops_per_rank per step,
    and the job's step time is the slowest rank's."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def max_over_ranks(value: float, world: int, device) -> float:
    """Max of a float over ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return value
    dev = device if torch.distributed.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------- CPU oracle

def oracle_band_step(orc, w, qn, kn, vn, head: int, band: int, n_blocks: int):
    """One bounded unit of the whole path on the oracle: for one head and
    the ``n_blocks`` query blocks starting at block ``band``, the fp32
    selection (pool Q of those blocks, pool K, score, select) and the fp64
    attention of every one of their query rows.  Returns (seconds, attention
    FLOPs of the unit): both measured on the same unit, nothing projected."""
    sl = slice(head, head + 1)
    r0 = band * 128
    r1 = min(w.Lq, r0 + n_blocks * 128)
    qh = np.ascontiguousarray(qn[:, sl, r0:r1])
    kh = np.ascontiguousarray(kn[:, sl])
    vh = np.ascontiguousarray(vn[:, sl])
    t0 = time.perf_counter()
    _, _, _, idx, cnt = orc.run_selection(qh, kh, w.text, w.image_ref, w.density)
    orc.attn_rows_f64(qh, kh, vh, idx, cnt, np.arange(r1 - r0, dtype=np.int64))
    dt = time.perf_counter() - t0
    return dt, attention_flops(idx, cnt, r1 - r0, w.Lk, w.D)


def _bands(w, n_units: int, n_blocks: int, seed: int):
    """Seeded (head, first query block) pairs; the first unit holds the
    last (possibly partial) query block."""
    rng = np.random.default_rng(seed)
    heads = w.B * w.H
    first = max(0, w.nQB - n_blocks)
    out = [(heads - 1, first)]
    while len(out) < n_units:
        out.append((int(rng.integers(0, heads)), int(rng.integers(0, first + 1))))
    return out


def cpu_baseline(w, qn, kn, vn, budget_s: float = 15.0, n_blocks: int = 2):
    """The oracle, as it stands, on this host's cores, on a bounded sample:
    whole-path units (one head, ``n_blocks`` query blocks) until the time
    budget is spent.  value = attention FLOPs of the units / their time."""
    import oracle as orc
    orc.lib()
    t_start = time.perf_counter()
    secs, flops, units = 0.0, 0.0, []
    for head, band in _bands(w, 10 ** 6, n_blocks, seed=7):
        dt, f = oracle_band_step(orc, w, qn, kn, vn, head, band, n_blocks)
        secs += dt
        flops += f
        units.append((head, band))
        if time.perf_counter() - t_start > budget_s and len(units) >= 2:
            break
    return {"value": flops / secs / 1e12, "unit": UNIT, "cores": orc.num_threads(),
            "kind": "oracle",
            "sample": ("%d units of the whole path (fp32 selection, then fp64 attention of every "
                       "row), each one head x %d query blocks (%d query rows): %.3g attention "
                       "FLOP in %.2f s; measured, not projected" % (
                           len(units), n_blocks, n_blocks * 128, flops, secs)),
            "wall_s": time.perf_counter() - t_start}


def run_reference(args, world, rank):
    """The comparison arm: the CPU oracle timed on this host's cores.  Each
    step is one bounded unit of the whole path (one head, a band of query
    blocks); value = attention FLOPs of the timed units / their time."""
    if rank != 0:
        return
    import oracle as orc
    orc.lib()
    w = bench_workload(args)
    q, k, v = synth.generate(w)
    qn, kn, vn = (synth.as_numpy(t) for t in (q, k, v))
    nb = args.ref_blocks
    units = _bands(w, args.warmup + args.steps, nb, seed=11)
    for head, band in units[:args.warmup]:
        oracle_band_step(orc, w, qn, kn, vn, head, band, nb)
    secs, flops = 0.0, 0.0
    for head, band in units[args.warmup:]:
        dt, f = oracle_band_step(orc, w, qn, kn, vn, head, band, nb)
        secs += dt
        flops += f
    value = flops / secs / 1e12
    sample = ("each step: one head x %d query blocks (%d rows) of the workload through the whole "
              "path (fp32 selection, fp64 attention of every row); %.3g attention FLOP per step "
              "on average; measured, not projected" % (nb, nb * 128, flops / args.steps))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle",
                         "cores": orc.num_threads(), "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, world):
    return {"workload": "%s: H=%d D=%d %s, keys text %d + image_ref %d + ref %d + cur %d = %d, "
                        "queries %d, density %g" % (w.name, w.H, w.D, w.dtype, w.text, w.image_ref,
                                                    w.ref, w.cur, w.Lk, w.Lq, w.density),
            "seq_len": w.Lq, "keys": w.Lk, "heads": w.H, "head_dim": w.D, "density": w.density,
            "seed": w.seed,
            "global_batch": w.B * world, "parallelism": "replicas" if world > 1 else "single",
            "l2": l2_note(w)}


def l2_note(w):
    """How the timed region treats L2 (no flush between steps): the note says
    whether this workload's inputs exceed the L2 or fit in it."""
    gb = w.B * (w.Lq + 2 * w.Lk) * w.H * w.D * (2 if w.dtype == "bf16" else 4) / 1e9
    l2 = 126 * 2 ** 20
    if torch.cuda.is_available():
        l2 = getattr(torch.cuda.get_device_properties(0), "L2_cache_size", l2) or l2
    if gb * 1e9 > 2 * l2:
        return "no flush: inputs (%.2f GB) larger than L2" % gb
    return ("no flush: inputs (%.3f GB) fit in L2, so the headline figure is L2-warm; the "
            "per_workload entry of this workload flushes L2 before each step" % gb)


# --------------------------------------------------------------- GPU arm

def fp32_peak_tflops(clocks):
    """FP32 FMA roofline: SMs x 128 lanes x 2 flops x the maximum SM clock."""
    mhz = clocks.get("sm_max_mhz") or 1965.0
    sms = torch.cuda.get_device_properties(0).multi_processor_count \
        if torch.cuda.is_available() else 148
    return sms * 128 * 2 * mhz * 1e6 / 1e12


def front_end_summary(w, per, peaks, clocks):
    """Rooflines of the selection kernels.  Pooling is HBM-bound: bytes = the
    Q and K reads + the mean writes.  The score is a fixed-order fp32 FMA
    product (2 * D flops per block pair): in the fused kernel it runs from
    shared memory and is bound by the FP32 pipes, peak = 148 SMs x 128 lanes
    x 2 flops x the SM clock; in the separate chain its S write and the
    select's S read go to memory."""
    esz = 2 if w.dtype == "bf16" else 4
    bh = w.B * w.H
    pool_bytes = ((w.Lq + w.Lk) * w.D * esz + (w.nQB + w.nKB) * w.D * 4) * bh
    score_flops = 2.0 * w.D * w.nQB * w.nKB * bh
    s_bytes = w.nQB * w.nKB * 4 * bh
    pool_ms = per["pool_qk"] if "pool_qk" in per else per["pool_q"] + per["pool_k"]
    pool_gbs = pool_bytes / (pool_ms * 1e-3) / 1e9
    out = {"pool": {"ms": pool_ms, "bytes": pool_bytes, "gbs": pool_gbs,
                    "frac_of_hbm": pool_gbs / peaks["hbm_gbs"], "bound": "hbm"}}
    fp32_peak = fp32_peak_tflops(clocks)
    if "score_select" in per:
        ms = per["score_select"]
        tf = score_flops / (ms * 1e-3) / 1e12
        out["score_select"] = {"ms": ms, "fp32_tflops": tf, "bound": "alu",
                               "peak_fp32_tflops": fp32_peak, "frac": tf / fp32_peak,
                               "s_bytes_kept_on_chip": s_bytes}
        # pool and score as one pair against HBM: the algorithmic bytes of
        # the two steps (Q, K read and means written; means read and S
        # written) over the time of the two fused launches.
        pair_bytes = pool_bytes + (w.nQB + w.nKB) * w.D * 4 * bh + s_bytes
        pair_ms = pool_ms + ms
        pair_gbs = pair_bytes / (pair_ms * 1e-3) / 1e9
        out["pool_score"] = {"ms": pair_ms, "bytes": pair_bytes, "gbs": pair_gbs,
                             "frac_of_hbm": pair_gbs / peaks["hbm_gbs"]}
    else:
        score_bytes = (w.nQB + w.nKB) * w.D * 4 * bh + s_bytes
        out["score"] = {"ms": per["score"], "bytes": score_bytes,
                        "gbs": score_bytes / (per["score"] * 1e-3) / 1e9,
                        "fp32_tflops": score_flops / (per["score"] * 1e-3) / 1e12}
        out["select"] = {"ms": per["select"], "bytes": s_bytes,
                         "gbs": s_bytes / (per["select"] * 1e-3) / 1e9}
    return out


def run_gpu(args, world, rank, local):
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU path)")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from block_sparse_attention_18_b200 import sparstar as sp

    w = bench_workload(args)
    q, k, v = synth.generate(w)
    qd, kd, vd = q.to(device), k.to(device), v.to(device)
    ws = sp.Workspace(w.B, w.H, w.D, w.text, w.image_ref, w.ref, w.cur, w.density, device)
    out = torch.empty_like(qd)
    lse = torch.empty(w.B, w.H, w.Lq, device=device, dtype=torch.float32)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    tau = sp.default_tau(w.D)
    stream = torch.cuda.current_stream(device)
    sep_names = ["pool_q", "pool_k", "score", "select", "attn"]
    fused_names = ["pool_qk", "score_select", "attn"]

    # The separate chain: five launches, S in device memory.
    def step_separate(st, ev=None):
        if ev: ev[0].record(st)
        sp.sparstar_block_pool(qd, ws.qbar, stream=st)
        if ev: ev[1].record(st)
        sp.sparstar_block_pool(kd, ws.kbar, stream=st)
        if ev: ev[2].record(st)
        sp.sparstar_block_score(ws.qbar, ws.kbar, tau, ws.S, stream=st)
        if ev: ev[3].record(st)
        sp.sparstar_select(ws.S, ws.n_forced, w.density, kv_idx=ws.kv_idx, kv_cnt=ws.kv_cnt,
                           stream=st)
        if ev: ev[4].record(st)
        sp.sparstar_attn_fwd(qd, kd, vd, ws.kv_idx, ws.kv_cnt, tau, out, lse, status, stream=st)
        if ev: ev[5].record(st)

    # The fused chain (the timed step): three launches, S never in memory.
    def step_fused(st, ev=None):
        if ev: ev[0].record(st)
        sp.sparstar_block_pool_qk(qd, kd, ws.qbar, ws.kbar, stream=st)
        if ev: ev[1].record(st)
        sp.sparstar_score_select(ws.qbar, ws.kbar, ws.n_forced, w.density, tau,
                                 kv_idx=ws.kv_idx, kv_cnt=ws.kv_cnt, stream=st)
        if ev: ev[2].record(st)
        sp.sparstar_attn_fwd(qd, kd, vd, ws.kv_idx, ws.kv_cnt, tau, out, lse, status, stream=st)
        if ev: ev[3].record(st)

    fused = args.chain == "fused"
    step, names = (step_fused, fused_names) if fused else (step_separate, sep_names)
    for _ in range(args.warmup):
        step(stream)
    torch.cuda.synchronize(device)
    if int(status.item()) != 0:
        raise SystemExit("attention kernel status %#x" % int(status.item()))
    flops = attention_flops(ws.kv_idx.cpu().numpy(), ws.kv_cnt.cpu().numpy(), w.Lq, w.Lk, w.D)

    def timed_steps(step_fn, n_names, use_graph):
        """K steps bracketed by events, per-kernel events inside.  With
        use_graph the K steps are captured into one CUDA graph (per-kernel
        events as external record nodes) and the timed region is its single
        replay, bracketed by events on the launching stream."""
        evs = [[torch.cuda.Event(enable_timing=True, external=use_graph)
                for _ in range(n_names + 1)] for _ in range(args.steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        graph = None
        if use_graph:
            graph = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(device)
            cap.wait_stream(stream)
            with torch.cuda.stream(cap), torch.cuda.graph(graph, stream=cap):
                for s_i in range(args.steps):
                    step_fn(cap, evs[s_i])
            stream.wait_stream(cap)
            graph.replay()  # upload; not timed
            torch.cuda.synchronize(device)
        with ClockSampler(local) as clk_:
            clk_.wait_first()
            barrier(world, device)
            torch.cuda.synchronize(device)
            h0 = time.monotonic()
            t0.record(stream)
            if graph is not None:
                graph.replay()
            else:
                for s_i in range(args.steps):
                    step_fn(stream, evs[s_i])
            t1.record(stream)
            torch.cuda.synchronize(device)
            h1 = time.monotonic()
            time.sleep(0.06)  # the sample taken at the region's end arrives
            # samples that arrive within one interval after the region ends
            # were taken inside it
            clk_.window = (h0, h1 + 0.05)
        barrier(world, device)
        total = max_over_ranks(t0.elapsed_time(t1), world, device)
        per_ = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps for i in range(n_names)]
        del graph
        return total / args.steps, per_, clk_

    ms_per_step, per_list, clk = timed_steps(step, len(names), fused and args.graph)
    per = dict(zip(names, per_list))
    if int(status.item()) != 0:
        raise SystemExit("attention kernel status %#x" % int(status.item()))
    # The other chain, eager, for comparison (same buffers, same results).
    other_step, other_names = (step_separate, sep_names) if fused else (step_fused, fused_names)
    other_step(stream)
    other_ms, other_list, _ = timed_steps(other_step, len(other_names), False)
    other = {"chain": "separate" if fused else "fused", "ms_per_step": other_ms,
             "kernel_ms": dict(zip(other_names, other_list))}

    # End to end through the C ABI from pinned host buffers.  Every step
    # copies its Q, K, V host->device and its O device->host inside the
    # timed region.  The copies run on their own streams with double-buffered
    # device inputs and outputs, so step s+1's upload and step s-1's download
    # overlap step s's compute (PCIe is full duplex).
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    out_h = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    qb = [qd, qd.clone()]
    kbuf = [kd, kd.clone()]
    vb = [vd, vd.clone()]
    ob = [out, torch.empty_like(out)]
    s_up = torch.cuda.Stream(device)
    s_down = torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    up_done, comp_done, down_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize(device)
    e0.record(stream)
    s_up.wait_event(e0)
    s_down.wait_event(e0)
    for step_i in range(args.steps):
        b = step_i % 2
        if step_i >= 2:
            s_up.wait_event(comp_done[b])      # buffer b's previous compute has read it
        with torch.cuda.stream(s_up):
            qb[b].copy_(qh, non_blocking=True)
            kbuf[b].copy_(kh, non_blocking=True)
            vb[b].copy_(vh, non_blocking=True)
            up_done[b].record(s_up)
        stream.wait_event(up_done[b])
        if step_i >= 2:
            stream.wait_event(down_done[b])    # out[b] of step-2 has been read back
        fwd = sp.sparstar_forward_fused if fused else sp.sparstar_forward
        fwd(qb[b], kbuf[b], vb[b], w.text, w.image_ref, w.ref, w.cur, w.density, workspace=ws,
            out=ob[b], lse=lse, status=status, stream=stream)
        comp_done[b].record(stream)
        s_down.wait_event(comp_done[b])
        with torch.cuda.stream(s_down):
            out_h[b].copy_(ob[b], non_blocking=True)
            down_done[b].record(s_down)
    stream.wait_event(down_done[(args.steps - 1) % 2])
    if args.steps >= 2:
        stream.wait_event(down_done[args.steps % 2])
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier(world, device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device) / args.steps
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = out_h[0].numel() * out_h[0].element_size()

    dense = dense_comparison(sp, w, qd, kd, vd, tau, per["attn"], stream) if args.dense else None
    mass = retained_mass(sp, w, qd, kd, ws, lse, args.mass_rows) if args.mass_rows > 0 else None
    reuse = None
    if args.reuse and args.mass_rows > 0:
        front_ms = sum(t for n, t in per.items() if n != "attn")
        reuse = reuse_across_scales(sp, w, qd, kd, vd, tau, ws.n_forced, per["attn"], front_ms,
                                    args.mass_rows, stream)

    if rank != 0:
        return
    peaks, peaks_src = read_peaks()
    value = job_throughput(flops, ms_per_step, world)
    attn_tflops = flops / (per["attn"] * 1e-3) / 1e12
    traffic = None
    if ATTN_TRAFFIC["source_sha256"] == attn_source_sha256():
        traffic = ATTN_TRAFFIC["bytes_per_launch"]
    front = front_end_summary(w, per, peaks, clk.summary())
    sel_ms = sum(t for n, t in per.items() if n != "attn")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, world),
        "attn_ms": per["attn"], "attn_tflops": attn_tflops,
        "attn_pct_of_bf16_peak": {"measured_burst": 100 * attn_tflops / peaks["bf16_tflops"],
                                  "measured_sustained": (
                                      100 * attn_tflops / peaks["bf16_tflops_sustained"]
                                      if peaks.get("bf16_tflops_sustained") else None),
                                  "datasheet_2250": 100 * attn_tflops / DATASHEET_BF16_TFLOPS},
        "chain": args.chain, "graph": bool(fused and args.graph),
        "kernel_ms": per, "selection_share_pct": 100 * sel_ms / sum(per.values()),
        "front_end": front, "other_chain": other,
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": attn_tflops / peaks["bf16_tflops"],
                     "traffic": traffic,
                     "peak_source": "%s bf16 burst (MEASURED_PEAKS.json)" % peaks_src},
        "e2e": {"value": job_throughput(flops, e2e_ms, world), "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": len(names) * args.steps,
        "clocks": clk.summary(),
        "flops_per_step_per_gpu": flops,
    }
    if dense is not None:
        line["dense_comparison"] = dense
    if mass is not None:
        line["retained_mass"] = mass
    if reuse is not None:
        line["reuse_across_scales"] = reuse
    if world == 1 and args.per_workload:
        line["per_workload"] = per_workload(sp, device, stream, peaks)
    if world == 1 and not args.no_cpu_baseline:
        qn, kn, vn = (synth.as_numpy(t) for t in (q, k, v))
        line["cpu_baseline"] = cpu_baseline(w, qn, kn, vn)
    print(json.dumps(line), flush=True)


def per_workload(sp, device, stream, peaks, steps=10, warmup=3):
    """Every workload of the synthetic suite through the fused chain (pool
    Q+K, score+select, attention): ``steps`` steps captured in one CUDA
    graph and replayed once, per-kernel CUDA events inside.  Workloads whose
    inputs fit in L2 get an L2 flush (a write of twice the L2 size) before
    each step, outside the timed kernels."""
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(2 * l2 // 4, dtype=torch.float32, device=device)
    res = {}
    for name, w in synth.WORKLOADS.items():
        q, k, v = synth.generate(w)
        qd, kd, vd = q.to(device), k.to(device), v.to(device)
        del q, k, v
        ws = sp.Workspace(w.B, w.H, w.D, w.text, w.image_ref, w.ref, w.cur, w.density, device,
                          scores=False)
        out = torch.empty_like(qd)
        lse = torch.empty(w.B, w.H, w.Lq, device=device, dtype=torch.float32)
        status = torch.zeros(1, dtype=torch.int32, device=device)
        tau = sp.default_tau(w.D)
        in_bytes = sum(t.numel() * t.element_size() for t in (qd, kd, vd))
        do_flush = in_bytes < 2 * l2

        def step(st, ev=None):
            if do_flush:
                flush.fill_(1.0)
            if ev: ev[0].record(st)
            sp.sparstar_block_pool_qk(qd, kd, ws.qbar, ws.kbar, stream=st)
            if ev: ev[1].record(st)
            sp.sparstar_score_select(ws.qbar, ws.kbar, ws.n_forced, w.density, tau,
                                     kv_idx=ws.kv_idx, kv_cnt=ws.kv_cnt, stream=st)
            if ev: ev[2].record(st)
            sp.sparstar_attn_fwd(qd, kd, vd, ws.kv_idx, ws.kv_cnt, tau, out, lse, status,
                                 stream=st)
            if ev: ev[3].record(st)

        for _ in range(warmup):
            step(stream)
        torch.cuda.synchronize(device)
        evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
               for _ in range(steps)]
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(device)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap), torch.cuda.graph(graph, stream=cap):
            for i in range(steps):
                step(cap, evs[i])
        stream.wait_stream(cap)
        graph.replay()
        torch.cuda.synchronize(device)
        with ClockSampler(device.index) as clk:
            clk.wait_first()
            h0 = time.monotonic()
            graph.replay()
            torch.cuda.synchronize(device)
            h1 = time.monotonic()
            time.sleep(0.06)
            clk.window = (h0, h1 + 0.05)
        del graph
        if int(status.item()) != 0:
            raise SystemExit("%s: attention kernel status %#x" % (name, int(status.item())))
        kms = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / steps for i in range(3)]
        flops = attention_flops(ws.kv_idx.cpu().numpy(), ws.kv_cnt.cpu().numpy(), w.Lq, w.Lk,
                                w.D)
        attn_tf = flops / (kms[2] * 1e-3) / 1e12
        fe = front_end_summary(w, {"pool_qk": kms[0], "score_select": kms[1]}, peaks,
                               clk.summary())
        res[name] = {
            "step_ms": sum(kms), "pool_qk_ms": kms[0], "score_select_ms": kms[1],
            "attn_ms": kms[2], "attn_tflops": attn_tf,
            "attn_frac_of_measured_burst": attn_tf / peaks["bf16_tflops"] if w.dtype == "bf16"
            else None,
            # fp32 inputs run the fp32 SIMT kernel: its roofline is the FP32 FMA rate.
            "attn_roofline": "bf16 tensor (measured burst)" if w.dtype == "bf16"
            else "fp32 FMA (SMs x 128 lanes x 2 x max clock)",
            "attn_frac_of_roofline": attn_tf / (peaks["bf16_tflops"] if w.dtype == "bf16"
                                                else fp32_peak_tflops(clk.summary())),
            "pool_score_frac_of_hbm": fe["pool_score"]["frac_of_hbm"],
            "front_end_share_pct": 100 * (kms[0] + kms[1]) / sum(kms),
            "sm_mhz": clk.summary().get("sm_mhz"), "l2_flushed": do_flush,
        }
        del qd, kd, vd, ws, out, lse
        torch.cuda.empty_cache()
    return res


def mass_rows(w, per_head, device, seed=0):
    """Per head: the first row, the last row and `per_head` seeded random
    query rows, as flat row indices (bh * Lq + r)."""
    rng = np.random.default_rng(seed)
    rows = []
    for bh in range(w.B * w.H):
        r = {0, w.Lq - 1, *rng.choice(w.Lq, per_head, replace=False).tolist()}
        rows.extend(bh * w.Lq + x for x in sorted(r))
    return torch.tensor(rows, dtype=torch.int64, device=device)


def reuse_across_scales(sp, w, qd, kd, vd, tau, n_forced, fresh_attn_ms, fresh_front_ms,
                        per_head, stream, reps=5):
    """Diagnostic, outside the timed region: the block lists selected at the
    previous scale of the schedule, carried to this scale by position
    (sparstar_transfer_lists), as a replacement for this scale's fresh
    selection.  The source-scale inputs are either an independent seeded
    draw of that scale's workload (no persistence of content between the
    scales) or this scale's own tokens taken at the source positions (full
    persistence under the same position map); the two bracket what real
    activations would give.  For each: the transfer's time and bytes, the
    attention's time over the reused lists, their density and the retained
    attention mass on the sampled rows, beside the fresh lists' mass."""
    prev = synth.PREVIOUS_SCALE.get(w.name)
    if prev is None:
        return None
    src = synth.WORKLOADS[prev]
    seg_s, seg_t = synth.segments(src), synth.segments(w)
    nF_s = sp.sparstar_forced_blocks(src.text, src.image_ref)
    rows_t = mass_rows(w, per_head, qd.device)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    def timed_graph(fn):
        # A short kernel: launched eagerly its time is the host's launch
        # overhead, so the repetitions are replayed from a CUDA graph.
        # fn(st) launches on stream st.
        fn(stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap), torch.cuda.graph(g, stream=cap):
            for _ in range(reps):
                fn(cap)
        stream.wait_stream(cap)
        with torch.cuda.stream(stream):
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    qs, ks, _ = synth.generate(src)
    sources = {"independent": (qs.cuda(), ks.cuda())}
    del qs, ks
    sources["subsampled"] = synth.coarser_scale(qd, kd, seg_t, seg_s)
    out = {"source_scale": prev, "source_density": src.density, "target_density": w.density,
           "map": "per-segment proportional token position (text, image_ref, ref, cur)",
           "fresh_front_end_ms": fresh_front_ms, "fresh_attn_ms": fresh_attn_ms}
    o = torch.empty_like(qd)
    for name, (a, b) in sources.items():
        qbar, kbar = sp.sparstar_block_pool_qk(a, b, stream=stream)
        sidx, scnt = sp.sparstar_score_select(qbar, kbar, nF_s, src.density, stream=stream)
        tidx, tcnt = sp.sparstar_transfer_lists(sidx, scnt, seg_s, seg_t, stream=stream)
        t_ms = timed_graph(lambda st: sp.sparstar_transfer_lists(sidx, scnt, seg_s, seg_t, tidx,
                                                                 tcnt, stream=st))
        a_ms = timed(lambda: sp.sparstar_attn_fwd(qd, kd, vd, tidx, tcnt, tau, o, None,
                                                  want_lse=False, stream=stream))
        m = sp.sparstar_retained_mass(qd, kd, tidx, tcnt, n_forced, rows_t)
        torch.cuda.synchronize()
        cnt = tcnt.double()
        moved = 4 * (sidx.numel() + scnt.numel() + tidx.numel() + tcnt.numel())
        out[name] = {
            "transfer_ms": t_ms, "transfer_bytes": moved,
            "transfer_gbs": moved / (t_ms * 1e-3) / 1e9,
            "attn_ms": a_ms,
            "attn_tflops": attention_flops(tidx.cpu().numpy(), tcnt.cpu().numpy(), w.Lq, w.Lk,
                                           w.D) / (a_ms * 1e-3) / 1e12,
            "mean_blocks_per_row": float(cnt.mean()),
            "density_of_candidates": float(((cnt - n_forced) / (w.nKB - n_forced)).mean()),
            "mass_block_mean": float(m["mass_block"].mean()),
            "mass_tok_mean": float(m["mass_tok"].mean()),
        }
        del qbar, kbar, sidx, scnt, tidx, tcnt
    return out


def retained_mass(sp, w, qd, kd, ws, lse, per_head, seed=0):
    """Diagnostic, outside the timed region: on a seeded sample of query rows
    (per head: the first row, the last row, and `per_head` random rows), the
    dense attention mass the block lists keep, the forced blocks' share, and
    the token-wise bound (the same forced blocks plus the M largest candidate
    weights, M = the lists' candidate tokens).  Also checks that the block
    mass equals exp(lse_sparse - lse_dense) with the attention kernel's LSE."""
    rows_t = mass_rows(w, per_head, qd.device, seed)
    rows = rows_t.tolist()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    got = sp.sparstar_retained_mass(qd, kd, ws.kv_idx, ws.kv_cnt, ws.n_forced, rows_t)
    b.record()
    torch.cuda.synchronize()
    mb = got["mass_block"].cpu().numpy()
    mt = got["mass_tok"].cpu().numpy()
    mf = got["mass_forced"].cpu().numpy()
    from_lse = np.exp(lse.reshape(-1)[rows_t].double().cpu().numpy()
                      - got["lse_dense"].cpu().numpy())
    return {"rows": len(rows),
            "sample": "per head: first row, last row and %d seeded random query rows" % per_head,
            "mass_block_mean": float(mb.mean()), "mass_tok_mean": float(mt.mean()),
            "mass_forced_mean": float(mf.mean()),
            "gap_pct_mean": float(np.mean(100.0 * (mt - mb) / mt)),
            "gap_pct_of_means": float(100.0 * (1.0 - mb.mean() / mt.mean())),
            "lse_identity_max_rel": float(np.max(np.abs(from_lse / mb - 1.0))),
            "ms": a.elapsed_time(b)}


def dense_comparison(sp, w, qd, kd, vd, tau, sparse_attn_ms, stream, reps=3):
    """Context for the sparse operator's speed: the same scale with every
    key block listed (this library's kernel at density 1) and torch's
    scaled_dot_product_attention on the same tensors."""
    nKB = w.nKB
    idx = torch.arange(nKB, device=qd.device, dtype=torch.int32).expand(w.B, w.H, w.nQB, nKB)
    idx = idx.contiguous()
    cnt = torch.full((w.B, w.H, w.nQB), nKB, device=qd.device, dtype=torch.int32)
    out = torch.empty_like(qd)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    ours = timed(lambda: sp.sparstar_attn_fwd(qd, kd, vd, idx, cnt, tau, out, None,
                                              want_lse=False, stream=stream))
    dense_flops = 4.0 * w.D * w.Lq * w.Lk * w.B * w.H
    sdpa = timed(lambda: torch.nn.functional.scaled_dot_product_attention(qd, kd, vd))
    return {"ours_density1_ms": ours, "ours_density1_tflops": dense_flops / (ours * 1e-3) / 1e12,
            "sdpa_ms": sdpa, "sdpa_tflops": dense_flops / (sdpa * 1e-3) / 1e12,
            "sparse_attn_ms": sparse_attn_ms, "speedup_vs_sdpa": sdpa / sparse_attn_ms,
            "speedup_vs_ours_dense": ours / sparse_attn_ms}


def bench_workload(args):
    """The workload named on the command line, with --seed replacing its
    seed when given (the synthetic inputs are drawn from that seed) and
    --heads its head count (a smaller launch of the same shapes, for
    profiling)."""
    w = synth.WORKLOADS[args.workload]
    seed = getattr(args, "seed", None)
    if seed is not None:
        w = synth.with_seed(w, seed)
    heads = getattr(args, "heads", None)
    if heads is not None:
        if heads < 1:
            raise SystemExit("--heads must be at least 1")
        w = dataclasses.replace(w, H=heads)
    return w


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=synth.BENCH_WORKLOAD, choices=list(synth.WORKLOADS))
    ap.add_argument("--seed", type=int, default=None,
                    help="seed of the synthetic inputs (default: the workload's own)")
    ap.add_argument("--heads", type=int, default=None,
                    help="head count replacing the workload's own (smaller launches of the "
                         "same per-head shapes, for profiling)")
    ap.add_argument("--ref-blocks", type=int, default=2,
                    help="query blocks (of one head) per step of the reference arm")
    ap.add_argument("--chain", choices=["fused", "separate"], default="fused",
                    help="timed step: pool_qk + score_select + attn (fused) or the five "
                         "separate calls; the other chain is timed eagerly beside it")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time the fused chain eagerly instead of replaying a CUDA graph")
    ap.add_argument("--mass-rows", type=int, default=64,
                    help="random query rows per head for the retained-mass diagnostic "
                         "(0 skips it)")
    ap.add_argument("--no-reuse", dest="reuse", action="store_false",
                    help="skip the mask-reuse diagnostic (lists of the previous scale carried "
                         "to this one)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", dest="per_workload", action="store_false",
                    help="skip the table of every workload (single GPU only)")
    ap.add_argument("--no-dense", dest="dense", action="store_false",
                    help="skip the dense comparison point (density 1 and torch SDPA)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
