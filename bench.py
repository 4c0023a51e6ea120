#!/usr/bin/env python3
"""Throughput of the DLRM hot path on B200, as one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload large] [--impl ours|reference]

A step is one forward pass of the whole hot path over one batch: bottom MLP,
fused embedding-bag gather + pairwise interaction + concat, top MLP and
sigmoid. Default workload: the large memory-bound configuration (B = 65536,
26 tables with log-spaced row counts 1e3 .. 4e7 = 29.6 GB of bf16, d = 128,
one-hot Zipf(1.05) bags, bottom MLP 13-512-256-128, top MLP
479-1024-1024-512-256-1). Inputs are seeded synthetic stand-ins for a click
log; the benchmark cycles a pool of 8 batches.

value:  samples/s with inputs resident in HBM, device time (CUDA events),
        max over ranks; each rank runs an independent replica (weak scaling).
e2e:    the same through dlrm_forward (dlrm_forward_cat for the concat-only
        interaction) with every step's batch copied from pinned host memory and
        y_hat copied back inside the timed region (the copy of step i+1 runs on
        a copy stream while step i computes; y_hat of step i goes back on a
        third stream while step i+1 computes, and the timing ends after the
        last one has arrived).
roofline: the fused gather + interaction kernel against measured HBM
        bandwidth, with algorithmic bytes = gathered rows + indices + offsets +
        x_dense read + concat write.
cpu_baseline: the fp64 CPU oracle on a bounded sample of the same workload.

--impl reference times that oracle alone (rank 0 only).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import CONFIGS, gen  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
POOL = 8


def workload_desc(cfg) -> str:
    rows = f"{min(cfg.rows)}..{max(cfg.rows)} rows" if len(set(cfg.rows)) > 1 else f"{cfg.rows[0]} rows each"
    tb = sum(cfg.rows) * table_row_bytes(cfg) / 1e9
    return (f"{cfg.name}: B={cfg.B}, K={cfg.K} tables ({rows}, {tb:.1f} GB {cfg.table_dtype}), d={cfg.d}, "
            f"bags={cfg.bag}, indices={cfg.index}, bottom={'-'.join(map(str, cfg.bottom))}, "
            f"top={'-'.join(map(str, cfg.top))}")


def table_row_bytes(cfg) -> int:
    """Bytes of one stored table row (row-wise 8-bit: d codes + fp32 scale and offset, padded to 16)."""
    if cfg.table_dtype == "u8row":
        return (cfg.d + 8 + 15) // 16 * 16
    return cfg.d * (4 if cfg.table_dtype == "f32" else 2)


def quantizer():
    """The library's row-wise 8-bit quantiser, for building uint8 tables on the device."""
    import embedding_bags_dot_b200 as E
    return lambda src, dst: E.dlrm_quantize_rows_u8(src, dst)


def algorithmic_bytes(cfg, batch) -> int:
    """Bytes the fused gather + interaction must move for one batch."""
    es_o = 4 if cfg.mlp_dtype == "f32" else 2
    rows = int(batch.indices.size) * table_row_bytes(cfg)
    return rows + 4 * batch.indices.size + 4 * (cfg.K * cfg.B + 1) + 4 * cfg.B * cfg.d + es_o * cfg.B * cfg.concat_width


def fused_kernel_name(cfg) -> str:
    """The gather + interaction kernel the library dispatches to for this workload."""
    if cfg.interaction == "cat":
        return "embbag_cat_bulk_kernel (dlrm_embbag_cat_fwd)"
    if cfg.table_dtype in ("bf16", "u8row") and cfg.K + (4 if cfg.table_dtype == "u8row" else 2) <= 64:
        return "embbag_interact_mma_kernel (dlrm_embbag_interact_fwd)"
    if cfg.table_dtype == "bf16" and cfg.mlp_dtype == "bf16" and cfg.d in (64, 128) and cfg.K <= 128:
        return "embbag_interact_wide_kernel (dlrm_embbag_interact_fwd)"
    if cfg.table_dtype == "f32" and cfg.d in (16, 32, 64, 128):
        return "embbag_interact_f32_kernel (dlrm_embbag_interact_fwd)"
    return "embbag_interact_kernel (dlrm_embbag_interact_fwd)"


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


# the files the fused gather + interaction kernel is compiled from (its traffic record is keyed on them)
K2_SOURCES = ("embedding_bags_dot_b200/csrc/embbag_mma.cu", "embedding_bags_dot_b200/csrc/async_copy.cuh",
              "embedding_bags_dot_b200/csrc/common.cuh")
CAT_SOURCES = ("embedding_bags_dot_b200/csrc/embbag_cat_bulk.cu", "embedding_bags_dot_b200/csrc/async_copy.cuh",
               "embedding_bags_dot_b200/csrc/common.cuh")
# full-size DRAM traffic records of the dominant kernel, per workload: (summary, the kernel's sources)
TRAFFIC = {"large": ("profiles/embbag_interact_large_traffic.json", K2_SOURCES),
           "large-cat": ("profiles/embbag_cat_large_traffic.json", CAT_SOURCES)}


def source_hash(src_rels) -> str:
    """sha256 over the concatenated bytes of the kernel's source files, in the given order."""
    h = hashlib.sha256()
    for rel in src_rels:
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()


def kernel_traffic(path_rel: str, src_rels):
    """dram bytes per launch from a committed ncu summary, if it was taken on the current kernel source."""
    p = os.path.join(ROOT, path_rel)
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    if j.get("source_sha256") != source_hash(src_rels):
        return None
    return j.get("dram_bytes_per_launch_full")


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples during the timed region."""
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (FileNotFoundError, OSError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], 0.0, set()
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = max(mx, float(parts[1]))
            except ValueError:
                continue
            for name, v in zip(self.REASONS, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- oracle (CPU baseline)

def oracle_rate(cfg, batch, n_samples: int, seed: int = 0):
    """samples/s of the fp64 oracle on n_samples drawn from the batch (excluding input prep): the forward, or for
    a training workload the forward and backward (loss, MLP and row gradients; the update itself is negligible)."""
    from oracle import oracle as O
    rng = np.random.default_rng(seed)
    samples = np.sort(rng.choice(cfg.B, size=min(n_samples, cfg.B), replace=False))
    Bs, dense, offs, idx, labels, rows, used = O.sub_batch(cfg, batch, samples)
    model = O.model_for_rows(cfg, used)
    t0 = time.perf_counter()
    if cfg.training:
        O.train_grads(model, dense, offs, idx, labels)
    else:
        (O.forward_cat if cfg.interaction == "cat" else O.forward)(model, dense, offs, idx)
    dt = time.perf_counter() - t0
    return Bs / dt, dt, O.threads(), Bs


def oracle_what(cfg) -> str:
    return "fp64 forward + backward" if cfg.training else "fp64 forward"


def cpu_baseline(cfg, batch, seconds: float) -> dict:
    """The oracle on all host cores and on one core, on bounded random samples of the batch."""
    rate, dt, cores, used = calibrated_oracle(cfg, batch, seconds)
    r1, dt1, c1, used1 = oracle_on_one_core(cfg, batch, seconds / 3)
    return {"value": rate, "unit": "samples/s", "cores": cores, "kind": "oracle",
            "sample": f"{used} random samples of batch 0, {oracle_what(cfg)} in {dt:.1f} s",
            "cpu_model": cpu_model(),
            "one_core": {"value": r1, "cores": c1,
                         "sample": f"{used1} random samples of batch 0, {oracle_what(cfg)} in {dt1:.1f} s"}}


def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_on_one_core(cfg, batch, target_s: float):
    """The same oracle measurement with its OpenMP pool cut to one thread."""
    from oracle import oracle as O
    lib = O.load()
    n_all = O.threads()
    lib.oracle_set_threads(1)
    try:
        rate, dt, cores, used = calibrated_oracle(cfg, batch, target_s)
    finally:
        lib.oracle_set_threads(n_all)
    return rate, dt, cores, used


def calibrated_oracle(cfg, batch, target_s: float):
    """The oracle on a sample sized to take about target_s: grown at most 8x per measurement, so that a rate
    that falls with the sample size (the training oracle's) cannot overshoot the time budget."""
    n = 64
    rate, dt, cores, used = oracle_rate(cfg, batch, n)
    seed = 1
    while dt < target_s / 2 and n < cfg.B:
        n = int(min(cfg.B, 8 * n, max(n + 1, rate * target_s)))
        rate, dt, cores, used = oracle_rate(cfg, batch, n, seed=seed)
        seed += 1
    return rate, dt, cores, used


def run_reference(args, cfg, rank):
    if rank != 0:
        return 0
    batch = gen.make_batches(cfg, (0,))[0]
    # size one step at 1/(steps + warmup) of ~2 minutes of CPU time, whatever the step count
    budget = 120.0 / max(1, args.steps + args.warmup)
    rate0, _, cores, _ = oracle_rate(cfg, batch, 32)
    n = int(min(cfg.B, max(16, rate0 * budget)))
    for w in range(args.warmup):
        oracle_rate(cfg, batch, n, seed=100 + w)
    total_s, total_n = 0.0, 0
    for s in range(args.steps):
        r, dt, cores, used = oracle_rate(cfg, batch, n, seed=s)
        total_s += dt
        total_n += used
    value = total_n / total_s
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "samples/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": workload_desc(cfg), "global_batch": cfg.B, "parallelism": "cpu-oracle"},
           "cpu_baseline": {"value": value, "unit": "samples/s", "cores": cores, "kind": "oracle",
                            "sample": f"{n} random samples of batch 0 per step ({oracle_what(cfg)}, host cores)",
                            "cpu_model": cpu_model()},
           "e2e": {"value": value, "unit": "samples/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


METRIC = "DLRM samples/s on 1 B200; EmbeddingBag+interaction HBM GB/s as % of peak"


# --------------------------------------------------------------------------- multi-rank plumbing (replicas)

def rank_batch_ids(rank: int) -> tuple:
    """Each rank benchmarks its own pool of seeded batches (independent replicas, weak scaling)."""
    return tuple(rank * POOL + j for j in range(POOL))


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest value over all ranks (the slowest rank's time bounds the whole job)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(samples_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job samples/s: every rank's samples over the slowest rank's time."""
    return samples_per_rank * world / (max_ms * 1e-3)


# --------------------------------------------------------------------------- GPU arm

def run_ours(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import embedding_bags_dot_b200 as E
    from synth import device as sd

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    E.lib()
    sd.build_fill()

    # model
    tables = sd.tables_on_device(cfg, device=dev, quantize=quantizer())
    T = E.Tables(tables, cfg.rows, cfg.d)
    bW, bb, bd = sd.mlp_on_device(cfg, "bottom", dev)
    tW, tb, td = sd.mlp_on_device(cfg, "top", dev)
    bot, top = E.MLP(bW, bb, bd), E.MLP(tW, tb, td)
    ws = E.alloc_workspace(E.dlrm_workspace_size(T, bot, top, cfg.B, 0), dev)

    # batch pool (independent per rank)
    ids = rank_batch_ids(rank)
    perms = {k: gen.table_permutation(cfg, k) for k in range(cfg.K)} if cfg.index.startswith("zipf") else None
    batches = gen.make_batches(cfg, ids, perms=perms)
    dev_b = [sd.batch_on_device(b, dev) for b in batches]
    host_b = [sd.batch_on_device(b, pin=True) for b in batches]
    algo_bytes = [algorithmic_bytes(cfg, b) for b in batches]
    pool_bytes = sum(sum(t.numel() * t.element_size() for t in d.values()) for d in dev_b)

    ldc = cfg.concat_ld
    out_t = sd.TORCH_DT[cfg.mlp_dtype]
    x_dense = torch.empty((cfg.B, cfg.d), dtype=torch.float32, device=dev)
    concat = torch.zeros((cfg.B, ldc), dtype=out_t, device=dev)
    y = torch.empty(cfg.B, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None):
        b = dev_b[i % POOL]
        if ev is not None:
            ev[0].record(stream)
        E.dlrm_mlp_fwd(bot, cfg.B, b["dense"], cfg.n_dense, x_dense, cfg.d, E.ACT_RELU, ws, stream)
        if ev is not None:
            ev[1].record(stream)
        if cfg.interaction == "cat":
            E.dlrm_embbag_cat_fwd(T, cfg.B, b["offsets"], b["indices"], x_dense, concat, ldc, cfg.mlp_dtype, ws, stream)
        else:
            E.dlrm_embbag_interact_fwd(T, cfg.B, b["offsets"], b["indices"], x_dense, concat, ldc, cfg.mlp_dtype, ws,
                                       stream)
        if ev is not None:
            ev[2].record(stream)
        E.dlrm_mlp_fwd(top, cfg.B, concat, ldc, y, 1, E.ACT_SIGMOID, ws, stream)
        if ev is not None:
            ev[3].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for i in range(args.warmup):
        step(i)
    st = E.dlrm_check_error(ws)
    if st[0] != 0:
        raise RuntimeError(f"device error record after warm-up: {st}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    barrier()
    clocks.start()
    n0 = E.dlrm_launch_count()
    for i in range(args.steps):
        step(i, evs[i])
    n1 = E.dlrm_launch_count()
    barrier()
    clk = clocks.stop()
    total_ms = evs[0][0].elapsed_time(evs[-1][3])
    k2_ms = [e[1].elapsed_time(e[2]) for e in evs]
    bot_ms = [e[0].elapsed_time(e[1]) for e in evs]
    top_ms = [e[2].elapsed_time(e[3]) for e in evs]
    st = E.dlrm_check_error(ws)
    if st[0] != 0:
        raise RuntimeError(f"device error record after timing: {st}")

    # End to end through dlrm_forward with host buffers: each step copies its batch from pinned host
    # memory (copy stream, two staging slots so the next batch's copy overlaps this step's forward)
    # and copies y_hat back.
    cstream = torch.cuda.Stream(dev)
    ostream = torch.cuda.Stream(dev)     # y_hat device -> host, overlapping the next step's forward
    in_keys = ("dense", "offsets", "indices")
    maxn = {k: max(hb[k].numel() for hb in host_b) for k in in_keys}
    slots = [{k: torch.empty(maxn[k], dtype=host_b[0][k].dtype, device=dev) for k in maxn} for _ in range(2)]
    y_dev = [torch.empty(cfg.B, dtype=torch.float32, device=dev) for _ in range(2)]
    y_host = [torch.empty(cfg.B, dtype=torch.float32).pin_memory() for _ in range(2)]
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]
    read_back = [torch.cuda.Event() for _ in range(2)]
    for ev in consumed + read_back:
        ev.record(stream)

    fwd = E.dlrm_forward_cat if cfg.interaction == "cat" else E.dlrm_forward

    def e2e_step(i):
        sl, hb = i & 1, host_b[i % POOL]
        cstream.wait_event(consumed[sl])
        with torch.cuda.stream(cstream):
            for k in in_keys:
                slots[sl][k][:hb[k].numel()].copy_(hb[k].view(-1), non_blocking=True)
        copied[sl].record(cstream)
        stream.wait_event(copied[sl])
        stream.wait_event(read_back[sl])          # y_dev[sl] of step i-2 has been copied out
        n = hb["indices"].numel()
        fwd(T, bot, top, cfg.B, slots[sl]["dense"], slots[sl]["offsets"], slots[sl]["indices"][:n],
            y_dev[sl], ws, stream)
        consumed[sl].record(stream)
        ostream.wait_event(consumed[sl])
        with torch.cuda.stream(ostream):
            y_host[sl].copy_(y_dev[sl], non_blocking=True)
        read_back[sl].record(ostream)

    for i in range(args.warmup):
        e2e_step(i)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cstream.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_stream(ostream)                   # the last step's y_hat is on the host
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    h2d = int(np.mean([sum(hb[k].numel() * hb[k].element_size() for k in in_keys) for hb in host_b]))
    d2h = cfg.B * 4

    # max over ranks
    total_ms = max_over_ranks(total_ms, world, dev)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    k2_avg = max_over_ranks(float(np.mean(k2_ms)), world, dev)
    peak_hbm, peak_bf16, peak_kind = read_peaks()
    avg_algo = float(np.mean([algo_bytes[i % POOL] for i in range(args.steps)]))
    achieved = avg_algo / (k2_avg * 1e-3) / 1e9
    samples = cfg.B * args.steps * world
    value = aggregate_rate(cfg.B * args.steps, world, total_ms)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, batches[0], args.cpu_seconds)

    if rank == 0:
        traffic = kernel_traffic(*TRAFFIC[cfg.name]) if cfg.name in TRAFFIC else None
        out = {
            "metric": METRIC, "value": value, "unit": "samples/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": cfg.table_dtype, "data": "synthetic",
            "config": {"workload": workload_desc(cfg), "global_batch": cfg.B * world, "per_gpu_batch": cfg.B,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": f"no flush: tables {sum(cfg.rows) * table_row_bytes(cfg) / 1e9:.1f} GB "
                             f"and a {POOL}-batch pool of {pool_bytes / 1e6:.0f} MB exceed the {L2_BYTES >> 20} MB L2"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak_hbm, "unit": "GB/s",
                         "frac": achieved / peak_hbm, "traffic": traffic, "peak_kind": peak_kind,
                         "kernel": fused_kernel_name(cfg),
                         "algorithmic_bytes_per_launch": avg_algo, "avg_launch_ms": k2_avg},
            "kernels_ms_per_step": {"bottom_mlp": float(np.mean(bot_ms)), "embbag_interact": float(np.mean(k2_ms)),
                                    "top_mlp": float(np.mean(top_ms))},
            "cpu_baseline": cpu,
            "e2e": {"value": aggregate_rate(cfg.B * args.steps, world, e2e_ms), "unit": "samples/s",
                    "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps},
            "gpu_launches": int(n1 - n0),
            "clocks": clk,
        }
        print(json.dumps(out), flush=True)
    return 0


def run_train(args, cfg, rank, world, local_rank):
    """Training workload: a step is dlrm_backward (forward with saved activations, BCE, backward, row sort)
    plus dlrm_sparse_sgd (touched rows and MLP parameters) on one batch."""
    import torch
    import torch.distributed as dist

    import embedding_bags_dot_b200 as E
    from synth import device as sd

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    E.lib()
    sd.build_fill()
    tables = sd.tables_on_device(cfg, device=dev, quantize=quantizer())
    T = E.Tables(tables, cfg.rows, cfg.d)
    bot = E.MLP(*sd.mlp_on_device(cfg, "bottom", dev))
    top = E.MLP(*sd.mlp_on_device(cfg, "top", dev))
    ws = E.alloc_workspace(E.dlrm_workspace_size(T, bot, top, cfg.B, 1), dev)
    ids = rank_batch_ids(rank)
    perms = {k: gen.table_permutation(cfg, k) for k in range(cfg.K)} if cfg.index.startswith("zipf") else None
    batches = gen.make_batches(cfg, ids, perms=perms)
    dev_b = [sd.batch_on_device(b, dev) for b in batches]
    nnz_max = max(b.indices.size for b in batches)
    grads = torch.zeros(max(E.dlrm_grads_size(T, bot, top, cfg.B, int(b.indices.size)) for b in batches),
                        dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    loss = torch.zeros(1, device=dev)

    def step(i, ev=None):
        b = dev_b[i % POOL]
        nnz = int(b["indices"].numel())
        if ev is not None:
            ev[0].record(stream)
        E.dlrm_backward(T, bot, top, cfg.B, b["dense"], b["offsets"], b["indices"], b["labels"], grads, ws, loss=loss,
                        stream=stream)
        if ev is not None:
            ev[1].record(stream)
        E.dlrm_sparse_sgd(T, bot, top, cfg.B, nnz, cfg.lr, grads, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for i in range(args.warmup):
        step(i)
    st = E.dlrm_check_error(ws)
    if st[0] != 0:
        raise RuntimeError(f"device error record after warm-up: {st}")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    n0 = E.dlrm_launch_count()
    for i in range(args.steps):
        step(i, evs[i])
    n1 = E.dlrm_launch_count()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    total_ms = max_over_ranks(evs[0][0].elapsed_time(evs[-1][2]), world, dev)
    bwd = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    sgd = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    # roofline of the dominant kernel, the 3xTF32 GEMM, on the largest layer of the step (top layer 2: the
    # batch x 1024 x 1024 forward product), timed alone right after the step loop
    I, J, R = cfg.B, cfg.top[2], cfg.top[1]
    gemm_ms = max_over_ranks(time_tf32x3(I, J, R, dev, stream), world, dev)
    _, peak_bf16, peak_kind = read_peaks()
    peak_tf32 = peak_bf16 * TF32_PER_BF16
    tensor_tflops = 3 * 2.0 * I * J * R / (gemm_ms * 1e-3) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, batches[0], args.cpu_seconds)
    if rank == 0:
        out = {"metric": "DLRM training samples/s on 1 B200 (forward + backward + sparse SGD)",
               "value": aggregate_rate(cfg.B * args.steps, world, total_ms), "unit": "samples/s", "n_gpus": world,
               "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
               "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
               "config": {"workload": workload_desc(cfg), "global_batch": cfg.B * world, "lr": cfg.lr,
                          "nnz_max": nnz_max},
               "kernels_ms_per_step": {"dlrm_backward": bwd, "dlrm_sparse_sgd": sgd},
               "roofline": {"bound": "tensor", "achieved": tensor_tflops, "peak": peak_tf32, "unit": "TFLOP/s",
                            "frac": tensor_tflops / peak_tf32, "traffic": None,
                            "peak_kind": f"{peak_kind} bf16 burst x {TF32_PER_BF16:.3f} (nominal TF32:BF16)",
                            "kernel": "gemm3x_kernel (dlrm_gemm_tf32x3)",
                            "shape": f"{I}x{J}x{R} K-major x K-major",
                            "flops_per_launch": "3 TF32 products x 2*I*J*R", "avg_launch_ms": gemm_ms,
                            "fp32_equiv_tflops": 2.0 * I * J * R / (gemm_ms * 1e-3) / 1e12},
               "cpu_baseline": cpu, "loss_last": float(loss.item()), "gpu_launches": int(n1 - n0), "clocks": clk}
        print(json.dumps(out), flush=True)
    return 0


TF32_PER_BF16 = 1.1 / 2.25   # nominal dense TF32 : BF16 tensor rate of B200


def time_tf32x3(I, J, R, dev, stream, reps=10, warmup=3):
    """Average launch time (ms) of the 3xTF32 GEMM kernel alone (dlrm_gemm_tf32x3, operands already in pair form,
    A [I][R] and B [J][R] K-major) on the given stream, CUDA events around each launch."""
    import torch
    import embedding_bags_dot_b200 as E
    g = torch.Generator(device=dev).manual_seed(7)
    A = torch.randn((I, R), device=dev, generator=g)
    B = torch.randn((J, R), device=dev, generator=g) / R ** 0.5
    Ah, Al, Bh, Bl = torch.empty_like(A), torch.empty_like(A), torch.empty_like(B), torch.empty_like(B)
    E.dlrm_tf32_split(I, R, A, R, Ah, Al, R, stream=stream)
    E.dlrm_tf32_split(J, R, B, R, Bh, Bl, R, stream=stream)
    del A, B
    C = torch.empty((I, J), device=dev)
    ws = E.alloc_workspace(E.dlrm_gemm_tf32x3_workspace_size(I, J, R), dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for _ in range(warmup):
        E.dlrm_gemm_tf32x3(I, J, R, Ah, Al, R, False, Bh, Bl, R, False, C, J, ws, stream=stream)
    torch.cuda.synchronize(dev)
    for a, b in ev:
        a.record(stream)
        E.dlrm_gemm_tf32x3(I, J, R, Ah, Al, R, False, Bh, Bl, R, False, C, J, ws, stream=stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    st = E.dlrm_check_error(ws)
    if st[0] != 0:
        raise RuntimeError(f"device error record after the GEMM timing: {st}")
    return float(np.mean([a.elapsed_time(b) for a, b in ev]))


def run_latency(args, cfg, rank, world, local_rank):
    """Latency-bounded inference: forward latency and throughput against batch size, and the
    aggregate throughput of several streams serving small batches side by side (batching and
    co-location, as the companion paper's CPU study measures them)."""
    import torch

    import embedding_bags_dot_b200 as E
    from synth import device as sd
    from synth import shrink

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    E.lib()
    sd.build_fill()
    T = E.Tables(sd.tables_on_device(cfg, device=dev, quantize=quantizer()), cfg.rows, cfg.d)
    bot = E.MLP(*sd.mlp_on_device(cfg, "bottom", dev))
    top = E.MLP(*sd.mlp_on_device(cfg, "top", dev))
    perms = {k: gen.table_permutation(cfg, k) for k in range(cfg.K)} if cfg.index.startswith("zipf") else None
    sizes = [b for b in (1, 8, 64, 256, 1024, 4096, 16384, 65536) if b <= cfg.B]
    rows = []
    for B in sizes:
        c = shrink(cfg, B=B)
        bt = sd.batch_on_device(gen.make_batches(c, (rank * 100 + 1,), perms=perms)[0], dev)
        ws = E.alloc_workspace(E.dlrm_workspace_size(T, bot, top, B, 0), dev)
        y = torch.empty(B, dtype=torch.float32, device=dev)
        st = torch.cuda.current_stream(dev)
        for _ in range(args.warmup):
            E.dlrm_forward(T, bot, top, B, bt["dense"], bt["offsets"], bt["indices"], y, ws, st)
        ms = []
        for _ in range(max(args.steps, 20)):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            E.dlrm_forward(T, bot, top, B, bt["dense"], bt["offsets"], bt["indices"], y, ws, st)
            e1.record(st)
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        ms.sort()
        med, p99 = ms[len(ms) // 2], ms[min(len(ms) - 1, int(0.99 * len(ms)))]
        row = {"batch": B, "latency_ms_p50": med, "latency_ms_p99": p99, "samples_per_s": B / (med * 1e-3)}
        # the same forward captured once in a CUDA graph and replayed: no per-call host work (argument checks,
        # tensor-map encoding, launches) between the events
        try:
            g = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(dev)
            side.wait_stream(st)
            with torch.cuda.stream(side):
                E.dlrm_forward(T, bot, top, B, bt["dense"], bt["offsets"], bt["indices"], y, ws, side)
            torch.cuda.synchronize(dev)
            with torch.cuda.graph(g):
                cs = torch.cuda.current_stream(dev)
                E.dlrm_forward(T, bot, top, B, bt["dense"], bt["offsets"], bt["indices"], y, ws, cs)
            for _ in range(args.warmup):
                g.replay()
            gms = []
            for _ in range(max(args.steps, 20)):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(st)
                g.replay()
                e1.record(st)
                e1.synchronize()
                gms.append(e0.elapsed_time(e1))
            gms.sort()
            row["graph_latency_ms_p50"] = gms[len(gms) // 2]
            row["graph_latency_ms_p99"] = gms[min(len(gms) - 1, int(0.99 * len(gms)))]
            del g
        except Exception as exc:  # report, keep the eager numbers
            row["graph_error"] = str(exc)[:200]
        rows.append(row)
    # co-location: S streams, each serving its own small batches
    coloc = []
    Bc = min(256, cfg.B)
    c = shrink(cfg, B=Bc)
    bts = [sd.batch_on_device(b, dev) for b in gen.make_batches(c, tuple(rank * 100 + 10 + j for j in range(4)),
                                                                perms=perms)]
    for S in (1, 2, 4):
        streams = [torch.cuda.Stream(dev) for _ in range(S)]
        wss = [E.alloc_workspace(E.dlrm_workspace_size(T, bot, top, Bc, 0), dev) for _ in range(S)]
        ys = [torch.empty(Bc, dtype=torch.float32, device=dev) for _ in range(S)]
        n_iter = max(args.steps, 20)

        def burst():
            for it in range(n_iter):
                for j in range(S):
                    b = bts[j]
                    E.dlrm_forward(T, bot, top, Bc, b["dense"], b["offsets"], b["indices"], ys[j], wss[j], streams[j])

        burst()
        torch.cuda.synchronize(dev)
        start = torch.cuda.Event(enable_timing=True)
        start.record(torch.cuda.current_stream(dev))
        for sj in streams:
            sj.wait_event(start)
        burst()
        ends = [torch.cuda.Event(enable_timing=True) for _ in streams]
        for e, sj in zip(ends, streams):
            e.record(sj)
        torch.cuda.synchronize(dev)
        dt = max(start.elapsed_time(e) for e in ends) * 1e-3
        coloc.append({"streams": S, "batch": Bc, "samples_per_s": S * n_iter * Bc / dt,
                      "ms_per_round": 1e3 * dt / n_iter})
    if rank == 0:
        print(json.dumps({"metric": "DLRM inference latency and throughput vs batch size on 1 B200",
                          "unit": "ms", "higher_is_better": False, "data": "synthetic",
                          "config": {"workload": workload_desc(cfg)}, "latency": rows, "colocation": coloc}),
              flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 1000 for a forward workload, 100 for training, 20 for the "
                         "reference arm and --latency; long enough for several clock samples)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="large", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None, help="smaller batch (profiling captures only)")
    ap.add_argument("--rows-cap", type=int, default=None, help="cap table rows (profiling captures only)")
    ap.add_argument("--latency", action="store_true", help="latency vs batch size and co-located streams")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = CONFIGS[args.workload]
    if args.steps is None:
        args.steps = 20 if args.impl == "reference" or args.latency else (100 if cfg.training else 1000)
    if args.steps < 1:
        ap.error("--steps must be >= 1")
    if args.batch or args.rows_cap:
        from synth import shrink
        cfg = shrink(cfg, B=args.batch, rows_cap=args.rows_cap, name=f"{cfg.name}-profile")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, cfg, rank)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.latency:
            return run_latency(args, cfg, rank, world, local_rank)
        if cfg.training:
            return run_train(args, cfg, rank, world, local_rank)
        return run_ours(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
