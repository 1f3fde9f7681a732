#!/usr/bin/env python
"""Sparse GQA benchmark on B200: prefill tokens/s at 128K (B=8, k=4096), decode tok/s at 1M.

One step is one pass of the whole layer (block-key compression, per-group block selection,
gated attention over the selected tokens) over one 131072-token sequence per GPU, inputs
resident in HBM (q, gate and out alone are 3.2 GB, far above the 126 MB L2, so no flush is
needed between steps). Launch:

    python bench.py [--gpus 1] [--steps 5] [--warmup 3]
    python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N ...
        (N > 1: the 128K sequence split over the GPUs by query, K/V/k_idx all-gathered over NCCL;
         decode: the 32 sequences split over the GPUs)
    python bench.py --impl reference ...   (the fp64 CPU oracle on a bounded sample, host cores)

Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from sgqa_inputs import CONFIGS, DECODE_NEW, gen_rows  # noqa: E402

METRIC = "Sparse GQA prefill tokens/s at 128K (B=8,k=4096); decode tok/s at 1M ctx"
CLOCK_FIELDS = ["pci.bus_id", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
                "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
                "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]


# DRAM bytes per stage call (dram__bytes_read.sum + dram__bytes_write.sum summed over the call's
# launches of the stage's kernels) from ncu captures, keyed by (stage, workload), each with the
# SHA-256 (first 16 hex digits) of the kernels' source file at capture time: an entry is reported
# only while that source is unchanged, else the traffic is null. The figures and the commands
# that produced them are under profiles/.
NCU_TRAFFIC: dict = {
    # profiles/traffic_prefill128k_decode1m.md, the bench's own 128K / 1M workloads
    ("attend", "128k"): (6508516608 + 1068875008, "0ae683a6e388e866"),   # one attend_tc launch
    ("select", "128k"): (96827136 + 350853632 + 311874560 + 824761856, "4c4c0517e456e378"),  # 4 select_tc + 4 sel_from_bits
    ("decode_scores", "decode_1m"): (1074967296 + 252742400, "0669c7900a2898e8"),
    ("decode_select", "decode_1m"): (45581824 + 512, "cc7074bb7dae8bdd"),
    ("decode_attend", "decode_1m"): (1072768256 + 274176, "f4009ea09891d2e4"),
}
STAGE_SOURCES = {"compress": "compress.cu", "select": "select_tc.cu", "attend": "attend_tc.cu",
                 "decode_scores": "decode_scores_tc.cu", "decode_select": "decode.cu",
                 "decode_attend": "decode_attend.cu"}


def source_sha(stage: str) -> str | None:
    import hashlib
    p = os.path.join(ROOT, "block_sparse_long_kbar_b200", "csrc", STAGE_SOURCES.get(stage, ""))
    if not os.path.isfile(p):
        return None
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def measured_traffic(stage: str, workload: str):
    e = NCU_TRAFFIC.get((stage, workload))
    if e is None or e[1] != source_sha(stage):
        return None
    return e[0]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "sm_max_mhz": d.get("sm_max_mhz", 1965.0),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
            "source": "fallback"}


# ---- analytic work counts (the definition's, not the kernels') -------------------------------

def work_counts(cfg):
    """Scored candidates, attended (query, group, token) visits and byte streams of one pass."""
    T, B, Kb = cfg.T, cfg.B, cfg.Kb
    t = np.arange(T, dtype=np.int64)
    c = t // B
    scored = int(c.sum()) * cfg.G * cfg.batch
    nsel = np.minimum(Kb, c + 1)
    visits_per_t = (nsel - 1) * B + (t % B) + 1
    visits = int(visits_per_t.sum()) * cfg.G * cfg.batch
    R = cfg.Hq // cfg.G
    nblk = T // B
    return {
        "scored": scored,
        "index_flops": 2 * cfg.d_idx * scored,
        "visits": visits,
        "attn_flops": 4 * cfg.d * R * visits,
        "gather_bytes": visits * 2 * cfg.d * 2,
        "qgo_bytes": 3 * cfg.batch * T * cfg.Hq * cfg.d * 2,
        "sel_bytes": cfg.batch * T * cfg.G * Kb * 4,
        "kv_bytes": 2 * cfg.batch * T * cfg.G * cfg.d * 2,
        "compress_bytes": cfg.batch * T * cfg.d_idx * 2 + cfg.batch * nblk * cfg.d_idx * 4,
    }


# Per-key instruction counts of the select kernel's epilogue (select_tc.cu), per pass over the
# scored candidates. The histogram passes work on the raw float bits: the first spends about 4
# thread-instructions per key (+0.0 add, top byte, bin address, shared reduction), a later one
# about 6 (+0.0 add, xor with the prefix, shift, min with the spare slot, address, reduction); the
# emit pass about 6 (two raw-bit compares, two bit updates, the bucket offset) plus a bitmap store
# per 32 keys; the tile's TMEM load adds 2 per key per pass. A typical 128K row (topic-clustered
# scores) resolves its threshold bucket after 2 histogram passes: the first isolates its topic's
# blocks, the second leaves a bucket of a few keys, collected in the emit pass.
SELECT_INSTR_PER_KEY = {"hist_first": 4 + 2, "hist_next": 6 + 2, "emit": 6 + 2}
SELECT_PASSES = {"hist_first": 1, "hist_next": 1, "emit": 1}


def select_ranges(cfg, nq: int) -> int:
    """Query ranges K2 runs in for nq query rows: bitmap rows of 4 words per 128 blocks, ranges of
    whole 128-query multiples within a 256 MiB bitmap budget (api.cu, select_bits_dims)."""
    nblk = cfg.T // cfg.B
    per_q = cfg.batch * cfg.G * 4 * ((nblk + 127) // 128) * 4
    q = max(128, (256 << 20) // per_q // 128 * 128) if per_q else nq
    q = min(q, cfg.T)
    return (nq + q - 1) // q


def forward_launches(cfg, nq: int) -> int:
    """Library kernel launches of one sgqa_forward(_rows) call over nq query rows: the block means,
    K2 and its list expansion per query range, the row plan (signature + 3 radix passes of 3
    kernels) and the attention."""
    return 1 + 2 * select_ranges(cfg, nq) + 10 + 1


def decode_launches(cfg, n_new: int, cache_len: int, fp8: bool) -> int:
    """Library kernel launches of one decode step (api.cu, sgqa_decode): the appends (K and V
    quantized for FP8 caches, k_idx), the block means when the new rows complete a block, K4, K5,
    the union, K6 and, when K6 splits a (sequence, group), the merge. K6 takes one wave of
    148 x (1 CTA per SM for FP8 caches, 2 for bf16) CTAs, split over the (sequence, group) units
    up to the union's 128-token tiles (decode_attend.cu, decode_attend_splits)."""
    appends = 3
    compress = 1 if (cache_len + n_new) // cfg.B > cache_len // cfg.B else 0
    units = cfg.batch * cfg.G
    max_tiles = -(-(n_new * cfg.Kb) // (128 // cfg.B))
    splits = min(max(1, 148 * (1 if fp8 else 2) // units), max_tiles)
    return appends + compress + 4 + (1 if splits > 1 else 0)


def select_alu_model(wc, sm_mhz):
    """Time the select's per-key epilogue work needs at full issue rate (148 SMs x 4 schedulers x
    32 lanes x clock): a kernel-specific ceiling, reported beside the tensor roofline."""
    instr = wc["scored"] * sum(SELECT_INSTR_PER_KEY[p] * SELECT_PASSES[p] for p in SELECT_PASSES)
    rate = 148 * 4 * 32 * sm_mhz * 1e6
    return {"thread_instructions": instr, "issue_rate_per_s": rate, "min_ms": instr / rate * 1e3,
            "model": "per-key instructions x passes (histogram 2, emit 1) / SM issue rate"}


# ---- clocks sampled during the timed region -------------------------------------------------

class ClockSampler:
    def __init__(self, bus_id: int | None):
        self.bus_id = bus_id
        self.f = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={','.join(CLOCK_FIELDS)}",
                                       "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        lines = open(self.f.name).read().strip().splitlines()
        os.unlink(self.f.name)
        sm, mx, reasons = [], [], set()
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < len(CLOCK_FIELDS):
                continue
            try:
                bus = int(f[0].split(":")[1], 16)
            except (IndexError, ValueError):
                bus = None
            if self.bus_id is not None and bus is not None and bus != self.bus_id:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names[1:], f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---- distributed plumbing --------------------------------------------------------------------

def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The step time every rank reports is the slowest rank's (weak scaling: one sequence per rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens(cfg, world: int) -> int:
    """Tokens one timed step processes across the job: every rank runs its own sequence(s)."""
    return world * cfg.batch * cfg.T


# ---- the CPU oracle on a bounded sample (cpu_baseline and the reference arm) ------------------

def oracle_inputs_host(cfg, rows):
    """Host bf16 inputs for the oracle: whole k, v, k_idx of sequence 0, the sampled rows' q,
    q_idx, gate (made by the shared seeded generator on the host)."""
    b = 0
    t_all = np.arange(cfg.T)
    full = {}
    for n in ("k", "v", "k_idx"):
        parts = [gen_rows(cfg, n, b, t_all[i:i + 8192]) for i in range(0, cfg.T, 8192)]
        full[n] = np.concatenate(parts).reshape((1, cfg.T, -1))
    ts = rows[:, 1]
    part = {n: gen_rows(cfg, n, b, ts) for n in ("q", "q_idx", "gate")}
    return full, part


def oracle_sample_time(cfg, stride, full, part, rows):
    import oracle
    dm = oracle.dims(1, cfg.T, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    t0 = time.perf_counter()
    kbar = oracle.compress(dm, full["k_idx"])
    sel, _, _ = oracle.select(dm, kbar, rows, part["q_idx"])
    oracle.attend(dm, rows, part["q"], full["k"], full["v"], part["gate"], sel)
    return time.perf_counter() - t0


def to_host(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def sample_rows_strided(cfg, stride, offset=0):
    ts = np.arange(offset % stride, cfg.T, stride, dtype=np.int32)
    return np.stack([np.zeros_like(ts), ts], axis=1)


# ---- our arm ---------------------------------------------------------------------------------

def run_ours(args, world, rank):
    import torch
    import block_sparse_long_kbar_b200 as sg
    from sgqa_inputs import gen_device
    cfg = CONFIGS[args.config]
    shape_of = lambda c, n, **kw: c.shape(n, **kw)
    peaks = load_peaks()
    dims = sg.sgqa_dims.of(cfg)
    s = torch.cuda.Stream()
    dev = {}
    for n in ("q", "k", "v", "gate", "q_idx", "k_idx"):
        dev[n] = torch.empty(shape_of(cfg, n), dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, dev[n])
    out = torch.empty(shape_of(cfg, "q"), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((cfg.batch, cfg.T, cfg.G, cfg.Kb), dtype=torch.int32, device="cuda")
    kbar = torch.empty((cfg.batch, cfg.T // cfg.B, cfg.d_idx), dtype=torch.float32, device="cuda")
    ws = sg.alloc_workspace(sg.sgqa_workspace_size(dims))
    sg.sgqa_reset_device_status(ws)
    torch.cuda.synchronize()

    def step():
        sg.sgqa_forward(dims, dev["q"], dev["k"], dev["v"], dev["q_idx"], dev["k_idx"], dev["gate"], out, ws,
                        sel_out=sel, stream=s)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    bus = getattr(torch.cuda.get_device_properties(torch.cuda.current_device()), "pci_bus_id", None)
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(bus)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(args.steps):
        step()
    e1.record(s)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    status = sg.sgqa_get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    tokens_step = job_tokens(cfg, world)
    value = tokens_step / (ms / 1e3)

    # per-stage times: the same kernels through the per-stage entry points, events on the launch stream
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    st = {"compress": [], "select": [], "attend": []}
    for _ in range(args.steps):
        ev[0].record(s)
        sg.sgqa_compress_keys(dims, dev["k_idx"], kbar, ws, stream=s)
        ev[1].record(s)
        sg.sgqa_select(dims, dev["q_idx"], kbar, sel, ws, stream=s)
        ev[2].record(s)
        sg.sgqa_attend(dims, dev["q"], dev["k"], dev["v"], dev["gate"], sel, out, ws, stream=s)
        ev[3].record(s)
        torch.cuda.synchronize()
        for i, k in enumerate(st):
            st[k].append(ev[i].elapsed_time(ev[i + 1]))
    stage_ms = {k: statistics.mean(v) for k, v in st.items()}
    wc = work_counts(cfg)
    sm_mhz = (clocks or {}).get("sm_mhz") or peaks["sm_max_mhz"]
    # Each stage is timed on its own (events around one launch), so the burst peaks apply.
    stage_roof = {
        "compress": {"bound": "hbm", "achieved": wc["compress_bytes"] / (stage_ms["compress"] / 1e3) / 1e9,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s"},
        # the indexer is a dense contraction: algorithmic flops (2 d_idx per scored candidate)
        # against the bf16 tensor peak
        "select": {"bound": "tensor", "achieved": wc["index_flops"] / (stage_ms["select"] / 1e3) / 1e12,
                   "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"},
        "attend": {"bound": "tensor", "achieved": wc["attn_flops"] / (stage_ms["attend"] / 1e3) / 1e12,
                   "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"},
    }
    for k, r in stage_roof.items():
        r["frac"] = r["achieved"] / r["peak"]
        r["ms"] = stage_ms[k]
        r["traffic"] = measured_traffic(k, cfg.name)
    # the select's own ceiling: its per-key epilogue work on the CUDA cores (a model of this
    # kernel, not of the definition): instructions per key and pass x keys x passes / issue rate
    stage_roof["select"]["alu_model"] = select_alu_model(wc, sm_mhz)
    dominant = max(stage_ms, key=stage_ms.get)
    roof = dict(stage_roof[dominant])
    roof.pop("ms")
    roof.pop("alu_model", None)
    roof["kernel"] = dominant
    roof["peak_source"] = f"{peaks['source']} (burst: the stage is timed on its own)"

    # end to end through the C ABI with host buffers: H2D of the step's inputs, D2H of its output
    host = {n: torch.empty(dev[n].shape, dtype=torch.bfloat16, pin_memory=True) for n in dev}
    for n in dev:
        host[n].copy_(dev[n])
    out_h = torch.empty(out.shape, dtype=torch.bfloat16, pin_memory=True)
    h2d = sum(t.numel() * 2 for t in host.values())
    d2h = out.numel() * 2
    torch.cuda.synchronize()

    # the host-buffer entry point: chunked copies in, compute, copies out, overlapped on three streams
    streams = (torch.cuda.Stream(), s, torch.cuda.Stream())
    dev_all = dict(dev, out=out)

    def e2e_step():
        sg.sgqa_forward_from_host(dims, host, dev_all, out_h, ws, chunks=32, streams=streams)

    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0.record(s)
    for _ in range(args.steps):
        e2e_step()
    e1.record(s)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)

    gather_gbs = wc["gather_bytes"] / (stage_ms["attend"] / 1e3) / 1e9
    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded topic-structured generator)",
        "config": {"workload": f"prefill {cfg.name}: batch {cfg.batch} per GPU, T={cfg.T}, Hq={cfg.Hq}, G={cfg.G}, "
                               f"d={cfg.d}, d_idx={cfg.d_idx}, B={cfg.B}, k={cfg.k}, topic span {cfg.span}, "
                               f"seed {cfg.seed}",
                   "global_batch": world * cfg.batch, "seq_len": cfg.T, "parallelism": f"dp{world} (one sequence per GPU)",
                   "l2": "inputs larger than L2 (q+gate+out 3.2 GB per step), no flush"},
        # per step: compress, select, the plan (signature + 3 radix passes of 3 kernels), attend
        "gpu_launches": forward_launches(cfg, cfg.T) * args.steps,
        "e2e": {"value": tokens_step / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "roofline": roof,
        "stages": stage_roof,
        "gather": {"per_query_kv_bytes": wc["gather_bytes"], "effective_gather_GBps": gather_gbs,
                   "compulsory_bytes": wc["kv_bytes"] + wc["qgo_bytes"] + wc["sel_bytes"]},
        "clocks": clocks,
    }
    cpu_in = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        # the bench's own output on a strided sample of rows, for the oracle check after the GPU work
        rows = sample_rows_strided(cfg, CPU_STRIDE)
        full = {n: to_host(dev[n][:1]) for n in ("k", "v", "k_idx")}
        ti = torch.from_numpy(rows[:, 1].astype(np.int64)).cuda()
        part = {n: to_host(dev[n][0].index_select(0, ti)).reshape(len(rows), -1) for n in ("q", "q_idx", "gate")}
        gpu_rows = {"sel": sel[0].index_select(0, ti).cpu().numpy(), "out": to_host(out[0].index_select(0, ti))}
        cpu_in = (rows, full, part, gpu_rows)
    # release the prefill buffers before the decode workload
    del dev, dev_all, out, sel, kbar, ws, host, out_h
    torch.cuda.empty_cache()
    if not args.no_decode:
        result["decode"] = run_decode(args, world, s)
        result["decode_fp8"] = run_decode_fp8(args, world, s)
    if not args.no_ablation and world == 1:
        result["ablation"] = run_ablation(args, world, s)
    if not args.no_backward and world == 1:
        result["backward"] = run_backward(args, world, s)
    if not args.no_swa:
        result["swa"] = run_swa(args, world, s)
    if cpu_in is not None:
        result["cpu_baseline"], result["errors"] = cpu_baseline(cfg, *cpu_in)
    return result


def run_sharded(args, world, rank):
    """N > 1: one 128K sequence split over the GPUs by query (zig-zag ranges), K, V and k_idx
    all-gathered over NCCL every step (each rank produces those of its own rows), then the layer
    for the rank's rows (sgqa_forward_rows). Strong scaling: the whole job is one sequence."""
    import torch
    import block_sparse_long_kbar_b200 as sg
    from block_sparse_long_kbar_b200.sharding import gather_sequence, prefill_rows, zigzag_ranges
    from sgqa_inputs import gen_device
    cfg = CONFIGS[args.config]
    dims = sg.sgqa_dims.of(cfg)
    s = torch.cuda.Stream()
    ranges = zigzag_ranges(cfg.T, world, rank)
    loc = {}
    for n in ("q", "gate", "q_idx", "k", "v", "k_idx"):
        loc[n] = []
        for t0, t1 in ranges:
            x = torch.empty(cfg.shape(n, T=t1 - t0), dtype=torch.bfloat16, device="cuda")
            gen_device(cfg, n, x, t0=t0, n_t=t1 - t0, dst_t0=0)
            loc[n].append(x)
    outs = [torch.empty_like(x) for x in loc["q"]]
    ws = sg.alloc_workspace(sg.sgqa_workspace_size(dims))
    sg.sgqa_reset_device_status(ws)
    torch.cuda.synchronize()

    def gather():
        return [gather_sequence(loc[n], world) for n in ("k", "v", "k_idx")]

    def step():
        k, v, k_idx = gather()
        prefill_rows(dims, ranges, loc["q"], loc["gate"], loc["q_idx"], k, v, k_idx, outs, ws, stream=s)

    with torch.cuda.stream(s):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    bus = getattr(torch.cuda.get_device_properties(torch.cuda.current_device()), "pci_bus_id", None)
    sampler = ClockSampler(bus)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(args.steps):
            step()
        e1.record(s)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    assert sg.sgqa_get_device_status(ws) == 0
    # the all-gather alone
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(args.steps):
            gather()
        e1.record(s)
    torch.cuda.synchronize()
    gather_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    # end to end: this rank's rows from pinned host buffers, the output back
    host = {n: [torch.empty(x.shape, dtype=torch.bfloat16, pin_memory=True).copy_(x) for x in loc[n]] for n in loc}
    out_h = [torch.empty(o.shape, dtype=torch.bfloat16, pin_memory=True) for o in outs]
    h2d = sum(x.numel() * 2 for xs in host.values() for x in xs)
    d2h = sum(o.numel() * 2 for o in outs)

    def e2e_step():
        for n in loc:
            for dst, src in zip(loc[n], host[n]):
                dst.copy_(src, non_blocking=True)
        step()
        for dst, src in zip(out_h, outs):
            dst.copy_(src, non_blocking=True)

    with torch.cuda.stream(s):
        e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e0.record(s)
        for _ in range(args.steps):
            e2e_step()
        e1.record(s)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    wc = work_counts(cfg)
    peaks = load_peaks()
    per_gpu_flops = (wc["attn_flops"] + wc["index_flops"]) / world
    result = {
        "metric": METRIC, "value": cfg.batch * cfg.T / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded topic-structured generator)",
        "config": {"workload": f"prefill {cfg.name}: batch {cfg.batch}, T={cfg.T}, Hq={cfg.Hq}, G={cfg.G}, "
                               f"d={cfg.d}, d_idx={cfg.d_idx}, B={cfg.B}, k={cfg.k}, topic span {cfg.span}, "
                               f"seed {cfg.seed}; queries split over {world} GPUs",
                   "global_batch": cfg.batch, "seq_len": cfg.T,
                   "parallelism": f"query-sharded x{world} (zig-zag ranges; all-gather of K, V, k_idx over NCCL)",
                   "l2": "inputs larger than L2, no flush"},
        "gpu_launches": sum(forward_launches(cfg, t1 - t0) for t0, t1 in ranges) * args.steps,
        "e2e": {"value": cfg.batch * cfg.T / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "roofline": {"bound": "tensor", "achieved": per_gpu_flops / (ms / 1e3) / 1e12, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": per_gpu_flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                     "traffic": None, "kernel": "whole step per GPU (indexer + attention flops / N)",
                     "peak_source": peaks["source"]},
        "allgather_ms": gather_ms,
        "clocks": clocks,
    }
    del loc, outs, ws, host, out_h
    torch.cuda.empty_cache()
    if not args.no_decode:
        result["decode"] = run_decode(args, world, s)
    return result


def run_decode(args, world, s):
    import torch
    import block_sparse_long_kbar_b200 as sg
    from sgqa_inputs import gen_device
    cfg = CONFIGS["decode_1m"]
    if world > 1:  # the 32 sequences split over the GPUs (data parallel, no exchange)
        cfg = cfg.replace(batch=cfg.batch // world)
    shape_of = lambda c, n, **kw: c.shape(n, **kw)
    n_new = DECODE_NEW
    cache_len = cfg.T
    T_cap = cache_len + cfg.B
    dims = sg.sgqa_dims(cfg.batch, T_cap, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    caches = {}
    for n in ("k", "v", "k_idx"):
        caches[n] = torch.zeros(shape_of(cfg, n, T=T_cap), dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, caches[n], t0=0, n_t=cache_len)
    kbar = torch.zeros((cfg.batch, T_cap // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(dims, caches["k_idx"], kbar, None)
    new = {}
    for n in ("q", "k", "v", "gate", "q_idx", "k_idx"):
        new[n] = torch.empty((cfg.batch, n_new) + shape_of(cfg, n)[2:], dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, new[n], t0=cache_len, n_t=n_new, dst_t0=0)
    out = torch.empty((cfg.batch, n_new, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
    ws = sg.alloc_workspace(sg.sgqa_decode_workspace_size(dims, n_new))
    sg.sgqa_reset_device_status(ws)
    torch.cuda.synchronize()

    def step():
        sg.sgqa_decode(dims, cache_len, n_new, caches["k"], caches["v"], caches["k_idx"], kbar, new["q"], new["k"],
                       new["v"], new["q_idx"], new["k_idx"], new["gate"], out, ws, stream=s)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = max(args.steps, 10)
    e0.record(s)
    for _ in range(steps):
        step()
    e1.record(s)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    assert sg.sgqa_get_device_status(ws) == 0
    toks = world * cfg.batch * n_new
    kbar_bytes = cfg.batch * (cache_len // cfg.B) * cfg.d_idx * 4
    visits = decode_visits(cfg, n_new, cache_len)
    gather = visits * 2 * cfg.d * 2
    res = {"metric": "decode query tokens/s at 1M context (32 seqs x 4 new tokens)", "value": toks / (ms / 1e3),
           "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
           "workload": f"decode: {cfg.batch} seqs per GPU x {n_new} new tokens after {cache_len} cached, Hq={cfg.Hq}, "
                       f"G={cfg.G}, d={cfg.d}, d_idx={cfg.d_idx}, B={cfg.B}, k={cfg.k}, span {cfg.span}, seed {cfg.seed}",
           "algorithmic_bytes": kbar_bytes + gather,
           "hbm_frac": (kbar_bytes + gather) / (ms / 1e3) / 1e9 / load_peaks()["hbm_gbs"],
           "kernel_traffic_bytes": {k: measured_traffic(k, "decode_1m")
                                    for k in ("decode_scores", "decode_select", "decode_attend")},
           "gpu_launches_per_step": decode_launches(cfg, n_new, cache_len, False)}
    del caches, kbar, new, out, ws
    torch.cuda.empty_cache()
    return res


def decode_visits(cfg, n_new, cache_len):
    """(query, group, token) visits of one decode step: every new token attends its k/B - 1 picked
    blocks (B tokens each) plus the tokens of its own block up to itself."""
    return cfg.batch * cfg.G * sum((cfg.Kb - 1) * cfg.B + (cache_len + i) % cfg.B + 1 for i in range(n_new))


def run_decode_fp8(args, world, s):
    """The same decode step over FP8 K/V caches (e4m3 codes + a power-of-two scale per (token,
    group) row, through sgqa_decode_fp8): the gathered cache bytes halve."""
    import torch
    import block_sparse_long_kbar_b200 as sg
    from sgqa_inputs import gen_device
    cfg = CONFIGS["decode_1m"]
    n_new = DECODE_NEW
    cache_len = cfg.T
    T_cap = cache_len + cfg.B
    dims = sg.sgqa_dims(cfg.batch, T_cap, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    c8 = {n: torch.zeros(cfg.shape(n, T=T_cap), dtype=torch.uint8, device="cuda") for n in ("k", "v")}
    csc = {n: torch.zeros((cfg.batch, T_cap, cfg.G), dtype=torch.float32, device="cuda") for n in ("k", "v")}
    chunk = 65536
    for t0 in range(0, cache_len, chunk):
        n = min(chunk, cache_len - t0)
        for name in ("k", "v"):
            tmp = torch.empty((cfg.batch, n, cfg.G, cfg.d), dtype=torch.bfloat16, device="cuda")
            gen_device(cfg, name, tmp, t0=t0, n_t=n, dst_t0=0)
            sg.sgqa_quantize_kv_fp8(dims, t0, n, tmp, c8[name], csc[name])
            del tmp
    kidx = torch.zeros(cfg.shape("k_idx", T=T_cap), dtype=torch.bfloat16, device="cuda")
    gen_device(cfg, "k_idx", kidx, t0=0, n_t=cache_len)
    kbar = torch.zeros((cfg.batch, T_cap // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(dims, kidx, kbar, None)
    new = {}
    for n in ("q", "k", "v", "gate", "q_idx", "k_idx"):
        new[n] = torch.empty((cfg.batch, n_new) + cfg.shape(n)[2:], dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, new[n], t0=cache_len, n_t=n_new, dst_t0=0)
    out = torch.empty((cfg.batch, n_new, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
    ws = sg.alloc_workspace(sg.sgqa_decode_workspace_size(dims, n_new))
    sg.sgqa_reset_device_status(ws)
    torch.cuda.synchronize()

    def step():
        sg.sgqa_decode_fp8(dims, cache_len, n_new, c8["k"], csc["k"], c8["v"], csc["v"], kidx, kbar, new["q"],
                           new["k"], new["v"], new["q_idx"], new["k_idx"], new["gate"], out, ws, stream=s)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = max(args.steps, 10)
    e0.record(s)
    for _ in range(steps):
        step()
    e1.record(s)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    assert sg.sgqa_get_device_status(ws) == 0
    toks = world * cfg.batch * n_new
    kbar_bytes = cfg.batch * (cache_len // cfg.B) * cfg.d_idx * 4
    visits = decode_visits(cfg, n_new, cache_len)
    gather = visits * 2 * (cfg.d + 4)  # codes + the row scale, K and V
    res = {"metric": "decode query tokens/s at 1M context, FP8 (e4m3) K/V caches (32 seqs x 4 new tokens)",
           "value": toks / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
           "workload": f"decode fp8: {cfg.batch} seqs x {n_new} new tokens after {cache_len} cached, Hq={cfg.Hq}, "
                       f"G={cfg.G}, d={cfg.d}, d_idx={cfg.d_idx}, B={cfg.B}, k={cfg.k}, span {cfg.span}, "
                       f"seed {cfg.seed}",
           "algorithmic_bytes": kbar_bytes + gather,
           "hbm_frac": (kbar_bytes + gather) / (ms / 1e3) / 1e9 / load_peaks()["hbm_gbs"],
           "gpu_launches_per_step": decode_launches(cfg, n_new, cache_len, True)}
    del c8, csc, kidx, kbar, new, out, ws
    torch.cuda.empty_cache()
    return res


def run_backward(args, world, s):
    """Gradients of the gated attention (dq, dk, dv, dgate, fp32) through the selection of the 128K
    prefill, via sgqa_attend_backward, inputs resident in HBM."""
    import torch
    import block_sparse_long_kbar_b200 as sg
    from sgqa_inputs import gen_device
    cfg = CONFIGS["128k"]
    dims = sg.sgqa_dims.of(cfg)
    dev = {}
    for n in ("q", "k", "v", "gate", "q_idx", "k_idx"):
        dev[n] = torch.empty(cfg.shape(n), dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, dev[n])
    out = torch.empty(cfg.shape("q"), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((cfg.batch, cfg.T, cfg.G, cfg.Kb), dtype=torch.int32, device="cuda")
    ws = sg.alloc_workspace(sg.sgqa_workspace_size(dims))
    sg.sgqa_reset_device_status(ws)
    sg.sgqa_forward(dims, dev["q"], dev["k"], dev["v"], dev["q_idx"], dev["k_idx"], dev["gate"], out, ws,
                    sel_out=sel, stream=s)
    del ws
    dy = torch.empty(cfg.shape("q"), dtype=torch.bfloat16, device="cuda")
    gen_device(cfg.replace(seed=cfg.seed + 1000), "q", dy)  # an independent N(0,1) output gradient
    grads = {n: torch.empty(cfg.shape("q" if n in ("dq", "dgate") else "k"), dtype=torch.float32, device="cuda")
             for n in ("dq", "dk", "dv", "dgate")}
    bws = sg.alloc_workspace(sg.sgqa_backward_workspace_size(dims))
    sg.sgqa_reset_device_status(bws)
    torch.cuda.synchronize()

    def step():
        sg.sgqa_attend_backward(dims, dev["q"], dev["k"], dev["v"], dev["gate"], sel, dy, grads["dq"], grads["dk"],
                                grads["dv"], grads["dgate"], bws, stream=s)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = 1  # a step takes seconds (CUDA-core kernels); one timed step after the warm-up
    e0.record(s)
    for _ in range(steps):
        step()
    e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    assert sg.sgqa_get_device_status(bws) == 0
    wc = work_counts(cfg)
    res = {"metric": "Sparse GQA backward (dq, dk, dv, dgate through the selection) tokens/s at 128K",
           "value": cfg.batch * cfg.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
           "workload": f"backward 128k: the 128K prefill's inputs and GPU selection, dout ~ N(0,1); fp32 gradients",
           "flops": 2 * wc["attn_flops"], "achieved_tflops": 2 * wc["attn_flops"] / (ms / 1e3) / 1e12,
           "note": "CUDA-core kernels (row-centric dq/dgate, a warp per head; key-centric dk/dv over a reverse "
                   "index); flops = 2x the forward attention's (the recomputations of z and p are not counted)",
           "gpu_launches_per_step": 6}
    del dev, out, sel, dy, grads, bws
    torch.cuda.empty_cache()
    return res


ABLATION_COV_STRIDE = 2048  # coverage rows: every 2048th query of the 64K sequence (all 32 heads)


def run_ablation(args, world, s):
    """The selection ablation on one 64K sequence (identical seeded inputs): B = 8, k = 4096 against
    B = 1, k = 2048. Throughput and stage times of the whole layer for both; the scored-candidate
    and attended-token ratios; and the token coverage per (query, head) of each GPU selection: the
    fraction of the query's top-2048 tokens by exact q.k that the selection holds (computed by the
    oracle's coverage function on sampled rows)."""
    import torch
    import block_sparse_long_kbar_b200 as sg
    from sgqa_inputs import gen_device
    import oracle
    res = {}
    dev = None
    cov_rows = None
    for name in ("64k_b8", "64k_b1"):
        cfg = CONFIGS[name]
        dims = sg.sgqa_dims.of(cfg)
        if dev is None:  # the generator does not depend on B or k: one set of inputs serves both
            dev = {}
            for n in ("q", "k", "v", "gate", "q_idx", "k_idx"):
                dev[n] = torch.empty(cfg.shape(n), dtype=torch.bfloat16, device="cuda")
                gen_device(cfg, n, dev[n])
        out = torch.empty(cfg.shape("q"), dtype=torch.bfloat16, device="cuda")
        sel = torch.empty((cfg.batch, cfg.T, cfg.G, cfg.Kb), dtype=torch.int32, device="cuda")
        kbar = torch.empty((cfg.batch, cfg.T // cfg.B, cfg.d_idx), dtype=torch.float32, device="cuda")
        ws = sg.alloc_workspace(sg.sgqa_workspace_size(dims))
        sg.sgqa_reset_device_status(ws)

        def step():
            sg.sgqa_forward(dims, dev["q"], dev["k"], dev["v"], dev["q_idx"], dev["k_idx"], dev["gate"], out, ws,
                            sel_out=sel, stream=s)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(args.steps):
            step()
        e1.record(s)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        st = {"select": [], "attend": []}
        for _ in range(args.steps):
            sg.sgqa_compress_keys(dims, dev["k_idx"], kbar, ws, stream=s)
            ev[0].record(s)
            sg.sgqa_select(dims, dev["q_idx"], kbar, sel, ws, stream=s)
            ev[1].record(s)
            sg.sgqa_attend(dims, dev["q"], dev["k"], dev["v"], dev["gate"], sel, out, ws, stream=s)
            ev[2].record(s)
            torch.cuda.synchronize()
            st["select"].append(ev[0].elapsed_time(ev[1]))
            st["attend"].append(ev[1].elapsed_time(ev[2]))
        assert sg.sgqa_get_device_status(ws) == 0
        wc = work_counts(cfg)
        entry = {"value": cfg.batch * cfg.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
                 "select_ms": statistics.mean(st["select"]), "attend_ms": statistics.mean(st["attend"]),
                 "scored_candidates": wc["scored"], "attended_visits": wc["visits"],
                 "B": cfg.B, "k": cfg.k}
        if not args.no_cpu_baseline:
            if cov_rows is None:
                ts = np.arange(ABLATION_COV_STRIDE - 1, cfg.T, ABLATION_COV_STRIDE, dtype=np.int32)
                cov_rows = np.stack([np.zeros_like(ts), ts], axis=1)
                ti = torch.from_numpy(ts.astype(np.int64)).cuda()
                cov_q = to_host(dev["q"][0].index_select(0, ti)).reshape(len(ts), -1)
                cov_k = to_host(dev["k"][:1])
            ti = torch.from_numpy(cov_rows[:, 1].astype(np.int64)).cuda()
            gsel = sel[0].index_select(0, ti).cpu().numpy()
            dm = oracle.dims(1, cfg.T, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
            cov = oracle.coverage(dm, cov_rows, cov_q, cov_k, gsel, ktop=2048)
            late = cov_rows[:, 1] >= 4096
            entry["coverage"] = {"mean": float(cov.mean()), "mean_t_ge_4096": float(cov[late].mean()),
                                 "rows": int(len(cov_rows)), "heads": cfg.Hq,
                                 "sample": f"every {ABLATION_COV_STRIDE}th query (t = {ABLATION_COV_STRIDE - 1} + "
                                           f"{ABLATION_COV_STRIDE} i), all heads; top-2048 by exact q.k"}
        res[name] = entry
        del out, sel, kbar, ws
        torch.cuda.empty_cache()
    del dev
    torch.cuda.empty_cache()
    b8, b1 = res["64k_b8"], res["64k_b1"]
    res["ratios"] = {"scored_b1_over_b8": b1["scored_candidates"] / b8["scored_candidates"],
                     "attended_b8_over_b1": b8["attended_visits"] / b1["attended_visits"],
                     "select_ms_b1_over_b8": b1["select_ms"] / b8["select_ms"],
                     "throughput_b8_over_b1": b8["value"] / b1["value"]}
    res["workload"] = ("selection ablation: batch 1, T=65536, Hq=32, G=4, d=128, d_idx=64, topic span 2048, seed 3; "
                       "B=8/k=4096 vs B=1/k=2048 on identical inputs")
    return res


SWA_WINDOW = 4096  # the pages give no window size for Gated SWA; this one matches the sparse budget


def run_swa(args, world, s):
    """Gated SWA (the efficient layer that alternates 3:1 with Sparse GQA) on the 128K prefill
    inputs: keys t - window < u <= t, through sgqa_gated_swa, inputs resident in HBM."""
    import torch
    import block_sparse_long_kbar_b200 as sg
    from sgqa_inputs import gen_device
    base = CONFIGS["128k"]
    cfg = base.replace(k=((SWA_WINDOW + 2 * base.B - 1) // base.B) * base.B)  # selection capacity
    dims = sg.sgqa_dims.of(cfg)
    dev = {}
    for n in ("q", "k", "v", "gate"):
        dev[n] = torch.empty(cfg.shape(n), dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, dev[n])
    out = torch.empty(cfg.shape("q"), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((cfg.batch, cfg.T, cfg.G, cfg.Kb), dtype=torch.int32, device="cuda")
    ws = sg.alloc_workspace(sg.sgqa_workspace_size(dims))
    sg.sgqa_reset_device_status(ws)
    torch.cuda.synchronize()

    def step():
        sg.sgqa_gated_swa(dims, SWA_WINDOW, dev["q"], dev["k"], dev["v"], dev["gate"], out, ws, sel_out=sel, stream=s)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(args.steps):
        step()
    e1.record(s)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    assert sg.sgqa_get_device_status(ws) == 0
    visits = cfg.batch * cfg.G * sum(min(t + 1, SWA_WINDOW) for t in range(cfg.T))  # (query, group, key)
    flops = visits * cfg.R * 4 * cfg.d
    peak = load_peaks()["bf16_tflops_sustained"]
    res = {"metric": "Gated SWA prefill tokens/s at 128K (window 4096)",
           "value": world * cfg.batch * cfg.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
           "steps": args.steps,
           "workload": f"gated swa 128k: batch {cfg.batch} per GPU, T={cfg.T}, Hq={cfg.Hq}, G={cfg.G}, d={cfg.d}, "
                       f"B={cfg.B}, window {SWA_WINDOW}, seed {cfg.seed} (the 128K prefill inputs)",
           "roofline": {"bound": "tensor", "achieved": flops / (ms / 1e3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                        "frac": flops / (ms / 1e3) / 1e12 / peak},
           "gpu_launches_per_step": 12}  # window selection, plan (10), attend
    del dev, out, sel, ws
    torch.cuda.empty_cache()
    return res


CPU_STRIDE = 64


NEAR_TIE_REL = 1e-4  # a selection may differ from the oracle's only where the swapped blocks' scores
                    # lie within this fraction of the m-th best score (the parity rule)


def cpu_baseline(cfg, rows, full, part, gpu_rows):
    """The oracle, as it stands, timed on the host cores on a strided sample of the same workload
    (the very bytes the GPU consumed); then, untimed, the bench's own GPU selection and output on
    those rows against it: selection mismatches (each must be a near-tie), and the output error
    (rows whose selection differs are compared with the oracle run on the GPU's selection)."""
    import oracle
    oracle.build()
    stride = CPU_STRIDE
    dm = oracle.dims(1, cfg.T, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    t0 = time.perf_counter()
    kbar = oracle.compress(dm, full["k_idx"])
    sel, s_m, _ = oracle.select(dm, kbar, rows, part["q_idx"])
    ref = oracle.attend(dm, rows, part["q"], full["k"], full["v"], part["gate"], sel)
    secs = time.perf_counter() - t0
    base = {"value": len(rows) / secs, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"every {stride}th query row of the {cfg.name} sequence ({len(rows)} rows, all heads and "
                      f"groups; block means of the whole sequence), {secs:.1f} s"}
    gsel = gpu_rows["sel"].reshape(sel.shape)
    diff = (gsel != sel).any(axis=2)
    near, bad = 0, 0
    for r, g in zip(*np.nonzero(diff)):
        t = int(rows[r, 1])
        c = t // cfg.B
        A = [int(j) for j in gsel[r, g] if j >= 0]
        O = [int(j) for j in sel[r, g] if j >= 0]
        ok = len(A) == len(O) and A == sorted(set(A)) and A[-1] == c
        if ok:
            sc = oracle.scores(dm, kbar, 0, part["q_idx"][r].reshape(cfg.G, cfg.d_idx)[g], c)
            thr = NEAR_TIE_REL * abs(s_m[r, g])
            ok = all(j < c and abs(sc[j] - s_m[r, g]) <= thr for j in set(A) ^ set(O))
        near += ok
        bad += not ok
    rr = np.nonzero(diff.any(axis=1))[0]
    if len(rr):
        ref[rr] = oracle.attend(dm, rows[rr], part["q"][rr], full["k"], full["v"], part["gate"][rr], gsel[rr])
    u = (gpu_rows["out"].reshape(ref.shape).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    dlt = np.abs(u - ref)
    errs = {"rows": int(len(rows)), "row_groups": int(diff.size), "selection_mismatches": int(diff.sum()),
            "near_tie_rows": int(near), "non_near_tie_mismatches": int(bad),
            "max_abs": float(dlt.max()), "mean_abs": float(dlt.mean()),
            "rel_rms": float(np.sqrt((dlt ** 2).sum() / max((ref ** 2).sum(), 1e-300))),
            "bounds": {"max_abs": 1e-2, "mean_abs": 1e-3, "near_tie_rel": NEAR_TIE_REL},
            "sample": f"the cpu_baseline rows; GPU output of the last timed step"}
    return base, errs


def run_reference(args, world, rank):
    """The fp64 oracle as it stands, on the host cores, on bounded strided samples of the workload."""
    import oracle
    oracle.build()
    cfg = CONFIGS[args.config]
    stride = 256
    rows0 = sample_rows_strided(cfg, stride)
    full, _ = oracle_inputs_host(cfg, rows0)
    times = []
    for i in range(args.warmup + args.steps):
        rows = sample_rows_strided(cfg, stride, offset=i * 37)
        part = {n: gen_rows(cfg, n, 0, rows[:, 1]) for n in ("q", "q_idx", "gate")}
        secs = oracle_sample_time(cfg, stride, full, part, rows)
        if i >= args.warmup:
            times.append((len(rows), secs))
    n = sum(r for r, _ in times)
    tot = sum(s for _, s in times)
    value = n / tot
    ms = 1e3 * cfg.T / value
    sample = (f"per step every {stride}th query row of the {cfg.name} sequence (rotating offset, "
              f"{len(rows0)} rows), fp64 oracle on {oracle.max_threads()} host threads")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded topic-structured generator)",
            "config": {"workload": f"prefill {cfg.name}: batch {cfg.batch}, T={cfg.T}, Hq={cfg.Hq}, G={cfg.G}, "
                                   f"d={cfg.d}, d_idx={cfg.d_idx}, B={cfg.B}, k={cfg.k}, topic span {cfg.span}, "
                                   f"seed {cfg.seed}", "global_batch": cfg.batch, "seq_len": cfg.T,
                       "parallelism": "host cores (OpenMP)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="128k", choices=["tiny", "32k", "128k", "64k_b8", "64k_b1"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-swa", action="store_true")
    ap.add_argument("--no-ablation", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--query-sharded", action="store_true",
                    help="split the sequence's queries over the ranks even at N = 1 (the N > 1 path)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world, rank)), flush=True)
        return
    world, rank, _ = dist_setup(args.gpus)
    try:
        sharded = world > 1 or args.query_sharded
        res = run_sharded(args, world, rank) if sharded else run_ours(args, world, rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
