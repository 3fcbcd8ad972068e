"""Benchmark of one paged decode step on B200.

A step is the whole hot path for one batch: copy-on-write block copies,
the cache write of each sequence's new token, and paged decode attention.
The headline workload is the largest single-GPU one, the Llama-2-13B-shaped
chat mix (128 sequences in 32 groups of n=4 samples sharing a 512-token
prompt prefix, 40 q / 40 kv heads, head_dim 128, block size 16, 24576-block
pool); its decode reads each group's shared tiles once
(pa_decode_shared_prefix).  The same line carries a ``per_config`` entry for
each other workload whose K/V exceeds L2 (Llama-2-7B-shaped, Llama-3-8B GQA,
long-context split), each timed the same way.

Prints one JSON line.  ``value`` is the step's algorithmic HBM bytes per
second (inputs resident in HBM, timed on the device with CUDA events, max
over ranks); the chat mix counts each shared K/V row once (the DRAM
minimum), its logical bytes (every sequence's whole history) are reported
beside.  ``e2e`` is the same metric measured through the public API with
pinned host buffers (host allocator append, host->device upload of the
step's inputs, copies, fused write + decode, output into host memory).
``roofline`` reports the decode call against the measured HBM copy peak;
``cpu_baseline`` is the fp64 oracle timed on this host's cores on a bounded
sample of the headline workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1..5] [--per-config 2,4,5]
    python bench.py --impl reference ...   (the oracle arm)
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "paged decode: achieved HBM GB/s (% of B200 peak) and KV tokens attended/sec"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0

WORKLOAD_NAMES = {
    1: "tiny paged decode: B=4, lens {1,16,33,47}, 4 q / 2 kv heads, d=64, bs=16, 32-block pool",
    2: "Llama-2-7B-shaped decode: B=64, 32 q / 32 kv heads, d=128, bs=16, lens U[128,2048], 16384-block pool",
    3: "Llama-2-13B-shaped chat mix: B=128 (32 groups x n=4), 40/40 heads, d=128, bs=16, "
       "len=U[100,2000]+U[50,500], 512-token shared prefix, CoW copies",
    4: "Llama-3-8B-shaped GQA decode: B=256, 32 q / 8 kv heads, d=128, bs=32, lognormal lens (median 800, cap 4096)",
    5: "long-context split-K decode: B=8, 64 q / 8 kv heads, d=128, bs=16, L=32768, 512-token partitions, "
       "1024 copy pairs",
}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def _measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _decode_traffic_record(cfg: int, kv_dtype: str, kernel: str):
    """ncu DRAM traffic of the decode call for this workload, KV dtype and entry point, if taken on the
    current device code."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            recs = json.load(f)["records"]
    except Exception:
        return None
    digest = kernel_src_sha256()
    for rec in recs:
        if (rec.get("kernel_src_sha256") == digest and rec.get("config") == cfg and rec.get("kv_dtype") == kv_dtype
                and rec.get("kernel", "").startswith(kernel)):
            return rec
    return None


def kernel_src_sha256() -> str:
    """Hash of the decode's device sources (kernel header + device helpers), in that order."""
    h = hashlib.sha256()
    for name in ("decode_kernels.cuh", "pa_common.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_349_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def step_bytes(case, kv_elem_bytes: int = 2):
    """Algorithmic bytes of one step: (copy, write, decode); fp8 pools hold 1 byte per value."""
    bs, d, Hkv = case.block_size, case.head_dim, case.num_kv_heads
    block_bytes = Hkv * bs * d * kv_elem_bytes
    copy = int(case.copy_pairs.shape[0]) * block_bytes * 2 * 2 + case.copy_pairs.size * 4
    T = int(case.slot_mapping.size)
    write = T * Hkv * d * (2 + kv_elem_bytes) * 2 + T * 4
    dec = W.algorithmic_decode_bytes(case, kv_elem_bytes=kv_elem_bytes)
    return copy, write, dec


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.samples = []
        self._stop = threading.Event()
        self._proc = None

    def start(self):
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.device_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self._proc = None
            return self
        self._thread = threading.Thread(target=self._read, daemon=True)
        self._thread.start()
        return self

    def _read(self):
        for line in self._proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append(parts)
            if self._stop.is_set():
                break

    def stop(self):
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()
        return self.summary()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for s in self.samples:
            for name, val in zip(names, s[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(self.samples)}


def _dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def _max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def _barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# CPU oracle baseline (the only place the bench runs the oracle)
# ---------------------------------------------------------------------------

def cpu_model() -> str:
    """The host CPU's model name (/proc/cpuinfo), or 'unknown'."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(case, budget_s: float = 12.0, threads=None):
    """Time the fp64 oracle on a bounded sample of (sequence, kv head) units of ``case``.

    Units are taken in a seeded order, in chunks, cycling over the whole
    workload until about ``budget_s`` seconds of oracle time have passed.
    Returns the oracle's throughput in the bench's unit (algorithmic GB/s),
    the threads it used, what the sample was, the seconds and bytes timed.
    Bytes are counted as the GPU arm counts them: for a workload whose
    sequences share blocks, the sample's logical bytes are scaled by the
    workload's ratio of unique to logical decode bytes.
    """
    import oracle
    threads = len(os.sched_getaffinity(0)) if threads is None else threads
    oracle.set_num_threads(threads)
    G = case.group_size
    rng = np.random.default_rng(7)
    units = [(int(b), int(h)) for b in rng.permutation(case.batch) for h in rng.permutation(case.num_kv_heads)]
    done_units, done_bytes, elapsed = 0, 0, 0.0
    chunk = max(1, threads)
    pos = 0
    while elapsed < budget_s:
        sel = [units[(pos + i) % len(units)] for i in range(min(chunk, len(units)))]
        pos = (pos + len(sel)) % len(units)
        rows = np.array([(b, h * G + g) for b, h in sel for g in range(G)], np.int32)
        t0 = time.perf_counter()
        oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.seq_lens,
                      num_kv_heads=case.num_kv_heads, block_size=case.block_size, scale=case.scale, rows=rows)
        dt = time.perf_counter() - t0
        elapsed += dt
        done_units += len(sel)
        done_bytes += sum(int(case.seq_lens[b]) * case.head_dim * 4 + G * case.head_dim * 6 for b, _ in sel)
        if dt < budget_s / 20:
            chunk *= 2
    scale = 1.0
    if case.groups is not None:
        scale = decode_bytes(case, 2, unique=True) / decode_bytes(case, 2, unique=False)
    counted = done_bytes * scale
    gbs = counted / elapsed / 1e9
    sample = (f"{done_units} (sequence, kv head) units ({done_units / len(units):.2f} passes over the "
              f"workload's {len(units)}), {done_units * G} query-head rows, {done_bytes / 1e9:.2f} GB of "
              f"K/V/q/out read"
              + (f", counted as {counted / 1e9:.2f} GB (x{scale:.3f}: shared rows once, as the GPU arm counts)"
                 if scale != 1.0 else "")
              + f", {elapsed:.1f} s of oracle time")
    return gbs, threads, sample, elapsed, counted


# ---------------------------------------------------------------------------
# native arm
# ---------------------------------------------------------------------------

def unique_kv_rows(case) -> int:
    """K/V rows (per kv head) a decode must read from DRAM at least: each physical block's rows
    counted once, as many as the furthest-reaching sequence reads from it."""
    bs = case.block_size
    rows = {}
    for b, L in enumerate(case.seq_lens):
        L = int(L)
        for j in range(-(-L // bs)):
            blk = int(case.block_tables[b, j])
            rows[blk] = max(rows.get(blk, 0), min(bs, L - j * bs))
    return sum(rows.values())


def decode_bytes(case, kv_elem_bytes: int, unique: bool) -> int:
    """Algorithmic decode bytes; with ``unique`` the K/V part counts each shared row once."""
    logical = W.algorithmic_decode_bytes(case, kv_elem_bytes=kv_elem_bytes)
    if not unique:
        return logical
    kv_row = case.num_kv_heads * case.head_dim * kv_elem_bytes * 2
    return logical - int(case.seq_lens.sum()) * kv_row + unique_kv_rows(case) * kv_row


def measure_workload(cfg, args, world, rank, pa, headline):
    """Time one workload's step (device-resident) and, unless disabled, its e2e step.

    Returns the fields of one bench entry (the headline line or a per_config entry)."""
    import torch

    base = 1000 + cfg if args.seed is None else args.seed
    seed = base + 7919 * rank  # weak scaling: every rank owns its own batch
    case = W.make_case(cfg, seed=seed, fill=W.BF16_ZERO, num_blocks=args.num_blocks,
                       block_size=args.block_size if cfg == 2 else None)
    fp8 = args.kv_dtype == "fp8"
    elem = 1 if fp8 else 2
    # Shared-prefix groups (the n=4 chat mix): the step decodes with pa_decode_shared_prefix,
    # which reads each group's shared tiles once; the plain fused decode (whose repeated prefix
    # reads L2 serves) is timed beside it, the two called in alternation, with L2 warm and with
    # L2 flushed before each call.
    has_groups = case.groups is not None and not fp8 and not args.unfused
    prefix = has_groups and args.decode == "shared-prefix"
    group_size = 4
    copy_b, write_b, _ = step_bytes(case, elem)
    shared_rows = case.groups is not None
    dec_b = decode_bytes(case, elem, unique=shared_rows)
    dec_logical = decode_bytes(case, elem, unique=False)
    total_b = copy_b + write_b + dec_b
    kv_tokens = int(case.seq_lens.sum())

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    def i32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()

    k, v = bf16(case.k_cache), bf16(case.v_cache)
    k_scale = v_scale = 1.0
    if fp8:
        # fp8 pools, quantised on the device by the library (per-pool scale = amax / 448)
        k_scale = max(float(k.float().abs().amax()) / 448.0, 1e-30)
        v_scale = max(float(v.float().abs().amax()) / 448.0, 1e-30)
        k8 = torch.empty(k.shape, dtype=torch.uint8, device="cuda")
        v8 = torch.empty(v.shape, dtype=torch.uint8, device="cuda")
        pa.pa_quantize_fp8(k, k8, k_scale)
        pa.pa_quantize_fp8(v, v8, v_scale)
        torch.cuda.synchronize()
        del k, v
        k, v = k8, v8
    q = bf16(case.q)
    k_new, v_new = bf16(case.k_new), bf16(case.v_new)
    slots = i32(case.slot_mapping)
    # Fused step: each sequence's token at L-1 is written by the decode launch itself;
    # any other new rows of the step (copy-on-write destinations) go through the cache write.
    k_last_np, v_last_np, other = W.split_last_tokens(case)
    k_last, v_last = bf16(k_last_np), bf16(v_last_np)
    k_other, v_other = bf16(case.k_new[other]), bf16(case.v_new[other])
    slots_other = i32(case.slot_mapping[other])
    fused = not args.unfused
    pairs = i32(case.copy_pairs.reshape(-1, 2))
    tables, lens = i32(case.block_tables), i32(case.seq_lens)
    out = torch.empty(case.q.shape, dtype=torch.float32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pt = case.partition_tokens
    resolved_pt = pa.pa_decode_partition_tokens(case.batch, case.num_q_heads, case.num_kv_heads,
                                                case.head_dim, case.block_size, case.max_seq_len, pt)
    ws_plain = pa.pa_decode_workspace_size(case.batch, case.num_q_heads, case.num_kv_heads, case.head_dim,
                                           case.block_size, case.max_seq_len, pt)
    ws_bytes = ws_plain
    prefix_lens = None
    if has_groups:
        prefix_lens = i32(case.shared_tokens[::group_size])
        ws_bytes = max(ws_bytes, pa.pa_decode_shared_prefix_workspace_size(
            case.batch, group_size, case.num_q_heads, case.num_kv_heads, case.head_dim, case.block_size,
            case.max_seq_len, pt))
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    dec_ev = []

    def decode_call(kind):
        if fp8:
            pa.pa_decode_fp8(out, q, k, v, tables, lens, max_seq_len=case.max_seq_len, scale=float(case.scale),
                             k_scale=k_scale, v_scale=v_scale, partition_tokens=pt, workspace=ws, err_flag=flag,
                             stream=stream, k_new=k_last, v_new=v_last)
        elif kind == "shared-prefix":
            pa.pa_decode_shared_prefix(out, q, k, v, tables, lens, prefix_lens, group_size=group_size,
                                       max_seq_len=case.max_seq_len, scale=float(case.scale), partition_tokens=pt,
                                       workspace=ws, err_flag=flag, stream=stream, k_new=k_last, v_new=v_last)
        elif fused:
            pa.pa_decode_append(out, q, k_last, v_last, k, v, tables, lens, max_seq_len=case.max_seq_len,
                                scale=float(case.scale), partition_tokens=pt, workspace=ws, err_flag=flag,
                                stream=stream)
        else:
            pa.pa_decode(out, q, k, v, tables, lens, max_seq_len=case.max_seq_len, scale=float(case.scale),
                         partition_tokens=pt, workspace=ws, err_flag=flag, stream=stream)

    kind_main = "shared-prefix" if prefix else "plain"

    def step(record=False, kind=kind_main, evs=dec_ev):
        if case.copy_pairs.shape[0]:
            (pa.pa_copy_blocks_fp8 if fp8 else pa.pa_copy_blocks)(k, v, pairs, err_flag=flag, stream=stream)
        if fused:
            if other.size:
                if fp8:
                    pa.pa_reshape_and_cache_fp8(k_other, v_other, k, v, slots_other, k_scale=k_scale,
                                                v_scale=v_scale, err_flag=flag, stream=stream)
                else:
                    pa.pa_reshape_and_cache(k_other, v_other, k, v, slots_other, err_flag=flag, stream=stream)
        else:
            pa.pa_reshape_and_cache(k_new, v_new, k, v, slots, err_flag=flag, stream=stream)
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        decode_call(kind)
        if record:
            e1.record(stream)
            evs.append((e0, e1))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert int(flag.item()) == 0, f"error flag {int(flag.item()):#x}"

    sampler = ClockSampler(torch.cuda.current_device()).start() if rank == 0 else None
    # The timed region lasts milliseconds, shorter than the sampling period: keep the
    # GPU under the same (untimed, idempotent) step for ~0.4 s first, so the clock
    # samples show the clocks under this load.
    load_steps = 0
    if sampler:
        t_load = time.perf_counter() + 0.4
        while time.perf_counter() < t_load:
            for _ in range(10):
                step()
            load_steps += 10
            torch.cuda.synchronize()
    _barrier(world)
    torch.cuda.synchronize()
    launches0 = pa.launch_count()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step(record=True)
    t1.record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    launches = int(_sum_over_ranks(float(pa.launch_count() - launches0), world))  # whole job, like value
    clocks = sampler.stop() if sampler else None
    if clocks is not None:
        clocks["untimed_load_steps_before_timing"] = load_steps
    ms_local = t0.elapsed_time(t1)
    ms = _max_over_ranks(ms_local, world)
    dec_ms = _max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in dec_ev), world)
    assert int(flag.item()) == 0, f"error flag {int(flag.item()):#x}"

    # The chat mix: both decodes of the same step, call by call in alternation (so both see
    # the same clocks), with L2 warm and with L2 flushed before each call.
    compare = None
    if has_groups:
        l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size

        def interleaved(flush=None):
            evs = {"plain": [], "shared-prefix": []}
            for _ in range(args.warmup):
                for kind in evs:
                    step(kind=kind)
            torch.cuda.synchronize()
            for _ in range(args.steps):
                for kind in evs:
                    if flush is not None:
                        flush.fill_(1)
                    step(record=True, kind=kind, evs=evs[kind])
            torch.cuda.synchronize()
            return {kind: round(_max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in e), world), 5)
                    for kind, e in evs.items()}

        compare = {"l2_warm": interleaved()}
        flush = torch.empty(2 * l2, dtype=torch.uint8, device="cuda")
        compare["l2_flushed"] = interleaved(flush)
        del flush
        assert int(flag.item()) == 0, f"error flag {int(flag.item()):#x}"

    all_bytes = _sum_over_ranks(float(total_b), world)
    all_tokens = _sum_over_ranks(float(kv_tokens), world)
    step_s = ms / 1e3 / args.steps
    value = all_bytes / step_s / 1e9
    peak, peak_kind = _measured_peak()
    achieved = dec_b / (dec_ms / 1e3) / 1e9

    e2e = None
    if not (args.no_e2e or args.unfused):
        e2e = run_e2e(args, case, pa, stream, world, k, v, (k_scale, v_scale) if fp8 else None,
                      (case.shared_tokens[::group_size], group_size) if prefix else None)

    kernel = ("pa_decode_append_fp8" if fp8 else "pa_decode_shared_prefix (fused write)" if prefix else
              "pa_decode_append" if fused else "pa_decode")
    rec = _decode_traffic_record(cfg, "fp8" if fp8 else "bf16", kernel)
    traffic = rec.get("traffic_bytes_per_launch") if rec else None
    split = prefix or resolved_pt > 0
    roof = {
        "kernel": kernel + (" (split decode + log-sum-exp reduce)" if split else " (single pass)"),
        "bound": "hbm",
        "achieved": round(achieved, 1),
        "peak": peak,
        "peak_kind": f"{peak_kind} (HBM copy)",
        "unit": "GB/s",
        "frac": round(achieved / peak, 4),
        "traffic": traffic,
        "algorithmic_bytes_per_launch": dec_b,
        "launch_ms": round(dec_ms, 5),
    }
    if shared_rows:
        roof["algorithmic_bytes_note"] = ("each shared K/V row counted once (DRAM minimum); logical bytes count "
                                          "it once per sequence")
        roof["logical_bytes_per_launch"] = dec_logical
        roof["logical_gbps"] = round(dec_logical / (dec_ms / 1e3) / 1e9, 1)
        if traffic:
            roof["traffic_vs_unique"] = round(traffic / dec_b, 4)
            roof["traffic_vs_logical"] = round(traffic / dec_logical, 4)
    if compare is not None:
        roof["decode_comparison_ms"] = compare
        roof["decode_comparison_note"] = (
            "pa_decode_append (plain: repeated prefix rows served by L2) against pa_decode_shared_prefix "
            "(each group's shared tiles read once), called in alternation; l2_flushed writes a "
            f"{2 * l2 >> 20} MiB buffer before each call")

    entry = {
        "value": round(value, 1),
        "unit": "GB/s",
        "ms_per_step": round(ms / args.steps, 4),
        "config": {
            "workload": workload_name(cfg, case),
            "config_index": cfg,
            "seed": base,
            "batch_per_gpu": case.batch,
            "global_batch": case.batch * world,
            "partition_tokens": case.partition_tokens,
            "parallelism": f"dp{world} (independent sequences per GPU, no collective)",
            "l2": f"inputs larger than L2: {dec_b / 1e9:.2f} GB of K/V per step vs 126 MB L2; no flush",
            "step": step_description(case, fp8, prefix, fused),
        },
        "pct_of_peak": {"nominal_8TBps": round(100 * value / NOMINAL_HBM_GBS, 1),
                        f"{peak_kind}_{peak:.0f}GBps": round(100 * value / peak, 1)},
        "kv_tokens_per_s": round(all_tokens / step_s, 1),
        "kv_head_tokens_per_s": round(all_tokens * case.num_kv_heads / step_s, 1),
        "kv_tokens_per_gpu": kv_tokens,
        "decode_partition_tokens": resolved_pt,
        "step_bytes": {"copy": copy_b, "write": write_b, "decode": dec_b},
        "gpu_launches": launches,
        "roofline": roof,
        "e2e": e2e,
        "clocks": clocks,
    }
    if fp8:
        entry["config"]["kv_scales"] = {"k": k_scale, "v": v_scale}
    cpu = None
    if headline and rank == 0 and world == 1 and not args.no_cpu_baseline and not fp8:
        gbs, cores, sample, _, _ = cpu_baseline(case, budget_s=args.cpu_budget)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample,
               "cpu_model": cpu_model()}
        if cores > 1:  # the same oracle on one thread, over a shorter sample
            gbs1, _, sample1, _, _ = cpu_baseline(case, budget_s=max(1.0, args.cpu_budget / 6), threads=1)
            cpu["single_thread"] = {"value": round(gbs1, 4), "unit": "GB/s", "sample": sample1}
    del k, v, q, ws
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return entry, cpu


def run_native(args):
    import paged_kv_cache_349_b200 as pa

    world, rank, local = _dist_setup()
    head, cpu = measure_workload(args.config, args, world, rank, pa, headline=True)
    per = {}
    for cfg in args.per_config:
        if cfg != args.config:
            e, _ = measure_workload(cfg, args, world, rank, pa, headline=False)
            per[str(cfg)] = e
    line = {
        "metric": METRIC,
        "value": head["value"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if args.kv_dtype == "bf16" else "e4m3 K/V (f16 mma), bf16 q",
        "accumulate": "fp32",
        "data": "synthetic (seeded bf16 N(0,1) K/V/q, seeded placement)",
    }
    line.update({k: v for k, v in head.items() if k not in ("value", "unit", "ms_per_step")})
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if per:
        line["per_config"] = per
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def replay_allocator(pa, case):
    """Rebuild the workload's tables with the host allocator (state before the step's append).

    Blocks are dealt in the generator's order; for the n=4 chat workload each
    group's prompt prefix is appended once, forked three times, and every
    member then appends its own tokens (members 0..2 copy the partial shared
    block on their first write, member 3 writes in place).
    """
    alloc = pa.Allocator(case.num_blocks, case.block_size, order=case.free_order)
    sids = np.zeros(case.batch, np.int32)
    if case.groups is None:
        for b, L in enumerate(case.seq_lens):
            s = alloc.create()
            sids[b] = s
            for _ in range(max(int(L) - 1, 0)):
                alloc.append(s)
        return alloc, sids
    for g in range(int(case.groups.max()) + 1):
        members = np.nonzero(case.groups == g)[0]
        root = alloc.create()
        for _ in range(int(case.shared_tokens[members[0]])):
            alloc.append(root)
        ids = [alloc.fork(root) for _ in range(len(members) - 1)] + [root]
        for b, s in zip(members, ids):
            sids[b] = s
            for _ in range(int(case.seq_lens[b]) - 1 - int(case.shared_tokens[b])):
                alloc.append(s)
    return alloc, sids


def run_e2e(args, case, pa, stream, world, k_pool, v_pool, kv_scales=None, prefix=None):
    """The same step through the public API with host buffers (pinned), timed end to end.

    Every step: the host allocator appends one token per sequence (and reports
    copy-on-write pairs) and exports the tables into pinned memory (one
    ``pa_alloc_step`` call); one ``pa_decode_step_plan_run`` call (the step is
    prepared once) then uploads the step's inputs, applies the copies and runs
    the fused cache write + decode, whose output lands in pinned host memory;
    the step ends when the output is on the host.  Byte counts are taken after
    the timed loop.  ``kv_scales`` = (k_scale, v_scale) for fp8 pools;
    ``prefix`` = (prefix lengths per group, group size) makes the step decode
    with ``pa_decode_shared_prefix`` (the replayed allocator forks each group's
    members from its first, so their shared tokens sit in the same blocks).
    """
    import torch
    bs = case.block_size
    steps, warm = args.steps, args.warmup
    grow = steps + warm + 1
    alloc, sids = replay_allocator(pa, case)
    max_blocks = case.max_blocks_per_seq + (grow + bs - 1) // bs + 1
    max_len_cap = case.max_seq_len + grow
    B = case.batch

    def pinned_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()

    # one new token per sequence and step (the case may carry extra rows for its first step)
    h_q = pinned_bf16(case.q)
    h_k = pinned_bf16(case.k_new[:B])
    h_v = pinned_bf16(case.v_new[:B])
    h_tables = torch.empty((B, max_blocks), dtype=torch.int32).pin_memory()
    h_lens = torch.empty(B, dtype=torch.int32).pin_memory()
    h_pairs = torch.zeros((B, 2), dtype=torch.int32).pin_memory()
    h_out = torch.empty(case.q.shape, dtype=torch.float32).pin_memory()
    tables_np, lens_np, pairs_np = h_tables.numpy(), h_lens.numpy(), h_pairs.numpy()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    if prefix is not None:
        size = pa.pa_decode_step_staging_size_shared_prefix(B, prefix[1], max_blocks, B, case.num_q_heads,
                                                            case.num_kv_heads, case.head_dim, bs, max_len_cap,
                                                            case.partition_tokens)
        h_prefix = torch.from_numpy(np.ascontiguousarray(prefix[0], dtype=np.int32)).pin_memory()
    else:
        size = pa.pa_decode_step_staging_size(B, max_blocks, B, case.num_q_heads, case.num_kv_heads, case.head_dim,
                                              bs, max_len_cap, case.partition_tokens)
        h_prefix = None
    staging = torch.empty(size, dtype=torch.uint8, device="cuda")
    if args.unfused:
        raise SystemExit("--unfused applies to the device-resident step only")
    run = pa.DecodeStepHost(out_host=h_out, q_host=h_q, k_new_host=h_k, v_new_host=h_v, tables_host=h_tables,
                            lens_host=h_lens, pairs_host=h_pairs, k_cache=k_pool, v_cache=v_pool,
                            scale=float(case.scale), max_seq_len_cap=max_len_cap,
                            partition_tokens=case.partition_tokens,
                            num_chunks=args.step_chunks, staging=staging,
                            err_flag=flag, stream=stream,
                            k_scale=kv_scales[0] if kv_scales else None, v_scale=kv_scales[1] if kv_scales else None,
                            prefix_lens_host=h_prefix, group_size=prefix[1] if prefix is not None else 0)
    elem = 1 if kv_scales else 2
    host_step = alloc.step_fn(sids, tables_np, lens_np, pairs_np)
    # per timed step: its max length and copy-pair count (the bytes are counted after the timed loop)
    steps_seen = []

    def e2e_step():
        n_pairs, max_len = host_step()  # append one token per sequence, export tables + lengths
        run(max_len, n_pairs)
        stream.synchronize()  # the step's output is on the host
        return n_pairs

    for _ in range(warm):
        e2e_step()
    lens0 = lens_np.copy()  # lengths after the warm-up steps; every timed step adds one token per sequence
    _barrier(world)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(steps):
        steps_seen.append(e2e_step())
    dt = time.perf_counter() - t0
    dt = _max_over_ranks(dt, world)
    assert int(flag.item()) == 0
    acc = {"h2d": 0, "d2h": 0, "alg": 0, "tokens": 0}
    # shared prefixes (forks) count once, as in the device-resident value
    share = (decode_bytes(case, elem, unique=True) / decode_bytes(case, elem, unique=False)
             if case.groups is not None else 1.0)
    for i, n_pairs in enumerate(steps_seen):
        lens_i = lens0 + i + 1
        acc["h2d"] += sum(t.numel() * t.element_size() for t in (h_q, h_k, h_v, h_tables, h_lens)) + n_pairs * 8
        acc["h2d"] += h_prefix.numel() * 4 if h_prefix is not None else 0
        acc["d2h"] += h_out.numel() * 4
        acc["tokens"] += int(lens_i.sum())
        c, w, d = step_bytes_from(case, lens_i, n_pairs, elem)
        acc["alg"] += c + w + d * share
    assert np.array_equal(lens0 + len(steps_seen), lens_np), "every timed step appends one token per sequence"
    alg = _sum_over_ranks(float(acc["alg"]), world)
    alloc.close()
    return {"value": round(alg / dt / 1e9, 1), "unit": "GB/s",
            "ms_per_step": round(dt * 1e3 / steps, 4),
            "h2d_bytes_per_step": acc["h2d"] // steps, "d2h_bytes_per_step": acc["d2h"] // steps,
            "kv_tokens_per_s": round(_sum_over_ranks(float(acc["tokens"]), world) / dt, 1),
            "step_chunks": args.step_chunks or "auto",
            "includes": "host allocator step (pa_alloc_step: batched append + table export into pinned memory), then one "
                        "pa_decode_step_plan_run call (a step prepared once with pa_decode_step_plan_create"
                        + (" over E4M3 pools" if kv_scales else "")
                        + (", in shared-prefix mode: pa_decode_step_plan_set_shared_prefix" if prefix is not None else "")
                        + "): upload of q/k_new/v_new/tables/lens" + ("/prefix lengths" if prefix is not None else "")
                        + "/copy pairs, block copies, fused cache write + "
                        + ("shared-prefix decode" if prefix is not None else "decode")
                        + ", out stored into pinned host memory; timed until out is on the host"}


def step_bytes_from(case, lens, n_pairs, kv_elem_bytes: int = 2):
    """Algorithmic bytes of one e2e step (copy, write, decode) from its lengths and copy-pair count."""
    bs, d, Hkv = case.block_size, case.head_dim, case.num_kv_heads
    copy = n_pairs * Hkv * bs * d * kv_elem_bytes * 2 * 2 + n_pairs * 8
    T = int(lens.size)
    write = T * Hkv * d * (2 + kv_elem_bytes) * 2 + T * 4
    dec = W.algorithmic_decode_bytes(lens, num_q_heads=case.num_q_heads, num_kv_heads=Hkv, head_dim=d,
                                     block_size=bs, kv_elem_bytes=kv_elem_bytes)
    return copy, write, dec


# ---------------------------------------------------------------------------
# reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------

def step_description(case, fp8: bool, prefix: bool, fused: bool) -> str:
    """What one timed step runs, in order."""
    copies = "block copies, " if case.copy_pairs.shape[0] else ""
    _, _, other = W.split_last_tokens(case)
    cow = "cache write of the copy-on-write rows, " if other.size else ""
    if fp8:
        return copies + cow + "pa_decode_append_fp8 (each new token quantised to E4M3 and written by the decode)"
    if prefix:
        return (copies + cow + "pa_decode_shared_prefix (each group's shared tiles read once; each new token "
                "written by the decode)")
    if fused:
        return copies + cow + "pa_decode_append (each sequence's new token written by the decode launch)"
    return copies + "pa_reshape_and_cache, pa_decode"


def workload_name(cfg: int, case) -> str:
    """WORKLOAD_NAMES[cfg], with the block size and pool of a re-paged workload 2."""
    name = WORKLOAD_NAMES[cfg]
    if cfg == 2 and case.block_size != 16:
        name = name.replace("bs=16", f"bs={case.block_size}").replace("16384-block", f"{case.num_blocks}-block")
    return name


def reference_config(case, cfg, base, world):
    """The reference arm's ``config``: the same keys and values as the native arm's headline."""
    prefix = case.groups is not None
    dec_b = decode_bytes(case, 2, unique=prefix)
    return {
        "workload": workload_name(cfg, case),
        "config_index": cfg,
        "seed": base,
        "batch_per_gpu": case.batch,
        "global_batch": case.batch * world,
        "partition_tokens": case.partition_tokens,
        "parallelism": f"dp{world} (independent sequences per GPU, no collective)",
        "l2": f"inputs larger than L2: {dec_b / 1e9:.2f} GB of K/V per step vs 126 MB L2; no flush",
        "step": step_description(case, False, case.groups is not None, True),
    }


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = args.config
    base = 1000 + cfg if args.seed is None else args.seed
    case = W.make_case(cfg, seed=base, fill=W.BF16_ZERO, block_size=args.block_size if cfg == 2 else None)
    per_step = max(1.0, args.cpu_budget / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(case, budget_s=per_step / 4)
    vals, secs, nbytes = [], 0.0, 0
    sample = ""
    cores = 0
    for _ in range(args.steps):
        gbs, cores, sample, el, by = cpu_baseline(case, budget_s=per_step)
        vals.append(gbs)
        secs += el
        nbytes += by
    value = nbytes / secs / 1e9
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs * 1e3 / args.steps, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded bf16 N(0,1) K/V/q, seeded placement)",
        "config": reference_config(case, cfg, base, world),
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": "per step: " + sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=3, choices=[1, 2, 3, 4, 5],
                    help="headline workload (default 3, the chat mix: the largest single-GPU workload)")
    ap.add_argument("--per-config", type=str, default=None,
                    help="comma-separated workloads timed after the headline into per_config "
                         "(default: 2,4,5 when --config is left at its default, none otherwise)")
    ap.add_argument("--decode", choices=["plain", "shared-prefix"], default="shared-prefix",
                    help="the chat mix's step: pa_decode_append (plain) or pa_decode_shared_prefix; the other "
                         "is timed beside it")
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--step-chunks", type=int, default=0,
                    help="e2e: chunks of sequences pa_decode_step_host pipelines (0 = the library's choice)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time")
    ap.add_argument("--kv-dtype", choices=["bf16", "fp8"], default="bf16",
                    help="fp8: E4M3 pools quantised by the library (per-pool scales)")
    ap.add_argument("--unfused", action="store_true",
                    help="time pa_reshape_and_cache + pa_decode instead of the fused pa_decode_append")
    ap.add_argument("--seed", type=int, default=None, help="input seed (default 1000 + config; + 7919 per rank)")
    ap.add_argument("--block-size", type=int, default=None, choices=[8, 16, 32, 64],
                    help="workload 2 only: re-page it with this block size (same lengths and pool bytes)")
    ap.add_argument("--num-blocks", type=int, default=None,
                    help="pool size override (same decode launch, smaller pool: for profiler captures)")
    args = ap.parse_args()
    explicit = any(a == "--config" or a.startswith("--config=") for a in sys.argv[1:])
    if args.per_config is None:
        args.per_config = [] if explicit else [2, 4, 5]
    else:
        args.per_config = [int(x) for x in args.per_config.split(",") if x.strip()]
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.block_size is not None and (args.config != 2 or args.per_config):
        ap.error("--block-size re-pages workload 2: use it with --config 2 alone")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus != world:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch N > 1 under torchrun "
              f"(one rank per GPU). Measuring {world} rank(s).", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
