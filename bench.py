#!/usr/bin/env python
"""Benchmark of one paged decode step (cache write of the appended tokens + split-context
decode attention + partition merge) on the llama3_8b_b64 workload: 64 sequences, 32 query /
8 KV heads, head_dim 128, bf16 KV in 16-token blocks drawn shuffled from a pool sized to
1.1x demand, contexts ~ U{512..4096}, 2048-token partitions.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  `value` is KV GB/s of the whole job (algorithmic K+V bytes
the step must read / device time of the step, CUDA events, inputs resident in HBM, L2
flushed between steps or inputs larger than L2).  `e2e` is the same metric through the binding's public calls with
pinned host inputs copied in and the output copied back inside the timed region.
`--impl reference` times the CPU oracle (the plain fp64 C implementation) on a bounded
sample of the same workload, on the host cores.

Multi-GPU (torchrun): weak scaling -- every rank runs its own batch of the same shape; the
units are independent, so no collective touches the data path.  The step time is the max
over ranks (device events), `value` the sum of all ranks' bytes over that time.
"""
from __future__ import annotations

import argparse
import datetime as _dt
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV GB/s & % of B200 HBM peak; decode tokens/s"
FALLBACK_HBM_GBS = 6650.0
DEFAULT_WORKLOAD = "llama3_8b_b64"
KERNEL_SOURCES = [os.path.join(ROOT, "paged_kv_cache_428_b200", "csrc", f)
                  for f in ("common.cuh", "decode.cuh", "decode_mma.cuh", "decode_q8.cuh", "decode_balanced.cuh")]
# the tcgen05 prefill kernel and every header it includes
PREFILL_SOURCES = [os.path.join(ROOT, "paged_kv_cache_428_b200", "csrc", f)
                   for f in ("common.cuh", "decode.cuh", "decode_mma.cuh", "prefill.cuh", "tc.cuh", "prefill_tc.cuh")]
PROFILES = os.path.join(ROOT, "profiles")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--partition", type=int, default=None, help="tokens per split-context partition")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill-line", action="store_true",
                    help="do not append the chunked-prefill measurement to the default decode line")
    ap.add_argument("--prefill-schedule", choices=("queue", "grid"), default="queue",
                    help="prefill workloads: pa_prefill_ws (one CTA per SM claiming work items) or "
                         "pa_prefill (one CTA per work item)")
    ap.add_argument("--l2", choices=["auto", "write", "write+read", "none"], default="auto",
                    help="between timed steps: write a 2x L2 buffer (write), then also read a second one so the "
                         "flush's dirty lines are written back before the step (write+read), or nothing (none, "
                         "for inputs larger than L2); auto = none when the step reads at least 4x L2 of distinct "
                         "K/V, else write+read")
    ap.add_argument("--warm-l2", action="store_true", help="same as --l2 none")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------------------- ranks
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=_dt.timedelta(seconds=120))
    return dist


def max_over_ranks(values, world: int, device):
    """Element-wise max over ranks (timing only; never on the data path)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def sum_over_ranks(values, world: int, device):
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.tolist()


def shard_seeds(seed: int, world: int):
    """Each rank draws its own batch of the workload shape (weak scaling)."""
    return [seed + 1000 * r for r in range(world)]


# ------------------------------------------------------------------------------------- metrics
def kv_bytes(case) -> int:
    return case.kv_bytes()


def distinct_kv_bytes(case) -> int:
    """K+V bytes of the step that are distinct in memory (shared prompt blocks counted once)."""
    if "unique_tokens" in case.meta:
        return case.meta["unique_tokens"] * case.h_kv * case.d * case.elem_bytes * 2
    return kv_bytes(case)


B200_L2_BYTES = 132120576          # what the device reports; used only where no GPU is visible


def l2_size() -> int:
    import torch
    if torch.cuda.is_available():
        return torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    return B200_L2_BYTES


def l2_plan(args, distinct_bytes: int, l2: int):
    """(mode, description) of what runs between timed steps; see L2Flush."""
    mode = "none" if args.warm_l2 else args.l2
    if mode == "auto":
        mode = "none" if distinct_bytes >= 4 * l2 else "write+read"
    desc = {
        "none": "no flush: every step reads %d distinct bytes of K/V, %.1fx L2 (%d B)"
                % (distinct_bytes, distinct_bytes / l2, l2),
        "write": "flushed between steps (2x L2 write, outside the events)",
        "write+read": "flushed between steps outside the events: 2x L2 written, then a second 2x L2 buffer "
                      "read so that the flush's dirty lines are written back before the step",
    }[mode]
    return mode, desc


def partition_kernel_bytes(case) -> int:
    """Algorithmic bytes of the partition pass: K+V of every context token (ctx*h_kv*d*b*2),
    q (B*h_q*d*2), the block-table entries used (4 per block) and context_lens (4 per seq).
    Split-context partials are implementation overhead and are not counted."""
    ctx = case.context_lens.to("cpu").tolist()
    blocks = sum(-(-c // case.bs) for c in ctx)
    return kv_bytes(case) + case.B * case.h_q * case.d * 2 + 4 * blocks + 4 * case.B


def ctx_desc(case) -> str:
    c = workloads_configs()[case.name]
    if "ctx_range" in c:
        return "U{%d..%d} incl. appended token" % tuple(c["ctx_range"])
    if "ctx_fixed" in c:
        return "%d incl. appended token" % c["ctx_fixed"]
    if "tail_range" in c:
        return "%d-token shared prompt + U{%d..%d} private tail + 1" % ((c["prompt_len"],) + tuple(c["tail_range"]))
    return str(case.context_lens.tolist())


def workloads_configs():
    import workloads
    return workloads.CONFIGS


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(sources=None) -> str:
    h = hashlib.sha256()
    for f in sources or KERNEL_SOURCES:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic_per_launch(workload: str, partition=None, schedule=None, sources=None):
    """DRAM bytes (read + write) of one launch of the workload's kernel from a committed ncu
    summary under profiles/ that names this workload and partition size (decode) or schedule
    (prefill), or None when there is none or the kernel sources changed since the counters were
    taken."""
    if not os.path.isdir(PROFILES):
        return None
    want = kernel_source_hash(sources)
    for name in sorted(os.listdir(PROFILES)):
        if not name.endswith(".md"):
            continue
        text = open(os.path.join(PROFILES, name)).read()
        w = re.search(r"^workload:\s*(\S+)", text, re.M)
        p = re.search(r"^partition:\s*(-?[0-9]+)", text, re.M)
        sc = re.search(r"^schedule:\s*(\S+)", text, re.M)
        m = re.search(r"^traffic_bytes_per_launch:\s*([0-9]+)", text, re.M)
        h = re.search(r"^kernel_source_sha256_16:\s*([0-9a-f]+)", text, re.M)
        if not (w and m and h) or w.group(1) != workload or h.group(1) != want:
            continue
        if partition is not None and not (p and int(p.group(1)) == partition):
            continue
        if schedule is not None and not (sc and sc.group(1) == schedule):
            continue
        return int(m.group(1))
    return None


# -------------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock, power and throttle reasons in the background."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), "pa_bench_clocks_%d.csv" % os.getpid())
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", gpu_id, "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self, t0: float, t1: float):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "nvidia-smi unavailable"}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = _dt.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), parts[4], parts[6:10]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1]
        window = "timed region"
        if not inside and rows:                          # very short timed region: nearest samples
            inside = sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))[:3]
            window = "nearest to timed region"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i in range(4) if r[4][i].lower().startswith("active")})
        pw = [float(r[3]) for r in inside if re.match(r"^[0-9.]+$", r[3])]
        return {"sm_mhz": statistics.median([r[1] for r in inside]) if inside else None,
                "sm_max_mhz": max(r[2] for r in inside) if inside else None,
                "reasons": reasons, "samples": len(inside), "window": window,
                "power_w_max": max(pw) if pw else None}


class NvmlPoller:
    """SM clock, power and clock-event reasons read through NVML every ~0.2 ms by a background
    thread: the timed region of a step loop lasts only milliseconds, shorter than nvidia-smi's
    sampling period, so these are the samples taken inside it."""
    REASONS = [("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap")]

    def __init__(self, uuid: str):
        import threading
        self.rows, self.ok = [], False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_sm = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv, h = self.nv, self.h
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.rows.append((time.time(), sm, rs, pw))
            except Exception:
                pass
            time.sleep(0.0002)

    def stop(self):
        if self.ok:
            self._stop.set()
            self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return None
        inside = [r for r in self.rows if t0 <= r[0] <= t1]
        if not inside:
            return None
        names = [n for n, c in self.REASONS if any(r[2] & getattr(self.nv, c) for r in inside)]
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": self.max_sm,
                "reasons": sorted(names), "samples": len(inside), "window": "timed region (NVML, ~0.2 ms)",
                "power_w_max": round(max(r[3] for r in inside), 1)}


# ---------------------------------------------------------------------------------- our arm
def cow_pairs(case):
    """(src, dst) block pairs of one copy-on-write event of a shared-prompt batch: each prompt's
    last shared block copied into a private block of every sharer but the first."""
    import torch
    pb = case.meta["prompt_blocks"]
    tab = case.block_tables.cpu()
    seen, pairs = set(), []
    for s in range(tab.shape[0]):
        src = int(tab[s, pb - 1])
        if src in seen and int(tab[s, pb]) >= 0:
            pairs.append([src, int(tab[s, pb])])
        seen.add(src)
    return torch.tensor(pairs, dtype=torch.int64).reshape(-1, 2)


def step_config(args, case, P, world, l2_desc):
    """The `config` object of the JSON line; both arms print the same one."""
    per_head = case.per_head_scales
    return {"workload": args.workload, "num_seqs": case.B, "h_q": case.h_q, "h_kv": case.h_kv, "head_dim": case.d,
            "block_size": case.bs, "ctx": ctx_desc(case), "partition": P,
            "num_blocks": case.num_blocks, "kv_bytes_per_step_per_gpu": kv_bytes(case),
            "step": ("pa_decode_step: reshape_and_cache(%d new tokens) + split-context decode with in-kernel "
                     "merge, the decode launched as a programmatic dependent of the write" % case.B
                     if not per_head else
                     "reshape_and_cache(%d new tokens) + split-context decode with in-kernel merge" % case.B),
            "scales": ("per KV head" if per_head else "per tensor") if case.quantised else None,
            "l2": l2_desc,
            "timing": ("one CUDA-event pair around the K back-to-back steps; step_ms_rank0 percentiles from a "
                       "second pass with an event pair per step" if l2_desc.startswith("no flush") else
                       "an event pair per step, the L2 flush between steps outside the events"),
            "parallelism": "replicas (weak scaling, no collective)" if world > 1 else "single GPU"}


def percentiles_ms(xs):
    """p10 / median / p90 of per-step times (ms), nearest-rank."""
    if not xs:
        return None
    v = sorted(xs)
    pick = lambda f: v[min(len(v) - 1, max(0, int(math.ceil(f * len(v))) - 1))]
    return {"p10": round(pick(0.10), 5), "p50": round(pick(0.50), 5), "p90": round(pick(0.90), 5)}


class L2Flush:
    """What runs between timed steps (outside the events).  Writing a buffer of 2x L2 evicts the
    step's data but leaves up to a whole L2 of dirty lines, whose write-back the next step would
    pay for (7 % of the 64-sequence decode); reading a second 2x L2 buffer after it leaves clean
    lines.  A step whose K/V read is several times L2 needs no flush at all."""

    def __init__(self, args, dev, distinct_bytes: int):
        import torch
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.mode, self.desc = l2_plan(args, distinct_bytes, l2)
        self.wbuf = (torch.empty(2 * l2, dtype=torch.uint8, device=dev)
                     if self.mode in ("write", "write+read") else None)
        self.rbuf = torch.ones(2 * l2 // 4, dtype=torch.float32, device=dev) if self.mode == "write+read" else None

    def __call__(self):
        if self.wbuf is not None:
            self.wbuf.zero_()
        if self.rbuf is not None:
            self.rbuf.sum()


def run_ours(args):
    import torch
    import workloads
    import paged_kv_cache_428_b200 as pa

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    seed = shard_seeds(args.seed, world)[rank]
    case = workloads.make_case(args.workload, seed, device=dev)
    P = case.partition if args.partition is None else args.partition
    B, h_q, d = case.B, case.h_q, case.d
    mcl = case.max_context_len
    per_head = case.per_head_scales
    if per_head:
        ks_dev, vs_dev = case.k_scale.to(dev), case.v_scale.to(dev)
        ks_arg, vs_arg = 1.0, 1.0                      # placeholders of the per-tensor arguments
    else:
        ks_arg, vs_arg = case.k_scale, case.v_scale
    if case.quantised:
        # quantise the cached tokens into code pools with the library's own cache write
        # (outside the timed region); the step then writes and quantises the appended tokens
        kc, vc = workloads.empty_quant_pool(case, dev)
        pa.pa_reshape_and_cache(case.fill_k_rows, case.fill_v_rows, kc, vc, case.fill_slots,
                                *((ks_dev, vs_dev) if per_head else (ks_arg, vs_arg)))
        case.fill_k_rows = case.fill_v_rows = None
    else:
        kc, vc = case.k_cache, case.v_cache
    q, k_new, v_new = case.q, case.key_new, case.value_new
    slots, tables, ctx = case.slot_mapping, case.block_tables, case.context_lens
    out = torch.empty((B, h_q, d), dtype=torch.bfloat16, device=dev)
    ws = pa.make_workspace(B, h_q, d, mcl, P, dev)
    flush = L2Flush(args, dev, distinct_kv_bytes(case))
    stream = torch.cuda.Stream(device=dev)

    # argument checks once; the timed loop calls the C ABI directly (which still validates),
    # so that the host stays ahead of the GPU
    L = pa.lib()
    sp = stream.cuda_stream
    rargs = pa.reshape_call_args(k_new, v_new, kc, vc, slots, ks_arg, vs_arg)
    dargs = pa.decode_call_args(out, q, kc, vc, tables, ctx, mcl, case.scale, P, ks_arg, vs_arg, workspace=ws)
    margs = pa.merge_call_args(out, ctx, mcl, P, ws)
    if per_head:
        # per-KV-head scales: the *_head_scales calls (their decode call includes the merge
        # pass, which launches nothing while every group has at most 16 partitions)
        hp = (ks_dev.data_ptr(), vs_dev.data_ptr())
        write_call = lambda ra, s_: L.pa_reshape_and_cache_head_scales(*ra[:-2], *hp, s_)
        part_call = lambda da, s_: L.pa_decode_head_scales(*da[:16], *hp, *da[18:], s_)
        decode_call = part_call
    else:
        write_call = lambda ra, s_: L.pa_reshape_and_cache(*ra, s_)
        part_call = lambda da, s_: L.pa_decode_partitions(*da, s_)
        decode_call = lambda da, s_: L.pa_decode(*da, s_)

    # the step: pa_decode_step (the decode overlaps the cache write) for per-tensor scales, the
    # separate calls for per-head scales
    sargs = None if per_head else pa.step_call_args(k_new, v_new, slots, out, q, kc, vc, tables, ctx, mcl, case.scale,
                                                    P, ks_arg, vs_arg, workspace=ws)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        if sargs is not None:
            rc = L.pa_decode_step(*sargs, sp)
        else:
            rc = write_call(rargs, sp)
            rc |= part_call(dargs, sp)
            rc |= L.pa_decode_merge(*margs, sp)
        if evs:
            evs[1].record(stream)
        if rc:
            raise SystemExit("library call failed: %d" % rc)

    def timed(body, n_ev, nvtx, per_step_events=False):
        """Run `body` for args.steps steps; returns the time of the steps (ms; with n_ev > 2, the
        summed intervals between consecutive events).  Barrier + synchronize on both sides.
        Without an L2 flush the steps run back to back between one pair of events, as a decode
        loop runs them; with a flush (or per_step_events) every step has its own event pair and
        the flush runs outside them."""
        if flush.mode == "none" and not per_step_events and n_ev == 2:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(dev)
            torch.cuda.nvtx.range_push(nvtx)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for i in range(args.steps):
                    body(None)
                e1.record(stream)
            torch.cuda.synchronize(dev)
            torch.cuda.nvtx.range_pop()
            if world > 1:
                dist.barrier()
            return [e0.elapsed_time(e1)]
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        torch.cuda.nvtx.range_push(nvtx)
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                flush()
                body(evs[i])
        torch.cuda.synchronize(dev)
        torch.cuda.nvtx.range_pop()
        if world > 1:
            dist.barrier()
        per_step[:] = [e[0].elapsed_time(e[n_ev - 1]) for e in evs]
        return [sum(e[k].elapsed_time(e[k + 1]) for e in evs) for k in range(n_ev - 1)]

    per_step = []                      # the last timed() call's per-step intervals (ms)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    poller = NvmlPoller(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    time.sleep(0.3)                    # the samplers start; the warm-up then runs right before the timing
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush()
            step()
    torch.cuda.synchronize(dev)
    t0 = time.time()
    # the timed region: K whole steps
    step_ms = timed(step, 2, "timed")[0]
    t1 = time.time()
    if flush.mode == "none":                 # per-step spread from a second pass, an event pair per step
        timed(step, 2, "per_step", per_step_events=True)
    step_pct = percentiles_ms(per_step)

    # each kernel alone over K launches (for the roofline and the per-kernel split); an event
    # pair itself reads about 2.7 us on this GPU, so these per-kernel times are slight overestimates
    def only(fn, args_):
        def body(evs):
            if evs:
                evs[0].record(stream)
            rc = fn(*args_, sp)
            if evs:
                evs[1].record(stream)
            if rc:
                raise SystemExit("library call failed: %d" % rc)
        return body
    write_ms = timed(only(lambda *a: write_call(a[:-1], a[-1]), rargs), 2, "kernel_write")[0]
    part_ms = timed(only(lambda *a: part_call(a[:-1], a[-1]), dargs), 2, "kernel_decode")[0]
    merge_launches = P > 0 and -(-mcl // P) > 16
    merge_ms = timed(only(L.pa_decode_merge, margs), 2, "kernel_merge")[0] if merge_launches else 0.0
    # shared prompts: one copy-on-write event (pa_copy_blocks), timed alone on a scratch copy of
    # the caches so that the attention workload above is untouched
    cow = cow_pairs(case) if "prompt_blocks" in case.meta and not case.quantised else None
    copy_ms = 0.0
    if cow is not None and cow.shape[0] > 0:
        kc_s, vc_s, cow_dev = kc.clone(), vc.clone(), cow.to(dev)

        def copy_body(evs):
            if evs:
                evs[0].record(stream)
            pa.pa_copy_blocks([kc_s], [vc_s], cow_dev, stream=stream)
            if evs:
                evs[1].record(stream)
        copy_ms = timed(copy_body, 2, "kernel_copy_blocks")[0]
        del kc_s, vc_s
    t2 = time.time()
    time.sleep(0.1)
    sampler.stop()
    poller.stop()
    clocks = poller.summary(t0, t1) or sampler.summary(t0, t1)
    clocks_kernels = poller.summary(t1, t2) or sampler.summary(t1, t2)

    # end to end through the public calls: pinned host inputs in, result out, every step
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, pa, L, case, kc, vc, q, k_new, v_new, slots, tables, ctx, mcl, P, ks_arg, vs_arg,
                      write_call, decode_call, per_head, stream, dev, world, dist, flush)

    errs = pa.pa_device_errors(clear=True)
    if errs:
        raise SystemExit("device error bits 0x%x during the benchmark" % errs)

    my_bytes = kv_bytes(case)
    mx = max_over_ranks([step_ms, part_ms, merge_ms, write_ms, e2e["ms"] if e2e else 0.0], world, dev)
    tot_bytes, tot_seqs = sum_over_ranks([float(my_bytes), float(B)], world, dev)
    step_ms, part_ms, merge_ms, write_ms, e2e_ms = mx
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return None

    K = args.steps
    per_step_s = step_ms / 1e3 / K
    # the kernel the library dispatches to for this cache type (the same switches as pa_lib.cu)
    if case.cache == "e4m3" and os.environ.get("PA_DECODE_E4M3_CUDA_CORES") == "1":
        kernel = "paged_decode_partition_kernel (E4M3, CUDA cores)"
    elif case.quantised:
        kernel = "paged_decode_partition_q8_kernel (%s codes converted in registers, tensor cores)" % case.cache.upper()
    elif os.environ.get("PA_DECODE_BF16_CUDA_CORES") == "1":
        kernel = "paged_decode_partition_kernel (bf16, CUDA cores)"
    elif P == -1 and os.environ.get("PA_DECODE_AUTO_WHOLE_BLOCK") == "1" and case.h_kv == 8 and case.bs in (16, 32):
        kernel = "paged_decode_allheads_kernel + paged_decode_allheads_merge_kernel"
    elif P == -1:
        kernel = "paged_decode_balanced_kernel"
    else:
        kernel = "paged_decode_partition_mma_kernel"
    value = tot_bytes / per_step_s / 1e9
    peak, peak_kind = measured_peaks()
    part_bytes = partition_kernel_bytes(case)
    achieved = part_bytes / (part_ms / 1e3 / K) / 1e9
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms / K, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 q/out, %s KV, fp32 accumulate" % case.cache,
        "data": "synthetic",
        "config": step_config(args, case, P, world, flush.desc),
        "tokens_per_s": round(tot_seqs / per_step_s, 1),
        "tokens_per_s_32_layer_attention_only": round(tot_seqs / per_step_s / 32, 1),
        "step_ms_rank0": step_pct,
        "pct_of_hbm_peak": round(value / world / peak, 4),
        "pct_of_nominal_8tbs": round(value / world / 8000.0, 4),
        "kernels_ms_alone": {"reshape_and_cache": round(write_ms / K, 5),
                             "decode (partitions + in-kernel merge)": round(part_ms / K, 5),
                             "note": ("each kernel timed alone over K back-to-back launches after the timed steps, "
                                      "one CUDA-event pair around them" if flush.mode == "none" else
                                      "each kernel timed alone over K launches after the timed steps, an event pair "
                                      "per launch (an empty pair reads ~2.7 us and is included)")},
        "roofline": {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 1),
                     "peak": peak, "peak_kind": peak_kind + " (hbm_gbs copy bandwidth)", "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": ncu_traffic_per_launch(args.workload, P),
                     "algorithmic_bytes_per_launch": part_bytes},
        "gpu_launches": K * (2 + (1 if P > 0 and -(-mcl // P) > 16 else 0)),
        "clocks": clocks,
        "clocks_kernel_loops": clocks_kernels,
    }
    if merge_launches:
        line["kernels_ms_alone"]["merge"] = round(merge_ms / K, 5)
    if "unique_tokens" in case.meta:      # shared prompts: bytes that are distinct in memory
        ub = case.meta["unique_tokens"] * case.h_kv * d * case.elem_bytes * 2
        line["unique_kv_GBs"] = round(ub * world / per_step_s / 1e9, 2)
    if cow is not None and cow.shape[0] > 0:
        moved = 2 * 2 * int(cow.shape[0]) * case.h_kv * case.bs * d * case.elem_bytes   # K and V, read + written
        line["copy_blocks"] = {"pairs_per_event": int(cow.shape[0]), "us_per_event": round(copy_ms / K * 1e3, 2),
                               "bytes_per_event": moved, "GBs": round(moved / (copy_ms / 1e3 / K) / 1e9, 1),
                               "event": "each prompt's last shared block copied for every sharer but one",
                               "note": "rank 0's time; an empty CUDA-event pair (~2.7 us) is included"}
    if e2e:
        line["e2e"] = {"value": round(tot_bytes / (e2e_ms / 1e3 / K) / 1e9, 2), "unit": "GB/s",
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": round(e2e_ms / K, 5),
                       "loop": "pa_decode_step through the C ABI; inputs copied in from pinned host memory and out "
                               "copied back every step, double-buffered on two copy streams so that copies overlap "
                               "the neighbouring steps' decode; timed from the first copy in to the last copy out; "
                               + ("L2: " + flush.desc if flush.mode == "none" else
                                  "L2 not flushed between steps: the step's %d distinct bytes of K/V stay partly in "
                                  "L2 (warm)" % distinct_kv_bytes(case))}
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case)
        line["cpu_baseline_omp"] = cpu_baseline_omp(case)
    if world > 1:
        dist.destroy_process_group()
    return line


def run_e2e(args, pa, L, case, kc, vc, q, k_new, v_new, slots, tables, ctx, mcl, P, ks_arg, vs_arg,
            write_call, decode_call, per_head, stream, dev, world, dist, flush):
    """The step end to end through the C ABI, as a decode loop runs it: each step's inputs (q, the
    new K/V rows, slot ids, block tables, context lengths) are copied in from one pinned host
    buffer, pa_decode_step runs, and `out` is copied back to pinned host memory.  Consecutive
    steps are pipelined: two input buffers and two outputs, the host-to-device copies on one
    stream and the device-to-host copies on another, ordered by events, so that step i+1's
    inputs arrive and step i-1's output leaves while step i decodes.  The loop never flushes L2
    (a flush would be work of its own inside the loop); where the step's distinct K/V is smaller
    than several L2s the line says so.  Returns the time of K steps (first copy in to last copy
    out)."""
    import torch
    B, h_q, d = case.B, case.h_q, case.d
    parts = [("q", q), ("k_new", k_new), ("v_new", v_new), ("slots", slots), ("tables", tables), ("ctx", ctx)]
    offs, total = {}, 0
    for n, t in parts:
        offs[n] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    view = lambda buf, n, t: buf[offs[n]: offs[n] + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
    host_in, dev_in, outs, out_host, sargs = [], [], [], [], []
    for _ in range(2):
        hb = torch.empty(total, dtype=torch.uint8).pin_memory()
        for n, t in parts:
            view(hb, n, t).copy_(t.cpu())
        db = torch.empty(total, dtype=torch.uint8, device=dev)
        dv = {n: view(db, n, t) for n, t in parts}
        o = torch.empty((B, h_q, d), dtype=torch.bfloat16, device=dev)
        ws = pa.make_workspace(B, h_q, d, mcl, P, dev)
        if per_head:
            ra = pa.reshape_call_args(dv["k_new"], dv["v_new"], kc, vc, dv["slots"], ks_arg, vs_arg)
            da = pa.decode_call_args(o, dv["q"], kc, vc, dv["tables"], dv["ctx"], mcl, case.scale, P, ks_arg, vs_arg,
                                     workspace=ws)
            sargs.append(("split", ra, da, ws))
        else:
            sa = pa.step_call_args(dv["k_new"], dv["v_new"], dv["slots"], o, dv["q"], kc, vc, dv["tables"], dv["ctx"],
                                   mcl, case.scale, P, ks_arg, vs_arg, workspace=ws)
            sargs.append(("step", sa, None, ws))
        host_in.append(hb)
        dev_in.append(db)
        outs.append(o)
        out_host.append(torch.empty((B, h_q, d), dtype=torch.bfloat16).pin_memory())
    h2d = sum(t.numel() * t.element_size() for _, t in parts)
    d2h = out_host[0].numel() * out_host[0].element_size()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    sp = stream.cuda_stream
    ev_in = [torch.cuda.Event() for _ in range(2)]          # inputs of the buffer's step have landed
    ev_dec = [torch.cuda.Event() for _ in range(2)]         # the buffer's step decoded (inputs read, out written)
    ev_out = [torch.cuda.Event() for _ in range(2)]         # the buffer's output copied out

    def loop(n):
        for i in range(n):
            b = i % 2
            if i >= 2:
                s_in.wait_event(ev_dec[b])                  # step i-2 has finished with this input buffer
            with torch.cuda.stream(s_in):
                dev_in[b].copy_(host_in[b], non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])                # step i-2's output has left this buffer
            kind, a1, a2, _ = sargs[b]
            if kind == "step":
                rc = L.pa_decode_step(*a1, sp)
            else:
                rc = write_call(a1, sp)
                rc |= decode_call(a2, sp)
            if rc:
                raise SystemExit("library call failed: %d" % rc)
            ev_dec[b].record(stream)
            s_out.wait_event(ev_dec[b])
            with torch.cuda.stream(s_out):
                out_host[b].copy_(outs[b], non_blocking=True)
            ev_out[b].record(s_out)

    loop(args.warmup)
    torch.cuda.synchronize(dev)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    torch.cuda.nvtx.range_push("timed_e2e")
    t_start.record(s_in)
    loop(args.steps)
    s_out.wait_event(ev_out[(args.steps - 1) % 2])
    t_end.record(s_out)
    torch.cuda.synchronize(dev)
    torch.cuda.nvtx.range_pop()
    got = out_host[(args.steps - 1) % 2]
    if not torch.equal(got.view(torch.int16), outs[(args.steps - 1) % 2].cpu().view(torch.int16)):
        raise SystemExit("e2e: the copied-out result differs from the device result")
    return {"ms": t_start.elapsed_time(t_end), "h2d": h2d, "d2h": d2h}


def oracle_step_state(case, orc):
    """The oracle's caches before the step (quantised by the oracle itself for E4M3 / INT8 caches,
    untimed) and the keyword arguments of its calls."""
    import numpy as np
    import torch
    import workloads
    u16 = lambda t: t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    ks, vs = case.k_scale, case.v_scale
    if case.per_head_scales:
        ks, vs = ks.numpy(), vs.numpy()
    kw = dict(h_kv=case.h_kv, bs=case.bs, cache=case.cache, k_scale=ks, v_scale=vs)
    if case.quantised:
        shape = (case.num_blocks, case.h_kv, case.bs, case.d)
        if case.cache == "int8":
            kc = np.full(shape, workloads.INT8_UNUSED, np.int8)
        else:
            kc = np.full(shape, workloads.E4M3_NAN, np.uint8)
        vc = kc.copy()
        orc.reshape_and_cache(u16(case.fill_k_rows), u16(case.fill_v_rows), kc, vc, case.fill_slots.cpu().numpy(),
                              d=case.d, num_blocks=case.num_blocks, **kw)
    else:
        kc, vc = u16(case.k_cache).copy(), u16(case.v_cache).copy()
    return kc, vc, kw


def cpu_baseline(case):
    """The oracle as it stands, single-threaded, on the host: the whole step (cache write of the
    appended tokens and every (sequence, query head) row of the decode), once."""
    import numpy as np
    import torch
    import oracle
    import workloads
    orc = oracle.load()
    u16 = lambda t: t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    if case.quantised:            # the bench's own copy dropped the fill rows: draw them again
        case = workloads.make_case(case.name, case.meta["seed"])
    kc, vc, kw = oracle_step_state(case, orc)
    q, kn, vn = u16(case.q), u16(case.key_new), u16(case.value_new)
    tab, ctx, sl = case.block_tables.cpu().numpy(), case.context_lens.cpu().numpy(), case.slot_mapping.cpu().numpy()
    t0 = time.perf_counter()
    orc.reshape_and_cache(kn, vn, kc, vc, sl, d=case.d, num_blocks=case.num_blocks, **kw)
    orc.paged_decode(q, kc, vc, tab, ctx, scale=case.scale, **kw)
    dt = time.perf_counter() - t0
    line = {"value": round(kv_bytes(case) / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "seconds": round(dt, 2), "host_cpus": os.cpu_count(),
            "sample": "one full step of the workload (cache write of %d tokens + all %d x %d decode rows), "
                      "single-threaded fp64 C" % (case.B, case.B, case.h_q)}
    return line


def cpu_baseline_omp(case):
    """The same oracle source built with OpenMP (rows shared out over the host's threads), on the
    same whole step: a second, multi-core reference point."""
    import numpy as np
    import torch
    import oracle
    import workloads
    orc = oracle.load(openmp=True)
    u16 = lambda t: t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    if case.quantised:
        case = workloads.make_case(case.name, case.meta["seed"])
    kc, vc, kw = oracle_step_state(case, orc)
    q, kn, vn = u16(case.q), u16(case.key_new), u16(case.value_new)
    tab, ctx, sl = case.block_tables.cpu().numpy(), case.context_lens.cpu().numpy(), case.slot_mapping.cpu().numpy()
    t0 = time.perf_counter()
    orc.reshape_and_cache(kn, vn, kc, vc, sl, d=case.d, num_blocks=case.num_blocks, **kw)
    orc.paged_decode(q, kc, vc, tab, ctx, scale=case.scale, **kw)
    dt = time.perf_counter() - t0
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": round(kv_bytes(case) / dt / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle, OpenMP build of the same source", "seconds": round(dt, 3),
            "sample": "one full step of the workload, the decode rows over %d host threads" % threads}


# ---------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The CPU oracle on the host cores, on a bounded sample of the same workload per step."""
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    import numpy as np
    import torch
    import oracle
    import workloads
    orc = oracle.load()
    case = workloads.make_case(args.workload, args.seed)
    u16 = lambda t: t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    kc, vc, kw = oracle_step_state(case, orc)
    q, kn, vn = u16(case.q), u16(case.key_new), u16(case.value_new)
    tab, ctx, sl = case.block_tables.numpy(), case.context_lens.numpy(), case.slot_mapping.numpy()
    orc.reshape_and_cache(kn, vn, kc, vc, sl, d=case.d, num_blocks=case.num_blocks, **kw)
    g = case.h_q // case.h_kv
    all_rows = [(s, h) for s in range(case.B) for h in range(case.h_q)]
    kw["scale"] = case.scale
    row_bytes = lambda r: int(ctx[r[0]]) * case.d * case.elem_bytes * 2 / g   # 1/g of the KV head's bytes
    probe = all_rows[:case.h_q]                                    # sequence 0's rows: the cost per byte
    t = time.perf_counter()
    orc.paged_decode_rows(probe, q, kc, vc, tab, ctx, **kw)
    per_byte = (time.perf_counter() - t) / max(1.0, sum(row_bytes(r) for r in probe))
    step_s = per_byte * sum(row_bytes(r) for r in all_rows)        # the whole workload, estimated
    budget = 150.0 / max(1, args.steps + args.warmup)             # whole run within a few minutes
    # the whole workload per step when it fits the budget, else a rotating sample of its rows
    n_rows = len(all_rows) if step_s <= budget else int(max(1, len(all_rows) * budget / step_s))
    pos = 0

    def take():
        nonlocal pos
        rows = [all_rows[(pos + i) % len(all_rows)] for i in range(n_rows)]
        pos = (pos + n_rows) % len(all_rows)
        return rows

    for _ in range(args.warmup):
        orc.paged_decode_rows(take(), q, kc, vc, tab, ctx, **kw)
    tot_s, tot_b = 0.0, 0.0
    whole = n_rows == len(all_rows)
    wkw = {k: v for k, v in kw.items() if k != "scale"}
    for _ in range(args.steps):
        rows = take()
        t = time.perf_counter()
        if whole:                  # the whole step: the appended tokens' cache write, then every row
            orc.reshape_and_cache(kn, vn, kc, vc, sl, d=case.d, num_blocks=case.num_blocks, **wkw)
        orc.paged_decode_rows(rows, q, kc, vc, tab, ctx, **kw)
        tot_s += time.perf_counter() - t
        tot_b += sum(row_bytes(r) for r in rows)
    value = tot_b / tot_s / 1e9
    if whole:
        sample = ("the whole workload every step: cache write of the %d appended tokens and all %d (sequence, "
                  "query head) decode rows, single-threaded fp64 C" % (case.B, len(all_rows)))
    else:
        sample = ("%d of %d (sequence, query head) decode rows per step, rotating through the batch"
                  % (n_rows, len(all_rows)))
    return {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_s / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": step_config(args, case, case.partition if args.partition is None else args.partition, world,
                                  l2_plan(args, distinct_kv_bytes(case), l2_size())[1]),
            "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------- prefill mode
def measured_bf16_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (cuBLAS bf16 burst)"
    return 1590.0, "fallback"


def prefill_kernel_name(schedule: str) -> str:
    """The prefill kernel the call dispatches to (PA_PREFILL_MMA_SYNC=1 selects the mma.sync one)."""
    if os.environ.get("PA_PREFILL_MMA_SYNC") == "1":
        return "paged_prefill_kernel (mma.sync bf16)"
    how = "one CTA per SM claiming work items" if schedule == "queue" else "one CTA per work item"
    return "paged_prefill_tc_kernel (tcgen05.mma bf16, fp32 accumulators in tensor memory; %s)" % how


def run_prefill(args):
    """--workload prefill_*: each step writes the chunks' K/V (pa_reshape_and_cache of every
    chunk token) and runs pa_prefill; reported as attention TFLOP/s against the bf16 peak."""
    import torch
    import workloads
    import paged_kv_cache_428_b200 as pa

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    seed = shard_seeds(args.seed, world)[rank]
    case = workloads.make_prefill_case(args.workload, seed, device=dev)
    kc, vc = case.k_cache, case.v_cache
    out = torch.empty_like(case.q)
    flush = L2Flush(args, dev, int(case.context_lens.sum().item()) * case.h_kv * case.d * 2 * 2)
    stream = torch.cuda.Stream(device=dev)
    L, sp = pa.lib(), stream.cuda_stream
    rargs = pa.reshape_call_args(case.key_new, case.value_new, kc, vc, case.slot_mapping)
    pargs = pa.prefill_call_args(out, case.q, kc, vc, case.block_tables, case.query_start, case.context_lens,
                                 case.max_query_len, case.scale)

    def timed(calls, n_steps):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            for i in range(n_steps):
                flush()
                evs[i][0].record(stream)
                rc = 0
                for fn, a in calls:
                    rc |= fn(*a, sp)
                evs[i][1].record(stream)
                if rc:
                    raise SystemExit("library call failed: %d" % rc)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        per_step[:] = [a.elapsed_time(b) for a, b in evs]
        return sum(per_step)

    per_step = []
    if args.prefill_schedule == "queue":
        ws = pa.make_prefill_workspace(dev)
        pcall = (L.pa_prefill_ws, pargs + (ws.data_ptr(), ws.numel()))
    else:
        pcall = (L.pa_prefill, pargs)
    step = [(L.pa_reshape_and_cache, rargs), pcall]
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    poller = NvmlPoller(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    time.sleep(0.3)                    # the samplers start; the warm-up then runs right before the timing
    timed(step, args.warmup)
    t0 = time.time()
    step_ms = timed(step, args.steps)
    step_pct = percentiles_ms(per_step)
    t1 = time.time()
    kern_ms = timed([pcall], args.steps)
    t2 = time.time()
    time.sleep(0.1)
    sampler.stop()
    poller.stop()
    errs = pa.pa_device_errors(clear=True)
    if errs:
        raise SystemExit("device error bits 0x%x during the benchmark" % errs)
    flops = float(case.attention_flops())
    T = float(case.q.shape[0])
    step_ms, kern_ms = max_over_ranks([step_ms, kern_ms], world, dev)
    tot_flops, tot_tok = sum_over_ranks([flops, T], world, dev)
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return None
    K = args.steps
    peak, kind = measured_bf16_peak()
    achieved = flops / (kern_ms / 1e3 / K) / 1e12
    line = {
        "metric": "chunked-prefill attention TFLOP/s over the paged KV cache; prefill tokens/s",
        "value": round(tot_flops / (step_ms / 1e3 / K) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(step_ms / K, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 in, fp32 accumulate", "data": "synthetic",
        "config": {"workload": args.workload, "num_seqs": case.B, "h_q": case.h_q, "h_kv": case.h_kv,
                   "head_dim": case.d, "block_size": case.bs, "chunk_tokens": int(T),
                   "cached_tokens": case.meta["cached"], "chunk_lens": case.meta["chunk"],
                   "attention_flops_per_step": int(flops),
                   "step": "reshape_and_cache(all chunk tokens) + %s" % pcall[0].__name__,
                   "schedule": args.prefill_schedule,
                   "l2": flush.desc},
        "tokens_per_s": round(tot_tok / (step_ms / 1e3 / K), 1),
        "step_ms_rank0": step_pct,
        "kernels_ms_alone": {"prefill": round(kern_ms / K, 5)},
        "roofline": {"bound": "tensor", "kernel": prefill_kernel_name(args.prefill_schedule), "achieved": round(achieved, 1),
                     "peak": peak, "peak_kind": kind, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": ncu_traffic_per_launch(args.workload, schedule=args.prefill_schedule,
                                                       sources=PREFILL_SOURCES),
                     "algorithmic_flops_per_launch": int(flops)},
        "gpu_launches": 2 * K,
        "clocks": poller.summary(t0, t1) or sampler.summary(t0, t1),
        "clocks_kernel_loops": poller.summary(t1, t2) or sampler.summary(t1, t2),
    }
    if world > 1:
        dist.destroy_process_group()
    return line


PREFILL_SIDE_WORKLOAD = "prefill_llama3_8b_b8_chunk512"


def prefill_side_line(args) -> dict:
    """The chunked-prefill row measured in the same run as the default decode line (one GPU):
    the same method as `--workload prefill_llama3_8b_b8_chunk512`, fewer steps.  A failure here is
    reported in the object and never costs the decode line."""
    try:
        pargs = parse_args(["--workload", PREFILL_SIDE_WORKLOAD, "--steps", "10", "--warmup", "3", "--no-cpu-baseline",
                            "--no-e2e", "--seed", str(args.seed)])
        pl = run_prefill(pargs)
        keep = ("metric", "value", "unit", "steps", "warmup", "ms_per_step", "tokens_per_s", "kernels_ms_alone",
                "roofline", "clocks")
        out = {k: pl[k] for k in keep if k in pl}
        out["config"] = {k: pl["config"][k] for k in ("workload", "schedule", "step", "attention_flops_per_step", "l2")
                         if k in pl["config"]}
        return out
    except Exception as e:                                      # pragma: no cover - reported, not raised
        return {"workload": PREFILL_SIDE_WORKLOAD, "error": repr(e)[:300]}


def main(argv=None):
    args = parse_args(argv)
    if args.impl != "reference" and args.workload.startswith("prefill_"):
        line = run_prefill(args)
    else:
        line = run_reference(args) if args.impl == "reference" else run_ours(args)
        if (line is not None and args.impl != "reference" and line.get("n_gpus") == 1 and not args.no_prefill_line
                and args.workload == DEFAULT_WORKLOAD):
            line["prefill"] = prefill_side_line(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
