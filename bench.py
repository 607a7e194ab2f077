#!/usr/bin/env python
"""Benchmark one decode step of the paged KV cache on B200: the new token's K/V
append (reshape_and_cache) followed by paged decode attention over every
running sequence, on a seeded synthetic batch resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 3] [--impl ours|reference]

Prints ONE JSON line (rank 0). ``value`` is the step's algorithmic bytes
(K/V tiles of every distinct referenced block, q, out, block tables and
seq_lens, plus the append's rows and slots) per second of device time, summed
over ranks (each rank runs its own replica: the path has no exchange step).
``roofline`` reports the decode kernel alone against the measured HBM copy
bandwidth. ``e2e`` repeats the step with every per-step input copied in from
pinned host memory and the output copied back inside the timed region.
``targets`` times the other points of the throughput target (long-context and
mixed-batch workloads with bf16 and E4M3 caches) the same way in the same run.
``--impl reference`` times the CPU oracle (fp64, one core) on the same
workload, a bounded sample per step.
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
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402
from paged_kv_cache_462_b200 import accounting as acct  # noqa: E402

METRIC = "paged decode KV GB/s & seq-steps/s vs B200 HBM roofline; oracle CPU time"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20   # > 126 MB of L2: read before every step so the step starts with a cold L2


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=int, default=3,
                    help="workload 0..4 (default 3: the mixed batch with shared prefixes, bf16, the largest)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--partitions", type=int, default=0, help="decode runs (0 = automatic)")
    ap.add_argument("--q-len", type=int, default=1,
                    help="new tokens per sequence: > 1 times the causal multi-query decode instead of the step")
    ap.add_argument("--kv-dtype", choices=["bf16", "e4m3", "e5m2", "int8"], default=None,
                    help="run the workload with this cache dtype instead of its own (configs 1-4)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle sample length for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--prefix-sharing", choices=["auto", "on", "off"], default="auto",
                    help="shared-prefix decode (blocks a plan shares read once per group): auto = on for "
                         "workloads whose sequences share prefix blocks (config 3) with a bf16 cache, off with "
                         "an 8-bit cache (there the plain step measured faster)")
    ap.add_argument("--num-seqs", type=int, default=None,
                    help="cut the workload down to its first N sequences' draw (same distributions; for profiling "
                         "captures that must stay small)")
    ap.add_argument("--fp8-kernel", choices=["mma", "tcgen05"], default="mma",
                    help="kernel for E4M3 / E5M2 caches (pkv_set_fp8_kernel): warp-level MMA on widened codes "
                         "(default) or tcgen05 on the 8-bit tiles")
    ap.add_argument("--no-targets", action="store_true",
                    help="skip the extra target points (long-context and mixed batch, bf16 and E4M3 caches)")
    return ap.parse_args()


# The throughput target names two workloads (long context: config 2; mixed batch with shared
# prefixes: config 3) with bf16 and FP8 E4M3 caches; the points other than the main line's are
# timed in the same run, with the same step count, and reported under "targets".
TARGET_POINTS = ((2, "bf16"), (2, "e4m3"), (3, "bf16"), (3, "e4m3"))


def workload_spec(args) -> W.Spec:
    """The config's workload, with the cache dtype replaced when --kv-dtype asks for it (q and the
    appended rows stay bf16; an E4M3 cache gets per-tensor absmax/448 scales)."""
    spec = W.config_spec(args.config)
    if args.num_seqs is not None:
        spec.num_seqs = args.num_seqs
        spec.name = f"{spec.name}_{args.num_seqs}seqs"
    if args.kv_dtype is not None:
        if spec.q_dtype != "bf16":
            raise SystemExit("--kv-dtype applies to the bf16-query workloads (configs 1-4)")
        spec.kv_dtype = args.kv_dtype
        spec.name = f"{spec.name}_{args.kv_dtype}kv" if args.kv_dtype not in spec.name else spec.name
    return spec


def describe(b: W.DecodeBatch) -> str:
    sp = b.spec
    return (f"{sp.name}: {sp.num_seqs} seqs, lengths {sp.lengths}, {sp.num_heads}q/{sp.num_kv_heads}kv heads, "
            f"head_dim {sp.head_dim}, block {sp.block_size}, pool {b.num_blocks} blocks, kv {sp.kv_dtype}, q {sp.q_dtype}"
            + (f", prefix groups of {sp.share_group} sharing <= {sp.share_blocks} blocks" if sp.share_group else ""))


def step_bytes(b: W.DecodeBatch, q_len: int = 1, plan=None):
    """Algorithmic bytes of the step: decode (q/out rows scale with q_len; with a shared-prefix
    plan the table entries of shared blocks are replaced by the plan's arrays), and the append
    (none in the multi-query form, whose new tokens are already in the cache)."""
    sp = b.spec
    dec = acct.decode_bytes(b.seq_lens, b.block_tables, sp.num_heads * q_len, sp.num_kv_heads, sp.head_dim,
                            sp.block_size, sp.kv_dtype, sp.q_dtype)
    if plan is not None:
        pb = acct.plan_bytes(b.seq_lens, sp.block_size, plan)
        dec["tables"] += pb["plan"] - pb["tables_saved"]
        dec["total"] += pb["plan"] - pb["tables_saved"]
    app = 0 if q_len > 1 else acct.append_bytes(int((b.new_slots >= 0).sum()), sp.num_kv_heads, sp.head_dim,
                                                sp.in_dtype, sp.kv_dtype)
    return dec, app


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_traffic(config: int, kv: str, prefix: bool):
    """DRAM bytes (read + written) per step of the decode kernels, from the committed ncu summary
    of this workload, if it was captured on this kernel build (else None)."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            recs = json.load(f)["records"]
    except Exception:
        return None
    for rec in recs:
        if (rec.get("kernel_sha") == kernel_sha() and int(rec.get("config", -1)) == config
                and rec.get("kv") == kv and bool(rec.get("prefix_sharing")) == prefix
                and rec.get("num_seqs") is None):
            return rec.get("dram_bytes_per_step")
    return None


def kernel_sha() -> str:
    h = hashlib.sha256()
    for name in ("decode_mma.cuh", "decode_kernel.cuh", "device.cuh", "decode_mma_dispatch.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_462_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock, power and throttle reasons sampled during the timed region (read-only queries).

    NVML is polled every ~1 ms from a thread (nvidia-smi's 20 ms loop saw no sample at all in a
    timed region of a few milliseconds); without NVML, ``nvidia-smi -lms 20`` is read instead.
    Every sample carries its time, and ``summary(t0, t1)`` keeps those inside [t0, t1]."""

    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: str, period_s: float = 0.001):
        self.samples = []          # (time, sm MHz, max sm MHz, set of active reason names)
        self.source = None
        self.proc = None
        self._stop = threading.Event()
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(int(device_index))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                         "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                         "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                         "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            self.source = "nvml"
            self.t = threading.Thread(target=self._poll_nvml, daemon=True)
        except Exception:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "20",
                     "-i", str(device_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi"
                self.t = threading.Thread(target=self._read_smi, daemon=True)
            except Exception:
                self.t = None
        if self.t is not None:
            self.t.start()

    def _poll_nvml(self):
        nv, h = self.nv, self.h
        while not self._stop.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                self.samples.append((time.perf_counter(), mhz, self.max_mhz,
                                     {n for n, b in self.bits.items() if r & b}))
            except Exception:
                pass
            time.sleep(self.period)

    def _read_smi(self):
        for line in self.proc.stdout:
            f = [x.strip() for x in line.split(",")]
            try:
                self.samples.append((time.perf_counter(), float(f[1]), float(f[2]),
                                     {n for n, v in zip(self.REASONS, f[5:9]) if v.lower() == "active"}))
            except (ValueError, IndexError):
                continue

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=5)

    def summary(self, t0: float, t1: float):
        """Median SM clock, max clock and the union of active reasons over samples in [t0, t1]."""
        inside = [x for x in self.samples if t0 <= x[0] <= t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source,
                    "window_ms": 1e3 * (t1 - t0)}
        reasons = set()
        for x in inside:
            reasons |= x[3]
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": max(x[2] for x in inside),
                "reasons": sorted(reasons), "samples": len(inside), "source": self.source,
                "window_ms": 1e3 * (t1 - t0)}


def smi_index(torch, dev: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        parts = [p.strip() for p in vis.split(",") if p.strip()]
        if dev < len(parts):
            return parts[dev]
    return str(dev)


# ----------------------------------------------------------------------------- ranks

MAX_KEYS = ("ms", "decode_ms", "e2e_ms", "errors")      # timed over ranks: the slowest rank counts
SUM_KEYS = ("step_bytes",)                               # work: every replica's bytes count


def aggregate_ranks(torch, dist, device, **vals):
    """Whole-job figures: the max over ranks of the times and error words, the sum of the bytes.

    With dist None (one process) the values are returned unchanged. Works on any process-group
    backend (NCCL with a CUDA device, gloo with the CPU)."""
    if dist is None:
        return dict(vals)
    keys = list(vals)
    t = torch.tensor([float(vals[k]) for k in keys], dtype=torch.float64, device=device)
    mx, tot = t.clone(), t.clone()
    dist.all_reduce(mx, op=dist.ReduceOp.MAX)
    dist.all_reduce(tot, op=dist.ReduceOp.SUM)
    out = {}
    for i, k in enumerate(keys):
        out[k] = tot[i].item() if k in SUM_KEYS else mx[i].item()
    return out


# ----------------------------------------------------------------------------- device state

class DeviceState:
    def __init__(self, torch, pkv, b: W.DecodeBatch, device, partitions: int):
        self.torch, self.pkv, self.b, self.dev = torch, pkv, b, device
        sp = b.spec
        self.q = self._dev(b.q, sp.q_dtype)
        self.bt = torch.from_numpy(b.block_tables).to(device)
        self.sl = torch.from_numpy(b.seq_lens).to(device)
        self.new_k = self._dev(b.new_k, sp.in_dtype)
        self.new_v = self._dev(b.new_v, sp.in_dtype)
        self.new_slots = torch.from_numpy(b.new_slots).to(device)
        cdt = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8, "e5m2": torch.float8_e5m2,
               "int8": torch.int8}[sp.kv_dtype]
        shape = (b.num_blocks, sp.num_kv_heads, sp.block_size, sp.head_dim)
        self.kc = torch.zeros(shape, dtype=cdt, device=device)
        self.vc = torch.zeros(shape, dtype=cdt, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.out = torch.empty_like(self.q)
        self.partitions = partitions
        self.q_len = 1
        self.plan = None
        self.ws = pkv.new_workspace(sp.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim, partitions, device)
        for i in range(0, b.hist_slots.size, 1 << 16):      # history already in the cache before the step
            pkv.reshape_and_cache(self._dev(b.hist_k[i:i + (1 << 16)], sp.in_dtype),
                                  self._dev(b.hist_v[i:i + (1 << 16)], sp.in_dtype), self.kc, self.vc,
                                  torch.from_numpy(b.hist_slots[i:i + (1 << 16)]).to(device),
                                  float(b.k_scale), float(b.v_scale), self.err)
        torch.cuda.synchronize(device)

    def _dev(self, a, name):
        t = self.torch
        if name == "bf16":
            return t.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(t.bfloat16).to(self.dev)
        return t.from_numpy(np.ascontiguousarray(a)).to(self.dev)

    def append(self):
        b = self.b
        self.pkv.reshape_and_cache(self.new_k, self.new_v, self.kc, self.vc, self.new_slots,
                                   float(b.k_scale), float(b.v_scale), self.err)

    def decode(self):
        b = self.b
        self.pkv.paged_attention_decode(self.out, self.q, self.kc, self.vc, self.bt, self.sl, float(b.scale),
                                        float(b.k_scale), float(b.v_scale), self.partitions, self.ws)

    def use_prefix_plan(self, max_group: int = 8):
        """Decode with the shared-prefix kernels: the plan of the batch's tables (pkv_prefix_plan,
        computed once on the host: the sharing structure changes when sequences fork or finish,
        not every step) copied to the device, and a workspace sized for its groups."""
        from paged_kv_cache_462_b200 import blocks
        t0 = time.perf_counter()
        plan = blocks.prefix_plan(self.b.block_tables, self.b.seq_lens, self.b.spec.block_size, max_group)
        self.plan_host_ms = 1e3 * (time.perf_counter() - t0)
        self.plan = self.pkv.DevicePrefixPlan(plan, max_group, self.dev)
        sp = self.b.spec
        self.ws = self.pkv.new_shared_prefix_workspace(sp.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim,
                                                       self.plan.num_groups, self.partitions, self.dev)
        return plan

    def step(self):
        """append + decode through paged_decode_step (one launch where the fused kernel applies);
        with a prefix plan paged_decode_step_shared_prefix (prefix pass, suffix pass with the
        append, merge); with q_len > 1 the causal multi-query decode of the last q_len tokens of
        every sequence"""
        b = self.b
        if self.plan is not None:
            self.pkv.paged_decode_step_shared_prefix(self.out, self.q, self.kc, self.vc, self.bt, self.sl, self.plan,
                                                     self.new_k, self.new_v, self.new_slots, float(b.scale),
                                                     float(b.k_scale), float(b.v_scale), self.partitions, self.ws)
            return
        if self.q_len > 1:
            self.pkv.paged_attention_decode_mq(self.out_mq, self.q_mq, self.kc, self.vc, self.bt, self.sl,
                                               float(b.scale), float(b.k_scale), float(b.v_scale), self.partitions,
                                               self.ws_mq)
            return
        self.pkv.paged_decode_step(self.out, self.q, self.kc, self.vc, self.bt, self.sl, self.new_k, self.new_v,
                                   self.new_slots, float(b.scale), float(b.k_scale), float(b.v_scale),
                                   self.partitions, self.ws)

    def set_q_len(self, q_len: int):
        """Multi-query mode: the history plus the appended token stand for the last q_len tokens."""
        self.q_len = q_len
        if q_len > 1:
            sp, t = self.b.spec, self.torch
            g = t.Generator(device="cpu").manual_seed(462)
            self.q_mq = t.randn((self.b.num_seqs, q_len, sp.num_heads, sp.head_dim), generator=g).to(
                t.bfloat16).to(self.dev)
            self.out_mq = t.empty_like(self.q_mq)
            self.ws_mq = self.pkv.new_workspace(sp.num_seqs, sp.num_heads * q_len, sp.num_kv_heads, sp.head_dim,
                                                self.partitions, self.dev)
            self.append()

    def errors(self):
        self.torch.cuda.synchronize(self.dev)
        e = int(self.err.item()) | self.pkv.read_device_error(self.ws)
        return e | (self.pkv.read_device_error(self.ws_mq) if self.q_len > 1 else 0)


# ----------------------------------------------------------------------------- oracle (CPU) timing

def oracle_pair_sampler(b: W.DecodeBatch):
    """Single (sequence, KV head 0) attention problems cut from the batch, for timing the oracle.

    Returns a list of (callable, bytes, seq_len, attention-only callable, its bytes). The
    data preparation (history fill through the oracle's own append, slicing of KV head 0)
    is done here, outside the timing.
    """
    import oracle
    sp = b.spec
    G = sp.num_heads // sp.num_kv_heads
    rng = np.random.default_rng(0)
    seqs = rng.permutation(b.num_seqs)[: min(b.num_seqs, 16)].tolist()
    _, kc, vc = oracle.run_step(b, seqs=seqs)
    kc0 = np.ascontiguousarray(kc[:, 0:1])
    vc0 = np.ascontiguousarray(vc[:, 0:1])
    q0 = np.ascontiguousarray(b.q[:, 0:G])
    nk0 = np.ascontiguousarray(b.new_k[:, 0:1])
    nv0 = np.ascontiguousarray(b.new_v[:, 0:1])
    items = []
    for s in seqs:
        L = int(b.seq_lens[s])
        attn_bytes = acct.decode_bytes(b.seq_lens[s:s + 1], b.block_tables[s:s + 1], G, 1, sp.head_dim,
                                       sp.block_size, sp.kv_dtype, sp.q_dtype)["total"]
        nbytes = attn_bytes + acct.append_bytes(1, 1, sp.head_dim, sp.in_dtype, sp.kv_dtype)

        def attend(s=s):
            oracle.paged_decode(q0, sp.q_dtype, kc0, vc0, sp.kv_dtype, b.block_tables, b.seq_lens, G, 1,
                                sp.head_dim, sp.block_size, b.num_blocks, b.scale, b.k_scale, b.v_scale, seqs=[s])

        def run(s=s):
            oracle.reshape_and_cache(nk0, nv0, sp.in_dtype, kc0, vc0, sp.kv_dtype, b.new_slots, 1, sp.head_dim,
                                     sp.block_size, b.num_blocks, b.k_scale, b.v_scale, rows=[s])
            attend(s)
        items.append((run, nbytes, L, attend, attn_bytes))
    return items


def time_oracle(items, seconds: float):
    done_bytes, n, t0 = 0, 0, time.perf_counter()
    while True:
        run, nbytes = items[n % len(items)][:2]
        run()
        done_bytes += nbytes
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            return done_bytes / el / 1e9, n, el


def time_oracle_threads(items, seconds: float, threads: int):
    """The attention-only problems on `threads` host threads at once (the C oracle runs with
    the interpreter lock released, and the problems only read shared arrays): aggregate
    GB/s, problems done, elapsed seconds."""
    import concurrent.futures as cf
    t0 = time.perf_counter()

    def worker(i):
        done, n = 0, 0
        while time.perf_counter() - t0 < seconds:
            _, _, _, attend, nbytes = items[(i + n) % len(items)]
            attend()
            done += nbytes
            n += 1
        return done, n

    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        res = list(ex.map(worker, range(threads)))
    el = time.perf_counter() - t0
    return sum(r[0] for r in res) / el / 1e9, sum(r[1] for r in res), el


# ----------------------------------------------------------------------------- arms

def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    b = W.build_batch(workload_spec(args))
    items = oracle_pair_sampler(b)
    # size each step to a bounded sample: one (sequence, kv head) pair, so the run stays within minutes
    for i in range(args.warmup):
        items[i % len(items)][0]()
    times, nbytes = [], 0
    for i in range(args.steps):
        run, nb = items[i % len(items)][:2]
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
        nbytes += nb
    total = sum(times)
    value = nbytes / total / 1e9
    sample = (f"one (sequence, KV head 0) attention problem per step, cycling over {len(items)} sequences "
              f"of the workload, append of its new token included; fp64 C oracle, single thread")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(b), "config_index": args.config},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def pack_step_inputs(torch, tensors: dict, dev):
    """One device buffer and one pinned host buffer holding copies of `tensors` at the same
    256-byte-aligned offsets: ({name: device view, "_buffer": device buffer}, {..host..})."""
    offs, total = {}, 0
    for n, t in tensors.items():
        offs[n] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    dbuf = torch.empty(total, dtype=torch.uint8, device=dev)
    hbuf = torch.empty(total, dtype=torch.uint8).pin_memory()
    dv, hv = {"_buffer": dbuf}, {"_buffer": hbuf}
    for n, t in tensors.items():
        nb = t.numel() * t.element_size()
        dv[n] = dbuf[offs[n]:offs[n] + nb].view(t.dtype).view(t.shape)
        hv[n] = hbuf[offs[n]:offs[n] + nb].view(t.dtype).view(t.shape)
        dv[n].copy_(t)
        hv[n].copy_(t.cpu())
    return dv, hv


def use_prefix_plan(args, spec) -> bool:
    """The shared-prefix decode for workloads whose sequences share prefix blocks (or when asked).

    By default only with a bf16 cache: there the step is HBM-bound and reading each shared block
    once per group saves its bytes (config 3: 398 against 418 us per step). With an 8-bit cache
    the decode is bound by its consumer warps, not HBM, so the bytes saved buy nothing while the
    prefix pass and its merge add work (config 3 with an E4M3 cache: 261 against 245 us)."""
    if args.q_len != 1 or args.prefix_sharing == "off" or spec.kv_dtype == "f32":
        return False
    if args.prefix_sharing == "on":
        return True
    return spec.share_group > 1 and spec.kv_dtype == "bf16"


def time_steps(torch, state, K: int, warmup: int, flush_l2, stream, dev):
    """W untimed steps, then K steps each bracketed by CUDA events on the launching stream, with
    the L2 flush between steps outside the events. Returns (per-step ms, wall start, wall end of
    the timed region)."""
    for _ in range(warmup):
        flush_l2()
        state.step()
    torch.cuda.synchronize(dev)
    if state.errors():
        raise SystemExit(f"device error word {state.errors()} after warm-up")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for i in range(K):
        flush_l2()                        # cold L2 for every step (outside the step's events)
        ev[i][0].record(stream)
        state.step()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.perf_counter()
    return [e[0].elapsed_time(e[1]) for e in ev], t0, t1


def ours_arm(args):
    import torch
    import paged_kv_cache_462_b200 as pkv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    pkv.load_library()
    pkv.set_fp8_kernel(pkv.FP8_KERNEL_TCGEN05 if args.fp8_kernel == "tcgen05" else pkv.FP8_KERNEL_MMA)

    spec = workload_spec(args)
    tc05 = args.fp8_kernel == "tcgen05" and spec.kv_dtype in ("e4m3", "e5m2")
    b = W.build_batch(spec, seed=spec.seed + 1000 * rank)
    state = DeviceState(torch, pkv, b, dev, args.partitions)
    state.set_q_len(args.q_len)
    plan = state.use_prefix_plan(spec.share_group) if use_prefix_plan(args, spec) else None
    plan_host_ms = state.plan_host_ms if plan is not None else None
    dec, app = step_bytes(b, args.q_len, plan)
    bytes_step = dec["total"] + app
    # a read (not a write) of a buffer twice the size of L2: the L2 ends up holding clean lines of
    # another buffer, as after the weight-streaming GEMMs that precede attention in a decode step
    flush_buf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_out = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        torch.sum(flush_buf, dim=0, out=flush_out)

    stream = torch.cuda.current_stream(dev)
    K = args.steps
    clocks = ClockSampler(smi_index(torch, local)) if rank == 0 else None
    if dist:
        dist.barrier()
    step_ms, t_on, t_off = time_steps(torch, state, K, args.warmup, flush_l2, stream, dev)
    if dist:
        dist.barrier()
    ms = sum(step_ms) / K
    fused = pkv.load_library() is not None and spec.kv_dtype != "f32" and spec.block_size in (16, 32)
    errs = state.errors()

    # end to end: per-step inputs from pinned host memory, output back to pinned host memory
    e2e = None
    if not args.no_e2e:
        names = ("q_mq", "sl", "bt") if args.q_len > 1 else ("q", "new_k", "new_v", "new_slots", "sl", "bt")
        owners = {n: state for n in names}
        if state.plan is not None:   # the plan's arrays travel with the tables they come from
            owners.update({n: state.plan for n in ("members", "offsets", "tables", "lens", "shared")})
        # the step's inputs live in one device buffer with a pinned host mirror of the same layout,
        # so each step's upload is a single copy
        dev_in, host_in = pack_step_inputs(torch, {n: getattr(o, n) for n, o in owners.items()}, dev)
        for n, o in owners.items():
            setattr(o, n, dev_in[n])
        dev_buf, host_buf = dev_in["_buffer"], host_in["_buffer"]
        dev_out = state.out_mq if args.q_len > 1 else state.out
        out_h = torch.empty(dev_out.shape, dtype=dev_out.dtype).pin_memory()
        h2d = host_buf.numel()
        d2h = out_h.numel() * out_h.element_size()
        # at least 100 timed steps after at least 10 warm-ups: over a handful of steps the host
        # side of this loop (pinned copies queued behind the step's launches) varies run to run
        Ke, We = max(K, 100), max(args.warmup, 10)
        ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Ke)]
        for i in range(Ke + We):
            flush_l2()
            rec = i >= We
            if rec:
                ee[i - We][0].record(stream)
            dev_buf.copy_(host_buf, non_blocking=True)
            state.step()
            out_h.copy_(dev_out, non_blocking=True)
            if rec:
                ee[i - We][1].record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = sum(a.elapsed_time(c) for a, c in ee) / Ke
        e2e = {"ms": e2e_ms, "h2d": h2d, "d2h": d2h, "steps": Ke}

    # the other points of the throughput target, timed the same way (same K and W), one at a time
    targets = []
    if (not args.no_targets and args.q_len == 1 and args.kv_dtype is None and args.partitions == 0
            and args.num_seqs is None):
        main_kv = spec.kv_dtype
        del state
        torch.cuda.empty_cache()
        batches = {args.config: b}
        for cfg, kv in TARGET_POINTS:
            if cfg == args.config and kv == main_kv:
                continue
            if cfg not in batches:
                batches = {args.config: b, cfg: W.build_batch(W.config_spec(cfg),
                                                              seed=W.config_spec(cfg).seed + 1000 * rank)}
            tb = W.with_cache_dtype(batches[cfg], kv)
            ts = DeviceState(torch, pkv, tb, dev, 0)
            tplan = ts.use_prefix_plan(tb.spec.share_group) if use_prefix_plan(args, tb.spec) else None
            tdec, tapp = step_bytes(tb, 1, tplan)
            tbytes = tdec["total"] + tapp
            if dist:
                dist.barrier()
            tms, t0, t1 = time_steps(torch, ts, K, args.warmup, flush_l2, stream, dev)
            terr = ts.errors()
            agg_t = aggregate_ranks(torch, dist, dev, ms=sum(tms) / K, step_bytes=float(tbytes), errors=float(terr))
            targets.append({"config_index": cfg, "kv_storage": kv, "workload": describe(tb),
                            "prefix_groups": tplan.num_groups if tplan is not None else 0,
                            "ms_per_step": agg_t["ms"], "value": agg_t["step_bytes"] / (agg_t["ms"] * 1e-3) / 1e9,
                            "unit": "GB/s", "algorithmic_bytes": tbytes,
                            "kv_logical_gbs": tdec["kv_logical"] / (sum(tms) / K * 1e-3) / 1e9,
                            "seq_steps_per_s": world * tb.spec.num_seqs / (agg_t["ms"] * 1e-3),
                            "device_errors": int(agg_t["errors"]),
                            "traffic": kernel_traffic(cfg, kv, tplan is not None),
                            "clocks": clocks.summary(t0, t1) if clocks else None})
            del ts
            torch.cuda.empty_cache()
    if clocks:
        clocks.stop()

    # aggregate over ranks: max time, summed bytes
    agg = aggregate_ranks(torch, dist, dev, ms=ms, decode_ms=ms,
                          e2e_ms=e2e["ms"] if e2e else 0.0, step_bytes=float(bytes_step), errors=float(errs))
    ms_max, dec_max, e2e_max = agg["ms"], agg["decode_ms"], agg["e2e_ms"]
    bytes_all, errs_all = agg["step_bytes"], int(agg["errors"])

    if rank == 0:
        peak, peak_kind = measured_peak()
        kern_bytes = dec["total"] + app          # the step kernel: decode plus the fused append
        kern_gbs = kern_bytes / (ms * 1e-3) / 1e9
        for t in targets:
            t["frac"] = t["value"] / world / peak
        line = {
            "metric": METRIC,
            "value": bytes_all / (ms_max * 1e-3) / 1e9,
            "unit": "GB/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": ms_max,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            # arithmetic of the products: bf16 for bf16 caches; 8-bit codes widened exactly to f16
            "dtype": {"f32": "f32", "bf16": "bf16", "e4m3": "f16", "e5m2": "f16", "int8": "f16"}[spec.kv_dtype],
            "data": "synthetic",
            "config": {
                "workload": describe(b), "config_index": args.config,
                "kv_storage": spec.kv_dtype, "partitions": args.partitions or pkv.default_partitions(
                    spec.head_dim, spec.block_size, spec.num_heads, spec.num_kv_heads,
                    {"f32": 0, "bf16": 1, "e4m3": 2, "e5m2": 3, "int8": 4}[spec.kv_dtype]),
                "step": (f"paged_attention_decode_mq: the last {args.q_len} tokens of every sequence as queries, "
                         "causal within the chunk (their K/V already cached)" if args.q_len > 1 else
                         f"paged_decode_step_shared_prefix: prefix pass over the {plan.num_groups} groups' shared "
                         f"blocks (plan made once on the host in {plan_host_ms:.2f} ms, outside the timed "
                         "region), suffix pass with the append fused, merge" if plan is not None else
                         "paged_decode_step: append of one new token per sequence fused into the paged "
                         "decode launch" if fused else
                         "paged_decode_step: reshape_and_cache then paged_attention_decode (two launches)"),
                "l2": "cold: a 256 MiB read before every step, outside the step's CUDA events",
                "replicas": world,
                **({"fp8_kernel": args.fp8_kernel} if spec.kv_dtype in ("e4m3", "e5m2") else {}),
            },
            "seq_steps_per_s": world * spec.num_seqs / (ms_max * 1e-3),
            "step_us": dec_max * 1e3,
            "kv_logical_gbs": dec["kv_logical"] / (ms * 1e-3) / 1e9,
            "step_bytes": bytes_step,
            "roofline": {
                "bound": "hbm",
                # events bracket the whole step: the decode kernel (append fused) and its merge kernel
                "kernel": ("paged_decode_mma_kernel prefix pass + suffix pass (append fused) + "
                           "paged_decode_prefix_merge_kernel" if plan is not None and plan.num_groups > 0 else
                           "paged_decode_tc05_kernel (append fused) + paged_decode_merge_kernel" if fused and tc05
                           else "paged_decode_mma_kernel (append fused) + paged_decode_merge_kernel" if fused
                           else "reshape_and_cache_kernel + paged_decode_kernel"),
                "achieved": kern_gbs,
                "peak": peak,
                "peak_kind": peak_kind,
                "unit": "GB/s",
                "frac": kern_gbs / peak,
                "traffic": (kernel_traffic(args.config, spec.kv_dtype, plan is not None)
                            if args.q_len == 1 and not tc05 else None),
                "algorithmic_bytes": kern_bytes,
            },
            # fused: the decode kernel (append inside) + the merge kernel; else append + decode
            "gpu_launches": (3 if plan is not None and plan.num_groups > 0 else 2) * K,
            "clocks": clocks.summary(t_on, t_off) if clocks else None,
            "device_errors": errs_all,
        }
        if targets:
            line["targets"] = targets
        if e2e:
            line["e2e"] = {"value": bytes_all / (e2e_max * 1e-3) / 1e9, "unit": "GB/s",
                           "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e_max,
                           "steps": e2e["steps"]}
        if world == 1 and not args.no_cpu_baseline:
            items = oracle_pair_sampler(b)
            v, n, el = time_oracle(items, args.cpu_seconds)
            line["cpu_baseline"] = {
                "value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                "sample": f"{n} single (sequence, KV head 0) problems of this workload cycled for {el:.1f} s "
                          f"(append + attention each), fp64 C oracle, one thread"}
            threads = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
            v, n, el = time_oracle_threads(items, args.cpu_seconds, threads)
            line["cpu_baseline_all_cores"] = {
                "value": v, "unit": "GB/s", "cores": threads, "kind": "oracle",
                "sample": f"{n} attention-only problems of the same sample on {threads} threads for {el:.1f} s, "
                          f"fp64 C oracle"}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return reference_arm(args)
    return ours_arm(args)


if __name__ == "__main__":
    sys.exit(main())
