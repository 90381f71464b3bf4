"""Benchmark of the paged decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl pkv|reference]

One step = one decode step of the whole path for a batch: the block manager's
append (slot mapping), the KV append kernel for the batch's new tokens, and
paged decode attention (plus its partition merge) over the updated cache.
Default workload: the Llama-2-7B-shaped decode batch (B=64, 32/32 heads,
D=128, bf16, block size 16, context lengths U[512,2048], random placement in
a 16384-block pool).

Printed metric (one JSON line on rank 0): achieved HBM GB/s of the step
(algorithmic bytes: every K/V byte of every context read once, Q, the output,
block tables and lengths, and the appended tokens read and written) with its
fraction of the measured HBM peak, plus decode tokens/s. `value` is timed with
per-step inputs already in HBM; `e2e` times the same steps through the public
API from host buffers (host block manager, pinned H2D copies of the step's
queries / new K,V / metadata, the kernels, D2H of the output).

Other operations, one JSON line each (`--op`): `swap` (preemption swap-out and
swap-in over the host link), `mq` (causal multi-query attention: chunked
prefill with --query-len 512, speculative verify with --query-len 5) and
`fork` (copy-on-write block copies when every sequence forks into --samples
samples).

Multi-GPU (torchrun): every rank runs its own replica of the batch (decode
batches are independent; there is no data exchange), times are the max over
ranks, and `value` is the sum of all ranks' bytes over that time.
"""
from __future__ import annotations

import argparse
import dataclasses
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

from paged_kv_cache_322_b200 import workloads as wl  # noqa: E402

L2_BYTES = 126 * 2 ** 20
BREAKDOWN_STEPS = 20           # e2e steps run again with the native step's phase timing on
SPEC_HBM_GBS = 8000.0          # B200 HBM3e, the spec sheet's 8 TB/s (the measured copy peak is the other denominator)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="pkv", choices=["pkv", "reference"])
    ap.add_argument("--op", default="decode", choices=["decode", "swap", "mq", "fork"],
                    help="decode: the decode step (append + attention); swap: preemption by swapping half the "
                         "workload's sequences to a page-locked host pool and back; mq: several causal query "
                         "tokens per sequence (--query-len: 512 = a chunked-prefill chunk, 5 = speculative verify); "
                         "fork: copy-on-write block copies when every sequence forks into --samples samples")
    ap.add_argument("--samples", type=int, default=4, help="samples per sequence (--op fork)")
    ap.add_argument("--query-len", type=int, default=512, help="query tokens per sequence and step (--op mq)")
    ap.add_argument("--workload", default="llama2_7b", choices=list(wl.WORKLOADS))
    ap.add_argument("--partition-tokens", type=int, default=-2,
                    help="-2: the workload's; 0: library-chosen partitions; -1: persistent schedule; >0: fixed")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-paging-overhead", action="store_true",
                    help="skip the random- vs identity-placement timing of the attention call")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU time of the oracle sample")
    ap.add_argument("--num-seqs", type=int, default=0, help="override the batch size (profiling a small case)")
    ap.add_argument("--num-blocks", type=int, default=0, help="override the pool size (profiling a small case)")
    ap.add_argument("--no-extra", action="store_true",
                    help="default run only: skip the 70B-shaped GQA sub-result")
    ap.add_argument("--block-size", type=int, default=0,
                    help="tokens per block (8, 16, 32, 64); the pool keeps the workload's token capacity")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_init(args):
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _all_reduce(x: float, ws: int, op: str) -> float:
    """Reduces a host float over all ranks (CUDA tensor under NCCL, CPU under gloo)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def all_max(x: float, ws: int) -> float:
    return _all_reduce(x, ws, "max")


def all_sum(x: float, ws: int) -> float:
    return _all_reduce(x, ws, "sum")


def override_workload(w: wl.Workload, args) -> wl.Workload:
    """--num-seqs / --num-blocks / --block-size applied to a workload (a block
    size change keeps the pool's token capacity)."""
    notes = []
    if args.block_size and args.block_size != w.block_size:
        nb = (args.num_blocks or w.num_blocks) * w.block_size // args.block_size
        w = dataclasses.replace(w, block_size=args.block_size, num_blocks=nb)
        notes.append(f"block_size={args.block_size}, pool={nb} blocks")
    if args.num_seqs or args.num_blocks:
        w = dataclasses.replace(w, num_seqs=args.num_seqs or w.num_seqs,
                                num_blocks=w.num_blocks if args.block_size else (args.num_blocks or w.num_blocks))
        notes.append(f"B={w.num_seqs}, pool={w.num_blocks}")
    if notes:
        w = dataclasses.replace(w, description=w.description + " [override: " + "; ".join(notes) + "]")
    return w


def replica_workload(w: wl.Workload, rank: int) -> wl.Workload:
    """Rank r's replica of the batch: same shapes, its own seed (decode batches
    are independent, so the replicas exchange no data)."""
    return w if rank == 0 else dataclasses.replace(w, seed=w.seed + 7919 * rank)


def aggregate(ms_local: float, bytes_local: float, tokens_local: float, ws: int):
    """Whole-job figures: time = max over ranks, bytes and tokens summed."""
    ms = all_max(ms_local, ws)
    nbytes = all_sum(bytes_local, ws)
    tokens = all_sum(tokens_local, ws)
    return ms, nbytes / (ms * 1e-3) / 1e9, tokens / (ms * 1e-3)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """Samples SM clock, max clock and throttle reasons through NVML every few
    milliseconds while the timed region runs (nvidia-smi as a fallback)."""

    def __init__(self, index: int, interval_s: float = 0.005):
        self.index, self.interval, self.samples, self._stop = index, interval_s, [], threading.Event()
        self._t = threading.Thread(target=self._run, daemon=True)
        self.source = "nvml"

    def _run(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            while True:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, mx, sorted(k for k, b in bits.items() if r & b)))
                if self._stop.wait(self.interval):
                    break
            pynvml.nvmlShutdown()
        except Exception:
            self.source = "nvidia-smi"
            self._run_smi()

    def _run_smi(self):
        fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        while True:
            try:
                r = subprocess.run(["nvidia-smi", f"--id={self.index}", f"--query-gpu={fields}",
                                    "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=5)
                v = [x.strip() for x in r.stdout.strip().split(",")]
                if r.returncode == 0 and len(v) == 6:
                    self.samples.append((float(v[0]), float(v[1]),
                                         [names[i] for i in range(4) if v[2 + i].lower() == "active"]))
            except Exception:
                pass
            if self._stop.wait(0.2):
                break

    def __enter__(self):
        self._t.start()
        time.sleep(0.02)                       # first sample lands before the timed region starts
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": max(s[1] for s in self.samples),
                "reasons": sorted({r for s in self.samples for r in s[2]}),
                "samples": len(self.samples), "source": self.source}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_tflops() -> float:
    """Measured dense bf16 TFLOP/s (burst), or the fallback figure."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"])
    return 1590.0


def traffic_record(workload: str):
    """ncu DRAM traffic of the attention kernel for this workload, if it was taken
    on the current device code (else None)."""
    path = os.path.join(ROOT, "profiles", "attention_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    entry = rec.get(workload)
    if not isinstance(entry, dict) or entry.get("source_sha1") != kernel_source_sha1():
        return None
    return entry


def kernel_source_sha1() -> str:
    """Hash of the decode attention kernel's device code: the shared device
    headers and the kernel template (the traffic records are ncu captures of
    paged_decode_kernel alone)."""
    csrc = os.path.join(ROOT, "paged_kv_cache_322_b200", "csrc")
    h = hashlib.sha1()
    for name in ("common.cuh", "attention_common.cuh", "paged_attention_kernel.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# ---------------------------------------------------------------------------
# byte accounting (algorithmic: each byte the method must move, once)
# ---------------------------------------------------------------------------
def attention_bytes(w: wl.Workload, lens_after: np.ndarray, out_elt: int) -> int:
    eb = w.elt_bytes
    kv = int(lens_after.sum()) * w.num_kv_heads * w.head_dim * eb * 2
    q = w.num_seqs * w.num_q_heads * w.head_dim * w.in_bytes
    out = w.num_seqs * w.num_q_heads * w.head_dim * out_elt
    tables = int(sum(-(-int(n) // w.block_size) for n in lens_after)) * 4
    return kv + q + out + tables + 4 * w.num_seqs


def mq_flops(lens_after, n: int, hq: int, d: int) -> int:
    """Causal multi-query attention flops: every sequence's n queries (positions
    c - n .. c - 1) against their visible tokens, 2 flops per multiply-add in
    Q K^T and in P V: 4 * Hq * D per (query, visible token)."""
    return sum(4 * hq * d * (n * (int(c) - n) + n * (n + 1) // 2) for c in lens_after)


def mq_attention_bytes(lens_after, n: int, hq: int, hkv: int, d: int, bs: int) -> int:
    """Algorithmic bytes of one multi-query attention launch (bf16): K and V of
    every cached token once, q in, out, the block tables."""
    T = n * len(lens_after)
    return (int(np.sum(lens_after)) * hkv * d * 2 * 2 + T * hq * d * 2 * 2 +
            int(sum(-(-int(c) // bs) for c in lens_after)) * 4)


def decode_launches(num_seqs: int, part: int, part_used: int, maxctx: int, block_size: int) -> int:
    """Kernels one decode attention call launches: the plan kernel when the
    library lists units longest first (two or more sequences, at most 65535
    units, partitions of at most 4096 blocks), the partition kernel, and the
    merge when the longest context spans more than one partition; the
    persistent schedule (part -1) is one kernel."""
    if part == -1:
        return 1
    parts = max(1, -(-maxctx // part_used))
    plan = 1 if (num_seqs >= 2 and num_seqs * parts <= 65535 and part_used // block_size <= 4096) else 0
    return plan + 1 + (1 if parts > 1 else 0)


def append_bytes(w: wl.Workload) -> int:
    n = w.num_kv_heads * w.head_dim
    return w.num_seqs * (2 * n * (w.in_bytes + w.elt_bytes) + 8)   # K and V rows read and written, slot ids


# ---------------------------------------------------------------------------
# the library arm
# ---------------------------------------------------------------------------
def run_pkv(args, ws, rank, local):
    import torch
    from paged_kv_cache_322_b200 import binding
    from paged_kv_cache_322_b200.engine import PagedKVCache

    dev = torch.device("cuda", local)
    w = wl.WORKLOADS[args.workload]
    w = override_workload(w, args)
    w = replica_workload(w, rank)
    part = w.partition_tokens if args.partition_tokens == -2 else args.partition_tokens
    K, W = args.steps, args.warmup
    total_steps = 3 * (K + W) + 2 + BREAKDOWN_STEPS
    lens0 = wl.context_lens(w)
    dt = torch.float32 if w.kv_dtype == "f32" else torch.bfloat16       # q and the appended K/V
    cdt = torch.uint8 if w.kv_dtype == "fp8" else dt                     # cache storage
    mb = -(-int(lens0.max() + total_steps) // w.block_size)

    # ---- set-up (untimed): prompts into the cache through the library ----
    cache = PagedKVCache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, cdt, dev,
                         free_order=wl.free_order(w), max_blocks_per_seq=mb, kv_scales=(w.kv_scale, w.kv_scale))
    kvs = wl.prompt_kv_all(w, lens0)
    for s in range(w.num_seqs):
        k, v = kvs[s]
        cache.add_sequence(s, torch.from_numpy(k).to(dev, dt), torch.from_numpy(v).to(dev, dt))
    ids = np.arange(w.num_seqs, dtype=np.int64)
    torch.cuda.synchronize()
    paging = None
    if not args.no_paging_overhead and part != -1:
        paging = paging_overhead(w, cache, kvs, dev, dt, cdt, mb, part, K, W)
    del kvs

    # ---- per-step inputs, resident in HBM before timing ----
    steps = []
    for i in range(K + W):
        slots, src, dst = cache.bm.append_slots(ids)
        assert src.size == 0
        tables, lens = cache.block_tables(ids)
        q = wl.decode_q(w, i)
        kn, vn = wl.decode_kv(w, i)
        steps.append(dict(
            q=torch.from_numpy(q).to(dev, dt), kn=torch.from_numpy(kn).to(dev, dt),
            vn=torch.from_numpy(vn).to(dev, dt), slots=torch.from_numpy(slots).to(dev),
            tables=torch.from_numpy(tables).to(dev), lens=torch.from_numpy(lens).to(dev),
            maxlen=int(lens.max()), bytes_attn=attention_bytes(w, lens, 2)))
    out = torch.empty((w.num_seqs, w.num_q_heads, w.head_dim), dtype=torch.bfloat16, device=dev)
    ws_bytes = binding.workspace_bytes(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, mb,
                                       max(s["maxlen"] for s in steps), part)
    workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    part_used = binding.partition_tokens(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, mb,
                                         max(s["maxlen"] for s in steps), part)
    stream = torch.cuda.current_stream(dev)
    maxctx = max(s["maxlen"] for s in steps)

    def step_device(st, ev0=None, ev1=None):
        cache.append(st["kn"], st["vn"], st["slots"])
        if ev0 is not None:
            ev0.record(stream)
        cache.attention(out, st["q"], st["tables"], st["lens"], w.scale, max_context_len=maxctx,
                        partition_tokens=part, workspace=workspace)
        if ev1 is not None:
            ev1.record(stream)

    for i in range(W):
        step_device(steps[i])
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for i in range(K):
            step_device(steps[W + i], *ev[i])
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    ms = t0.elapsed_time(t1)
    attn_ms = [a.elapsed_time(b) for a, b in ev]
    assert binding.get_device_error() == 0
    timed = steps[W:]
    bytes_step = [s["bytes_attn"] + append_bytes(w) for s in timed]
    local_bytes = float(sum(bytes_step))
    ms_max, gbs, tokens_s = aggregate(ms, local_bytes, float(w.num_seqs * K), ws)
    peak, peak_kind = measured_peaks()
    attn_avg_ms = statistics.mean(attn_ms)
    attn_bytes_avg = statistics.mean(s["bytes_attn"] for s in timed)
    achieved = attn_bytes_avg / (attn_avg_ms * 1e-3) / 1e9
    launches_per_step = 1 + decode_launches(w.num_seqs, part, part_used, maxctx, w.block_size)   # + the append
    del steps

    # ---- end to end through the C ABI from host buffers: pkv_decode_step ----
    e2e = None
    if not args.no_e2e:
        host = []
        for i in range(K + W):
            q = wl.decode_q(w, 1000 + i)
            kn, vn = wl.decode_kv(w, 1000 + i)
            host.append(tuple(torch.from_numpy(x).to(dt).pin_memory() for x in (q, kn, vn)))
        out_hosts = [torch.empty((w.num_seqs, w.num_q_heads, w.head_dim), dtype=torch.bfloat16).pin_memory()
                     for _ in range(2)]
        out_host = out_hosts[0]
        native = binding.DecodeStep(cache.bm, cache.k_cache, cache.v_cache, max_seqs=w.num_seqs,
                                    num_q_heads=w.num_q_heads, max_blocks_per_seq=mb, out_dtype=torch.bfloat16,
                                    partition_tokens=part, kv_scales=(w.kv_scale, w.kv_scale))
        lens_cur = np.array([cache.bm.seq_len(int(s)) for s in ids])

        def run_steps(count, pipelined):
            """count steps through pkv_decode_step; returns (ms, bytes). Pipelined:
            step j's result is read (its event waited for) after step j + 1 is
            issued, so host work and copies overlap the previous step's kernels;
            serial: each step's result is waited for before the next is issued."""
            nonlocal lens_cur
            nbytes, evs = 0, []
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for j in range(count):
                hq, hk, hv = host[j % len(host)]
                native(ids, hq, hk, hv, out_hosts[j % 2], w.scale, stream=stream)
                lens_cur = lens_cur + 1
                nbytes += attention_bytes(w, lens_cur, 2) + append_bytes(w)
                ev = torch.cuda.Event()
                ev.record(stream)
                evs.append(ev)
                if not pipelined:
                    ev.synchronize()                  # the step's result is on the host
                elif j >= 1:
                    evs[j - 1].synchronize()          # the previous step's result is on the host
            evs[-1].synchronize()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1), nbytes

        run_steps(W, True)
        barrier(ws)
        torch.cuda.synchronize()
        ms_p, bytes_p = run_steps(K, True)
        barrier(ws)
        ms_s, bytes_s = run_steps(K, False)
        barrier(ws)
        assert binding.get_device_error() == 0
        e_ms, e_gbs, e_tok = aggregate(ms_p, float(bytes_p), float(w.num_seqs * K), ws)
        s_ms, s_gbs, _ = aggregate(ms_s, float(bytes_s), float(w.num_seqs * K), ws)
        eb = w.in_bytes
        h2d = (w.num_seqs * w.num_q_heads * w.head_dim * eb + 2 * w.num_seqs * w.num_kv_heads * w.head_dim * eb +
               w.num_seqs * (3 * 8 + mb * 4 + 4))
        d2h = w.num_seqs * w.num_q_heads * w.head_dim * 2
        e2e = {"value": round(e_gbs, 1), "unit": "GB/s",
               "decode_tokens_per_s": round(e_tok, 1),
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(e_ms / K, 4),
               "path": "pkv_decode_step (C ABI, host buffers): block manager, H2D, kernels, D2H; each step's result "
                       "waited for on the host after the next step is issued (the context overlaps one step's copies "
                       "with its neighbours' kernels)",
               "serial": {"value": round(s_gbs, 1), "ms_per_step": round(s_ms / K, 4),
                          "what": "the same steps, each step's result waited for before the next is issued"}}
        # where the end-to-end step's time goes: the same steps again with the
        # context's phase timing on (host clock + events), medians, after the timed loop
        native.set_timing(True)
        phases = []
        for i in range(BREAKDOWN_STEPS):
            t_w = time.perf_counter()
            native(ids, *host[i % len(host)], out_host, w.scale, stream=stream)
            stream.synchronize()
            ph = native.last_timing()
            ph["wall"] = (time.perf_counter() - t_w) * 1e3
            phases.append(ph)
        native.set_timing(False)
        bd = {k: round(statistics.median(x[k] for x in phases), 4) for k in phases[0]}
        bd["other"] = round(bd["wall"] - bd["host_block_manager"] - bd["h2d"] - bd["kernels"] - bd["d2h"], 4)
        bd["what"] = ("medians over %d steps, ms: host block manager (host clock), H2D, kernels, D2H (events on the "
                      "stream); wall = the Python call + stream sync; other = wall minus the four (API, launch and "
                      "sync latency)" % BREAKDOWN_STEPS)
        e2e["breakdown_ms"] = bd

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds)

    tr = traffic_record(args.workload) if part != -1 else None
    result = {
        "metric": "paged decode attention achieved HBM GB/s (% of B200 peak); decode tokens/s",
        "value": round(gbs, 1), "unit": "GB/s", "n_gpus": ws, "steps": K, "warmup": W,
        "ms_per_step": round(ms_max / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.kv_dtype, "data": "synthetic",
        "pct_of_peak": round(100 * gbs / ws / peak, 1),
        "pct_of_peak_spec": round(100 * gbs / ws / SPEC_HBM_GBS, 1),
        "decode_tokens_per_s": round(tokens_s, 1),
        "attention_layer_tokens_per_s_per_32_layers": round(tokens_s / 32, 1),
        "config": {"workload": w.description, "global_batch": w.num_seqs * ws, "seq_len": f"U[{w.lo},{w.hi}]",
                   "block_size": w.block_size,
                   "schedule": ("persistent" if part == -1 else f"partitions of {part_used} tokens"),
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
                   "l2": f"inputs larger than L2 ({int(lens0.sum()) * w.num_kv_heads * w.head_dim * w.elt_bytes * 2 / 1e9:.2f} GB KV per step vs 126 MB L2); no flush",
                   "seed": w.seed},
        "roofline": {"bound": "hbm", "kernel": "paged_decode_kernel + merge_partitions_kernel (one attention call)",
                     "achieved": round(achieved, 1), "peak": peak, "peak_source": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "frac_of_spec": round(achieved / SPEC_HBM_GBS, 4),
                     "avg_launch_ms": round(attn_avg_ms, 5),
                     "algorithmic_bytes_per_launch": int(attn_bytes_avg),
                     "traffic": (int(tr["traffic_per_algorithmic_byte"] * attn_bytes_avg) if tr else None),
                     "traffic_source": (tr["captured_on"] if tr else None)},
        "e2e": e2e,
        "paging_overhead": paging,
        "gpu_launches": launches_per_step * K,
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
    }
    return result


def unique_attention_bytes(w: wl.Workload, tables: np.ndarray, lens: np.ndarray, out_elt: int) -> int:
    """Algorithmic bytes of one attention call counting each distinct physical
    block once: a block shared by several sequences (a common prompt prefix) is
    charged the tokens its longest reader uses, once. Plus q, out, the block
    tables and the lengths, as in attention_bytes."""
    bs = w.block_size
    used = {}
    for s in range(len(lens)):
        n = int(lens[s])
        for j in range(-(-n // bs)):
            b = int(tables[s][j])
            used[b] = max(used.get(b, 0), min(bs, n - j * bs))
    kv = sum(used.values()) * w.num_kv_heads * w.head_dim * w.elt_bytes * 2
    q = len(lens) * w.num_q_heads * w.head_dim * w.in_bytes
    out = len(lens) * w.num_q_heads * w.head_dim * out_elt
    nt = int(sum(-(-int(n) // bs) for n in lens)) * 4
    return kv + q + out + nt + 4 * len(lens)


def run_shared_prefix(args, ws, rank, local):
    """The shared-prefix decode step (parallel sampling: 32 sequences share the
    64 blocks of a 1024-token prompt, ref count 32, plus private tails).

    One step: copy_blocks forks the last shared block (logical 63) for the 31
    sequences that diverge (the 32nd keeps the original), reshape_and_cache
    appends one token per sequence, and decode attention runs over the updated
    contexts. The fork's copy list comes from the block manager's copy-on-write
    of logical block 63 before the first step; every step replays it (the source
    block is full and never written again, so each replay rewrites the same
    bytes), so every timed step does a fork step's work.

    Bytes: the attention is charged both ways, logical (every sequence's context
    read once, prefix included 32 times) and unique (each physical block once);
    `value` and % of peak use unique bytes. Timed twice: as a stream of steps with
    no flush (the 16 MiB prefix stays in L2 between steps), and with L2 flushed
    before every step (events around the step only)."""
    import torch
    from paged_kv_cache_322_b200 import binding
    from paged_kv_cache_322_b200.engine import PagedKVCache

    dev = torch.device("cuda", local)
    w = override_workload(wl.WORKLOADS[args.workload], args)
    w = replica_workload(w, rank)
    part = w.partition_tokens if args.partition_tokens == -2 else args.partition_tokens
    K, W = args.steps, args.warmup
    B, bs, p = w.num_seqs, w.block_size, w.shared_prefix
    dt = torch.bfloat16 if w.kv_dtype != "f32" else torch.float32
    lens0 = wl.context_lens(w)
    total_steps = 2 * (W + 2 * K) + 2
    mb = -(-int(lens0.max() + total_steps) // bs)
    ids = np.arange(B, dtype=np.int64)

    # ---- set-up (untimed): the shared prompt once, forked to every sequence, then the private tails ----
    cache = PagedKVCache(w.num_blocks, bs, w.num_kv_heads, w.head_dim, dt, dev, free_order=wl.free_order(w),
                         max_blocks_per_seq=mb)

    def tdev(x):
        return torch.from_numpy(x).to(dev, dt)

    k0, v0 = wl.prompt_kv(w, 0, int(lens0[0]))
    cache.add_sequence(-1, tdev(k0[:p]), tdev(v0[:p]))
    for s in range(B):
        cache.fork(-1, s)
    cache.free(-1)
    for s in range(B):
        n = int(lens0[s])
        k, v = wl.prompt_kv(w, s, n)
        slots = np.concatenate([cache.bm.append_slots([s])[0] for _ in range(n - p)])
        cache.append(tdev(k[p:]), tdev(v[p:]), torch.from_numpy(slots).to(dev))
    last = p // bs - 1
    assert cache.bm.ref_count(int(cache.block_tables([0])[0][0][last])) == B
    pairs = [x for x in (cache.bm.make_writable(int(s), last) for s in ids) if x is not None]
    assert len(pairs) == B - 1
    pa = np.asarray(pairs, dtype=np.int64)
    src_d, dst_d = torch.from_numpy(pa[:, 0].copy()).to(dev), torch.from_numpy(pa[:, 1].copy()).to(dev)
    block_bytes = bs * w.num_kv_heads * w.head_dim * w.elt_bytes
    copy_bytes = 2 * len(pairs) * block_bytes * 2 + 16 * len(pairs)      # K and V blocks read + written, the ids
    torch.cuda.synchronize()

    def make_steps(n, step0):
        out = []
        for i in range(n):
            slots, src, dst = cache.bm.append_slots(ids)
            assert src.size == 0
            tables, lens = cache.block_tables(ids)
            q = wl.decode_q(w, step0 + i)
            kn, vn = wl.decode_kv(w, step0 + i)
            out.append(dict(q=tdev(q), kn=tdev(kn), vn=tdev(vn), slots=torch.from_numpy(slots).to(dev),
                            tables=torch.from_numpy(tables).to(dev), lens=torch.from_numpy(lens).to(dev),
                            maxlen=int(lens.max()), logical=attention_bytes(w, lens, 2),
                            unique=unique_attention_bytes(w, tables, lens, 2)))
        return out

    steps = make_steps(W + 2 * K, 0)
    maxctx = max(st["maxlen"] for st in steps) + (W + K + 2)
    out = torch.empty((B, w.num_q_heads, w.head_dim), dtype=torch.bfloat16, device=dev)
    ws_bytes = binding.workspace_bytes(B, w.num_q_heads, w.num_kv_heads, w.head_dim, bs, mb, maxctx, part)
    workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    part_used = binding.partition_tokens(B, w.num_q_heads, w.num_kv_heads, w.head_dim, bs, mb, maxctx, part)
    stream = torch.cuda.current_stream(dev)
    flush_w = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    flush_r = torch.ones(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)

    def step_device(st, e_step=None, e_attn=None):
        if e_step is not None:
            e_step[0].record(stream)
        binding.copy_blocks(cache.k_cache, cache.v_cache, src_d, dst_d, stream=stream)
        cache.append(st["kn"], st["vn"], st["slots"], stream=stream)
        e_attn[0].record(stream)
        cache.attention(out, st["q"], st["tables"], st["lens"], w.scale, max_context_len=maxctx,
                        partition_tokens=part, workspace=workspace, stream=stream)
        e_attn[1].record(stream)
        if e_step is not None:
            e_step[1].record(stream)

    def evpair():
        return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    for i in range(W):
        step_device(steps[i], None, evpair())
    torch.cuda.synchronize()
    # (a) a stream of steps, no flush
    ev_a = [evpair() for _ in range(K)]
    t0, t1 = evpair()
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for i in range(K):
            step_device(steps[W + i], None, ev_a[i])
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    ms_a = t0.elapsed_time(t1)
    attn_a = [a.elapsed_time(b) for a, b in ev_a]
    # (b) L2 flushed before every step (write 2x L2, then read another 2x L2), each step timed alone
    ev_b = [(evpair(), evpair()) for _ in range(K)]
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks_b:
        for i in range(K):
            flush_w.fill_(i)
            flush_r.sum()
            step_device(steps[W + K + i], *ev_b[i])
        torch.cuda.synchronize()
    barrier(ws)
    ms_b = sum(a.elapsed_time(b) for (a, b), _ in ev_b)
    attn_b = [a.elapsed_time(b) for _, (a, b) in ev_b]
    assert binding.get_device_error() == 0

    ta, tb = steps[W:W + K], steps[W + K:]
    step_bytes = lambda st, key: st[key] + copy_bytes + append_bytes(w)        # noqa: E731
    uniq_a, logi_a = sum(step_bytes(st, "unique") for st in ta), sum(step_bytes(st, "logical") for st in ta)
    uniq_b, logi_b = sum(step_bytes(st, "unique") for st in tb), sum(step_bytes(st, "logical") for st in tb)
    ms_max, gbs, tokens_s = aggregate(ms_a, float(uniq_a), float(B * K), ws)
    _, gbs_logical, _ = aggregate(ms_a, float(logi_a), 0.0, ws)
    msb_max, gbs_b, _ = aggregate(ms_b, float(uniq_b), 0.0, ws)
    _, gbs_b_logical, _ = aggregate(ms_b, float(logi_b), 0.0, ws)
    peak, peak_kind = measured_peaks()
    au = statistics.mean(st["unique"] for st in ta)
    al = statistics.mean(st["logical"] for st in ta)
    aa, ab = statistics.mean(attn_a), statistics.mean(attn_b)
    ach = au / (aa * 1e-3) / 1e9
    ach_b = statistics.mean(st["unique"] for st in tb) / (ab * 1e-3) / 1e9
    del steps

    # ---- the same attention calls as a cascade that reads the shared prefix once ----
    cascade = None
    if w.kv_dtype == "bf16" and w.head_dim == 128 and B * w.group >= 32:
        pre = (p // bs - 1) * bs            # blocks still shared by every sequence after the fork of the last one
        cws = torch.empty(binding.shared_prefix_workspace_bytes(B, w.num_q_heads, w.num_kv_heads, w.head_dim, pre),
                          dtype=torch.uint8, device=dev)
        cout = torch.empty_like(out)

        def casc(st):
            binding.paged_attention_decode_shared_prefix(cout, st["q"], cache.k_cache, cache.v_cache, st["tables"],
                                                         st["lens"], pre, w.scale, maxctx, workspace=cws,
                                                         stream=stream)

        st = ta[-1]                          # guard: the same result as the regular call
        cache.attention(out, st["q"], st["tables"], st["lens"], w.scale, max_context_len=maxctx,
                        partition_tokens=part, workspace=workspace, stream=stream)
        casc(st)
        torch.cuda.synchronize()
        assert binding.get_device_error() == 0
        assert float((cout.float() - out.float()).abs().max()) <= 1e-2
        for st in ta[:3]:
            casc(st)
        ev_c = [evpair() for _ in ta]
        with ClockSampler(local) as clocks_c:
            for st, (e0, e1) in zip(ta, ev_c):
                e0.record(stream)
                casc(st)
                e1.record(stream)
            torch.cuda.synchronize()
        ev_cf = [evpair() for _ in tb]
        for i, (st, (e0, e1)) in enumerate(zip(tb, ev_cf)):
            flush_w.fill_(i)
            flush_r.sum()
            e0.record(stream)
            casc(st)
            e1.record(stream)
        torch.cuda.synchronize()
        cms = statistics.mean(a.elapsed_time(b) for a, b in ev_c)
        cms_f = statistics.mean(a.elapsed_time(b) for a, b in ev_cf)

        # both calls replayed from CUDA graphs (10 calls a graph): the GPU time without host launch gaps
        def graph_ms(fn, n=10, reps=10):
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(torch.cuda.current_stream(dev))
            with torch.cuda.stream(side):
                for _ in range(2):
                    fn(side)
            torch.cuda.current_stream(dev).wait_stream(side)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                cs = torch.cuda.current_stream(dev)
                for _ in range(n):
                    fn(cs)
            torch.cuda.synchronize()
            ts = []
            for _ in range(reps):
                e0, e1 = evpair()
                e0.record(stream)
                with torch.cuda.stream(stream):
                    g.replay()
                e1.record(stream)
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1) / n)
            del g
            return statistics.median(ts)

        st = ta[-1]
        g_casc = graph_ms(lambda s: binding.paged_attention_decode_shared_prefix(
            cout, st["q"], cache.k_cache, cache.v_cache, st["tables"], st["lens"], pre, w.scale, maxctx,
            workspace=cws, stream=s))
        g_plain = graph_ms(lambda s: cache.attention(out, st["q"], st["tables"], st["lens"], w.scale,
                                                     max_context_len=maxctx, partition_tokens=part,
                                                     workspace=workspace, stream=s))
        assert binding.get_device_error() == 0
        au_b = statistics.mean(st["unique"] for st in tb)
        cascade = {"attention_ms": round(cms, 5), "attention_achieved_unique": round(au / (cms * 1e-3) / 1e9, 1),
                   "attention_frac_unique": round(au / (cms * 1e-3) / 1e9 / peak, 4),
                   "speedup_vs_per_sequence": round(aa / cms, 3),
                   "l2_flushed": {"attention_ms": round(cms_f, 5),
                                  "attention_achieved_unique": round(au_b / (cms_f * 1e-3) / 1e9, 1),
                                  "attention_frac_unique": round(au_b / (cms_f * 1e-3) / 1e9 / peak, 4),
                                  "speedup_vs_per_sequence": round(ab / cms_f, 3)},
                   "graph": {"attention_ms": round(g_casc, 5), "per_sequence_ms": round(g_plain, 5),
                             "attention_achieved_unique": round(st["unique"] / (g_casc * 1e-3) / 1e9, 1),
                             "attention_frac_unique": round(st["unique"] / (g_casc * 1e-3) / 1e9 / peak, 4),
                             "speedup_vs_per_sequence": round(g_plain / g_casc, 3),
                             "how": "10 calls captured in a CUDA graph, replayed; L2 not flushed"},
                   "prefix_tokens": pre, "clocks": clocks_c.summary(),
                   "path": "pkv_paged_attention_decode_shared_prefix: the shared prefix once for all 32 queries "
                           "(tcgen05 multi-query kernel, no causal mask, cut into partitions), each tail (decode "
                           "kernel), then an exact log-sum-exp merge of the partials; same steps, same unique bytes"}

    # ---- e2e: public API calls from pinned host buffers ----
    e2e = None
    if not args.no_e2e:
        hsteps = []
        for i in range(W + K):
            q = wl.decode_q(w, 1000 + i)
            kn, vn = wl.decode_kv(w, 1000 + i)
            hsteps.append(tuple(torch.from_numpy(x).to(dt).pin_memory() for x in (q, kn, vn)))
        h_src = torch.from_numpy(pa[:, 0].copy()).pin_memory()
        h_dst = torch.from_numpy(pa[:, 1].copy()).pin_memory()
        h_out = torch.empty((B, w.num_q_heads, w.head_dim), dtype=torch.bfloat16).pin_memory()
        d_q = torch.empty((B, w.num_q_heads, w.head_dim), dtype=dt, device=dev)
        d_k = torch.empty((B, w.num_kv_heads, w.head_dim), dtype=dt, device=dev)
        d_v = torch.empty_like(d_k)
        d_src = torch.empty(len(pairs), dtype=torch.int64, device=dev)
        d_dst = torch.empty(len(pairs), dtype=torch.int64, device=dev)
        h_slots = torch.empty(B, dtype=torch.int64).pin_memory()
        h_tables = torch.empty((B, mb), dtype=torch.int32).pin_memory()
        h_lens = torch.empty(B, dtype=torch.int32).pin_memory()
        d_slots = torch.empty(B, dtype=torch.int64, device=dev)
        d_tables = torch.empty((B, mb), dtype=torch.int32, device=dev)
        d_lens = torch.empty(B, dtype=torch.int32, device=dev)
        e2e_bytes = []

        def step_host(hq, hk, hv):
            slots, src, dst = cache.bm.append_slots(ids)                  # host block manager
            tables, lens = cache.block_tables(ids)
            h_slots.numpy()[:] = slots
            h_tables.numpy()[:] = tables
            h_lens.numpy()[:] = lens
            for d, h in ((d_q, hq), (d_k, hk), (d_v, hv), (d_src, h_src), (d_dst, h_dst), (d_slots, h_slots),
                         (d_tables, h_tables), (d_lens, h_lens)):
                d.copy_(h, non_blocking=True)
            binding.copy_blocks(cache.k_cache, cache.v_cache, d_src, d_dst, stream=stream)
            cache.append(d_k, d_v, d_slots, stream=stream)
            cache.attention(out, d_q, d_tables, d_lens, w.scale, max_context_len=maxctx, partition_tokens=part,
                            workspace=workspace, stream=stream)
            h_out.copy_(out, non_blocking=True)
            stream.synchronize()
            return unique_attention_bytes(w, tables, lens, 2) + copy_bytes + append_bytes(w)

        for i in range(W):
            step_host(*hsteps[i])
        barrier(ws)
        torch.cuda.synchronize()
        e0, e1 = evpair()
        e0.record(stream)
        for i in range(K):
            e2e_bytes.append(step_host(*hsteps[W + i]))
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
        assert binding.get_device_error() == 0
        e_ms, e_gbs, e_tok = aggregate(e0.elapsed_time(e1), float(sum(e2e_bytes)), float(B * K), ws)
        eb = w.in_bytes
        h2d = (B * w.num_q_heads * w.head_dim * eb + 2 * B * w.num_kv_heads * w.head_dim * eb +
               16 * len(pairs) + B * (8 + mb * 4 + 4))
        e2e = {"value": round(e_gbs, 1), "unit": "GB/s", "decode_tokens_per_s": round(e_tok, 1),
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(B * w.num_q_heads * w.head_dim * 2),
               "ms_per_step": round(e_ms / K, 4),
               "path": "host block manager append, H2D of q / new K,V / copy list / slots / tables / lengths, "
                       "copy_blocks, reshape_and_cache, paged_attention_decode, D2H of the output, stream sync "
                       "(unique bytes)"}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds)
    return {
        "metric": "paged decode attention achieved HBM GB/s (% of B200 peak); decode tokens/s",
        "value": round(gbs, 1), "unit": "GB/s", "n_gpus": ws, "steps": K, "warmup": W,
        "ms_per_step": round(ms_max / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.kv_dtype, "data": "synthetic",
        "bytes_basis": "unique: each physical block's K/V once (the shared prefix once per step)",
        "pct_of_peak": round(100 * gbs / ws / peak, 1), "pct_of_peak_spec": round(100 * gbs / ws / SPEC_HBM_GBS, 1),
        "value_logical": round(gbs_logical, 1),
        "decode_tokens_per_s": round(tokens_s, 1),
        "bytes_per_step": {"attention_unique": int(au), "attention_logical": int(al), "copy_blocks": copy_bytes,
                           "append": append_bytes(w), "copies": len(pairs), "block_bytes": block_bytes},
        "l2_flushed": {"value": round(gbs_b, 1), "value_logical": round(gbs_b_logical, 1),
                       "ms_per_step": round(msb_max / K, 4), "attention_achieved_unique": round(ach_b, 1),
                       "attention_frac_unique": round(ach_b / peak, 4), "avg_attention_ms": round(ab, 5),
                       "clocks": clocks_b.summary()},
        "config": {"workload": w.description, "global_batch": B * ws, "seq_len": f"{p} shared + U[{w.lo},{w.hi}]",
                   "block_size": bs, "schedule": f"partitions of {part_used} tokens" if part != -1 else "persistent",
                   "step": f"copy_blocks of {len(pairs)} copy-on-write pairs (logical block {last}), "
                           f"reshape_and_cache of {B} tokens, paged decode attention",
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
                   "l2": "value: no flush between steps (the 16 MiB prefix stays in L2); l2_flushed: L2 flushed "
                         "before every step (write of 2x L2 then read of another 2x L2), outside the events",
                   "seed": w.seed},
        "roofline": {"bound": "hbm", "kernel": "paged_decode_kernel (one attention call)",
                     "achieved": round(ach, 1), "peak": peak, "peak_source": peak_kind, "unit": "GB/s",
                     "frac": round(ach / peak, 4), "frac_of_spec": round(ach / SPEC_HBM_GBS, 4),
                     "achieved_logical": round(al / (aa * 1e-3) / 1e9, 1), "avg_launch_ms": round(aa, 5),
                     "algorithmic_bytes_per_launch": int(au), "bytes_basis": "unique", "traffic": None},
        "e2e": e2e,
        "cascade": cascade,
        "gpu_launches": (2 + decode_launches(B, part, part_used, maxctx, bs)) * K,   # + copy_blocks, append
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
    }


def run_swap(args, ws, rank, local):
    """Swap-out and swap-in of every other sequence of the workload through the
    cache's public calls (block manager + block-id staging + one swap kernel per
    direction), timed with CUDA events; the kernel alone on the same block sets;
    and, as the host-link roofline, one contiguous page-locked copy of the same
    bytes per direction by the copy engine."""
    import torch
    from paged_kv_cache_322_b200 import binding
    from paged_kv_cache_322_b200.engine import PagedKVCache

    dev = torch.device("cuda", local)
    w = replica_workload(wl.WORKLOADS[args.workload], rank)
    w = override_workload(w, args)
    K, W = args.steps, args.warmup
    lens = wl.context_lens(w)
    bs = w.block_size
    group = list(range(0, w.num_seqs, 2))
    nblk = int(sum(-(-int(lens[s]) // bs) for s in group))
    cdt = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.uint8}[w.kv_dtype]
    cache = PagedKVCache(w.num_blocks, bs, w.num_kv_heads, w.head_dim, cdt, dev, free_order=wl.free_order(w),
                         host_blocks=nblk)
    for s in range(w.num_seqs):
        cache.bm.allocate(s, int(lens[s]))
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    for c in (cache.k_cache, cache.v_cache):           # synthetic pool contents (a copy does not read values)
        c.view(torch.uint8).copy_(torch.randint(0, 256, c.view(torch.uint8).shape, device=dev, dtype=torch.uint8,
                                                generator=g))
    stream = torch.cuda.current_stream(dev)
    block_bytes = bs * w.num_kv_heads * w.head_dim * w.elt_bytes
    moved = 2 * nblk * block_bytes                       # K and V, one direction

    def ev():
        return torch.cuda.Event(enable_timing=True)

    # ---- through the cache's calls ----
    t_out, t_in = [], []
    for i in range(W + K):
        e0, e1, e2 = ev(), ev(), ev()
        e0.record(stream)
        pairs_out = cache.swap_out(group)
        e1.record(stream)
        pairs_in = cache.swap_in(group)
        e2.record(stream)
        if i >= W:
            t_out.append((e0, e1))
            t_in.append((e1, e2))
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0 and len(pairs_out) == nblk and len(pairs_in) == nblk
    api_out = statistics.median(a.elapsed_time(b) for a, b in t_out)
    api_in = statistics.median(a.elapsed_time(b) for a, b in t_in)

    # ---- the kernel alone, same block sets (device ids of the last swap-in) ----
    dblk = torch.tensor([d for _, d in pairs_in], dtype=torch.int64, device=dev)
    hblk = torch.tensor([h for h, _ in pairs_in], dtype=torch.int64, device=dev)
    k_out, k_in = [], []
    for i in range(W + K):
        e0, e1, e2 = ev(), ev(), ev()
        e0.record(stream)
        binding.swap_blocks(cache.k_cache, cache.v_cache, cache.k_host, cache.v_host, dblk, hblk)
        e1.record(stream)
        binding.swap_blocks(cache.k_host, cache.v_host, cache.k_cache, cache.v_cache, hblk, dblk)
        e2.record(stream)
        if i >= W:
            k_out.append((e0, e1))
            k_in.append((e1, e2))
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    kern_out = statistics.median(a.elapsed_time(b) for a, b in k_out)
    kern_in = statistics.median(a.elapsed_time(b) for a, b in k_in)

    # ---- roofline: one contiguous page-locked copy of the same bytes per direction ----
    hbuf = torch.empty(moved, dtype=torch.uint8, pin_memory=True)
    dbuf = torch.empty(moved, dtype=torch.uint8, device=dev)
    c_out, c_in = [], []
    for i in range(W + K):
        e0, e1, e2 = ev(), ev(), ev()
        e0.record(stream)
        hbuf.copy_(dbuf, non_blocking=True)
        e1.record(stream)
        dbuf.copy_(hbuf, non_blocking=True)
        e2.record(stream)
        if i >= W:
            c_out.append((e0, e1))
            c_in.append((e1, e2))
    torch.cuda.synchronize()
    copy_out = statistics.median(a.elapsed_time(b) for a, b in c_out)
    copy_in = statistics.median(a.elapsed_time(b) for a, b in c_in)

    def gbs(ms):
        return round(moved / (ms * 1e-3) / 1e9, 2)

    ms_step = api_out + api_in
    ms_max, total_gbs, _ = aggregate(ms_step * K, 2.0 * moved * K, float(len(group) * K), ws)
    ach = 2.0 * moved / ((kern_out + kern_in) * 1e-3) / 1e9
    peak = 2.0 * moved / ((copy_out + copy_in) * 1e-3) / 1e9
    return {
        "metric": "swap_blocks: preemption swap-out + swap-in GB/s over the host link (device <-> page-locked host)",
        "value": round(total_gbs, 2), "unit": "GB/s", "n_gpus": ws, "steps": K, "warmup": W,
        "ms_per_step": round(ms_max / K, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.kv_dtype, "data": "synthetic",
        "config": {"workload": f"swap every other sequence of: {w.description}", "sequences_swapped": len(group),
                   "blocks_per_direction": nblk, "bytes_per_direction": moved,
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"},
        "api": {"swap_out_ms": round(api_out, 4), "swap_in_ms": round(api_in, 4), "swap_out_gbs": gbs(api_out),
                "swap_in_gbs": gbs(api_in)},
        "kernel": {"swap_out_ms": round(kern_out, 4), "swap_in_ms": round(kern_in, 4),
                   "swap_out_gbs": gbs(kern_out), "swap_in_gbs": gbs(kern_in)},
        "roofline": {"bound": "host_link", "achieved": round(ach, 2), "peak": round(peak, 2), "unit": "GB/s",
                     "frac": round(ach / peak, 4),
                     "peak_source": "measured in this run: one contiguous page-locked copy of the same bytes per "
                                    f"direction (copy engine; out {gbs(copy_out)} GB/s, in {gbs(copy_in)} GB/s)",
                     "traffic": None},
        "gpu_launches": 2 * K,
    }


def fork_pairs(bm, B: int, samples: int):
    """One parallel-sampling fork of every sequence 0..B-1 through the block
    manager: samples - 1 children per parent, each child appending its first own
    token (a shared, partly filled last block is copied on that write), then the
    children freed. Returns the copy lists (src, dst) int64."""
    kids = np.arange(B, B * samples, dtype=np.int64)
    for c in kids:
        bm.fork(int((c - B) // (samples - 1)), int(c))
    _, src, dst = bm.append_slots(kids)
    for c in kids:
        bm.free(int(c))
    return src.copy(), dst.copy()


def run_fork(args, ws, rank, local):
    """copy_blocks under parallel sampling: every sequence of the workload forks
    into --samples samples; each child's first divergent token copies the shared
    last block (copy-on-write). The copy kernel is timed alone on the block
    manager's copy lists, L2 flushed before each step; the e2e leg runs the fork,
    the copy lists' H2D, the kernel and the error-word read per step."""
    import torch
    from paged_kv_cache_322_b200 import binding
    from paged_kv_cache_322_b200.engine import PagedKVCache

    dev = torch.device("cuda", local)
    w = replica_workload(wl.WORKLOADS[args.workload], rank)
    w = override_workload(w, args)
    K, W, n = args.steps, args.warmup, args.samples
    if n < 2:
        raise SystemExit("--samples must be >= 2")
    lens = wl.context_lens(w)
    bs, B = w.block_size, w.num_seqs
    cdt = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.uint8}[w.kv_dtype]
    cache = PagedKVCache(w.num_blocks, bs, w.num_kv_heads, w.head_dim, cdt, dev, free_order=wl.free_order(w))
    for s in range(B):
        cache.bm.allocate(s, int(lens[s]))
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    for c in (cache.k_cache, cache.v_cache):           # synthetic pool contents (a copy does not read values)
        c.view(torch.uint8).copy_(torch.randint(0, 256, c.view(torch.uint8).shape, device=dev, dtype=torch.uint8,
                                                generator=g))
    block_bytes = bs * w.num_kv_heads * w.head_dim * w.elt_bytes
    sets = [fork_pairs(cache.bm, B, n) for _ in range(W + K)]   # the free list rotates: new dst blocks each step
    npairs = int(sets[0][0].size)
    assert all(s.size == npairs for s, _ in sets)
    moved = 2 * npairs * block_bytes * 2 + 16 * npairs   # K and V read once and written once; the two ids
    dsets = [(torch.from_numpy(s).to(dev), torch.from_numpy(d).to(dev)) for s, d in sets]
    # L2 flush: write a buffer of 2x L2, then read another one, so that the timed
    # copy starts from an L2 holding only clean, unrelated lines (a write-only
    # flush leaves ~L2 of dirty lines whose write-back would land in the copy)
    flush_w = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    flush_r = torch.ones(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def flush(i):
        flush_w.fill_(i)
        return flush_r.sum()

    for i in range(W):
        flush(i)
        binding.copy_blocks(cache.k_cache, cache.v_cache, *dsets[i])
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(K):
            flush(W + i)
            ev[i][0].record(stream)
            binding.copy_blocks(cache.k_cache, cache.v_cache, *dsets[W + i])
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    assert binding.get_device_error() == 0
    ms = sum(a.elapsed_time(b) for a, b in ev)
    ms_max, total_gbs, _ = aggregate(ms, float(moved * K), float(npairs * K), ws)
    copy_ms = ms / K
    ach = moved / (copy_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    del dsets, flush_w, flush_r

    # ---- e2e: fork in the block manager, copy lists H2D, kernel, error word D2H ----
    e2e = None
    if not args.no_e2e:
        hs = torch.empty(npairs, dtype=torch.int64, pin_memory=True)
        hd = torch.empty(npairs, dtype=torch.int64, pin_memory=True)
        ds, dd = torch.empty(npairs, dtype=torch.int64, device=dev), torch.empty(npairs, dtype=torch.int64, device=dev)

        def step_host():
            src, dst = fork_pairs(cache.bm, B, n)
            hs.numpy()[:] = src
            hd.numpy()[:] = dst
            ds.copy_(hs, non_blocking=True)
            dd.copy_(hd, non_blocking=True)
            binding.copy_blocks(cache.k_cache, cache.v_cache, ds, dd, stream=stream)
            if binding.get_device_error() != 0:         # D2H of the error word; synchronises the stream
                raise RuntimeError("copy_blocks flagged a bad block id")

        for _ in range(W):
            step_host()
        barrier(ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            step_host()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
        e_ms, e_gbs, _ = aggregate(e0.elapsed_time(e1), float(moved * K), float(npairs * K), ws)
        e2e = {"value": round(e_gbs, 2), "unit": "GB/s", "h2d_bytes_per_step": 16 * npairs,
               "d2h_bytes_per_step": 4, "ms_per_step": round(e_ms / K, 4),
               "path": "block manager fork + append_slots, H2D of the copy lists, copy_blocks, error word D2H"}

    return {
        "metric": "copy_blocks: copy-on-write block copies under parallel sampling, GB/s (K and V read + written)",
        "value": round(total_gbs, 2), "unit": "GB/s", "n_gpus": ws, "steps": K, "warmup": W,
        "ms_per_step": round(ms_max / K, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.kv_dtype, "data": "synthetic",
        "config": {"workload": f"parallel sampling, {n} samples per sequence, of: {w.description}",
                   "samples": n, "copies_per_step": npairs, "block_bytes": block_bytes,
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
                   "l2": "L2 flushed before each step, outside the timed events: a write of 2x L2, then a read "
                         "of another 2x L2 buffer (no dirty lines left to write back inside the copy)"},
        "roofline": {"bound": "hbm", "kernel": "block_copy_kernel", "achieved": round(ach, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(ach / peak, 4), "avg_launch_ms": round(copy_ms, 5),
                     "algorithmic_bytes_per_launch": moved, "peak_source": peak_kind, "traffic": None},
        "e2e": e2e,
        "gpu_launches": K,
        "clocks": clocks.summary(),
    }


def run_mq(args, ws, rank, local):
    """Causal multi-query steps: every sequence appends --query-len tokens (a
    prefill chunk, or draft tokens to verify) and attends with them over its
    cache. Device-timed: the append kernel + the multi-query attention over
    inputs already in HBM; the attention launches alone give the roofline
    (tensor FLOP/s when the step's FLOP per algorithmic byte is above the
    measured ridge, HBM GB/s otherwise). e2e: the same steps through
    PagedKVCache.extend from page-locked host buffers, output read back."""
    import torch
    from paged_kv_cache_322_b200 import binding
    from paged_kv_cache_322_b200.engine import PagedKVCache

    dev = torch.device("cuda", local)
    w = replica_workload(override_workload(wl.WORKLOADS[args.workload], args), rank)
    if w.kv_dtype != "bf16":
        raise SystemExit("--op mq runs bf16 caches")
    n, K, W = args.query_len, args.steps, args.warmup
    part = 0 if args.partition_tokens in (-2, -1) else args.partition_tokens
    lens0 = wl.context_lens(w)
    bs, B = w.block_size, w.num_seqs
    grow = 2 * (K + W) * n                              # device loop, then the e2e loop
    mb = -(-int(lens0.max() + grow) // bs)
    nb = max(w.num_blocks, int(sum(-(-(int(c) + grow) // bs) for c in lens0)) + 64)
    cache = PagedKVCache(nb, bs, w.num_kv_heads, w.head_dim, torch.bfloat16, dev, free_order=wl.free_order(
        dataclasses.replace(w, num_blocks=nb)), max_blocks_per_seq=mb)
    kvs = wl.prompt_kv_all(w, lens0)
    for s in range(B):
        cache.add_sequence(s, torch.from_numpy(kvs[s][0]).to(dev, torch.bfloat16),
                           torch.from_numpy(kvs[s][1]).to(dev, torch.bfloat16))
    del kvs
    ids = np.arange(B, dtype=np.int64)
    hq, hkv, d = w.num_q_heads, w.num_kv_heads, w.head_dim
    T = B * n
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)

    def rnd(shape):
        return torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)

    def flops_and_bytes(lens_after):
        return mq_flops(lens_after, n, hq, d), mq_attention_bytes(lens_after, n, hq, hkv, d, bs)

    steps = []
    order = np.repeat(ids, n)
    for i in range(K + W):
        slots, src, dst = cache.bm.append_slots(order)
        assert src.size == 0
        tables, lens = cache.block_tables(ids)
        fl, by = flops_and_bytes(lens)
        steps.append(dict(q=rnd((T, hq, d)), k=rnd((T, hkv, d)), v=rnd((T, hkv, d)),
                          slots=torch.from_numpy(slots).to(dev), tables=torch.from_numpy(tables).to(dev),
                          lens=torch.from_numpy(lens).to(dev), maxlen=int(lens.max()), flops=fl, bytes=by))
    qs = torch.from_numpy(np.arange(0, T + 1, n, dtype=np.int32)).to(dev)
    out = torch.empty((T, hq, d), dtype=torch.bfloat16, device=dev)
    maxctx = max(st["maxlen"] for st in steps)
    wsb = binding.multi_query_workspace_bytes(B, T, hq, hkv, d, bs, mb, n, maxctx, part)
    workspace = torch.empty(max(wsb, 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step_device(st, e0=None, e1=None):
        cache.append(st["k"], st["v"], st["slots"])
        if e0 is not None:
            e0.record(stream)
        binding.paged_attention_multi_query(out, st["q"], cache.k_cache, cache.v_cache, st["tables"], st["lens"], qs,
                                            w.scale, max_query_len=n, max_context_len=maxctx, partition_tokens=part,
                                            workspace=workspace)
        if e1 is not None:
            e1.record(stream)

    for i in range(W):
        step_device(steps[i])
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for i in range(K):
            step_device(steps[W + i], *ev[i])
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    assert binding.get_device_error() == 0
    ms = t0.elapsed_time(t1)
    attn_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    timed = steps[W:]
    fl = statistics.mean(st["flops"] for st in timed)
    by = statistics.mean(st["bytes"] for st in timed)
    ms_max, _, tok_s = aggregate(ms, 0.0, float(T * K), ws)
    flop_total = all_sum(float(sum(st["flops"] for st in timed)), ws)
    peak_gbs, peak_kind = measured_peaks()
    peak_tf = measured_tflops()
    ridge = peak_tf * 1e12 / (peak_gbs * 1e9)
    tensor = fl / by > ridge
    ach = (fl / (attn_ms * 1e-3) / 1e12) if tensor else (by / (attn_ms * 1e-3) / 1e9)
    peak = peak_tf if tensor else peak_gbs
    del steps

    # ---- e2e: PagedKVCache.extend from page-locked host buffers ----
    e2e = None
    if not args.no_e2e:
        host = [tuple(torch.empty(shape, dtype=torch.bfloat16).normal_().pin_memory()
                      for shape in ((T, hq, d), (T, hkv, d), (T, hkv, d))) for _ in range(2)]
        dq, dk, dv = (torch.empty(x.shape, dtype=torch.bfloat16, device=dev) for x in host[0])
        out_h = torch.empty((T, hq, d), dtype=torch.bfloat16).pin_memory()

        def step_host(hb):
            for dst_t, src_t in zip((dq, dk, dv), hb):
                dst_t.copy_(src_t, non_blocking=True)
            cache.extend(ids, [n] * B, dq, dk, dv, w.scale, out=out, partition_tokens=part, stream=stream)
            out_h.copy_(out, non_blocking=True)
            stream.synchronize()

        for i in range(W):
            step_host(host[i % 2])
        barrier(ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(K):
            step_host(host[i % 2])
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
        assert binding.get_device_error() == 0
        e_ms, _, e_tok_s = aggregate(e0.elapsed_time(e1), 0.0, float(T * K), ws)
        e2e = {"value": round(e_tok_s, 1), "unit": "query tokens/s",
               "h2d_bytes_per_step": int(T * (hq + 2 * hkv) * d * 2 + T * 8 + B * (mb * 4 + 8)),
               "d2h_bytes_per_step": int(T * hq * d * 2), "ms_per_step": round(e_ms / K, 4),
               "path": "PagedKVCache.extend (block manager, H2D, append, multi-query attention), D2H, sync"}

    return {
        "metric": f"multi-query paged attention ({'chunked prefill' if n >= 64 else 'speculative verify'}): "
                  "query tokens/s per step (append + causal attention)",
        "value": round(tok_s, 1), "unit": "query tokens/s", "n_gpus": ws, "steps": K,
        "warmup": W, "ms_per_step": round(ms_max / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "attention_tflops": round(flop_total / (ms_max * 1e-3) / 1e12, 2),
        "config": {"workload": w.description, "query_len": n, "global_batch": B * ws, "block_size": bs,
                   "partition_tokens": part or "library-chosen",
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
                   "l2": "KV per step larger than L2; no flush", "seed": w.seed},
        "roofline": {"bound": "tensor" if tensor else "hbm",
                     "kernel": ("tc::paged_mq_tc_kernel (tcgen05)" if d == 128 and n * (hq // hkv) >= 32
                                else "paged_mq_kernel (mma.sync)") + " (+ merge_mq_kernel when partitioned)",
                     "achieved": round(ach, 2), "peak": peak, "unit": "TFLOP/s" if tensor else "GB/s",
                     "frac": round(ach / peak, 4), "avg_launch_ms": round(attn_ms, 5),
                     "flops_per_launch": int(fl), "algorithmic_bytes_per_launch": int(by),
                     "flop_per_byte": round(fl / by, 1), "ridge_flop_per_byte": round(ridge, 1),
                     "peak_source": ("measured bf16 dense (cuBLAS burst)" if tensor else peak_kind), "traffic": None},
        "e2e": e2e,
        "gpu_launches": 2 * K + (K if part and maxctx > part else 0),
        "clocks": clocks.summary(),
    }


def paging_overhead(w, cache, kvs, dev, dt, cdt, mb, part, K, W):
    """The same attention call over the same prompts stored twice: blocks in the
    workload's random physical placement (the bench cache) and in identity
    placement (each sequence's blocks consecutive in the pool). Calls alternate,
    each timed with CUDA events; ratio = random / identity time."""
    import torch
    from paged_kv_cache_322_b200 import binding
    from paged_kv_cache_322_b200.engine import PagedKVCache
    ident = PagedKVCache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, cdt, dev,
                         free_order=np.arange(w.num_blocks, dtype=np.int32), max_blocks_per_seq=mb,
                         kv_scales=(w.kv_scale, w.kv_scale))
    for s in range(w.num_seqs):
        k, v = kvs[s]
        ident.add_sequence(s, torch.from_numpy(k).to(dev, dt), torch.from_numpy(v).to(dev, dt))
    ids = np.arange(w.num_seqs, dtype=np.int64)
    legs = []
    for c in (cache, ident):
        tables, lens = c.block_tables(ids)
        legs.append((c, torch.from_numpy(tables).to(dev), torch.from_numpy(lens).to(dev), int(lens.max())))
    q = torch.from_numpy(wl.decode_q(w, 0)).to(dev, dt)
    out = torch.empty((w.num_seqs, w.num_q_heads, w.head_dim), dtype=torch.bfloat16, device=dev)
    ws_bytes = binding.workspace_bytes(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, mb,
                                       legs[0][3], part)
    workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    times = ([], [])
    for i in range(W + K):
        for j, (c, t, l, mx) in enumerate(legs):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            c.attention(out, q, t, l, w.scale, max_context_len=mx, partition_tokens=part, workspace=workspace)
            e1.record(stream)
            if i >= W:
                times[j].append((e0, e1))
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    r_ms, i_ms = (statistics.median(a.elapsed_time(b) for a, b in t) for t in times)
    del ident
    torch.cuda.empty_cache()
    return {"random_placement_ms": round(r_ms, 5), "identity_placement_ms": round(i_ms, 5),
            "ratio": round(r_ms / i_ms, 4),
            "what": "median attention-call time over the prompts (no append), random vs identity block placement"}


def cpu_baseline(w: wl.Workload, target_s: float):
    """The oracle, as it stands, on a bounded sample of the same workload: whole
    sequences (their logical K/V regenerated from the seeded generator, written
    into an oracle pool, attention in fp64), sequence after sequence and step
    after step, until ~target_s seconds of CPU time."""
    from oracle import cache_ops as ocache
    from oracle import paged_attention as oattn
    from oracle.block_manager import BlockManager as OracleBM
    lens = wl.context_lens(w)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    done, nbytes, t_total, step = 0, 0, 0.0, 0
    while t_total < target_s:
        q = wl.decode_q(w, step)
        for s in range(w.num_seqs):
            n = int(lens[s])
            k, v = wl.prompt_kv(w, s, n)
            nblk = -(-n // w.block_size)
            bm = OracleBM(nblk, w.block_size)
            kc = np.zeros((nblk, w.block_size, w.num_kv_heads, w.head_dim), np.float32)
            vc = np.zeros_like(kc)
            t0 = time.perf_counter()
            if w.kv_dtype == "fp8":
                kc, vc = kc.astype(np.uint8), vc.astype(np.uint8)
                ocache.reshape_and_cache_fp8(k, v, kc, vc, np.asarray(bm.allocate(0, n)), w.kv_scale, w.kv_scale)
                oattn.paged_attention_decode_fp8(q[s:s + 1], kc, vc, [bm.block_table(0)], [n], w.scale,
                                                 w.block_size, w.kv_scale, w.kv_scale)
            else:
                ocache.reshape_and_cache(k, v, kc, vc, np.asarray(bm.allocate(0, n)))
                oattn.paged_attention_decode(q[s:s + 1], kc, vc, [bm.block_table(0)], [n], w.scale, w.block_size)
            t_total += time.perf_counter() - t0
            done += 1
            nbytes += n * w.num_kv_heads * w.head_dim * w.elt_bytes * 2 + 2 * w.num_q_heads * w.head_dim * w.in_bytes
            if t_total >= target_s:
                break
        step += 1
    return {"value": round(nbytes / t_total / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} sequence-steps of the bench workload ({w.num_seqs} sequences per step; KV append "
                      f"into an oracle pool + fp64 attention), {t_total:.1f} s of CPU time",
            "decode_tokens_per_s": round(done / t_total, 2)}


def step_bytes_cpu(w: wl.Workload) -> int:
    """Bytes cpu_baseline counts for one whole step of the workload (every
    sequence's K and V read once, its q in and out)."""
    return int(sum(int(n) * w.num_kv_heads * w.head_dim * w.elt_bytes * 2 + 2 * w.num_q_heads * w.head_dim *
                   w.in_bytes for n in wl.context_lens(w)))


def run_reference(args, ws, rank):
    """The reference arm: the CPU oracle, timed per step on a bounded sample of
    the same workload (with the same overrides) as the library arm."""
    w = override_workload(wl.WORKLOADS[args.workload], args)
    if rank != 0:
        return None
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    per_step_s = max(0.5, min(10.0, 90.0 / max(1, args.steps + args.warmup)))
    vals = []
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(w, per_step_s)
        if i >= args.warmup:
            vals.append(r)
    v = statistics.mean(x["value"] for x in vals)
    return {"impl": "reference", "metric": "paged decode attention achieved HBM GB/s (% of B200 peak); decode tokens/s",
            "value": round(v, 4), "unit": "GB/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(step_bytes_cpu(w) / (v * 1e9) * 1e3, 3),
            "ms_per_step_basis": "one whole step of the workload at the sampled rate",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "decode_tokens_per_s": round(statistics.mean(x["decode_tokens_per_s"] for x in vals), 2),
            "config": {"workload": w.description, "global_batch": w.num_seqs, "block_size": w.block_size,
                       "parallelism": "CPU oracle on rank 0's host cores", "seed": w.seed},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"per step: {vals[0]['sample']}"},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def sub_result(workload: str, args) -> dict:
    """The same decode-step measurement on another workload, run as a child
    process on the same GPU (its own caches; no e2e, CPU baseline or paging
    run), reduced to its throughput, roofline and clocks."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--workload", workload, "--steps", str(args.steps),
           "--warmup", str(args.warmup), "--no-e2e", "--no-cpu-baseline", "--no-paging-overhead", "--no-extra"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=900)
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    if r.returncode != 0 or not lines:
        return {"workload": workload, "error": (r.stderr or r.stdout)[-500:]}
    d = json.loads(lines[-1])
    keep = ("value", "unit", "ms_per_step", "pct_of_peak", "pct_of_peak_spec", "decode_tokens_per_s", "roofline",
            "clocks", "gpu_launches")
    out = {"workload": d["config"]["workload"], "schedule": d["config"]["schedule"]}
    out.update({k: d[k] for k in keep if k in d})
    return out


def main():
    args = parse()
    if args.impl == "reference":
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        r = run_reference(args, ws, rank)
        if r is not None:
            print(json.dumps(r), flush=True)
        return
    ws, rank, local = dist_init(args)
    try:
        run = {"swap": run_swap, "mq": run_mq, "fork": run_fork}.get(args.op, run_pkv)
        if args.op == "decode" and wl.WORKLOADS[args.workload].ctx == "shared_prefix":
            run = run_shared_prefix
        r = run(args, ws, rank, local)
        if (rank == 0 and ws == 1 and args.op == "decode" and args.workload == "llama2_7b" and not args.no_extra
                and not (args.num_seqs or args.num_blocks or args.block_size)):
            r["gqa_70b"] = sub_result("gqa_70b", args)
        if rank == 0:
            print(json.dumps(r), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
