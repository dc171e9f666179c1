#!/usr/bin/env python3
"""Benchmark of the Dual-QK decode hot path (libdualqk) on B200.

One step = one pass of the whole path over the batch: dqk_append of the step's
new K/V row per sequence (position L-1), then dqk_decode (query transform and
channel selection, split-K pruned attention over the INT2 cache, LSE combine).

Default workload: batch 4, 32 q / 8 kv heads, head_dim 128, 128K context,
16-token pages in seeded random order, 40 % query-channel sparsity.  The cache
(411 MB) is larger than L2, so no flush is needed between steps.

Prints ONE JSON line (rank 0).  --impl reference times the CPU oracle on a
bounded sample of the same workload instead.  --gpus N without an outer
launcher re-runs this script under torch.distributed.run with N ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode KV-tokens/s and achieved HBM GB/s (% of roofline) at 128K ctx, 1 B200"
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------
# helpers shared with the multi-process tests
# ----------------------------------------------------------------------------
def world():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(tokens_per_rank: int, elapsed_s: float, steps: int, n_ranks: int, device=None) -> dict:
    """Whole-job throughput: all ranks' tokens / the slowest rank's time."""
    t = reduce_max(elapsed_s, device)
    return {"value": tokens_per_rank * steps * n_ranks / t, "ms_per_step": 1e3 * t / steps, "elapsed_s": t}


def rank_workload(w, rank: int):
    """Weak scaling: every rank decodes its own independent batch of sequences
    (same layer shapes, its own seeded contents); nothing crosses ranks."""
    return w if rank == 0 else w.with_(seed=w.seed + 7919 * rank)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_kv_cache_dqk_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh")):
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if the kernel sources
    have not changed since it was taken (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(f"{kernel}/{workload}")
    if not rec or rec.get("source_hash") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """NVML SM clock / throttle-reason sampler, run during the timed region."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int, period_s: float = 0.001):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        for bit, name in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.nv or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# the layer on the device
# ----------------------------------------------------------------------------
class Layer:
    def __init__(self, w, dev):
        import torch
        from bit_kv_cache_dqk_b200 import dualqk as Q
        from bit_kv_cache_dqk_b200 import inputs as I
        self.Q, self.I, self.torch, self.w, self.dev = Q, I, torch, w, dev
        self.lens = I.lengths(w)
        self.table, self.num_pages = I.page_table(w, self.lens)
        self.max_pages = self.table.shape[1]
        from bit_kv_cache_dqk_b200 import calibrate as Cb
        tk, tq, _, _ = Cb.layer_transforms(w)
        self.t_k = torch.from_numpy(tk).to(dev)
        self.t_q = torch.from_numpy(tq).to(dev)
        probe = Q.layer_desc(w.d, w.hq, w.hkv, 0, 0, 0, 1, group_size=w.group_size)
        self.bb = Q.dqk_block_bytes(probe)
        self.pool = torch.empty(self.num_pages * w.hkv * self.bb, dtype=torch.uint8, device=dev)
        self.desc = Q.layer_desc(w.d, w.hq, w.hkv, self.t_k, self.t_q, self.pool, self.num_pages,
                                 group_size=w.group_size)
        self.table_d = torch.from_numpy(self.table).to(dev)
        self.lens_d = torch.from_numpy(self.lens).to(dev)
        self.ws_bytes = Q.dqk_decode_workspace_size(self.desc, w.batch, self.max_pages)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.keep = w.d - (w.pct * w.d) // 100
        self.out = torch.empty((w.batch, w.hq, w.d), dtype=torch.float32, device=dev)
        self.sel = torch.empty((w.batch, w.hq, self.keep), dtype=torch.int16, device=dev)

    def prefill(self, chunk=8192):
        torch, Q, I, w = self.torch, self.Q, self.I, self.w
        done = np.zeros(w.batch, np.int32)
        target = self.lens - 1                 # the last row is appended by every step
        while (done < target).any():
            new = np.minimum(chunk, target - done).astype(np.int32)
            ks, vs = zip(*[I.kv_rows(w, b, int(done[b]), int(done[b] + new[b])) for b in range(w.batch)])
            k = torch.from_numpy(np.concatenate(ks)).to(torch.bfloat16).to(self.dev)
            v = torch.from_numpy(np.concatenate(vs)).to(torch.bfloat16).to(self.dev)
            Q.dqk_append(self.desc, k, v, Q.DQK_BF16, w.batch, torch.from_numpy(new).to(self.dev),
                         torch.from_numpy(done.copy()).to(self.dev), int(new.max()), self.table_d,
                         self.max_pages)
            done += new
        torch.cuda.synchronize(self.dev)
        # the step's inputs: the row at position L-1 and the query
        ks, vs = zip(*[I.kv_rows(w, b, int(self.lens[b]) - 1, int(self.lens[b])) for b in range(w.batch)])
        self.k_host = torch.from_numpy(np.concatenate(ks)).to(torch.bfloat16).pin_memory()
        self.v_host = torch.from_numpy(np.concatenate(vs)).to(torch.bfloat16).pin_memory()
        self.q_host = torch.from_numpy(I.queries(w, self.lens)).to(torch.bfloat16).pin_memory()
        self.k_step = self.k_host.to(self.dev)
        self.v_step = self.v_host.to(self.dev)
        self.q_step = self.q_host.to(self.dev)
        self.out_host = torch.empty(self.out.shape, dtype=torch.float32).pin_memory()
        self.ones = torch.ones(w.batch, dtype=torch.int32, device=self.dev)
        self.before = (self.lens_d - 1).contiguous()

    def step(self):
        """One fused decode step: append 1 row per sequence + decode
        (dqk_decode_step: the append and the query preparation overlap)."""
        Q, w = self.Q, self.w
        Q.dqk_decode_step(self.desc, self.k_step, self.v_step, Q.DQK_BF16, self.ones, self.before, 1,
                          self.q_step, Q.DQK_BF16, w.batch, self.lens_d, self.table_d, self.max_pages, w.pct,
                          self.out, self.sel, self.ws, self.ws_bytes)

    def decode(self):
        """dqk_decode alone (the query and the cache as they are)."""
        Q, w = self.Q, self.w
        Q.dqk_decode(self.desc, self.q_step, Q.DQK_BF16, w.batch, self.lens_d, self.table_d, self.max_pages, w.pct,
                     self.out, self.sel, self.ws, self.ws_bytes)

    def per_launch_ms(self, fn, n):
        """Mean device time of one call of fn (one kernel launch), each call
        bracketed by its own CUDA events on the current stream."""
        torch = self.torch
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for a, b in ev:
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize(self.dev)
        return statistics.mean(a.elapsed_time(b) for a, b in ev)

    def step_e2e(self):
        """The same step from pinned host buffers: H2D inputs, D2H result."""
        self.k_step.copy_(self.k_host, non_blocking=True)
        self.v_step.copy_(self.v_host, non_blocking=True)
        self.q_step.copy_(self.q_host, non_blocking=True)
        self.step()
        self.out_host.copy_(self.out, non_blocking=True)

    def algorithmic_bytes(self) -> tuple[float, float]:
        return algorithmic_bytes(self.w, self.sel.cpu().numpy(), self.lens)


def algorithmic_bytes(w, sel: np.ndarray, lens: np.ndarray) -> tuple[float, float]:
    """Bytes the attend kernel must touch per launch (retained-channel key
    codes for the union of the GQA group's kept channels, K scale/min of
    touched groups, K channel 0, V codes, V scale/min) and per token-kv-head."""
    G, ns = w.group, w.d // w.group_size
    total = 0.0
    for b in range(len(lens)):
        for j in range(w.hkv):
            kept = np.zeros(w.d, bool)
            kept[sel[b, j * G:(j + 1) * G].ravel()] = True
            kept[0] = False
            u = int(kept.sum())
            groups = int(kept.reshape(ns, w.group_size).any(axis=1).sum())
            per_tok = -(-u // 4) + 4 * groups + 2 + w.d // 4 + 4 * ns
            total += per_tok * int(lens[b])
    return total, total / (w.hkv * float(np.sum(lens)))


def run_dqk(args):
    import torch
    import torch.distributed as dist
    rank, nranks, local = world()
    if nranks > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from bit_kv_cache_dqk_b200 import inputs as I
    w = rank_workload(I.CONFIGS[args.workload], rank)
    layer = Layer(w, dev)
    layer.prefill()
    tokens = int(layer.lens.sum())

    for _ in range(args.warmup):
        layer.step()
    torch.cuda.synchronize(dev)
    algo_bytes, per_tok = layer.algorithmic_bytes()
    try:
        nvml_index = torch.cuda._get_nvml_device_index(dev)
    except Exception:
        nvml_index = local

    with ClockSampler(nvml_index) as clk:
        # device-timed steps (one launch each, back to back, as a serving loop runs them)
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if nranks > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        start.record()
        for _ in range(args.steps):
            layer.step()
        stop.record()
        torch.cuda.synchronize(dev)
        if nranks > 1:
            dist.barrier()
        elapsed = start.elapsed_time(stop) / 1e3
        agg = aggregate(tokens, elapsed, args.steps, nranks, dev)

        # the kernel's own duration: each launch between its own events
        step_ms = reduce_max(layer.per_launch_ms(layer.step, args.steps), dev)
        for _ in range(3):
            layer.decode()
        decode_ms = reduce_max(layer.per_launch_ms(layer.decode, args.steps), dev)

        # end to end from host buffers
        for _ in range(2):
            layer.step_e2e()
        torch.cuda.synchronize(dev)
        if nranks > 1:
            dist.barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record()
        for _ in range(args.steps):
            layer.step_e2e()
        e2.record()
        torch.cuda.synchronize(dev)
        e2e = aggregate(tokens, s2.elapsed_time(e2) / 1e3, args.steps, nranks, dev)

    peak, peak_kind = measured_peaks()
    achieved = algo_bytes / (step_ms / 1e3) / 1e9
    decode_achieved = algo_bytes / (decode_ms / 1e3) / 1e9
    traffic = recorded_traffic("k_decode", w.name)
    cpu = None
    if rank == 0 and nranks == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, layer.q_host.float().numpy(), args.cpu_seconds)
    if nranks > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": agg["value"], "unit": "KV-tokens/s", "n_gpus": nranks,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": agg["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int2-kv/f16-mma/f32-acc",
            "data": "synthetic",
            "config": {"workload": f"{w.name}: batch {w.batch}, {w.hq}/{w.hkv} heads, head_dim {w.d}, "
                                   f"context {int(layer.lens.max())}, 16-token pages ({w.page_order} order), "
                                   f"{w.pct}% query-channel sparsity, 1 appended row per sequence per step",
                       "global_batch": w.batch * nranks, "seq_len": int(layer.lens.max()),
                       "parallelism": f"dp{nranks} (independent sequences per GPU)",
                       "l2": "inputs larger than L2 (packed cache %.0f MB per step), no flush" %
                             (layer.pool.numel() / 1e6)},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "peak_kind": peak_kind,
                         "kernel": "k_decode (the whole decode step: append + query prep + attend + merge)",
                         "kernel_ms": step_ms,
                         "algorithmic_bytes_per_launch": algo_bytes,
                         "bytes_per_token_kv_head": per_tok},
            "decode_call": {"kernel": "k_decode (dqk_decode: query prep + attend + merge)", "ms": decode_ms,
                            "achieved_gbs": decode_achieved, "frac": decode_achieved / peak},
            "e2e": {"value": e2e["value"], "unit": "KV-tokens/s",
                    "h2d_bytes_per_step": int(layer.k_host.numel() * 2 + layer.v_host.numel() * 2 + layer.q_host.numel() * 2),
                    "d2h_bytes_per_step": int(layer.out_host.numel() * 4)},
            "gpu_launches": args.steps,
            "kernel_timing": "one launch per step; kernel_ms = mean of CUDA-event times around each launch "
                             "in a second pass of the same steps (decode_call: dqk_decode alone, same way)",
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if nranks > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_cpu_selftest(args):
    """The multi-rank path without a GPU (gloo): every rank times K steps of a
    CPU stand-in step ((rank+1) ms of sleep), rank 0 prints the aggregate."""
    import torch.distributed as dist
    rank, nranks, _ = world()
    if nranks > 1:
        from datetime import timedelta
        dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    for _ in range(args.warmup):
        time.sleep(0.001 * (rank + 1))
    if nranks > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time.sleep(0.001 * (rank + 1))
    agg = aggregate(1000, time.perf_counter() - t0, args.steps, nranks)
    if nranks > 1:
        dist.barrier()
    if rank == 0:
        print(json.dumps({"metric": "launcher self-test", "value": agg["value"], "unit": "tokens/s",
                          "n_gpus": nranks, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": agg["ms_per_step"], "scaling": "weak"}), flush=True)
    if nranks > 1:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch_under_torchrun(n: int, argv) -> int:
    """--gpus N > 1 with no outer launcher: run this script as N ranks (one
    per GPU of this node) under torch.distributed.run and return its status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


# ----------------------------------------------------------------------------
# CPU oracle (the reported CPU baseline, and the --impl reference arm)
# ----------------------------------------------------------------------------
class OracleSample:
    """Bounded sample of the workload for the CPU oracle: sequence 0, all kv
    heads, the first `ctx` tokens; the oracle quantizes the rows itself."""

    def __init__(self, w, ctx: int, q=None):
        from concurrent.futures import ThreadPoolExecutor
        from bit_kv_cache_dqk_b200 import inputs as I
        from oracle import oracle as O
        self.O, self.w, self.ctx = O, w, ctx
        from bit_kv_cache_dqk_b200 import calibrate as Cb
        tk, tq, _, _ = Cb.layer_transforms(w)
        self.tq = tq
        k, v = I.kv_rows(w, 0, 0, ctx)
        with ThreadPoolExecutor(min(w.hkv, os.cpu_count() or 1)) as ex:
            parts = list(ex.map(lambda j: O.append(tk[j:j + 1], np.ascontiguousarray(k[:, j:j + 1]),
                                                   np.ascontiguousarray(v[:, j:j + 1])), range(w.hkv)))
        self.cache = O.Cache({key: np.ascontiguousarray(np.concatenate([p[key] for p in parts], axis=1))
                              for key in parts[0]})
        lens = np.full(w.batch, ctx, np.int32)
        self.q = (q[0] if q is not None else I.queries(w, lens)[0]).astype(np.float32)
        self.threads = min(w.hkv, os.cpu_count() or 1)

    def step(self):
        self.O.decode_seq(self.cache, self.q, self.tq, self.w.hq, self.w.pct, threads=self.threads)


def cpu_baseline(w, q=None, seconds: float = 10.0, ctx: int = 16384):
    s = OracleSample(w, ctx, q)
    s.step()
    n, t0 = 0, time.perf_counter()
    while True:
        s.step()
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = (time.perf_counter() - t0) / n
    return {"value": ctx / dt, "unit": "KV-tokens/s", "cores": s.threads, "kind": "oracle",
            "sample": f"sequence 0, all {w.hkv} kv heads / {w.hq} q heads, first {ctx} tokens of the "
                      f"{w.name} workload, fp64 oracle decode (quantized by the oracle, untimed), "
                      f"{n} repetitions"}


def run_reference(args):
    rank, nranks, _ = world()
    if rank != 0:
        return
    from bit_kv_cache_dqk_b200 import inputs as I
    w = I.CONFIGS[args.workload]
    s = OracleSample(w, args.ref_ctx)
    for _ in range(args.warmup):
        s.step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        s.step()
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = args.ref_ctx * args.steps / total
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "KV-tokens/s", "n_gpus": nranks,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name} (bounded sample: sequence 0, {args.ref_ctx} tokens, all heads)",
                   "global_batch": 1, "seq_len": args.ref_ctx, "parallelism": "cpu threads over kv heads"},
        "cpu_baseline": {"value": value, "unit": "KV-tokens/s", "cores": s.threads, "kind": "oracle",
                         "sample": f"sequence 0, first {args.ref_ctx} tokens, all {w.hkv} kv heads"},
        "e2e": {"value": value, "unit": "KV-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ----------------------------------------------------------------------------
# the sparsity x batch x context sweep against the BF16 comparison decode, and
# the 64-row append of the ragged Qwen-shaped workload
# ----------------------------------------------------------------------------
def _event_time_us(torch, fn, reps, flush):
    ts = []
    for r in range(reps):
        flush.fill_(r & 255)             # L2 flush: 256 MB write
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    # trimmed mean: event timestamps come in steps of about 2 us, which a median would keep
    ts.sort()
    cut = len(ts) // 10
    return statistics.mean(ts[cut:len(ts) - cut])


def run_sweep(args):
    import torch
    from bit_kv_cache_dqk_b200 import dualqk as Q
    from bit_kv_cache_dqk_b200 import inputs as I
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = I.CONFIGS["sweep"]
    Bmax, Lmax = w.batch, w.ctx
    lens = np.full(Bmax, Lmax, np.int32)
    table, num_pages = I.page_table(w, lens)
    max_pages = table.shape[1]
    tk, tq, _, _ = I.transforms(w)
    t_k, t_q = torch.from_numpy(tk).to(dev), torch.from_numpy(tq).to(dev)
    probe = Q.layer_desc(w.d, w.hq, w.hkv, 0, 0, 0, 1)
    pool = torch.empty(num_pages * w.hkv * Q.dqk_block_bytes(probe), dtype=torch.uint8, device=dev)
    pool_b = torch.empty(num_pages * w.hkv * Q.dqk_bf16_block_bytes(probe), dtype=torch.uint8, device=dev)
    desc = Q.layer_desc(w.d, w.hq, w.hkv, t_k, t_q, pool, num_pages)
    desc_b = Q.layer_desc(w.d, w.hq, w.hkv, 0, 0, pool_b, num_pages)
    table_d = torch.from_numpy(table).to(dev)
    chunk = 4096
    new_d = torch.full((Bmax,), chunk, dtype=torch.int32, device=dev)
    for t0 in range(0, Lmax, chunk):
        k, v = I.kv_rows_device(w, range(Bmax), t0, t0 + chunk, dev)
        before = torch.full((Bmax,), t0, dtype=torch.int32, device=dev)
        Q.dqk_append(desc, k, v, Q.DQK_BF16, Bmax, new_d, before, chunk, table_d, max_pages)
        Q.dqk_bf16_append(desc_b, k, v, Q.DQK_BF16, Bmax, new_d, before, chunk, table_d, max_pages)
    torch.cuda.synchronize(dev)
    q = torch.from_numpy(I.queries(w, lens)).to(torch.bfloat16).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peak, peak_kind = measured_peaks()
    points = []
    for B in (1, 4, 16):
        ws_bytes = max(Q.dqk_decode_workspace_size(desc, B, max_pages),
                       Q.dqk_bf16_decode_workspace_size(desc_b, B, max_pages))
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        out = torch.empty((B, w.hq, w.d), dtype=torch.float32, device=dev)
        for L in (8192, 32768, 131072):
            lens_d = torch.full((B,), L, dtype=torch.int32, device=dev)
            t_b16 = _event_time_us(torch, lambda: Q.dqk_bf16_decode(desc_b, q, Q.DQK_BF16, B, lens_d, table_d,
                                                                     max_pages, out, ws, ws_bytes), args.reps, flush)
            b16_bytes = B * L * w.hkv * Q.dqk_bf16_block_bytes(probe) / 16
            for pct in (0, 20, 40, 60):
                keep = w.d - (pct * w.d) // 100
                sel = torch.empty((B, w.hq, keep), dtype=torch.int16, device=dev)
                t_dqk = _event_time_us(torch, lambda: Q.dqk_decode(desc, q, Q.DQK_BF16, B, lens_d, table_d,
                                                                   max_pages, pct, out, sel, ws, ws_bytes),
                                       args.reps, flush)
                algo, per_tok = algorithmic_bytes(w, sel.cpu().numpy(), np.full(B, L))
                points.append({"batch": B, "context": L, "sparsity_pct": pct, "dqk_decode_us": t_dqk,
                               "bf16_decode_us": t_b16, "speedup": t_b16 / t_dqk,
                               "dqk_kv_tokens_per_s": B * L / (t_dqk * 1e-6),
                               "dqk_algorithmic_gbs": algo / (t_dqk * 1e-6) / 1e9,
                               "dqk_bytes_per_token_kv_head": per_tok,
                               "bf16_gbs": b16_bytes / (t_b16 * 1e-6) / 1e9})
    # whole decode steps (append one row per sequence, then decode) at 128K context, 40 %
    steps = []
    k1, v1 = I.kv_rows_device(w, range(Bmax), Lmax - 1, Lmax, dev)
    for B in (4, 16):
        L = Lmax
        ws_bytes = max(Q.dqk_decode_workspace_size(desc, B, max_pages),
                       Q.dqk_bf16_decode_workspace_size(desc_b, B, max_pages))
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        out = torch.empty((B, w.hq, w.d), dtype=torch.float32, device=dev)
        lens_d = torch.full((B,), L, dtype=torch.int32, device=dev)
        ones = torch.ones(B, dtype=torch.int32, device=dev)
        before = torch.full((B,), L - 1, dtype=torch.int32, device=dev)
        kb, vb = k1[:B].contiguous(), v1[:B].contiguous()
        sel = torch.empty((B, w.hq, w.d - (40 * w.d) // 100), dtype=torch.int16, device=dev)

        def dqk_step():
            Q.dqk_decode_step(desc, kb, vb, Q.DQK_BF16, ones, before, 1, q, Q.DQK_BF16, B, lens_d, table_d,
                              max_pages, 40, out, sel, ws, ws_bytes)

        def bf16_step():
            Q.dqk_bf16_append(desc_b, kb, vb, Q.DQK_BF16, B, ones, before, 1, table_d, max_pages)
            Q.dqk_bf16_decode(desc_b, q, Q.DQK_BF16, B, lens_d, table_d, max_pages, out, ws, ws_bytes)

        t_dqk = _event_time_us(torch, dqk_step, args.reps, flush)
        t_b16 = _event_time_us(torch, bf16_step, args.reps, flush)
        steps.append({"batch": B, "context": L, "sparsity_pct": 40, "dqk_step_us": t_dqk, "bf16_step_us": t_b16,
                      "speedup": t_b16 / t_dqk, "dqk_kv_tokens_per_s": B * L / (t_dqk * 1e-6)})
    print(json.dumps({"metric": "decode time vs BF16 decode over sparsity x batch x context", "unit": "us",
                      "peak_hbm_gbs": peak, "peak_kind": peak_kind, "reps": args.reps,
                      "timing": "10 %-trimmed mean of CUDA-event times of one dqk_decode / dqk_bf16_decode call each, "
                                "256 MB L2 flush before every call",
                      "data": "synthetic, drawn on the device (torch Philox), random page order",
                      "config": {"workload": "sweep: 32/8 heads, head_dim 128, BF16 K/V, batch {1,4,16} x "
                                             "context {8K,32K,128K} x sparsity {0,20,40,60}%"},
                      "points": points,
                      "steps": steps,
                      "step_timing": "one decode step each: dqk_decode_step (append 1 row per sequence + "
                                     "decode, overlapped) vs dqk_bf16_append of the same row + "
                                     "dqk_bf16_decode; 10 %-trimmed mean of CUDA-event times, 256 MB L2 flush before each"}),
          flush=True)


def run_append64(args):
    """dqk_append of 64 rows per sequence on the ragged Qwen-shaped layer
    (batch 16, lengths 4K..64K, Student-t keys), timed alone."""
    import torch
    from bit_kv_cache_dqk_b200 import dualqk as Q
    from bit_kv_cache_dqk_b200 import inputs as I
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = I.CONFIGS["qwen"]
    lens = I.lengths(w)
    table, num_pages = I.page_table(w, lens)
    max_pages = table.shape[1]
    tk, tq, _, _ = I.transforms(w)
    t_k, t_q = torch.from_numpy(tk).to(dev), torch.from_numpy(tq).to(dev)
    probe = Q.layer_desc(w.d, w.hq, w.hkv, 0, 0, 0, 1)
    bb = Q.dqk_block_bytes(probe)
    pool = torch.empty(num_pages * w.hkv * bb, dtype=torch.uint8, device=dev)
    desc = Q.layer_desc(w.d, w.hq, w.hkv, t_k, t_q, pool, num_pages)
    table_d = torch.from_numpy(table).to(dev)
    n = w.append_new
    before = (lens - n).astype(np.int32)
    ks, vs = zip(*[I.kv_rows(w, b, int(before[b]), int(lens[b])) for b in range(w.batch)])
    k = torch.from_numpy(np.concatenate(ks)).to(torch.bfloat16).to(dev)
    v = torch.from_numpy(np.concatenate(vs)).to(torch.bfloat16).to(dev)
    new_d = torch.full((w.batch,), n, dtype=torch.int32, device=dev)
    before_d = torch.from_numpy(before).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    call = lambda: Q.dqk_append(desc, k, v, Q.DQK_BF16, w.batch, new_d, before_d, n, table_d, max_pages)
    for _ in range(3):
        call()
    t = _event_time_us(torch, call, args.reps, flush)
    rows = w.batch * n * w.hkv
    pages_touched = int(sum(((int(lens[b]) - 1) // 16) - (int(before[b]) // 16) + 1 for b in range(w.batch)))
    print(json.dumps({"metric": "append of 64 rows per sequence (transform + INT2 pack)", "value": t, "unit": "us",
                      "rows_per_s": rows / (t * 1e-6),
                      "bytes_in": rows * w.d * 2 * 2, "bytes_out": pages_touched * w.hkv * bb,
                      "achieved_gbs": (rows * w.d * 4 + 2 * pages_touched * w.hkv * bb) / (t * 1e-6) / 1e9,
                      "reps": args.reps, "timing": "10 %-trimmed mean of CUDA-event times, 256 MB L2 flush before each call",
                      "config": {"workload": f"qwen: batch {w.batch}, 32/8 heads, head_dim 128, lengths "
                                             f"{int(lens.min())}..{int(lens.max())}, {n} rows appended per "
                                             f"sequence"}}), flush=True)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["dqk", "reference"], default="dqk")
    ap.add_argument("--workload", default="long")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-ctx", type=int, default=16384)
    ap.add_argument("--sweep", action="store_true", help="sparsity x batch x context sweep vs the BF16 decode")
    ap.add_argument("--append64", action="store_true", help="time the 64-row append of the qwen workload")
    ap.add_argument("--reps", type=int, default=10)
    ap.add_argument("--cpu-selftest", action="store_true", help="the multi-rank launcher path on CPU (gloo)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch_under_torchrun(args.gpus, argv))
    if args.cpu_selftest:
        run_cpu_selftest(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    elif args.append64:
        run_append64(args)
    else:
        run_dqk(args)


if __name__ == "__main__":
    main()
