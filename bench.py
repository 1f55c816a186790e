#!/usr/bin/env python
"""Benchmark of the CSA forward path (libcsa.so) on B200.

One step = one whole CSA forward pass (projections, compression, indexer +
top-k, sparse MQA) over one batch of seeded synthetic input already resident
in device memory.  Default workload: prefill, batch 1, n = 8192, d = 4096,
c = 512, m = 4, c^I = 128, n_h^I = 64, n_h = 64, d_c = 1536, k = 512, bf16
with fp32 accumulation.  Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun) every rank runs an independent replica of the workload
(one sequence per GPU, no data-path collective): weak scaling; the timed
region is bracketed by a barrier and the time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on the host cores instead (rank
0 only), on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import compressed_sparse_attention_09_b200 as csa  # noqa: E402
from compressed_sparse_attention_09_b200 import synth  # noqa: E402

METRIC = "CSA forward tokens/s (prefill n=8192, decode) at 1 B200; % of roofline per stage"
FLUSH_BYTES = 512 << 20   # > 4x the 126 MB L2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm=j["hbm_gbs"], bf16=j["bf16_tflops"], bf16_sustained=j["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ------------------------------------------------------------------ work model
def causal_counts(seqlens, m, k):
    """sum_t floor(t/m) (indexer pairs) and sum_t min(k, floor(t/m)) (selections)."""
    pairs = sel = 0
    for L in seqlens:
        a = np.arange(L) // m
        pairs += int(a.sum())
        sel += int(np.minimum(a, k).sum())
    return pairs, sel


def stage_work(dims, seqlens):
    """Algorithmic FLOPs (or bytes for compression) of each stage of one step."""
    T = sum(seqlens)
    NB = sum(L // dims.m for L in seqlens)
    es = 2 if dims.dtype == csa.CSA_BF16 else 4
    N1 = 4 * dims.c + 4 * dims.cI + dims.dc + dims.nhI
    N2 = dims.nhI * dims.cI + dims.nh * dims.c
    pairs, sel = causal_counts(seqlens, dims.m, dims.topk)
    return {
        "A1_project_hidden": ("tensor", 2.0 * T * dims.d * N1),
        "A2_project_query": ("tensor", 2.0 * T * dims.dc * N2),
        "A3_compress": ("hbm", 4.0 * T * (dims.c + dims.cI) * es + NB * (dims.c + dims.cI) * es),
        "A4_indexer_topk": ("tensor", 2.0 * dims.nhI * dims.cI * pairs),
        "A5_sparse_mqa": ("tensor", 4.0 * dims.c * dims.nh * sel),
    }


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self, wait_s=5.0):
        """Starts sampling every 50 ms and waits (at most wait_s) for the first sample."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
            return
        t_end = time.monotonic() + wait_s
        while not self.lines and time.monotonic() < t_end:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def stop(self, t0=None, t1=None):
        """Summary of the samples taken in [t0, t1] (monotonic seconds; all when not given)."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = [ln for t, ln in self.lines if (t0 is None or t >= t0) and (t1 is None or t <= t1)]
        if not lines and self.lines and t0 is not None:   # none inside a short window: the next one after it
            later = [ln for t, ln in self.lines if t >= t0]
            lines = later[:1]
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ timing helpers
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# a stage's kernel, from one ncu capture of the current kernel version on the
# named workload (profiles/<kernel>_<workload>.md).  A kernel change makes the
# figure stale: it is then removed until the next capture.
MEASURED_TRAFFIC = {
    ("prefill", "A4_indexer_topk"): 102_976_512 + 7_183_104,
}


def timed_steps(fn, steps, flush, stream):
    """Per-step CUDA-event durations (ms) of fn(), with an L2 flush before each step."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for s, e in evs:
        flush()
        s.record(stream)
        fn()
        e.record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in evs]


class PrefillRunner:
    def __init__(self, w, dev):
        self.w, self.dims, self.dev = w, w.dims, dev
        d = self.dims
        self.T = sum(w.seqlens)
        self.nseq = len(w.seqlens)
        self.maxlen = max(w.seqlens)
        W = synth.make_weights(d, w.seed)
        self.packed = torch.empty(csa.csa_packed_weights_bytes(d), dtype=torch.uint8, device=dev)
        csa.csa_pack_weights(d, {k: v.to(dev) for k, v in W.items()}, self.packed)
        del W
        self.H_host = synth.make_hidden(self.T, d, w.seed).pin_memory()
        self.H = self.H_host.to(dev)
        cu, cb = csa.cu_from_lengths(w.seqlens, d.m)
        self.NB = int(cb[-1])
        self.cu, self.cb = cu.to(dev), cb.to(dev)
        dt = self.H.dtype
        self.O = torch.empty(self.T, d.nh * d.c, dtype=dt, device=dev)
        self.O_host = None   # pinned host copy of O, made on first end-to-end use
        self.ws = torch.empty(csa.csa_forward_workspace_bytes(d, self.T, self.nseq), dtype=torch.uint8,
                              device=dev)
        # stage buffers (separate from the workspace so stages can be timed one by one)
        self.Y1 = torch.empty(self.T, csa.csa_hidden_row_elems(d), dtype=dt, device=dev)
        self.wI = torch.empty(self.T, d.nhI, dtype=torch.float32, device=dev)
        self.Y2 = torch.empty(self.T, csa.csa_query_row_elems(d), dtype=dt, device=dev)
        self.Cc = torch.empty(max(self.NB, 1), d.c, dtype=dt, device=dev)
        self.KI = torch.empty(max(self.NB, 1), d.cI, dtype=dt, device=dev)
        self.idx = torch.empty(self.T, d.topk, dtype=torch.int32, device=dev)
        self.iws = torch.empty(csa.csa_indexer_workspace_bytes(d, self.T, self.nseq, self.maxlen), dtype=torch.uint8,
                               device=dev)

    def forward(self):
        d = self.dims
        csa.csa_forward(d, self.packed, self.H, self.cu, self.cb, self.nseq, self.T, self.NB, self.maxlen,
                        self.O, None, None, None, self.ws)

    def forward_e2e(self):
        if self.O_host is None:
            self.O_host = torch.empty(self.T, self.dims.nh * self.dims.c, dtype=self.O.dtype).pin_memory()
        self.H.copy_(self.H_host, non_blocking=True)
        self.forward()
        self.O_host.copy_(self.O, non_blocking=True)

    def stages(self):
        d, T = self.dims, self.T
        es = self.Y1.element_size()
        c, cI = d.c, d.cI
        N1b = self.Y1.shape[1]
        Y1 = self.Y1

        def col(j):
            return Y1.data_ptr() + j * es

        def a3():   # both key sets in one launch, as csa_forward runs the stage
            csa.csa_compress_kv(d, self.packed, self.Y1, T, self.cu, self.cb, self.nseq, self.NB, self.Cc, self.KI)
        return {
            "A1_project_hidden": lambda: csa.csa_project_hidden(d, self.packed, self.H, T, self.Y1, self.wI),
            "A2_project_query": lambda: csa.csa_project_query(d, self.packed, col(4 * c + 4 * cI), N1b, T, self.Y2),
            "A3_compress": a3,
            "A4_indexer_topk": lambda: csa.csa_indexer_topk(d, self.Y2, self.Y2.shape[1], self.wI, d.nhI, self.KI,
                                                            self.cu, self.cb, self.nseq, T, self.NB, self.maxlen,
                                                            self.idx, self.iws),
            "A5_sparse_mqa": lambda: csa.csa_sparse_mqa(d, self.Y2.data_ptr() + d.nhI * cI * es, self.Y2.shape[1],
                                                        self.Cc, self.idx, self.cu, self.cb, self.nseq, T,
                                                        self.NB, self.O),
        }


class DecodeRunner:
    """One decode step of B independent sequences over a cached C^Comp/K^IComp."""

    def __init__(self, w, dev):
        d = w.dims
        self.w, self.dims, self.B = w, d, w.decode_batch
        W = synth.make_weights(d, w.seed)
        self.packed = torch.empty(csa.csa_packed_weights_bytes(d), dtype=torch.uint8, device=dev)
        csa.csa_pack_weights(d, {k: v.to(dev) for k, v in W.items()}, self.packed)
        del W
        dt = synth.torch_dtype(d)
        g = torch.Generator(device=dev).manual_seed(w.seed + 1)
        cap = w.cache_cap
        self.cap = cap
        self.Cc = torch.randn(self.B, cap, d.c, device=dev, generator=g, dtype=torch.float32).to(dt)
        self.Kc = torch.randn(self.B, cap, d.cI, device=dev, generator=g, dtype=torch.float32).to(dt)
        self.ring = torch.randn(self.B, 2 * d.m, csa.csa_ring_row_elems(d), device=dev, generator=g).to(dt)
        self.h = torch.randn(self.B, d.d, device=dev, generator=g).to(dt)
        self.pos = torch.full((self.B,), w.decode_pos, dtype=torch.int32, device=dev)
        self.clen = torch.full((self.B,), w.decode_pos // d.m, dtype=torch.int32, device=dev)
        self.O = torch.empty(self.B, d.nh * d.c, dtype=dt, device=dev)
        self.ws = torch.empty(csa.csa_decode_workspace_bytes(d, self.B, self.cap), dtype=torch.uint8, device=dev)

    def step(self):
        csa.csa_decode(self.dims, self.packed, self.h, self.pos, self.ring, self.Cc, self.Kc, self.clen,
                       self.cap, self.B, self.O, None, self.ws)

    def bytes_per_step(self):
        d = self.dims
        N1 = 4 * d.c + 4 * d.cI + d.dc + d.nhI
        N2 = d.nhI * d.cI + d.nh * d.c
        avail = self.w.decode_pos // d.m
        es = 2
        weights = (d.d * N1 + d.dc * N2) * es
        keys = self.B * avail * d.cI * es
        gathered = self.B * min(d.topk, avail) * d.c * es
        return weights + keys + gathered


# ------------------------------------------------------------------ oracle baseline
class OracleSampler:
    """Times the fp64 oracle on bounded samples of a workload, extrapolated to
    tokens/s.  The per-token part (projections of every token and the
    compression) is timed once in full by `base()`; each `sample()` then runs
    one oracle forward with eqs. 5-11 on `rows_sample` seeded query rows and
    extrapolates its per-row cost to every row."""

    def __init__(self, w, rows_sample):
        from oracle import csa_oracle as orc
        self.orc, self.w = orc, w
        d = w.dims
        self.W = {k: v.double().numpy() for k, v in synth.make_weights(d, w.seed).items()}
        self.T = sum(w.seqlens)
        self.H = synth.make_hidden(self.T, d, w.seed).double().numpy()
        self.od = dict(m=d.m, topk=d.topk, nh=d.nh, nhI=d.nhI, c=d.c, cI=d.cI)
        self.store = "bf16" if d.dtype == csa.CSA_BF16 else "f32"
        self.rows_sample = min(rows_sample, self.T)
        self.base_s = None

    def _forward(self, rows):
        t0 = time.perf_counter()
        self.orc.csa_forward(self.H, self.W, self.od, list(self.w.seqlens), store=self.store, rows=rows)
        return time.perf_counter() - t0

    def base(self):
        self.base_s = self._forward(np.zeros(0, dtype=np.int64))
        return self.base_s

    def sample(self, seed):
        if self.base_s is None:
            self.base()
        rows = np.sort(np.random.default_rng(seed).choice(self.T, size=self.rows_sample, replace=False))
        t = self._forward(rows)
        per_row = max(t - self.base_s, 0.0) / len(rows)
        return self.T / (self.base_s + per_row * self.T), dict(base_s=self.base_s, per_row_s=per_row,
                                                               rows=len(rows), wall_s=t)


def oracle_sample(w, rows_sample, seed=0):
    """One bounded oracle sample of the workload (base part timed in full,
    eqs. 5-11 on `rows_sample` rows), extrapolated to tokens/s."""
    return OracleSampler(w, rows_sample).sample(seed)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def max_over_ranks(ms, dev, world):
    """The slowest rank's device time (every rank takes part; world 1: ms itself)."""
    if world == 1:
        return ms
    t = torch.tensor([ms], device=dev, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step, steps, world, max_ms):
    """Whole-job tokens/s: the tokens every rank processed over the slowest rank's time."""
    return tokens_per_rank_step * steps * world / (max_ms / 1000.0)


# ------------------------------------------------------------------ arms
def run_reference(args, rank, world):
    if rank != 0:
        return
    w = synth.workloads()[args.workload]
    sampler = OracleSampler(w, args.ref_rows)
    sampler.base()                      # the token-parallel part, timed in full once
    times = []
    info = None
    for i in range(args.warmup + args.steps):
        tps, info = sampler.sample(seed=i)
        if i >= args.warmup:
            times.append(tps)
    value = statistics.mean(times)
    sample = (f"oracle forward per step with eqs. 5-11 on {info['rows']} seeded query rows, extrapolated "
              f"to all {sum(w.seqlens)} rows; projections + compression of every token timed in full "
              f"({info['base_s']:.2f} s) before the steps")
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * sum(w.seqlens) / value, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(w, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(w, world):
    d = w.dims
    return {"workload": f"{w.name}: batch {len(w.seqlens)}, n={max(w.seqlens)}, d={d.d}, c={d.c}, m={d.m}, "
                        f"cI={d.cI}, nhI={d.nhI}, nh={d.nh}, dc={d.dc}, topk={d.topk}, "
                        f"{'bf16 (fp32 accumulation)' if d.dtype == csa.CSA_BF16 else 'fp32'}",
            "global_batch": len(w.seqlens) * world, "seq_len": max(w.seqlens),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed before every timed step (512 MiB write)"}


def run_ours(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks = load_peaks()
    w = synth.workloads()[args.workload]
    runner = PrefillRunner(w, dev)
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.fill_(1)

    # clock sampling starts before the warm-up: nvidia-smi's first sample takes a while
    sampler = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                           else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    sampler.start()
    for _ in range(args.warmup):
        runner.forward()
    torch.cuda.synchronize()
    st = csa.csa_get_device_status()
    if st != 0:
        sampler.stop()
        raise RuntimeError(f"device status after warm-up: {csa.status_string(st)}")

    # ---- timed region: exactly K steps (clock samples kept from inside it only)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_sample0 = time.monotonic()
    n0 = csa.csa_launch_count()
    step_ms = timed_steps(runner.forward, args.steps, flush, stream)
    launches = csa.csa_launch_count() - n0
    torch.cuda.synchronize()
    t_sample1 = time.monotonic()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop(t_sample0, t_sample1)
    total_ms = max_over_ranks(sum(step_ms), dev, world)
    tokens = runner.T * args.steps * world
    value = job_throughput(runner.T, args.steps, world, total_ms)
    ms_per_step = total_ms / args.steps

    # ---- end to end through host buffers (H2D of H, forward, D2H of O)
    e2e = None
    if not args.no_e2e:
        for _ in range(2):
            runner.forward_e2e()
        e2e_ms = max_over_ranks(sum(timed_steps(runner.forward_e2e, args.steps, flush, stream)), dev, world)
        e2e = {"value": tokens / (e2e_ms / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": runner.H.numel() * runner.H.element_size(),
               "d2h_bytes_per_step": runner.O.numel() * runner.O.element_size()}

    # ---- stages, each timed alone (per-stage roofline)
    stages = {}
    work = stage_work(w.dims, w.seqlens)
    if not args.no_stages:
        fns = runner.stages()
        for name, fn in fns.items():
            for _ in range(2):
                fn()
            ms = statistics.mean(timed_steps(fn, max(3, min(args.steps, 10)), flush, stream))
            bound, amount = work[name]
            if bound == "hbm":
                ach = amount / (ms / 1000.0) / 1e9
                peak = peaks["hbm"]
                stages[name] = {"ms": ms, "bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                                "frac": ach / peak, "algorithmic": amount}
            else:
                ach = amount / (ms / 1000.0) / 1e12
                peak = peaks["bf16"]
                stages[name] = {"ms": ms, "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                                "frac": ach / peak, "algorithmic": amount}
        st = csa.csa_get_device_status()
        if st != 0:
            raise RuntimeError(f"device status after stages: {csa.status_string(st)}")
    roofline = None
    if stages:
        top = max(stages, key=lambda k: stages[k]["ms"])
        s = stages[top]
        roofline = {"kernel": top, "bound": s["bound"], "achieved": s["achieved"], "peak": s["peak"],
                    "unit": s["unit"], "frac": s["frac"], "traffic": MEASURED_TRAFFIC.get((args.workload, top)),
                    "peak_source": f"{peaks['source']} ({'hbm_gbs' if s['bound'] == 'hbm' else 'bf16_tflops'})"}

    # ---- decode workload, same build
    decode = None
    if not args.no_decode:
        del runner
        torch.cuda.empty_cache()
        dr = DecodeRunner(synth.workloads()["decode"], dev)
        for _ in range(3):
            dr.step()
        dms = statistics.mean(timed_steps(dr.step, args.steps, flush, stream))
        st = csa.csa_get_device_status()
        if st != 0:
            raise RuntimeError(f"device status after decode: {csa.status_string(st)}")
        gbs = dr.bytes_per_step() / (dms / 1000.0) / 1e9
        decode = {"value": dr.B / (dms / 1000.0), "unit": "tokens/s", "ms_per_step": dms,
                  "workload": "64 sequences x 1 new token over 16384 cached entries (t=65536), nh=128, k=2048",
                  "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                               "frac": gbs / peaks["hbm"], "algorithmic_bytes": dr.bytes_per_step()}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, info = oracle_sample(w, rows_sample=args.ref_rows)
        cpu = {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": (f"projections + compression of all {runner_T(w)} tokens in full "
                          f"({info['base_s']:.1f} s), eqs. 5-11 on {info['rows']} seeded query rows "
                          f"({info['per_row_s'] * 1e3:.1f} ms/row), extrapolated")}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16" if w.dims.dtype == csa.CSA_BF16 else "f32",
                "data": "synthetic (seeded normal H, N(0,1/fan_in) weights)", "config": workload_config(w, world),
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
                "clocks": clocks, "stages": stages, "decode": decode}
        print(json.dumps(line), flush=True)


def run_stage(args):
    """Runs one stage of the prefill workload (after one full forward that fills
    its inputs) warmup + steps times; for profiling a single kernel."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = synth.workloads()[args.workload]
    runner = PrefillRunner(w, dev)
    fn = runner.stages()[args.stage]
    # inputs of every stage: one pass of the stages in order
    for name, f in runner.stages().items():
        f()
        if name == args.stage:
            break
    for _ in range(args.warmup + args.steps):
        fn()
    torch.cuda.synchronize()
    st = csa.csa_get_device_status()
    print(json.dumps({"stage": args.stage, "workload": args.workload, "launches": args.warmup + args.steps,
                      "status": csa.status_string(st)}), flush=True)
    if st != 0:
        raise SystemExit(1)


def runner_T(w):
    return sum(w.seqlens)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill", "tiny", "long", "ragged"], default="prefill")
    ap.add_argument("--ref-rows", type=int, default=64, help="query rows the oracle runs per sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-stages", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--stage", choices=["A1_project_hidden", "A2_project_query", "A3_compress", "A4_indexer_topk",
                                        "A5_sparse_mqa"], help="run only this stage (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.stage:
        run_stage(args)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
