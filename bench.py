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
        "A1A3_project_compress": ("tensor", 2.0 * T * dims.d * N1),
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
# a stage's kernel, taken from one ncu capture of the current kernel version
# on the named workload.  A kernel change makes the figure stale: it is then
# removed until the kernel is captured again.
MEASURED_TRAFFIC = {
    ("prefill", "A4_indexer_topk"): 102_978_816 + 7_641_088,
    ("prefill", "A5_sparse_mqa"): 556_276_992 + 493_239_040,
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
    def __init__(self, w, dev, stage_buffers=True):
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
        self.e2e_bufs = None   # second H / O buffers, pinned host O and copy streams, made on first use
        self.ws = torch.empty(csa.csa_forward_workspace_bytes(d, self.T, self.nseq), dtype=torch.uint8,
                              device=dev)
        if not stage_buffers:
            return
        # stage buffers (separate from the workspace so stages can be timed one by one)
        self.Y1 = torch.empty(self.T, csa.csa_hidden_row_elems(d), dtype=dt, device=dev)
        self.wI = torch.empty(self.T, d.nhI, dtype=torch.float32, device=dev)
        self.Y2 = torch.empty(self.T, csa.csa_query_row_elems(d), dtype=dt, device=dev)
        self.Cc = torch.empty(max(self.NB, 1), d.c, dtype=dt, device=dev)
        self.KI = torch.empty(max(self.NB, 1), d.cI, dtype=dt, device=dev)
        self.idx = torch.empty(self.T, d.topk, dtype=torch.int32, device=dev)
        self.iws = torch.empty(csa.csa_indexer_workspace_bytes(d, self.T, self.nseq, self.maxlen), dtype=torch.uint8,
                               device=dev)
        fb = csa.csa_project_compress_workspace_bytes(d, self.T)
        self.fws = torch.empty(fb, dtype=torch.uint8, device=dev) if fb else None

    def forward(self, H=None, O=None):
        d = self.dims
        csa.csa_forward(d, self.packed, self.H if H is None else H, self.cu, self.cb, self.nseq, self.T, self.NB,
                        self.maxlen, self.O if O is None else O, None, None, None, self.ws)

    def forward_staged(self, events):
        d = self.dims
        csa.csa_forward_staged(d, self.packed, self.H, self.cu, self.cb, self.nseq, self.T, self.NB, self.maxlen,
                               self.O, None, None, None, self.ws, events)

    def e2e_pipeline(self, steps, flush):
        """`steps` end-to-end steps through host buffers; returns the device
        time in ms from the first step's H2D copy to the last step's D2H copy.
        Step i copies H from pinned host memory into device buffer i % 2 (copy
        stream), runs the forward on the compute stream into O buffer i % 2,
        and copies that O to pinned host memory (second copy stream), so that
        step i's forward overlaps step i+1's H2D and step i-1's D2H.  The L2
        is flushed before every forward."""
        if self.e2e_bufs is None:
            self.e2e_bufs = {"H": [self.H, torch.empty_like(self.H)], "O": [self.O, torch.empty_like(self.O)],
                             "O_host": torch.empty(self.O.shape, dtype=self.O.dtype).pin_memory(),
                             "s_in": torch.cuda.Stream(), "s_out": torch.cuda.Stream()}
        b = self.e2e_bufs
        comp, s_in, s_out = torch.cuda.current_stream(), b["s_in"], b["s_out"]
        ready = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        freed = [torch.cuda.Event() for _ in range(2)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(s_in)
        for i in range(steps):
            k = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done[k])        # step i-2's forward has read H[k]
                b["H"][k].copy_(self.H_host, non_blocking=True)
                ready[k].record(s_in)
            comp.wait_event(ready[k])
            if i >= 2:
                comp.wait_event(freed[k])           # step i-2's D2H has read O[k]
            flush()
            self.forward(b["H"][k], b["O"][k])
            done[k].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[k])
                b["O_host"].copy_(b["O"][k], non_blocking=True)
                freed[k].record(s_out)
        end.record(s_out)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

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
        out = {}
        if self.fws is not None:   # A1 with A3 in its epilogue, as csa_forward runs it
            out["A1A3_project_compress"] = lambda: csa.csa_project_hidden_compress(
                d, self.packed, self.H, T, self.cu, self.cb, self.nseq, self.NB, self.Y1, self.wI, self.Cc, self.KI,
                self.fws)
        return out | {
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

    def step_staged(self, events):
        csa.csa_decode_staged(self.dims, self.packed, self.h, self.pos, self.ring, self.Cc, self.Kc, self.clen,
                              self.cap, self.B, self.O, None, self.ws, events)

    def quantise_keys(self):
        """The key cache as E4M3 codes + per-entry scales (for the q8 steps)."""
        d = self.dims
        self.Kq = torch.empty(self.B, self.cap, d.cI, dtype=torch.uint8, device=self.Kc.device)
        self.Ks = torch.empty(self.B, self.cap, dtype=torch.float32, device=self.Kc.device)
        csa.csa_quantize_keys_e4m3(self.Kc, d.cI, self.B * self.cap, d.cI, self.Kq, self.Ks)

    def step_q8(self):
        csa.csa_decode_q8(self.dims, self.packed, self.h, self.pos, self.ring, self.Cc, self.Kq, self.Ks, self.clen,
                          self.cap, self.B, self.O, None, self.ws)

    def step_q8_staged(self, events):
        csa.csa_decode_q8_staged(self.dims, self.packed, self.h, self.pos, self.ring, self.Cc, self.Kq, self.Ks,
                                 self.clen, self.cap, self.B, self.O, None, self.ws, events)

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
    """Times the fp64 oracle on bounded samples of a workload.  The
    token-parallel half (eqs. 1-4: projections and compression of every
    token) is timed once in full by `base()`; `rows(n, seed)` times the
    per-query half (eqs. 5-11) on n seeded query rows, on its own.  The
    whole-workload rate is then T / (base + per-row cost x T)."""

    def __init__(self, w):
        from oracle import csa_oracle as orc
        self.orc, self.w = orc, w
        d = w.dims
        self.W = {k: v.double().numpy() for k, v in synth.make_weights(d, w.seed).items()}
        self.T = sum(w.seqlens)
        self.H = synth.make_hidden(self.T, d, w.seed).double().numpy()
        self.od = dict(m=d.m, topk=d.topk, nh=d.nh, nhI=d.nhI, c=d.c, cI=d.cI)
        self.store = "bf16" if d.dtype == csa.CSA_BF16 else "f32"
        self.base_s = None
        self.entries = None

    def base(self):
        t0 = time.perf_counter()
        self.entries = self.orc.compressed_entries(self.H, self.W, self.od, list(self.w.seqlens), self.store)
        self.base_s = time.perf_counter() - t0
        return self.base_s

    def rows(self, n, seed):
        """Seconds the per-query half takes on n seeded rows (distinct, sorted)."""
        if self.entries is None:
            self.base()
        rows = np.sort(np.random.default_rng(seed).choice(self.T, size=min(n, self.T), replace=False))
        Cc, Kc, cu, cb = self.entries
        t0 = time.perf_counter()
        self.orc.query_rows(self.H, self.W, self.od, Cc, Kc, cu, cb, rows, self.store)
        return time.perf_counter() - t0, len(rows)

    def tokens_per_s(self, per_row_s):
        return self.T / (self.base_s + per_row_s * self.T)


def oracle_baseline(w, budget_s=15.0, chunk=16):
    """cpu_baseline of the default line: the token-parallel half in full, then
    seeded query rows in chunks until about budget_s of row time (at least
    two chunks); per-row cost = row time / rows, measured, not differenced."""
    smp = OracleSampler(w)
    smp.base()
    t_rows, n_rows, seed = 0.0, 0, 0
    while (t_rows < budget_s or seed < 2) and n_rows < smp.T:
        dt, n = smp.rows(chunk, seed)
        t_rows += dt
        n_rows += n
        seed += 1
    per_row = t_rows / n_rows
    return smp.tokens_per_s(per_row), dict(base_s=smp.base_s, per_row_s=per_row, rows=n_rows, rows_s=t_rows)


def oracle_tiny_one_thread():
    """The tiny fp32 workload, whole forward (every row), on one BLAS thread."""
    from threadpoolctl import threadpool_limits
    from oracle import csa_oracle as orc
    w = synth.workloads()["tiny"]
    d = w.dims
    W = {k: v.double().numpy() for k, v in synth.make_weights(d, w.seed).items()}
    T = sum(w.seqlens)
    H = synth.make_hidden(T, d, w.seed).double().numpy()
    od = dict(m=d.m, topk=d.topk, nh=d.nh, nhI=d.nhI, c=d.c, cI=d.cI)
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        orc.csa_forward(H, W, od, list(w.seqlens), store="f32")
        dt = time.perf_counter() - t0
    return {"value": T / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"tiny fp32 workload ({T} tokens), whole forward, every row, one BLAS thread ({dt:.2f} s)"}


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
    smp = OracleSampler(w)
    smp.base()                      # the token-parallel half, timed in full once, before the steps
    values, step_s = [], []
    for i in range(args.warmup + args.steps):
        dt, n = smp.rows(args.ref_rows, seed=i)
        if i >= args.warmup:
            values.append(smp.tokens_per_s(dt / n))
            step_s.append(dt)
    value = statistics.mean(values)
    T = sum(w.seqlens)
    sample = (f"each step: the oracle's per-query half (eqs. 5-11) on {args.ref_rows} seeded query rows, timed "
              f"on its own ({1e3 * statistics.mean(step_s) / args.ref_rows:.1f} ms/row); the token-parallel half "
              f"(eqs. 1-4, all {T} tokens) timed in full once before the steps ({smp.base_s:.2f} s); value = "
              f"{T} / (that + per-row cost x {T}); ms_per_step = the measured sampled step")
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * statistics.mean(step_s), "higher_is_better": True,
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


def stage_entry(name, ms, work, peaks, peak_key="bf16"):
    """Roofline record of one stage timed for `ms` milliseconds."""
    bound, amount = work[name]
    if bound == "hbm":
        ach = amount / (ms / 1000.0) / 1e9
        return {"ms": ms, "bound": "hbm", "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s",
                "frac": ach / peaks["hbm"], "algorithmic": amount}
    ach = amount / (ms / 1000.0) / 1e12
    return {"ms": ms, "bound": "tensor", "achieved": ach, "peak": peaks[peak_key], "unit": "TFLOP/s",
            "frac": ach / peaks[peak_key], "algorithmic": amount}


STAGES = ("A1_project_hidden", "A2_project_query", "A3_compress", "A4_indexer_topk", "A5_sparse_mqa")


def staged_step_ms(step_fn, nstages, steps, flush, stream):
    """Mean in-step duration of each stage over `steps` steps of step_fn(events)
    (L2 flushed before each step; events recorded between the stages)."""
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nstages + 1)] for _ in range(steps)]
    for ev in evs:
        for e in ev:
            e.record(stream)   # creates the handles
    torch.cuda.synchronize()
    for ev in evs:
        flush()
        step_fn(ev)
    torch.cuda.synchronize()
    return [statistics.mean(ev[k].elapsed_time(ev[k + 1]) for ev in evs) for k in range(nstages)]


def measure_stages(runner, w, args, peaks, flush, stream, reps):
    """Each stage timed alone (inputs from one pass of the stages), and the
    same stages timed inside the real step (csa_forward_staged)."""
    work = stage_work(w.dims, w.seqlens)
    alone = {}
    for name, fn in runner.stages().items():
        for _ in range(2):
            fn()
        alone[name] = stage_entry(name, statistics.mean(timed_steps(fn, reps, flush, stream)), work, peaks)
    in_step_ms = staged_step_ms(runner.forward_staged, len(STAGES), reps, flush, stream)
    names = list(STAGES)
    if runner.fws is not None:   # the compression runs inside the A1 kernel; its own interval is empty
        names[0] = "A1A3_project_compress"
    in_step = {}
    for n, ms in zip(names, in_step_ms):
        if n == "A3_compress" and runner.fws is not None:
            in_step[n] = {"ms": ms, "note": "fused into A1A3_project_compress"}
        else:
            in_step[n] = stage_entry(n, ms, work, peaks, "bf16_sustained")
    st = csa.csa_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status after stages: {csa.status_string(st)}")
    return alone, in_step


def decode_stage_bytes(w):
    """Algorithmic HBM bytes of each stage of one decode step."""
    d = w.dims
    B, avail = w.decode_batch, w.decode_pos // d.m
    es = 2
    N1 = 4 * d.c + 4 * d.cI + d.dc + d.nhI
    N2 = d.nhI * d.cI + d.nh * d.c
    ring = 4 * d.c + 4 * d.cI
    return {
        "A1_project_hidden": d.d * N1 * es + B * d.d * es + B * N1 * es,
        "A6_cache_append": B * (2 * d.m * ring * es + (d.c + d.cI) * es),
        "A2_project_query": d.dc * N2 * es + B * d.dc * es + B * N2 * es,
        "A4_indexer_scores": B * avail * d.cI * es + B * avail * 4,
        "A4_topk_select": B * avail * 4 + B * d.topk * 4,
        "A5_sparse_mqa": B * min(d.topk, avail) * d.c * es + 2 * B * d.nh * d.c * es + B * d.topk * 4,
    }


def run_decode(dev, args, peaks, flush, stream):
    """The decode step, timed back to back without an L2 flush: every step
    reads 1.34 GB of caches and 261 MB of weights, far more than the 126 MB
    L2, so nothing a step leaves in L2 serves the next one (a 512 MB flush
    would instead charge the write-back of its dirty lines to the step)."""
    w = synth.workloads()["decode"]
    dr = DecodeRunner(w, dev)
    for _ in range(3):
        dr.step()
    no_flush = lambda: None   # noqa: E731
    dms = statistics.mean(timed_steps(dr.step, args.steps, no_flush, stream))
    dms_flushed = statistics.mean(timed_steps(dr.step, max(3, min(args.steps, 50)), flush, stream))
    names = ("A1_project_hidden", "A2_project_query", "A6_cache_append", "A4_indexer_scores", "A4_topk_select",
             "A5_sparse_mqa")
    in_step_ms = staged_step_ms(dr.step_staged, len(names), max(3, min(args.steps, 50)), no_flush, stream)
    st = csa.csa_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status after decode: {csa.status_string(st)}")
    nbytes = decode_stage_bytes(w)
    stages = {}
    for n, ms in zip(names, in_step_ms):
        gbs = nbytes[n] / (ms / 1000.0) / 1e9
        stages[n] = {"ms": ms, "bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm"], "algorithmic_bytes": nbytes[n]}
    gbs = dr.bytes_per_step() / (dms / 1000.0) / 1e9
    # the same step over the E4M3 key cache (codes + per-entry scales)
    dr.quantise_keys()
    for _ in range(3):
        dr.step_q8()
    qms = statistics.mean(timed_steps(dr.step_q8, args.steps, no_flush, stream))
    q_in_step = staged_step_ms(dr.step_q8_staged, len(names), max(3, min(args.steps, 50)), no_flush, stream)
    st = csa.csa_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status after the e4m3-key decode: {csa.status_string(st)}")
    d = w.dims
    avail = w.decode_pos // d.m
    qbytes = dict(nbytes)
    qbytes["A4_indexer_scores"] = dr.B * avail * (d.cI + 4) + dr.B * avail * 4   # codes + scales read, scores written
    q_total = dr.bytes_per_step() - dr.B * avail * d.cI * 2 + dr.B * avail * (d.cI + 4)
    q_stages = {}
    for n, ms in zip(names, q_in_step):
        sgbs = qbytes[n] / (ms / 1000.0) / 1e9
        q_stages[n] = {"ms": ms, "bound": "hbm", "achieved": sgbs, "peak": peaks["hbm"], "unit": "GB/s",
                       "frac": sgbs / peaks["hbm"], "algorithmic_bytes": qbytes[n]}
    qgbs = q_total / (qms / 1000.0) / 1e9
    e4m3 = {"value": dr.B / (qms / 1000.0), "unit": "tokens/s", "ms_per_step": qms,
            "cache": "K^IComp as E4M3 codes + one fp32 scale per entry; C^Comp bf16",
            "roofline": {"bound": "hbm", "achieved": qgbs, "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": qgbs / peaks["hbm"], "algorithmic_bytes": q_total},
            "stages_in_step": q_stages}
    out = {"value": dr.B / (dms / 1000.0), "unit": "tokens/s", "ms_per_step": dms,
           "ms_per_step_l2_flushed": dms_flushed, "e4m3_keys": e4m3,
           "l2": "not flushed: each step reads 1.6 GB (> 126 MB L2); ms_per_step_l2_flushed = the same with a "
                 "512 MiB write before each step",
           "workload": "64 sequences x 1 new token over 16384 cached entries (t=65536), nh=128, k=2048",
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                        "frac": gbs / peaks["hbm"], "algorithmic_bytes": dr.bytes_per_step()},
           "stages_in_step": stages}
    del dr
    torch.cuda.empty_cache()
    return out


def run_extra_workload(name, dev, args, peaks, flush, stream):
    """Step time, throughput and per-stage rooflines of another prefill workload."""
    w = synth.workloads()[name]
    runner = PrefillRunner(w, dev, stage_buffers=True)
    for _ in range(3):
        runner.forward()
    steps = max(3, min(args.steps, 5))
    ms = statistics.mean(timed_steps(runner.forward, steps, flush, stream))
    alone, in_step = measure_stages(runner, w, args, peaks, flush, stream, 3)
    out = {"workload": workload_config(w, 1)["workload"], "tokens": runner.T, "steps": steps, "ms_per_step": ms,
           "value": runner.T / (ms / 1000.0), "unit": "tokens/s", "stages": alone, "stages_in_step": in_step}
    del runner
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks = load_peaks()
    w = synth.workloads()[args.workload]
    runner = PrefillRunner(w, dev, stage_buffers=not args.no_stages)
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
    value = job_throughput(runner.T, args.steps, world, total_ms)
    ms_per_step = total_ms / args.steps

    # ---- end to end through host buffers: every step copies its H in from
    # pinned host memory and its O out to pinned host memory; the copies run
    # on their own streams, overlapped with the neighbouring steps' compute
    e2e = None
    if not args.no_e2e:
        runner.e2e_pipeline(2, flush)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(runner.e2e_pipeline(args.steps, flush), dev, world)
        e2e = {"value": runner.T * args.steps * world / (e2e_ms / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": runner.H.numel() * runner.H.element_size(),
               "d2h_bytes_per_step": runner.O.numel() * runner.O.element_size(),
               "how": "H2D of step i+1 and D2H of step i-1 on copy streams, overlapped with step i's forward; "
                      "timed from the first H2D to the last D2H"}

    # ---- stages: each alone (per-stage roofline) and inside the step
    stages, stages_in_step = {}, {}
    if not args.no_stages:
        stages, stages_in_step = measure_stages(runner, w, args, peaks, flush, stream, max(3, min(args.steps, 10)))
    roofline = None
    if stages:
        top = max(stages, key=lambda k: stages[k]["ms"])
        s = stages[top]
        roofline = {"kernel": top, "bound": s["bound"], "achieved": s["achieved"], "peak": s["peak"],
                    "unit": s["unit"], "frac": s["frac"], "traffic": MEASURED_TRAFFIC.get((args.workload, top)),
                    "peak_source": f"{peaks['source']} ({'hbm_gbs' if s['bound'] == 'hbm' else 'bf16_tflops'})"}
    del runner
    torch.cuda.empty_cache()

    # ---- decode workload, same build
    decode = None if args.no_decode else run_decode(dev, args, peaks, flush, stream)

    # ---- the long and ragged prefill workloads (step, stages, rooflines)
    workloads = {}
    if not args.no_workloads and world == 1:
        for name in ("long", "ragged"):
            if name != args.workload:
                workloads[name] = run_extra_workload(name, dev, args, peaks, flush, stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, info = oracle_baseline(w, budget_s=args.cpu_budget)
        cpu = {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": (f"token-parallel half (eqs. 1-4) of all {runner_T(w)} tokens in full "
                          f"({info['base_s']:.1f} s), per-query half (eqs. 5-11) timed on its own on "
                          f"{info['rows']} seeded query rows ({info['per_row_s'] * 1e3:.1f} ms/row), "
                          f"tokens/s = T / (base + per-row x T)"),
               "tiny_1thread": oracle_tiny_one_thread()}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16" if w.dims.dtype == csa.CSA_BF16 else "f32",
                "data": "synthetic (seeded normal H, N(0,1/fan_in) weights)", "config": workload_config(w, world),
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
                "clocks": clocks, "stages": stages, "stages_in_step": stages_in_step, "decode": decode,
                "workloads": workloads}
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


def run_indexer_only(args):
    """csa_indexer_topk alone on seeded q^I, w^I and K^IComp with the sizes of
    a workload (no projections: a few GB on the device even at n = 131072),
    warmup + steps launches; for DRAM-traffic captures of the indexer."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = synth.workloads()[args.workload]
    d = w.dims
    T, nseq, maxlen = sum(w.seqlens), len(w.seqlens), max(w.seqlens)
    cu, cb = csa.cu_from_lengths(w.seqlens, d.m)
    NB = int(cb[-1])
    g = torch.Generator(device=dev).manual_seed(w.seed + 11)
    qI = torch.randn(T, d.nhI * d.cI, device=dev, generator=g).to(torch.bfloat16)
    wI = torch.randn(T, d.nhI, device=dev, generator=g)
    KI = (0.5 * torch.randn(NB, d.cI, device=dev, generator=g)).to(torch.bfloat16)
    idx = torch.empty(T, d.topk, dtype=torch.int32, device=dev)
    ws = torch.empty(csa.csa_indexer_workspace_bytes(d, T, nseq, maxlen), dtype=torch.uint8, device=dev)
    cu, cb = cu.to(dev), cb.to(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for i in range(args.warmup + args.steps):
        if i == args.warmup:
            ev[0].record()
        csa.csa_indexer_topk(d, qI, d.nhI * d.cI, wI, d.nhI, KI, cu, cb, nseq, T, NB, maxlen, idx, ws)
    ev[1].record()
    torch.cuda.synchronize()
    st = csa.csa_get_device_status()
    ms = ev[0].elapsed_time(ev[1]) / max(args.steps, 1)
    print(json.dumps({"stage": "A4_indexer_topk (seeded inputs)", "workload": args.workload, "ms": ms,
                      "scratch_bytes": ws.numel(), "status": csa.status_string(st)}), flush=True)
    if st != 0:
        raise SystemExit(1)


def run_decode_only(args):
    """warmup + steps decode steps of the decode workload (bf16 key cache, then
    the E4M3 key cache); for profiling the decode kernels."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dr = DecodeRunner(synth.workloads()["decode"], dev)
    for _ in range(args.warmup + args.steps):
        dr.step()
    dr.quantise_keys()
    for _ in range(args.warmup + args.steps):
        dr.step_q8()
    torch.cuda.synchronize()
    st = csa.csa_get_device_status()
    print(json.dumps({"decode_steps": 2 * (args.warmup + args.steps), "status": csa.status_string(st)}), flush=True)
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
    ap.add_argument("--ref-rows", type=int, default=16, help="query rows the reference arm runs per step")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle row time for cpu_baseline")
    ap.add_argument("--no-workloads", action="store_true", help="skip the long and ragged workload lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-stages", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--stage", choices=["A1_project_hidden", "A2_project_query", "A3_compress", "A4_indexer_topk",
                                        "A5_sparse_mqa", "A1A3_project_compress"],
                    help="run only this stage (profiling)")
    ap.add_argument("--decode-only", action="store_true", help="run decode steps only (profiling)")
    ap.add_argument("--indexer-only", action="store_true",
                    help="run csa_indexer_topk alone on seeded inputs of the workload's sizes (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.indexer_only:
        run_indexer_only(args)
        return
    if args.decode_only:
        run_decode_only(args)
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
