#!/usr/bin/env python
"""Benchmark of MLA decoding over a paged latent KV cache on B200.

One step = one pass of the whole decode path on one batch of synthetic input:
the tile scheduler (metadata kernel), the split-KV kernel and the combine
kernel.  The headline workload is the compute-bound decode (batch 64, s_q 1,
h_q 128, d_qk 576, d_v 512, cache lengths uniform in [1024, 8192], 64-token
pages, shuffled block table, bf16 N(0,1), scale 1/sqrt(576)).  The other decode
workloads (the four other configurations, and the compute one over an FP8-with-scale
cache) are timed in the same run and reported under "workloads".

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronisation; each step replays one captured CUDA graph holding the
three kernels with timing events around them (on the launching stream; a second
graph with events between the kernels gives each kernel's own time); L2
is flushed between steps (a write of 2 x L2), outside the events.  For N > 1 GPUs each rank runs an independent replica
(the path needs no collective) and rank 0 reports the maximum step time over
ranks.

Prints one JSON line (rank 0).  ``--impl reference`` times the FP64 CPU oracle
on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_decode_attention_12_b200 import workloads as W  # noqa: E402

METRIC = "MLA decode TFLOPS and KV-cache GB/s (fraction of roofline), µs/call, 1×B200"
DESCR = {
    "tiny": "tiny MLA decode: batch 2, s_q=1, h_q=16, h_kv=1, d_qk=576, d_v=512, cache_seqlens {256,193}, "
            "page 64, shuffled block_table, bf16 N(0,1), scale 1/sqrt(576), non-causal",
    "compute": "compute-bound MLA decode: batch 64, s_q=1, h_q=128, h_kv=1, d_qk=576, d_v=512, "
               "cache_seqlens uniform in [1024,8192], page 64, shuffled block_table, bf16 N(0,1), scale 1/sqrt(576)",
    "spec_padded": "speculative MLA decode with padded heads: batch 128, s_q=2, causal, h_q=64 (first 16 active, "
                   "rest zero), d_qk=576, d_v=512, cache_seqlens 4096 +- 512, page 64, bf16 N(0,1)",
    "long_split": "long-context split-KV MLA decode: batch 4, s_q=1, h_q=128, d_qk=576, d_v=512, "
                  "cache_seqlens {65536,49152,32768,8192}, page 64, shuffled block_table, bf16 N(0,1)",
    "fp16_norope": "fp16 MLA decode without the rope part: batch 32, s_q=4, causal, h_q=64, d_qk=d_v=512, "
                   "cache_seqlens log-uniform in [512,16384], page 64, shuffled block_table, fp16 N(0,0.5), "
                   "scale 1/sqrt(512)",
    "fp8_compute": "compute-bound MLA decode over an FP8-with-scale cache: batch 64, s_q=1, h_q=128, h_kv=1, "
                   "d_qk=576, d_v=512, cache_seqlens uniform in [1024,8192], page 64, shuffled block_table, "
                   "bf16 N(0,1) q, 656-byte cache rows (512 e4m3 latent + 4 fp32 scales + 64 bf16 rope, "
                   "|value| <= 3.5), scale 1/sqrt(576)",
    "sparse_fp8": "token-level sparse MLA decode over an FP8-with-scale cache: batch 64, s_q=2, h_q=128, h_kv=1, "
                  "d_qk=576, d_v=512, topk=2048 entries per query token drawn without repetition from its "
                  "request's cache (cache_seqlens uniform in [8192,16384]), 656-byte cache rows, bf16 N(0,1) q, "
                  "scale 1/sqrt(576)",
    "sparse_prefill": "sparse MLA prefill: s_q=2048 query tokens, h_q=128, h_kv=1, d_qk=576, d_v=512, s_kv=16384 "
                      "kv rows, topk=2048 distinct rows per token drawn uniformly, bf16 N(0,1) q and kv, "
                      "sm_scale 1/sqrt(576); outputs out, base-2 max_logits and lse",
}
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NVML_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
                0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=W.WORKLOADS, default="compute")
    ap.add_argument("--extra-workloads", default="all",
                    help="comma-separated other workloads to time too ('all' or 'none')")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle baseline")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


def _code_tokens(text: str) -> str:
    """C / CUDA source without comments, whitespace runs collapsed (string literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":  # string or character literal, copied with its escapes
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_sha() -> str:
    """Hash of the CUDA sources' code (comments and whitespace excluded): it changes exactly
    when the compiled kernels can, so recorded counters stay attached to the code they measured."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mla_decode_attention_12_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_tokens(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per split-KV launch from a committed ncu summary, if it matches the current source."""
    path = os.path.join(ROOT, "profiles", "splitkv_dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        ent = d.get(workload)
        if ent and d.get("source_sha") == kernel_source_sha():
            return float(ent["bytes_per_launch"])
    except Exception:
        pass
    return None


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML while running."""

    def __init__(self, device_index: int, uuid: str | None, period_s: float = 0.001):
        self.samples = []
        self.max_mhz = None
        self.err = None
        self._stop = threading.Event()
        self.period = period_s
        try:
            import pynvml

            pynvml.nvmlInit()
            h = None
            if uuid:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report that instead of clocks
            self.nv = None
            self.err = str(e)

    def sample(self) -> bool:
        """One reading of the SM clock and the clock-event reasons (False once NVML fails)."""
        nv, h = self.nv, self.h
        if nv is None:
            return False
        try:
            mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            try:
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            except Exception:
                reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
            self.samples.append((mhz, int(reasons), None))
            return True
        except Exception as e:
            self.err = str(e)
            self.nv = None
            return False

    def _run(self):
        while not self._stop.is_set() and self.sample():
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.nv is not None:
            self._stop.set()
            self._t.join()
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": self.err or "no samples"}
        # Every sample is taken inside the timed region, which keeps the GPU busy (NVML's
        # utilization counter averages over a longer window, so it is not used to filter).
        reasons = set()
        for _, r, _ in self.samples:
            for bit, name in NVML_REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[0] for s in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- GPU arm
class PrefillRunner:
    """The sparse prefill's step (the metadata kernel, then split-KV and combine in one call),
    captured like Runner's; the breakdown has two stages: metadata, split-KV + combine."""

    def __init__(self, torch, mla, p, dev):
        self.torch, self.mla, self.p, self.dev = torch, mla, p, dev
        dt = torch.bfloat16 if p.dtype == W.BF16 else torch.float16
        self.q = torch.from_numpy(p.q.view(np.int16)).view(dt).to(dev)
        self.kv = torch.from_numpy(p.kv.view(np.int16)).view(dt).to(dev)
        self.ind = torch.from_numpy(p.indices).to(dev)
        self.parts = mla.num_sm_parts(dev)
        _, n_ns = mla.metadata_sizes(p.s_q, p.h_q, 1, self.parts)
        self.md = torch.zeros(self.parts, 8, dtype=torch.int32, device=dev)
        self.ns = torch.zeros(n_ns, dtype=torch.int32, device=dev)
        self.out = torch.empty(p.s_q, p.h_q, p.dv, dtype=dt, device=dev)
        self.mx = torch.empty(p.s_q, p.h_q, dtype=torch.float32, device=dev)
        self.lse = torch.empty(p.s_q, p.h_q, dtype=torch.float32, device=dev)
        self.ws = torch.zeros(mla.workspace_bytes(p.s_q, 1, p.h_q, 1, self.parts), dtype=torch.uint8, device=dev)
        from mla_decode_attention_12_b200 import _lib
        lib, topk = _lib.load(), p.indices.shape[2]
        ptr = lambda t: t.data_ptr()

        def metadata():
            _lib.check(lib.mla_get_metadata_sparse(p.s_q, topk, p.h_q, 1, self.parts, ptr(self.md), ptr(self.ns),
                                                   torch.cuda.current_stream(dev).cuda_stream), "metadata")

        def prefill():
            _lib.check(lib.mla_sparse_prefill(ptr(self.q), p.s_q, p.h_q, p.d_qk, ptr(self.kv), p.s_kv, 1, ptr(self.ind),
                                              topk, p.dv, p.dtype, p.sm_scale, ptr(self.md), self.parts, ptr(self.ns),
                                              ptr(self.out), ptr(self.mx), ptr(self.lse), ptr(self.ws),
                                              self.ws.numel(), torch.cuda.current_stream(dev).cuda_stream), "prefill")

        stages = [metadata, prefill]
        self.launches_per_step = 3
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            for _ in range(2):
                for f in stages:
                    f()
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize(dev)
        self.events = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.events[0].record()
            for f in stages:
                f()
            self.events[1].record()
        self.stage_events = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
        self.stage_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.stage_graph):
            self.stage_events[0].record()
            for i, f in enumerate(stages):
                f()
                self.stage_events[i + 1].record()
        torch.cuda.synchronize(dev)

    def step(self):
        self.graph.replay()

    def step_staged(self):
        self.stage_graph.replay()

    def times_ms(self):
        return self.events[0].elapsed_time(self.events[1])

    def stage_times_ms(self):
        """(metadata, split-KV + combine, 0): the prefill's two kernels run in one call."""
        e = self.stage_events
        return (e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), 0.0)

    def status(self):
        return self.mla.read_device_status(self.ws, clear=True)


class Runner:
    """Device tensors and the three launches of one decode step for one workload.

    Each launch is captured once in its own CUDA graph, so replaying a step costs
    the host a few microseconds and the GPU never waits for Python between kernels.
    """

    def __init__(self, torch, mla, p: W.Problem, dev):
        self.torch, self.mla, self.p, self.dev = torch, mla, p, dev
        dt = torch.bfloat16 if p.dtype == W.BF16 else torch.float16
        self.q = torch.from_numpy(p.q.view(np.int16)).view(dt).to(dev)
        self.kv = (torch.from_numpy(p.kvcache) if p.fp8_kv else torch.from_numpy(p.kvcache.view(np.int16)).view(dt)).to(dev)
        self.bt = torch.from_numpy(p.block_table).to(dev)
        self.sl = torch.from_numpy(p.cache_seqlens).to(dev)
        self.rows = p.s_q * p.h_q
        parts = mla.num_sm_parts(dev)
        sparse = p.indices is not None  # token-level sparse decode: the entry lists replace the block table
        self.ind = torch.from_numpy(p.indices).to(dev) if sparse else None
        md_kw = dict(h_q=p.h_q, topk=p.indices.shape[2]) if sparse else dict(is_fp8_kvcache=p.fp8_kv)
        n_md, n_ns = mla.metadata_sizes(p.batch * p.s_q if sparse else p.batch, p.h_q if sparse else self.rows, 1,
                                        parts)
        self.md = torch.zeros(parts, 8, dtype=torch.int32, device=dev)
        self.ns = torch.zeros(n_ns, dtype=torch.int32, device=dev)
        mla.get_mla_metadata(self.sl, self.rows, 1, out=(self.md, self.ns), **md_kw)
        ws_b, ws_s = (p.batch * p.s_q, 1) if sparse else (p.batch, p.s_q)
        ws = torch.zeros(mla.workspace_bytes(ws_b, ws_s, p.h_q, 1, parts), dtype=torch.uint8, device=dev)
        # padding heads (the spec_padded workload) are declared, so their outputs are skipped
        self.call = mla.DecodeCall(self.q, self.kv, self.bt, self.sl, p.dv, self.md, self.ns, causal=p.causal,
                                   softmax_scale=p.scale, workspace=ws, active_heads=p.active_heads,
                                   is_fp8_kvcache=p.fp8_kv, indices=self.ind)
        self.launches_per_step = 3
        stages = [lambda: mla.get_mla_metadata(self.sl, self.rows, 1, out=(self.md, self.ns), **md_kw),
                  self.call.splitkv, self.call.combine]
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            for _ in range(2):
                for f in stages:
                    f()
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize(dev)
        # Two graphs of one step each, so a replay costs one launch.  The step graph has
        # timing events only around the three kernels: consecutive kernels keep their
        # programmatic launch edges, so each one's set-up overlaps the previous one's end.
        # The staged graph has an event between kernels (event record nodes serialise
        # them) and gives each kernel's own duration.
        self.events = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.events[0].record()
            for f in stages:
                f()
            self.events[1].record()
        self.stage_events = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
        self.stage_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.stage_graph):
            self.stage_events[0].record()
            for i, f in enumerate(stages):
                f()
                self.stage_events[i + 1].record()
        torch.cuda.synchronize(dev)

    def step(self):
        self.graph.replay()

    def step_staged(self):
        self.stage_graph.replay()

    def times_ms(self):
        """Duration of the last step replay; call after synchronising."""
        return self.events[0].elapsed_time(self.events[1])

    def stage_times_ms(self):
        """(metadata, split-KV, combine) of the last staged replay; call after synchronising."""
        e = self.stage_events
        return (e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3]))

    def status(self):
        return self.mla.read_device_status(self.call.workspace, clear=True)


def time_steps(torch, runner, flush, steps, warmup, barrier, sampler=None, staged_steps=None):
    """Times `steps` step replays (after `warmup`), then `staged_steps` staged replays for
    the per-kernel breakdown.  Returns ms rows: step, metadata, split-KV, combine (the
    breakdown columns come from the staged replays, cycled over the step rows)."""
    for _ in range(warmup):
        flush.zero_()
        runner.step()
        flush.zero_()
        runner.step_staged()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t = []
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        for _ in range(steps):
            flush.zero_()  # L2 flush between steps, outside the events
            runner.step()
            if sampler is not None:
                sampler.sample()  # while the step runs (the launch is asynchronous)
            torch.cuda.synchronize()
            t.append(runner.times_ms())
    barrier()
    st = []
    for _ in range(min(steps, 100) if staged_steps is None else staged_steps):
        flush.zero_()
        runner.step_staged()
        torch.cuda.synchronize()
        st.append(runner.stage_times_ms())
    st = np.array(st)
    rows = np.zeros((len(t), 4))
    rows[:, 0] = t
    rows[:, 1:] = st[np.arange(len(t)) % len(st)]
    return rows  # ms: step, metadata, splitkv, combine


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank number over all ranks (the job is as slow as its slowest replica)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_replica: float, world: int, step_ms: float) -> float:
    """Throughput of N independent replicas, each doing one decode step per step time."""
    return world * flops_per_replica / (step_ms * 1e-3) / 1e12


def roofline(p: W.Problem, t_splitkv_ms: float, peaks, src: str, traffic):
    flops, nbytes = p.flops(), p.io_bytes()
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    t = t_splitkv_ms * 1e-3
    if t_hbm >= t_tc:
        ach, peak, unit, bound = nbytes / t / 1e9, peaks["hbm_gbs"], "GB/s", "hbm"
    else:
        ach, peak, unit, bound = flops / t / 1e12, peaks["bf16_tflops"], "TFLOP/s", "tensor"
    return {"bound": bound, "achieved": round(ach, 2), "peak": peak, "unit": unit, "frac": round(ach / peak, 4),
            "traffic": traffic, "peak_source": f"{src} (MEASURED_PEAKS.json burst)" if src == "measured" else src,
            "kernel": "mla_splitkv_kernel", "algorithmic_bytes": nbytes, "algorithmic_flops": flops}


def workload_line(p, t, peaks, src):
    step_ms = float(t[:, 0].mean())
    sk_ms = float(t[:, 2].mean())
    flops, nbytes = p.flops(), p.io_bytes()
    rf = roofline(p, sk_ms, peaks, src, recorded_traffic(p.name))
    out = {
        "us_per_call": round(step_ms * 1e3, 2),
        "us_per_call_median": round(float(np.median(t[:, 0])) * 1e3, 2),
        "us_per_call_p10": round(float(np.percentile(t[:, 0], 10)) * 1e3, 2),
        "us_per_call_p90": round(float(np.percentile(t[:, 0], 90)) * 1e3, 2),
        "us_splitkv": round(sk_ms * 1e3, 2),
        "us_combine": round(float(t[:, 3].mean()) * 1e3, 2),
        "us_metadata": round(float(t[:, 1].mean()) * 1e3, 2),
        "tflops": round(flops / (step_ms * 1e-3) / 1e12, 2),
        "kv_gbs": round(p.kv_bytes() / (step_ms * 1e-3) / 1e9, 1),
        "io_gbs": round(nbytes / (step_ms * 1e-3) / 1e9, 1),
        "roofline": rf,
    }
    if p.active_heads is not None:
        out["tflops_active_heads"] = round(flops * p.active_heads / p.h_q / (step_ms * 1e-3) / 1e12, 2)
    return out


def workload_config(p: W.Problem, world: int) -> dict:
    """The ``config`` object of a JSON line: the same keys and values in both arms for one workload."""
    return {"workload": DESCR[p.name], "batch": p.batch, "s_q": p.s_q, "h_q": p.h_q, "h_kv": 1,
            "d_qk": p.d_qk, "d_v": p.dv, "page_size": 64, "causal": p.causal,
            "l2": "flushed between steps (write of 2 x L2 outside the timed events)",
            "parallelism": f"{world} independent replica(s), no collective"}


def oracle_rows(oracle, p: W.Problem, ids):
    """The oracle on flat query rows `ids` (an FP8 cache is dequantized by the oracle itself)."""
    if p.fp8_kv:
        return oracle.decode_rows_fp8(p.q, p.kvcache, p.block_table, p.cache_seqlens, ids, dv=p.dv,
                                      causal=p.causal, scale=p.scale)
    return oracle.decode_rows(p.q, p.kvcache, p.block_table, p.cache_seqlens, ids, dv=p.dv, dtype=p.dtype,
                              causal=p.causal, scale=p.scale)


def cpu_baseline(p: W.Problem, target_s: float, seed=0):
    """The FP64 oracle on a bounded sample of rows of the same workload."""
    import oracle

    oracle.build()
    rows_total = p.batch * p.s_q * p.h_q
    vis = np.repeat(p.visible()[:, :, None], p.h_q, axis=2).reshape(-1)
    rng = np.random.default_rng(seed)
    order = rng.permutation(rows_total)

    def run(n):
        ids = np.sort(order[:n]).astype(np.int64)
        t0 = time.perf_counter()
        oracle_rows(oracle, p, ids)
        dt = time.perf_counter() - t0
        return dt, float(2.0 * (p.d_qk + p.dv) * vis[ids].sum())

    threads = oracle.num_threads()
    n = max(1, min(rows_total, threads))
    dt, fl = run(n)
    while dt < 0.5 and n < rows_total:
        n = min(rows_total, n * 4)
        dt, fl = run(n)
    n = max(1, min(rows_total, int(n * target_s / max(dt, 1e-3))))
    dt, fl = run(n)
    return {"value": fl / dt / 1e12, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
            "sample": f"{n} of {rows_total} query rows of the {p.name} workload (seeded random subset), FP64, "
                      f"{dt:.1f} s", "seconds": round(dt, 2)}


def e2e(torch, mla, p: W.Problem, steps: int):
    """Same metric through the public call with pinned host buffers, copies inside the timed region."""
    dt = torch.bfloat16 if p.dtype == W.BF16 else torch.float16
    q = torch.from_numpy(p.q.view(np.int16)).view(dt).pin_memory()
    kv = (torch.from_numpy(p.kvcache) if p.fp8_kv else torch.from_numpy(p.kvcache.view(np.int16)).view(dt)).pin_memory()
    bt = torch.from_numpy(p.block_table).pin_memory()
    sl = torch.from_numpy(p.cache_seqlens).pin_memory()
    rows = p.s_q * p.h_q

    def one():
        md, ns = mla.get_mla_metadata(sl.cuda(non_blocking=True), rows, 1)
        return mla.flash_mla_with_kvcache(q, kv, bt, sl, p.dv, md, ns, causal=p.causal, softmax_scale=p.scale,
                                          is_fp8_kvcache=p.fp8_kv)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        o, lse = one()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = float(np.mean(times))
    h2d = q.numel() * 2 + kv.numel() * kv.element_size() + bt.numel() * 4 + 2 * sl.numel() * 4
    d2h = o.numel() * 2 + lse.numel() * 4
    return {"value": round(p.flops() / (ms * 1e-3) / 1e12, 3), "unit": "TFLOPS", "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "path": "flash_mla_with_kvcache with pinned host tensors (C ABI), H2D + kernels + D2H"}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import mla_decode_attention_12_b200 as mla
    from mla_decode_attention_12_b200 import _lib

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    _lib.load()  # fails loudly if the CUDA library is missing

    def barrier():
        if world > 1:
            dist.barrier()

    peaks, src = load_peaks()
    props = torch.cuda.get_device_properties(dev)
    flush = torch.empty(max(2 * props.L2_cache_size, 256 << 20), dtype=torch.uint8, device=dev)

    p = W.make_workload(args.workload)
    runner = Runner(torch, mla, p, dev)
    sampler = ClockSampler(local, getattr(props, "uuid", None) and str(props.uuid))
    t = time_steps(torch, runner, flush, args.steps, args.warmup, barrier, sampler)
    status = runner.status()
    step_ms = max_over_ranks(float(t[:, 0].mean()), device=dev)
    main = workload_line(p, t, peaks, src)

    extra = {}
    names = [] if args.extra_workloads == "none" else (
        [w for w in W.WORKLOADS + W.SPARSE_WORKLOADS + W.PREFILL_WORKLOADS if w != args.workload]
        if args.extra_workloads == "all"
        else [w for w in args.extra_workloads.split(",") if w and w != args.workload])
    if rank == 0:
        for name in names:
            if name in W.PREFILL_WORKLOADS:
                pw = W.make_prefill_workload(name)
                r = PrefillRunner(torch, mla, pw, dev)
                tw = time_steps(torch, r, flush, min(args.steps, 50), min(args.warmup, 5), lambda: None)
                extra[name] = workload_line(pw, tw, peaks, src)
                extra[name]["workload"] = DESCR[name]
                extra[name]["device_status"] = r.status()
                extra[name]["note"] = "us_splitkv is split-KV + combine (one call); the kv is L2-resident and counted once"
                del r
                torch.cuda.empty_cache()
                continue
            pw = W.make_workload(name)
            r = Runner(torch, mla, pw, dev)
            tw = time_steps(torch, r, flush, min(args.steps, 200), min(args.warmup, 10), lambda: None)
            extra[name] = workload_line(pw, tw, peaks, src)
            extra[name]["workload"] = DESCR[name]
            extra[name]["device_status"] = r.status()
            del r
            torch.cuda.empty_cache()
    e2e_line = None if args.no_e2e or rank != 0 else e2e(torch, mla, p, steps=min(args.steps, 10))
    base = cpu_baseline(p, args.cpu_seconds) if (rank == 0 and world == 1 and args.cpu_seconds > 0) else None

    if rank == 0:
        value = whole_job_tflops(p.flops(), world, step_ms)
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "TFLOPS",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(step_ms, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if p.dtype == W.BF16 else "fp16",
            "data": "synthetic (seeded, shapes and distributions of the workload)",
            "config": workload_config(p, world),
            "us_per_call": main["us_per_call"],
            "us_per_call_p10_median_p90": [main["us_per_call_p10"], main["us_per_call_median"],
                                           main["us_per_call_p90"]],
            "kv_gbs": main["kv_gbs"],
            "tflops": main["tflops"],
            "breakdown_us": {"metadata": main["us_metadata"], "splitkv": main["us_splitkv"],
                             "combine": main["us_combine"],
                             "note": "each kernel alone: replays with an event between kernels, "
                                     "which removes the launch overlap the timed steps have"},
            "roofline": main["roofline"],
            "cpu_baseline": base,
            "e2e": e2e_line,
            "gpu_launches": runner.launches_per_step * args.steps,
            "clocks": sampler.summary(),
            "device_status": status,
            "workloads": extra,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The FP64 CPU oracle, as it stands, on a bounded sample of the same workload per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle

    oracle.build()
    p = W.make_workload(args.workload)
    budget_s = 150.0
    per_step = min(2.0, budget_s / max(1, args.steps + args.warmup))
    rows_total = p.batch * p.s_q * p.h_q
    vis = np.repeat(p.visible()[:, :, None], p.h_q, axis=2).reshape(-1)
    order = np.random.default_rng(0).permutation(rows_total)
    # calibrate the sample size to about per_step seconds
    n = max(1, oracle.num_threads())
    while True:
        ids = np.sort(order[:n]).astype(np.int64)
        t0 = time.perf_counter()
        oracle_rows(oracle, p, ids)
        dt = time.perf_counter() - t0
        if dt >= per_step / 4 or n >= rows_total:
            break
        n = min(rows_total, n * 2)
    n = max(1, min(rows_total, int(n * per_step / max(dt, 1e-4))))
    ids = np.sort(order[:n]).astype(np.int64)
    flops = float(2.0 * (p.d_qk + p.dv) * vis[ids].sum())
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle_rows(oracle, p, ids)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    s = float(np.mean(times))
    value = flops / s / 1e12
    sample = f"{n} of {rows_total} query rows of the {p.name} workload per step (seeded subset), FP64"
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(s * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
        # the GPU arm's config object for the same workload and N (the oracle has no L2 flush
        # of its own to state; the keys stay identical so the two lines compare directly)
        "config": workload_config(p, int(os.environ.get("WORLD_SIZE", str(args.gpus)))),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
