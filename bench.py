"""Benchmark of the HySparse2 hybrid sparse attention step on B200.

One step = one hs2_step call (full attention -> GQA-max log-softmax score -> top-k +
window -> sparse attention with KV Reuse) over one batch of the chosen workload.  The
default workload is the long-context decode at N = 128K (B=1, Hq=64, Hkv=8, d=128,
T=1, k=4096, W=512), the configuration the sparse-attention queries/s and HBM GB/s
metric is quoted on.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long] [--impl reference]
                    [--workloads batched,prefill,...|none]

Under torchrun (N > 1) every rank runs an independent replica of the workload on its own
GPU (the step has no cross-GPU exchange); timing is the max over ranks.  Prints one JSON
line on rank 0.  ``--impl reference`` times the fp64 CPU oracle instead (rank 0 only).

On one GPU the same line also carries a ``workloads`` block: the other benchmark shapes
(tiny and batched decode, chunked prefill, 1M-token decode at T = 1 and 16) and the headline shapes
with the cache stored as FP8 E4M3 or in a paged pool, each with its step time, queries/s,
roofline, clocks and a bounded CPU-oracle baseline.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn queries/s and achieved HBM GB/s (% of 8 TB/s) at N=128K, 1xB200"
# DRAM bytes (read + write) per launch of the roofline kernel, from an ncu capture of the same
# kernel binary on the same workload; None where no capture matches the current kernel.
NCU_TRAFFIC = {("long", "full_attn_keep_logits"): 536944384 + 8409600}
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 1000 * 1000
L2_FLUSH_BYTES = 256 << 20


# Workloads the default run measures besides the headline one: the other benchmark shapes and
# the headline shapes with the cache stored as FP8 E4M3 or in a paged pool.
#   name -> (shape, cache dtype, page size)
EXTRA_WORKLOADS = {
    "tiny": ("tiny", "bf16", 0),
    "batched": ("batched", "bf16", 0),
    "prefill": ("prefill", "bf16", 0),
    "1m_t1": ("1m_t1", "bf16", 0),
    "1m_t16": ("1m_t16", "bf16", 0),
    "long_fp8": ("long", "fp8_e4m3", 0),
    "long_paged": ("long", "bf16", 64),
    "1m_t1_fp8": ("1m_t1", "fp8_e4m3", 0),
}


def elem_bytes(kv_dtype):
    return 1 if kv_dtype == "fp8_e4m3" else 2


def kv_bytes(w, kv_dtype="bf16"):
    return 2 * w.B * w.Hkv * w.N * w.d * elem_bytes(kv_dtype)


def kv_fits_l2(w, kv_dtype="bf16"):
    """K and V together no larger than L2: the timed steps then flush L2 in between."""
    return kv_bytes(w, kv_dtype) <= L2_BYTES
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def workload(name):
    from long_context_sparse_hs2_b200.inputs import WORKLOADS

    return WORKLOADS[name]


def flop_model(w):
    """Tensor FLOPs of the full-attention layer (QK^T and PV over every visible key)."""
    visible = sum(w.N - w.T + t + 1 for t in range(w.T))
    return 4.0 * w.B * w.Hq * w.d * visible


def byte_model(w, kv_dtype="bf16"):
    """Algorithmic bytes per step.

    literal: K read once + the gathered K/V rows of the selection (the metric's formula);
    minimum: K and V read once + gathered rows + Q in, O/LSE/idx out.
    kv_once: K and V read once -- the algorithmic bytes of the full-attention kernel.
    A cache row is d elements of 2 bytes (bf16) or 1 byte (FP8 E4M3)."""
    B, Hq, Hkv, d, N, T, k, W = w.B, w.Hq, w.Hkv, w.d, w.N, w.T, w.k, w.W
    kv_row = d * elem_bytes(kv_dtype)
    k_bytes = B * Hkv * N * kv_row
    sel = 0
    for t in range(T):
        pos = N - T + t
        sel += min(k, max(0, pos - W + 1)) + min(W, pos + 1)
    gathered = B * Hkv * sel * 2 * kv_row
    q_o = B * Hq * T * d * 2 * 4 + B * Hq * T * 4 * 2 + B * Hkv * T * (k + W + 1) * 4
    return dict(literal=k_bytes + gathered, minimum=2 * k_bytes + gathered + q_o, kv_once=2 * k_bytes,
                gathered=gathered)


class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed region runs.

    NVML is polled every millisecond from a background thread (a decode step is ~0.1 ms, so
    nvidia-smi's 100 ms polling would miss a short timed region entirely); one sample is also
    taken on entry and on exit.  Without NVML it falls back to `nvidia-smi -lms 100`.
    """

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvmlClocksEventReason*)
    REASON_BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
                   0x40: "hw_thermal_slowdown"}

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.nvml = None
        self.samples = []
        self.lines = []

    # -- NVML path
    def _nvml_sample(self):
        nv, h = self.nvml, self.handle
        try:
            clk = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.samples.append((float(clk), int(get_reasons(h))))
        except Exception:
            pass

    def _nvml_loop(self):
        while True:
            self._nvml_sample()
            if self.stop.wait(0.001):
                break

    def __enter__(self):
        try:
            import pynvml
            import threading

            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self._nvml_sample()
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.nvml is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            self._nvml_sample()
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
            return
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        if self.samples:
            for clk, bits in self.samples:
                sm.append(clk)
                for bit, nm in self.REASON_BITS.items():
                    if bits & bit:
                        reasons.add(nm)
            mx = self.max_mhz
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "source": "nvml" if self.samples else "nvidia-smi"}


# ----------------------------------------------------------------------------- oracle (CPU) arm

def oracle_rows(w, kv=("bf16", 0)):
    from dataclasses import replace

    from long_context_sparse_hs2_b200.inputs import bf16_cache, fp8_e4m3_cache, generate, paged_cache

    inp = generate(w)
    kv_dtype, page_size = kv
    if kv_dtype != "bf16" or page_size:
        c = fp8_e4m3_cache(inp.K, inp.V) if kv_dtype == "fp8_e4m3" else bf16_cache(inp)
        if page_size:
            c = paged_cache(c, page_size, seed=w.seed, spare_pages=0)
        inp = replace(inp, cache=c)
    rows = [(b, h, t) for t in range(w.T) for b in range(w.B) for h in range(w.Hkv)]
    return inp, rows


def oracle_time(w, budget_s, inp_rows=None, kv=("bf16", 0)):
    """Time the fp64 oracle on a bounded sample of the workload's selection rows."""
    import oracle.hs2_oracle as O

    inp, rows = inp_rows or oracle_rows(w, kv)
    done, t0 = 0, time.perf_counter()
    for r in rows:
        O.step_rows(inp, [r])
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    el = time.perf_counter() - t0
    per_row = el / done
    queries_per_s = 1.0 / (per_row * w.B * w.Hkv)   # one query = all B*Hkv rows of one t
    sample = f"{done} of {len(rows)} (b, kv head, t) rows of the '{w.name}' workload, full step per row"
    return queries_per_s, el, sample


def oracle_steps(w, steps, warmup):
    """Reference arm: each step runs the oracle on one (b, kv head, t) row (cycling)."""
    import oracle.hs2_oracle as O

    inp, rows = oracle_rows(w)
    for i in range(warmup):
        O.step_rows(inp, [rows[i % len(rows)]])
    t0 = time.perf_counter()
    for i in range(steps):
        O.step_rows(inp, [rows[(warmup + i) % len(rows)]])
    el = time.perf_counter() - t0
    queries = steps / (w.B * w.Hkv)
    sample = (f"{steps} timed steps, each one (b, kv head, t) row of the '{w.name}' workload "
              f"(1/{w.B * w.Hkv} of a query), after {warmup} warm-up rows")
    return queries / el, el, sample


def max_over_ranks(x, dist, device=None):
    """Max of a float over all ranks (the slowest rank sets the step time); identity without dist."""
    if dist is None:
        return x
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(n_ranks, queries_per_replica_step, steps, max_ms):
    """Whole-job queries/s: every rank ran `steps` replica steps; time is the max over ranks."""
    return n_ranks * queries_per_replica_step * steps / (max_ms / 1000.0)


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


# ----------------------------------------------------------------------------- GPU arm

def run_gpu(w, kv_dtype, page_size, steps, warmup, e2e_steps, local_rank, dist):
    """Time `steps` hs2 steps of workload w (cache stored as kv_dtype, paged if page_size) on
    this rank's GPU, after `warmup` untimed ones; e2e_steps > 0 also times the public call with
    host buffers and the copies inside the timed region."""
    import numpy as np
    import torch
    from long_context_sparse_hs2_b200 import build, hs2
    from long_context_sparse_hs2_b200.inputs import bf16_cache, fp8_e4m3_cache, generate, paged_cache

    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    inp = generate(w)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    Qf, Qs = to_dev(inp.Qf), to_dev(inp.Qs)
    pos = torch.from_numpy(inp.pos).to(dev)
    cache = None
    if kv_dtype == "bf16" and not page_size:
        K, V = to_dev(inp.K), to_dev(inp.V)
        dims = hs2.dims_of(Qf, K, w.k, w.W)
        ws = hs2.alloc_workspace(dims, dev)
    else:
        c = fp8_e4m3_cache(inp.K, inp.V) if kv_dtype == "fp8_e4m3" else bf16_cache(inp)
        if page_size:
            c = paged_cache(c, page_size, seed=w.seed, spare_pages=0)
        t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
        kv = (to_dev(c.K), to_dev(c.V)) if kv_dtype == "bf16" else (t(c.K), t(c.V))
        cache = hs2.KVCache(K=kv[0], V=kv[1], N=c.N, dtype=c.dtype, k_scale=t(c.k_scale), v_scale=t(c.v_scale),
                            page_size=c.page_size, page_table=t(c.page_table))
        del c
        dims = hs2.dims_kv(Qf, cache, w.k, w.W)
        ws = hs2.alloc_workspace_kv(dims, cache, dev)
    del inp
    out = hs2.alloc_step_outputs(dims, dev)
    stream = torch.cuda.Stream(device=dev)

    def one_step():
        if cache is None:
            hs2.step(Qf, Qs, K, V, pos, k=w.k, W=w.W, out=out, ws=ws, stream=stream)
        else:
            hs2.step_kv(Qf, Qs, cache, pos, k=w.k, W=w.W, out=out, ws=ws, stream=stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    # K and V smaller than L2: write a buffer larger than L2 between timed steps, outside the
    # events, so that no step finds the previous step's data in L2
    flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev) if kv_fits_l2(w, kv_dtype) else None

    def timed(n):
        torch.cuda.synchronize(dev)
        barrier()
        if flush_buf is None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                one_step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            barrier()
            return e0.elapsed_time(e1)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for e0, e1 in evs:
            flush_buf.fill_(1)
            e0.record(stream)
            one_step()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        return sum(e0.elapsed_time(e1) for e0, e1 in evs)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            one_step()
    torch.cuda.synchronize(dev)
    assert hs2.read_device_status(ws, stream) == 0, "device status bits set during warm-up"

    # main timed region (headline number), clocks sampled meanwhile
    l0 = hs2.launch_count()
    with ClockSampler(local_rank) as clk:
        ms = timed(steps)
    launches = hs2.launch_count() - l0
    clocks = clk.summary()

    # traced timed region: per-kernel CUDA-event durations on the launch stream
    hs2.trace_enable(True)
    ms_traced = timed(steps)
    kern = hs2.trace_collect()
    hs2.trace_enable(False)
    assert hs2.read_device_status(ws, stream) == 0, "device status bits set during the timed region"

    ms_e2e, h2d, d2h = None, 0, 0
    if e2e_steps > 0:
        # end to end through the public API with host buffers (pinned), copies inside the timed region
        src = {"Qf": Qf, "Qs": Qs, "pos": pos}
        if cache is None:
            src.update(K=K, V=V)
        else:
            src.update({"cache_" + n: t for n, t in cache.tensors().items()})
        host_in = {n: t.cpu().pin_memory() for n, t in src.items()}
        dev_in = {n: torch.empty_like(t, device=dev) for n, t in host_in.items()}
        host_out = {n: torch.empty_like(t, device="cpu").pin_memory() for n, t in out.as_dict().items()}
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out.values())
        dev_cache = None
        if cache is not None:
            dev_cache = hs2.KVCache(K=dev_in["cache_K"], V=dev_in["cache_V"], N=cache.N, dtype=cache.dtype,
                                    k_scale=dev_in.get("cache_k_scale"), v_scale=dev_in.get("cache_v_scale"),
                                    page_size=cache.page_size, page_table=dev_in.get("cache_page_table"))

        def e2e_step():
            for n in dev_in:
                dev_in[n].copy_(host_in[n], non_blocking=True)
            if dev_cache is None:
                hs2.step(dev_in["Qf"], dev_in["Qs"], dev_in["K"], dev_in["V"], dev_in["pos"], k=w.k, W=w.W, out=out,
                         ws=ws, stream=stream)
            else:
                hs2.step_kv(dev_in["Qf"], dev_in["Qs"], dev_cache, dev_in["pos"], k=w.k, W=w.W, out=out, ws=ws,
                            stream=stream)
            for n, t in out.as_dict().items():
                host_out[n].copy_(t, non_blocking=True)

        with torch.cuda.stream(stream):
            e2e_step()
            torch.cuda.synchronize(dev)
            barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(e2e_steps):
                e2e_step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            barrier()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1), dist, dev)
        assert hs2.read_device_status(ws, stream) == 0, "device status bits set during the end-to-end region"

    ms = max_over_ranks(ms, dist, dev)
    return dict(w=w, ms=ms, ms_traced=ms_traced, ms_e2e=ms_e2e, kern=kern, launches=launches, clocks=clocks,
                h2d=h2d, d2h=d2h, dims=dims)


def kernel_table(r, steps):
    return {k: {"avg_us": 1000.0 * v[0] / v[1], "launches": v[1], "share": v[0] / max(r["ms_traced"], 1e-9)}
            for k, v in r["kern"].items()}


def roofline(w, kv_dtype, kern, peaks, peak_src, name):
    """Roofline of the dominant kernel (the full-attention sweep) from its live CUDA-event time."""
    bm = byte_model(w, kv_dtype)
    top = max((k for k in kern if k.startswith("full_attn") or k in ("umma_attn", "decode_fused")),
              key=lambda k: kern[k]["avg_us"], default=None)
    if top is None:
        return None
    secs = kern[top]["avg_us"] * 1e-6
    if top == "decode_fused":
        # the whole decode step in one launch: K and V once, then the gathered selection rows
        alg = bm["kv_once"] + bm["gathered"]
        achieved = alg / secs / 1e9
        return {"bound": "hbm", "kernel": top, "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": NCU_TRAFFIC.get((name, top)),
                "peak_source": f"{peak_src} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                "algorithmic_bytes_per_launch": alg}
    # the tcgen05 sweep is a dense contraction; it is tensor-bound when its FLOPs take longer at
    # the measured GEMM peak than its K/V bytes at the measured copy bandwidth (chunked prefill),
    # HBM-bound otherwise (16 decode queries: 128 FLOPs per byte, below the ridge)
    tensor_bound = top == "umma_attn" and (flop_model(w) / (peaks["bf16_tflops"] * 1e12) >
                                           bm["kv_once"] / (peaks["hbm_gbs"] * 1e9))
    if top == "umma_attn" and not tensor_bound:
        achieved = bm["kv_once"] / secs / 1e9
        flops = flop_model(w) / secs / 1e12
        return {"bound": "hbm", "kernel": top, "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": NCU_TRAFFIC.get((name, top)),
                "peak_source": f"{peak_src} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                "algorithmic_bytes_per_launch": bm["kv_once"],
                "tensor": {"achieved_tflops": flops, "frac_of_burst": flops / peaks["bf16_tflops"]}}
    if tensor_bound:
        achieved = flop_model(w) / secs / 1e12
        return {"bound": "tensor", "kernel": top, "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                "peak_source": f"{peak_src} bf16 dense (MEASURED_PEAKS.json bf16_tflops, burst)",
                "algorithmic_flops_per_launch": flop_model(w),
                "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])}
    achieved = bm["kv_once"] / secs / 1e9
    return {"bound": "hbm", "kernel": top, "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": NCU_TRAFFIC.get((name, top)),
            "peak_source": f"{peak_src} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
            "algorithmic_bytes_per_launch": bm["kv_once"]}


def hbm_block(w, kv_dtype, step_s, peaks):
    bm = byte_model(w, kv_dtype)
    return {"literal_bytes_per_step": bm["literal"], "literal_gbs": bm["literal"] / step_s / 1e9,
            "literal_frac_of_8tbs": bm["literal"] / step_s / 1e9 / NOMINAL_HBM_GBS,
            "min_bytes_per_step": bm["minimum"], "min_gbs": bm["minimum"] / step_s / 1e9,
            "min_frac_of_8tbs": bm["minimum"] / step_s / 1e9 / NOMINAL_HBM_GBS,
            "min_frac_of_measured": bm["minimum"] / step_s / 1e9 / peaks["hbm_gbs"]}


def extra_workloads(args, names, peaks, peak_src):
    """The `workloads` block: each extra workload timed on its own (one GPU, rank 0)."""
    import torch

    out = {}
    for name in names:
        shape, kv_dtype, page_size = EXTRA_WORKLOADS[name]
        w = workload(shape)
        t0 = time.perf_counter()
        r = run_gpu(w, kv_dtype, page_size, args.extra_steps, args.warmup, 0, 0, None)
        torch.cuda.empty_cache()
        step_s = r["ms"] / 1000.0 / args.extra_steps
        kern = kernel_table(r, args.extra_steps)
        entry = {"workload": shape, "kv_cache": kv_dtype + (f", paged ({page_size}-token pages)" if page_size else ""),
                 "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "N": w.N, "T": w.T, "k": w.k, "W": w.W,
                 "steps": args.extra_steps, "ms_per_step": step_s * 1000.0,
                 "value": w.B * w.T / step_s, "unit": "queries/s",
                 "roofline": roofline(w, kv_dtype, kern, peaks, peak_src, name),
                 "hbm": hbm_block(w, kv_dtype, step_s, peaks), "kernels": kern, "clocks": r["clocks"],
                 "l2": "flush between steps" if kv_fits_l2(w, kv_dtype) else "no flush (K/V exceed L2)"}
        if not args.no_cpu_baseline:
            qps_cpu, el, sample = oracle_time(w, args.extra_cpu_budget, kv=(kv_dtype, page_size))
            entry["cpu_baseline"] = {"value": qps_cpu, "unit": "queries/s", "cores": cores(), "kind": "oracle",
                                     "sample": sample, "seconds": el}
        entry["wall_s"] = time.perf_counter() - t0
        out[name] = entry
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long")
    ap.add_argument("--impl", default="hs2", choices=["hs2", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kv-dtype", default="bf16", choices=["bf16", "fp8_e4m3"],
                    help="how the headline workload's cache is stored")
    ap.add_argument("--page-size", type=int, default=0, help="paged cache for the headline workload (0: contiguous)")
    ap.add_argument("--workloads", default=",".join(EXTRA_WORKLOADS),
                    help="comma-separated extra workloads timed after the headline one (one GPU), or 'none'")
    ap.add_argument("--extra-steps", type=int, default=20)
    ap.add_argument("--extra-cpu-budget", type=float, default=3.0, help="seconds of oracle time per extra workload")
    args = ap.parse_args()
    if args.workloads != "none":
        unknown = [x for x in args.workloads.split(",") if x and x not in EXTRA_WORKLOADS]
        if unknown:
            ap.error(f"unknown workloads {unknown}; choose from {sorted(EXTRA_WORKLOADS)}")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = workload(args.workload)
    cfg = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "N": w.N, "T": w.T, "k": w.k,
           "W": w.W, "global_batch": w.B * w.T * max(world, args.gpus), "seq_len": w.N,
           "parallelism": f"replicas x{max(world, args.gpus)}",
           "l2": (("flush: a %d MiB buffer is written between timed steps (K and V, %.1f MiB, fit in the 126 MB L2)"
                   % (L2_FLUSH_BYTES >> 20, kv_bytes(w, args.kv_dtype) / 2**20)) if kv_fits_l2(w, args.kv_dtype) else
                  "no flush: K and V (%d MiB) exceed the 126 MB L2" % (kv_bytes(w, args.kv_dtype) >> 20))}

    if args.impl == "reference":
        if rank != 0:
            return
        qps, el, sample = oracle_steps(w, args.steps, args.warmup)
        line = {"impl": "reference", "metric": METRIC, "value": qps, "unit": "queries/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * el / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": cfg,
                "cpu_baseline": {"value": qps, "unit": "queries/s", "cores": cores(), "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": qps, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_mod

        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_mod
    try:
        r = run_gpu(w, args.kv_dtype, args.page_size, args.steps, args.warmup, args.e2e_steps, local_rank, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    n = max(world, 1)
    step_s = r["ms"] / 1000.0 / args.steps
    qps = replica_throughput(n, w.B * w.T, args.steps, r["ms"])
    kern = kernel_table(r, args.steps)
    line = {
        "metric": METRIC, "value": qps, "unit": "queries/s", "n_gpus": n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_s * 1000.0, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if args.kv_dtype == "bf16" else "bf16 queries, fp8 e4m3 KV cache",
        "data": "synthetic (seeded N(0,1) Q/K/V, needles, AR(1) drift)",
        "config": dict(cfg, kv_cache=args.kv_dtype + (f", paged ({args.page_size}-token pages)" if args.page_size
                                                      else "")),
        "hbm": hbm_block(w, args.kv_dtype, step_s, peaks),
        "roofline": roofline(w, args.kv_dtype, kern, peaks, peak_src, w.name if args.kv_dtype == "bf16" and
                             not args.page_size else None),
        "kernels": kern,
        "traced_ms_per_step": r["ms_traced"] / args.steps,
        "e2e": ({"value": replica_throughput(n, w.B * w.T, args.e2e_steps, r["ms_e2e"]), "unit": "queries/s",
                 "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                 "ms_per_step": r["ms_e2e"] / args.e2e_steps, "steps": args.e2e_steps}
                if args.e2e_steps > 0 else None),
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
    }
    if not args.no_cpu_baseline and n == 1:
        qps_cpu, el, sample = oracle_time(w, args.cpu_budget)
        line["cpu_baseline"] = {"value": qps_cpu, "unit": "queries/s", "cores": cores(), "kind": "oracle",
                                "sample": sample, "seconds": el}
    # the other benchmark shapes and cache formats, one GPU only (a multi-GPU run times the
    # headline workload alone)
    extras = [x for x in args.workloads.split(",") if x] if args.workloads != "none" else []
    if n == 1 and extras:
        t0 = time.perf_counter()
        line["workloads"] = extra_workloads(args, extras, peaks, peak_src)
        line["workloads_wall_s"] = time.perf_counter() - t0
    print(json.dumps(line))


if __name__ == "__main__":
    main()
