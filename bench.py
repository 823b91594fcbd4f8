#!/usr/bin/env python
"""SALS latent-sparse decode benchmark on B200: microseconds per layer-step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl salsc|reference]
                    [--workload NAME] [--layers L]

One step is one decoded token through L layers (default 32): every layer has
its own latent cache Kc/Vc, projections Pk/Pv, query and output buffers, so the
step reads 32 distinct layer sets (4 GiB at the default workload, far above
the 126 MB L2) and no layer finds the previous one's data in L2.  Each layer
runs the whole hot path through the C ABI (salsc_decode_step: latent query,
scoring, top-k, gather/reconstruct/RoPE/attention, merge).  The metric is the
step time divided by L.  The timed steps are CUDA-graph replays of the L
decode calls, timed with CUDA events on the replay stream, max over ranks.

For N > 1 each rank decodes its own batch of sequences (replicas: the path
needs no exchange between GPUs), so per-GPU work is fixed ("weak" scaling)
and the reported time per layer-step is the slowest rank's.

``--impl reference`` times the fp64 CPU oracle (the only other executable
statement of the method) on the host cores, one bounded sample per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from latent_space_sparse_b200 import synth, workloads  # noqa: E402

METRIC = "latent-sparse decode µs/layer-step at 4K/32K ctx; achieved HBM GB/s vs peak"
UNIT = "us/layer-step"

# DRAM bytes (read + write) of one launch, from an ncu capture of the named
# kernel on the named workload (the summary under profiles/ gives the command).
# The capture keeps the caches as the bench's own kernel order leaves them
# (--cache-control none), as in the timed step. An entry is removed whenever
# its kernel changes after the capture.
PROFILED_TRAFFIC: dict[tuple[str, str], float] = {
    # (the attention kernel's entry, 31.89 MB per launch in the bench's kernel
    # order, was removed when its tile partition changed after the capture)
}
TRAFFIC_HOW = ("ncu dram__bytes_read.sum + dram__bytes_write.sum per launch, mean of two launches "
               "in the bench's own kernel order, --cache-control none")
DEFAULT_WORKLOAD = workloads.MISTRAL_32K_B4.name
THROTTLE_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["salsc", "reference"], default="salsc")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.BY_NAME))
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle timing on the host cores")
    ap.add_argument("--no-compress", action="store_true",
                    help="skip the prefill compression GEMM timing")
    ap.add_argument("--compress-only", action="store_true",
                    help="time only the prefill compression GEMM and print its JSON object")
    ap.add_argument("--compress-rows", type=int, default=0,
                    help="rows of K and V for the compression GEMM (default: 16 x 4096)")
    ap.add_argument("--no-side-workloads", action="store_true",
                    help="time only the chosen workload (no `workloads` object)")
    ap.add_argument("--side-steps", type=int, default=20,
                    help="timed steps of each other decode workload")
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_bf16_peak(sustained: bool = False):
    """bf16 dense GEMM TFLOP/s: the burst figure (a kernel timed alone), or the
    sustained one (GEMMs back to back under the power cap)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            peaks = json.load(f)
        key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
        if key in peaks:
            return float(peaks[key]), "measured"
    return (1400.0 if sustained else 1590.0), "fallback"


def bench_compress(salsc, dev, reps: int = 20, warmup: int = 3, rows: int = 0):
    """The prefill compression GEMM of the LLaMA2-7B-shaped batch (16 x 4096
    rows of K and V, hidden 4096, r 512), both halves in one salsc_compress
    call, timed alone with CUDA events; torch.matmul (cuBLAS) on the same
    operands is timed beside it as a library reference point."""
    w = workloads.LLAMA2_4K_B16
    n, hid, r = rows or w.compress_rows, w.hidden, w.rank
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    K = torch.randn(n, hid, device=dev, generator=g).to(torch.bfloat16)
    V = torch.randn(n, hid, device=dev, generator=g).to(torch.bfloat16)
    Pk = torch.linalg.qr(torch.randn(hid, r, device=dev, generator=g))[0].to(torch.bfloat16)
    Pv = torch.linalg.qr(torch.randn(hid, r, device=dev, generator=g))[0].to(torch.bfloat16)
    Kc = torch.empty(n, r, dtype=torch.bfloat16, device=dev)
    Vc = torch.empty_like(Kc)
    flop = 2 * 2 * n * hid * r

    def timed(fn):
        for _ in range(warmup):
            fn()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        for i in range(reps):
            ev[i].record()
            fn()
            ev[i + 1].record()
        torch.cuda.synchronize(dev)
        ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(reps)]
        return statistics.median(ms)

    def isolated(fn):
        # each launch after the GPU has idled for a few ms, so that it runs at
        # the clocks a kernel timed alone gets (the back-to-back loop above
        # settles under the power cap)
        for _ in range(warmup):
            fn()
        ms = []
        for _ in range(reps):
            torch.cuda.synchronize(dev)
            time.sleep(0.004)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        return statistics.median(ms)

    ours = lambda: salsc.salsc_compress(K, V, Pk, Pv, Kc, Vc)  # noqa: E731
    lib = lambda: (torch.matmul(K, Pk, out=Kc), torch.matmul(V, Pv, out=Vc))  # noqa: E731
    with ClockSampler(dev.index if dev.index is not None else 0) as sampler:
        ms = timed(ours)
        ms_lib = timed(lib)
    ms_iso, ms_iso_lib = isolated(ours), isolated(lib)
    peak, kind = measured_bf16_peak()
    peak_s, kind_s = measured_bf16_peak(sustained=True)
    tf = flop / (ms * 1e-3) / 1e12
    tf_iso = flop / (ms_iso * 1e-3) / 1e12
    return {"workload": f"{w.name} prefill: 2 x [{n} x {hid}] . [{hid} x {r}] bf16",
            "us": ms_iso * 1e3, "achieved": tf_iso, "peak": peak, "unit": "TFLOP/s",
            "bound": "tensor", "frac": tf_iso / peak, "peak_kind": kind,
            "torch_matmul_us": ms_iso_lib * 1e3,
            "torch_matmul_tflops": flop / (ms_iso_lib * 1e-3) / 1e12,
            "how": f"median of {reps} launches, each after {4} ms of idle GPU (a kernel timed "
                   "alone, against the burst peak); back_to_back: the same launches in a loop, "
                   "against the sustained peak",
            "back_to_back": {"us": ms * 1e3, "achieved": tf, "peak": peak_s, "frac": tf / peak_s,
                             "peak_kind": kind_s, "torch_matmul_us": ms_lib * 1e3,
                             "torch_matmul_tflops": flop / (ms_lib * 1e-3) / 1e12,
                             "clocks": sampler.summary()}}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only)."""

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.h, self.err = None, str(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in THROTTLE_BITS.items():
                    if bits & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.h is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if self.h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


def max_over_ranks(value: float, device) -> float:
    """The largest ``value`` over the ranks of the default process group (a
    job's time is its slowest rank's); ``value`` itself without one.  Every
    rank must call it (a collective)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ inputs

def make_layers(w, L, device):
    """L layer buffer sets; layer 0 is the canonical numpy-seeded draw."""
    layers = []
    for l in range(L):
        if l == 0:
            x = {k: v.to(device) for k, v in synth.decode_inputs(w).items()}
        else:
            x = synth.decode_inputs_device(w, l, device)
        layers.append(x)
    return layers


def distinct_rows(w, idx):
    """Distinct selected token rows of each sequence (union over its units)."""
    return sum(np.unique(idx[b].reshape(-1)[idx[b].reshape(-1) >= 0]).size
               for b in range(w.batch))


def algorithmic_bytes(w, idx_list, elem):
    """Algorithmic HBM bytes of one layer-step per layer: Kc once, the distinct
    kept Vc rows of each sequence, Pk and Pv once, q and out."""
    N, r, hid = w.n_tokens, w.rank, w.hidden
    return [N * r * elem + distinct_rows(w, idx) * r * elem + 2 * hid * r * elem
            + 2 * w.batch * w.n_q_heads * w.head_dim * elem for idx in idx_list]


def kernel_bytes(w, idx_list, elem):
    """Algorithmic bytes of one launch of each kernel (mean over layers): what
    the kernel must read and write at least once, counting no re-reads.

    latent_q: q, Pk, q_lat (fp32) and its hi/lo bf16 split.
    score:    Kc, the hi/lo latent queries, the fp32 scores.
    topk:     the fp32 scores, the int32 indices.
    attend:   the distinct selected Kc and Vc rows of each sequence, Pk, q,
              the indices (its fp32 per-segment partials are not counted).
    combine:  Pv and out (the partials it reads are not counted)."""
    B, U, r, k, N = w.batch, w.n_kv_heads, w.rank, w.top_k, w.n_tokens
    hid, qo = w.hidden, w.batch * w.n_q_heads * w.head_dim * elem
    npad = (2 * U + 15) // 16 * 16
    split = B * npad * r * 2
    rows = float(np.mean([distinct_rows(w, idx) for idx in idx_list]))
    return {
        "latent_q": qo + hid * r * elem + B * U * r * 4 + split,
        "score": N * r * elem + split + N * U * 4,
        "topk": N * U * 4 + B * U * k * 4,
        "attend": 2 * rows * r * elem + hid * r * elem + qo + B * U * k * 4,
        "combine": hid * r * elem + qo,
    }


# ------------------------------------------------------------------ oracle timing

def oracle_inputs(w, units: int):
    """The first `units` selection units of sequence 0 as their own problem."""
    import oracle
    x = synth.decode_inputs(w, seq_lens=(w.seq_lens[0],))
    G = w.group
    units = min(units, w.n_kv_heads)
    p = oracle.Problem(1, units * G, units, w.head_dim, w.rank, w.top_k,
                       np.array([0, w.seq_lens[0]], dtype=np.int64), w.rope_base)
    return (p, x["q"][:, :units * G], x["Kc"], x["Vc"], x["Pk"][:units * w.head_dim],
            x["Pv"][:units * w.head_dim]), units


def oracle_time(inputs, n_threads: int) -> float:
    import oracle
    t0 = time.perf_counter()
    oracle.decode(*inputs, n_threads=n_threads)
    return time.perf_counter() - t0


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w, n_threads, min_seconds: float = 10.0, single_seconds: float = 5.0):
    """The oracle on all units of sequence 0 with every host core, repeated for at
    least `min_seconds`, and on one unit single-threaded for at least
    `single_seconds`; each extrapolated (units scaled linearly) to one
    layer-step of the whole batch, and labelled as such."""
    total_units = w.batch * w.n_kv_heads
    inputs, units = oracle_inputs(w, w.n_kv_heads)
    secs = []
    while sum(secs) < min_seconds:
        secs.append(oracle_time(inputs, n_threads))
    scale = total_units / units
    mean = statistics.mean(secs)
    inputs1, units1 = oracle_inputs(w, 1)
    secs1 = []
    while sum(secs1) < single_seconds:
        secs1.append(oracle_time(inputs1, 1))
    mean1 = statistics.mean(secs1)
    scale1 = total_units / units1
    return {"value": mean * scale * 1e6, "unit": UNIT, "cores": n_threads, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"oracle.decode of sequence 0 ({units} of {total_units} selection units, "
                      f"n={w.seq_lens[0]}), {len(secs)} runs in {sum(secs):.1f} s, mean "
                      f"{mean:.3f} s, extrapolated x{scale:g} to one layer-step",
            "extrapolated": {"sampled_units": units, "total_units": total_units,
                             "scale": scale, "measured_s_per_sample": mean},
            "single_thread": {"value": mean1 * scale1 * 1e6, "unit": UNIT, "cores": 1,
                              "sample": f"oracle.decode of 1 of {total_units} units of sequence "
                                        f"0, {len(secs1)} runs in {sum(secs1):.1f} s, mean "
                                        f"{mean1:.3f} s, extrapolated x{scale1:g}",
                              "extrapolated": {"sampled_units": units1,
                                               "total_units": total_units, "scale": scale1,
                                               "measured_s_per_sample": mean1}}}


def run_reference(args, w):
    """The oracle timed on the host cores: one bounded sample per step.

    A timed step is the oracle on the first units of sequence 0 (as many as the
    host has cores, at most all of the sequence's units); ``ms_per_step`` is
    that sample's measured time, and ``value`` extrapolates it linearly in the
    units to one layer-step of the whole batch (labelled in ``extrapolated``)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    n_threads = oracle.default_threads()
    inputs, units = oracle_inputs(w, max(1, min(w.n_kv_heads, n_threads)))
    for _ in range(args.warmup):
        oracle_time(inputs, n_threads)
    secs = [oracle_time(inputs, n_threads) for _ in range(args.steps)]
    total_units = w.batch * w.n_kv_heads
    scale = total_units / units
    mean = statistics.mean(secs)
    value = mean * scale * 1e6
    extrap = {"sampled_units": units, "total_units": total_units, "scale": scale,
              "measured_s_per_sample": mean,
              "how": "value = measured seconds per sample x scale, in us per layer-step; "
                     "ms_per_step is the measured sample time"}
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean * 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(args, w),
        "extrapolated": extrap,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": n_threads, "kind": "oracle",
                         "cpu_model": cpu_model(),
                         "sample": f"per step: oracle.decode of {units} of {total_units} units "
                                   f"(sequence 0), extrapolated x{scale:g}",
                         "extrapolated": extrap},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(args, w):
    return {"workload": w.name, "batch": w.batch, "seq_lens": list(w.seq_lens),
            "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
            "rank": w.rank, "top_k": w.top_k, "rope_base": w.rope_base, "layers": args.layers,
            "parallelism": f"replicas x{args.gpus}",
            "l2": f"inputs larger than L2: {args.layers} distinct layer buffer sets per step"}


# ------------------------------------------------------------------ main

# The other decode workloads timed beside the headline (the metric's 4K points
# and the long-context ragged batch); each gets a `workloads` entry.
SIDE_WORKLOADS = (workloads.LLAMA2_4K_B1.name, workloads.LLAMA2_4K_B16.name,
                  workloads.LLAMA31_RAGGED_128K.name)


def timeline_summary(tr, stages):
    """Critical path of traced layer-steps.  tr: int64 [layers][stage][cta][3] global-timer
    stamps (start, dependency wait returned, end; 0 = not recorded).  For each stage that
    recorded: `critical_us` = its last CTA's end minus the previous recorded stage's last end
    (the previous layer's last stage for the first), `wait_us` = its first returned
    dependency wait minus that same previous end (the kernel boundary), and `span_us` = its
    last end minus its first returned wait; means over the layers after the first."""
    tr = np.asarray(tr, dtype=np.float64)
    crit = {n: [] for n in stages}
    wait = {n: [] for n in stages}
    span = {n: [] for n in stages}
    prev_end = None
    step_us = []
    for l in range(tr.shape[0]):
        layer_start = prev_end
        for k, n in enumerate(stages):
            rows = tr[l, k]
            ok = rows[:, 2] > 0
            if not ok.any():
                continue
            end = rows[ok, 2].max()
            waited = rows[ok & (rows[:, 1] > 0), 1].min() if (ok & (rows[:, 1] > 0)).any() \
                else rows[ok, 0].min()
            if prev_end is not None and l > 0:
                crit[n].append((end - prev_end) / 1e3)
                wait[n].append((waited - prev_end) / 1e3)
                span[n].append((end - waited) / 1e3)
            prev_end = end
        if layer_start is not None and l > 0:
            step_us.append((prev_end - layer_start) / 1e3)

    def mean(d):
        return {n: float(np.mean(v)) for n, v in d.items() if v}

    return {"critical_us": mean(crit), "wait_us": mean(wait), "span_us": mean(span),
            "layer_step_us": float(np.mean(step_us)) if step_us else None,
            "how": "salsc_decode_step_traced in a CUDA graph of all layers; per-CTA "
                   "%globaltimer stamps (start, dependency wait returned, end); critical_us = "
                   "stage's last CTA end minus the previous stage's last end, wait_us = first "
                   "returned dependency wait minus that end, span_us = last end minus first "
                   "returned wait; means over layers 1..L-1"}


def step_timeline(salsc, dec, layers, outs, idxs, stream, dev, reps=3):
    """Per-stage critical path of the decode step from a traced graph replay."""
    L = len(layers)
    traces = [salsc.trace_buffer(dev) for _ in range(L)]

    def traced():
        for l, x in enumerate(layers):
            salsc.salsc_decode_step_traced(dec.desc, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"],
                                           outs[l], idxs[l], dec.ws, traces[l])

    with torch.cuda.stream(stream):
        traced()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
        traced()
    with torch.cuda.stream(stream):
        for _ in range(reps):
            g.replay()
    torch.cuda.synchronize(dev)
    del g
    tr = torch.stack(traces).cpu().numpy()
    return timeline_summary(tr, salsc.DECODE_KERNELS)


def time_decode(salsc, w, L, steps, warmup, dev, local, dist, kernel_reps=None, e2e=False,
                timeline=False):
    """Times `steps` graph replays of one decoded token through L layers of
    workload w (CUDA events on the replay stream, max over ranks).  Returns a
    dict: us per layer-step, per-kernel event times, byte counts, clocks, and
    (with e2e) the end-to-end time through the public API with host buffers."""
    dt = synth.torch_dtype(w.dtype)
    elem = 2 if w.dtype == "bf16" else 4
    layers = make_layers(w, L, dev)
    # every layer's query (and output) is a view into one buffer, so the end-to-end
    # run moves a step's inputs and results with one copy each way
    q_all = torch.stack([x["q"] for x in layers])
    for l, x in enumerate(layers):
        x["q"] = q_all[l]
    dec = salsc.Decoder(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank, w.top_k,
                        w.seq_lens, rope_base=w.rope_base, dtype=dt, device=dev)
    out_all = torch.empty_like(q_all)
    outs = list(out_all.unbind(0))
    idxs = [torch.empty((w.batch, w.n_kv_heads, w.top_k), dtype=torch.int32, device=dev)
            for _ in range(L)]
    stream = torch.cuda.Stream(device=dev)

    def step(timed_events=None):
        for l, x in enumerate(layers):
            if timed_events is None:
                salsc.salsc_decode_step(dec.desc, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"],
                                        outs[l], idxs[l], dec.ws)
            else:
                salsc.salsc_decode_step_timed(dec.desc, x["q"], x["Kc"], x["Vc"], x["Pk"],
                                              x["Pv"], outs[l], idxs[l], dec.ws, timed_events[l])

    # eager warm-up (sets kernel attributes, first-touch), then capture
    with torch.cuda.stream(stream):
        step()
    stream.synchronize()
    assert dec.flags() == 0, "device-side anomaly flag set"
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream, capture_error_mode="thread_local"):
        step()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            graph.replay()
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            t0.record(stream)
            for _ in range(steps):
                graph.replay()
            t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), dev)
    res = {"ms_per_step": ms / steps, "us_layer": ms / steps * 1e3 / L,
           "clocks": clocks.summary()}
    del graph

    # per-kernel times: the same work with event marks between the kernels (the
    # marks end the programmatic-launch overlap, so each time includes its
    # kernel's own launch latency)
    nk = len(salsc.DECODE_KERNELS)
    if kernel_reps:
        kev = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(L)]
        with torch.cuda.stream(stream):
            for evs in kev:
                for e in evs:
                    e.record(stream)
        graph_t = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_t, stream=stream, capture_error_mode="thread_local"):
            step(kev)
        per_kernel = np.zeros(nk)
        for _ in range(kernel_reps):
            with torch.cuda.stream(stream):
                graph_t.replay()
            torch.cuda.synchronize(dev)
            for evs in kev:
                for i in range(nk):
                    per_kernel[i] += evs[i].elapsed_time(evs[i + 1])
        res["per_kernel_us"] = per_kernel * 1e3 / (kernel_reps * L)
        del graph_t

    if timeline:
        res["timeline"] = step_timeline(salsc, dec, layers, outs, idxs, stream, dev)

    assert dec.flags() == 0, "device-side anomaly flag set"
    idx_host = [i.cpu().numpy() for i in idxs]
    res["bytes_layer"] = float(np.mean(algorithmic_bytes(w, idx_host, elem)))
    res["kbytes"] = kernel_bytes(w, idx_host, elem)
    res["launches"] = salsc.salsc_decode_launch_count(dec.desc)

    if e2e:
        # end to end through the public API with host buffers
        q_host = q_all.cpu().pin_memory()
        out_host = torch.empty(out_all.shape, dtype=out_all.dtype).pin_memory()
        e2e_steps = max(3, min(steps, 50))
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(e2e_steps):
                q_all.copy_(q_host, non_blocking=True)  # all layers' queries of this step
                step()
                out_host.copy_(out_all, non_blocking=True)
                stream.synchronize()  # the host reads the step's result
            e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        res["e2e"] = {"value": e_ms * 1e3 / (e2e_steps * L), "unit": UNIT,
                      "h2d_bytes_per_step": q_host.numel() * q_host.element_size(),
                      "d2h_bytes_per_step": out_host.numel() * out_host.element_size(),
                      "steps": e2e_steps,
                      "how": "eager salsc_decode_step per layer; every step copies all layers' "
                             "q in from pinned host memory (one copy) and all outputs back (one "
                             "copy); the host waits for each step"}
    del layers, q_all, out_all, outs, idxs, dec
    torch.cuda.empty_cache()
    return res


def step_roofline(res, peak):
    gbs = res["bytes_layer"] / (res["us_layer"] * 1e-6) / 1e9
    return {"bound": "hbm", "algorithmic_bytes_per_layer_step": res["bytes_layer"],
            "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
            "frac_of_8tbs": gbs / 8000.0}


def main():
    args = parse_args()
    w = workloads.BY_NAME[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
        return

    from latent_space_sparse_b200 import salsc
    if args.compress_only:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        print(json.dumps(bench_compress(salsc, torch.device("cuda"), rows=args.compress_rows)),
              flush=True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    L = args.layers
    peak, peak_kind = measured_peaks()
    # ---- headline: K graph replays of the default workload
    reps = max(3, min(20, args.steps // 10))
    res = time_decode(salsc, w, L, args.steps, args.warmup, dev, local, dist, kernel_reps=reps,
                      e2e=True, timeline=True)
    per_kernel_us = res["per_kernel_us"]
    kbytes = res["kbytes"]
    dominant = int(np.argmax(per_kernel_us))
    name = salsc.DECODE_KERNELS[dominant]
    ach = kbytes[name] / (per_kernel_us[dominant] * 1e-6) / 1e9
    roofline = {"kernel": name, "bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                "frac": ach / peak, "traffic": PROFILED_TRAFFIC.get((w.name, name)),
                "traffic_how": TRAFFIC_HOW if (w.name, name) in PROFILED_TRAFFIC else None,
                "peak_kind": peak_kind, "algorithmic_bytes_per_launch": kbytes[name],
                "time": "per_kernel_us (event-separated: includes the kernel's launch latency)"}

    line = {
        "metric": METRIC, "value": res["us_layer"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic", "config": config_of(args, w),
        "clocks": res["clocks"],
        "gpu_launches": res["launches"] * L * args.steps,
        "roofline": roofline,
        "step_roofline": step_roofline(res, peak),
        "per_kernel_us": {n: float(v) for n, v in zip(salsc.DECODE_KERNELS, per_kernel_us)},
        "per_kernel_gbs": {n: (kbytes[n] / (v * 1e-6) / 1e9 if kbytes[n] else 0.0)
                           for n, v in zip(salsc.DECODE_KERNELS, per_kernel_us)},
        "e2e": res["e2e"],
        "timeline": res["timeline"],
    }
    # ---- the other decode workloads (the metric's 4K points, long context)
    if not args.no_side_workloads:
        side = {}
        for name_w in SIDE_WORKLOADS:
            if name_w == w.name:
                continue
            ws = workloads.BY_NAME[name_w]
            r2 = time_decode(salsc, ws, L, args.side_steps, args.warmup, dev, local, dist,
                             kernel_reps=3, timeline=True)
            side[name_w] = {
                "value": r2["us_layer"], "unit": UNIT, "steps": args.side_steps,
                "ms_per_step": r2["ms_per_step"], "clocks": r2["clocks"],
                "step_roofline": step_roofline(r2, peak),
                "per_kernel_us": {n: float(v)
                                  for n, v in zip(salsc.DECODE_KERNELS, r2["per_kernel_us"])},
                "gpu_launches": r2["launches"] * L * args.side_steps,
                "timeline": r2["timeline"],
                "config": config_of(args, ws)}
        line["workloads"] = side
    if not args.no_compress:
        line["compress"] = bench_compress(salsc, dev, rows=args.compress_rows)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        line["cpu_baseline"] = cpu_baseline(w, oracle.default_threads())
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
