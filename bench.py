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
# An entry is removed whenever its kernel changes after the capture.
PROFILED_TRAFFIC: dict[tuple[str, str], float] = {
    ("mistral_7b_gqa32x8_d128_r256_n32768_b4_k2048_bf16", "attend"): 54.450432e6 + 1.064192e6,
}
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
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_bf16_peak():
    """Burst bf16 dense GEMM TFLOP/s (a kernel timed alone)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


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

    ms = timed(lambda: salsc.salsc_compress(K, V, Pk, Pv, Kc, Vc))
    ms_lib = timed(lambda: (torch.matmul(K, Pk, out=Kc), torch.matmul(V, Pv, out=Vc)))
    peak, kind = measured_bf16_peak()
    tf = flop / (ms * 1e-3) / 1e12
    return {"workload": f"{w.name} prefill: 2 x [{n} x {hid}] . [{hid} x {r}] bf16",
            "us": ms * 1e3, "achieved": tf, "peak": peak, "unit": "TFLOP/s", "bound": "tensor",
            "frac": tf / peak, "peak_kind": kind,
            "torch_matmul_us": ms_lib * 1e3,
            "torch_matmul_tflops": flop / (ms_lib * 1e-3) / 1e12}


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


def cpu_baseline(w, n_threads, min_seconds: float = 10.0):
    """The oracle on all units of sequence 0, repeated for at least
    `min_seconds`, scaled to one layer-step of the whole batch."""
    total_units = w.batch * w.n_kv_heads
    inputs, units = oracle_inputs(w, w.n_kv_heads)
    secs = []
    while sum(secs) < min_seconds:
        secs.append(oracle_time(inputs, n_threads))
    scale = total_units / units
    mean = statistics.mean(secs)
    return {"value": mean * scale * 1e6, "unit": UNIT, "cores": n_threads, "kind": "oracle",
            "sample": f"oracle.decode of sequence 0 ({units} of {total_units} selection units, "
                      f"n={w.seq_lens[0]}), {len(secs)} runs in {sum(secs):.1f} s, mean "
                      f"{mean:.3f} s scaled x{scale:g} to one layer-step"}


def run_reference(args, w):
    """The oracle timed on the host cores: one bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    n_threads = oracle.default_threads()
    inputs, units = oracle_inputs(w, max(1, min(w.n_kv_heads, n_threads)))
    for _ in range(args.warmup):
        oracle_time(inputs, n_threads)
    secs = [oracle_time(inputs, n_threads) for _ in range(args.steps)]
    scale = w.batch * w.n_kv_heads / units
    value = statistics.mean(secs) * scale * 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": value * args.layers / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(args, w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": n_threads, "kind": "oracle",
                         "sample": f"per step: oracle.decode of {units} of "
                                   f"{w.batch * w.n_kv_heads} units (sequence 0), scaled "
                                   f"x{scale:g}"},
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
    nk = len(salsc.DECODE_KERNELS)
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(L)]
    with torch.cuda.stream(stream):
        for evs in kev:
            for e in evs:
                e.record(stream)
    graph_t = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_t, stream=stream, capture_error_mode="thread_local"):
        step(kev)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # ---- headline: K graph replays
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            t0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), dev)
    ms_per_step = ms / args.steps
    us_layer = ms_per_step * 1e3 / L

    # ---- per-kernel times (same work, with event marks between kernels)
    reps = max(3, min(20, args.steps // 10))
    per_kernel = np.zeros(nk)
    for _ in range(reps):
        with torch.cuda.stream(stream):
            graph_t.replay()
        torch.cuda.synchronize(dev)
        for evs in kev:
            for i in range(nk):
                per_kernel[i] += evs[i].elapsed_time(evs[i + 1])
    per_kernel_us = per_kernel * 1e3 / (reps * L)
    dominant = int(np.argmax(per_kernel_us))

    # ---- bytes
    assert dec.flags() == 0, "device-side anomaly flag set"
    idx_host = [i.cpu().numpy() for i in idxs]
    step_bytes = algorithmic_bytes(w, idx_host, elem)
    bytes_layer = float(np.mean(step_bytes))
    peak, peak_kind = measured_peaks()
    launches = salsc.salsc_decode_launch_count(dec.desc)
    kbytes = kernel_bytes(w, idx_host, elem)
    name = salsc.DECODE_KERNELS[dominant]
    ach = kbytes[name] / (per_kernel_us[dominant] * 1e-6) / 1e9
    roofline = {"kernel": name, "bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                "frac": ach / peak, "traffic": PROFILED_TRAFFIC.get((w.name, name)),
                "peak_kind": peak_kind, "algorithmic_bytes_per_launch": kbytes[name]}
    step_gbs = bytes_layer / (us_layer * 1e-6) / 1e9

    # ---- end to end through the public API with host buffers
    q_host = q_all.cpu().pin_memory()
    out_host = torch.empty(out_all.shape, dtype=out_all.dtype).pin_memory()
    e2e_steps = max(3, min(args.steps, 50))
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
    e2e_us = e_ms * 1e3 / (e2e_steps * L)
    qbytes = q_host.numel() * q_host.element_size()
    obytes = out_host.numel() * out_host.element_size()

    line = {
        "metric": METRIC, "value": us_layer, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic", "config": config_of(args, w),
        "clocks": clocks.summary(),
        "gpu_launches": launches * L * args.steps,
        "roofline": roofline,
        "step_roofline": {"bound": "hbm", "algorithmic_bytes_per_layer_step": bytes_layer,
                          "achieved": step_gbs, "peak": peak, "unit": "GB/s",
                          "frac": step_gbs / peak, "frac_of_8tbs": step_gbs / 8000.0},
        "per_kernel_us": {n: float(v) for n, v in zip(salsc.DECODE_KERNELS, per_kernel_us)},
        "per_kernel_gbs": {n: (kbytes[n] / (v * 1e-6) / 1e9 if kbytes[n] else 0.0)
                           for n, v in zip(salsc.DECODE_KERNELS, per_kernel_us)},
        "e2e": {"value": e2e_us, "unit": UNIT, "h2d_bytes_per_step": qbytes,
                "d2h_bytes_per_step": obytes, "steps": e2e_steps,
                "how": "eager salsc_decode_step per layer; every step copies all layers' q in "
                       "from pinned host memory (one copy) and all outputs back (one copy); "
                       "the host waits for each step"},
    }
    if not args.no_compress:
        line["compress"] = bench_compress(salsc, dev, rows=args.compress_rows)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        line["cpu_baseline"] = cpu_baseline(w, oracle.default_threads())
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph, graph_t
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
