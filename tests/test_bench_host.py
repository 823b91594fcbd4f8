"""Host logic of bench.py on CPU: the algorithmic byte counts behind the
roofline fields, the clock sampler's decoding of clock-event reasons (against
a fake NVML: nothing here reads or sets a real GPU), and the max-over-ranks
timing on gloo ranks."""
import os
import socket
import sys
import time
import types

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from latent_space_sparse_b200 import workloads as W

SMALL = W.Workload(name="bytes_small", batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64, rank=64,
                   top_k=4, seq_lens=(10, 7), dtype="bf16", rope_base=10000.0, low_rank=8, seed=1)


def test_distinct_rows_union_over_units_without_pads():
    idx = np.array([[[0, 3, 5, -1], [3, 9, 0, 1]],     # sequence 0: {0, 1, 3, 5, 9}
                    [[6, 6, -1, -1], [2, -1, -1, -1]]],  # sequence 1: {2, 6}
                   dtype=np.int32)
    assert bench.distinct_rows(SMALL, idx) == 7


def test_algorithmic_and_kernel_bytes():
    idx = np.array([[[0, 3, 5, -1], [3, 9, 0, 1]], [[6, 6, -1, -1], [2, -1, -1, -1]]],
                   dtype=np.int32)
    e, r, N, hid = 2, 64, 17, 128
    qo = 2 * 4 * 64 * e
    assert bench.algorithmic_bytes(SMALL, [idx], e) == [N * r * e + 7 * r * e + 2 * hid * r * e
                                                        + 2 * qo]
    kb = bench.kernel_bytes(SMALL, [idx, idx], e)
    split = 2 * 16 * r * 2  # B x npad (2U rounded up to 16) x r bf16
    assert kb["latent_q"] == qo + hid * r * e + 2 * 2 * r * 4 + split
    assert kb["score"] == N * r * e + split + N * 2 * 4
    assert kb["topk"] == N * 2 * 4 + 2 * 2 * 4 * 4
    assert kb["attend"] == 2 * 7 * r * e + hid * r * e + qo + 2 * 2 * 4 * 4
    assert kb["combine"] == hid * r * e + qo


class FakeNvml(types.ModuleType):
    """Read-only NVML stand-in: a fixed handle, a clock trace and reason bits."""
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, bits, fail_init=False):
        super().__init__("pynvml")
        self.clocks, self.bits, self.fail_init, self.i = list(clocks), bits, fail_init, 0

    def nvmlInit(self):
        if self.fail_init:
            raise RuntimeError("NVML library not found")

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        assert bus == b"00000000:1b:00.0"
        return "handle"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        v = self.clocks[self.i % len(self.clocks)]
        self.i += 1
        return v

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.bits


@pytest.fixture
def fake_gpu(monkeypatch):
    props = types.SimpleNamespace(pci_domain_id=0, pci_bus_id=0x1b, pci_device_id=0)
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: props)

    def install(**kw):
        monkeypatch.setitem(sys.modules, "pynvml", FakeNvml(**kw))
    return install


def test_clock_sampler_reasons_and_median(fake_gpu):
    # gpu_idle | sw_power_cap | hw_slowdown: the idle bit is not reported
    fake_gpu(clocks=[1965, 1900, 1965], bits=0x1 | 0x4 | 0x8)
    with bench.ClockSampler(0, period_s=0.001) as c:
        time.sleep(0.05)
    s = c.summary()
    assert s["sm_max_mhz"] == 1965
    assert s["sm_mhz"] in (1900, 1965)
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert s["samples"] >= 3


def test_clock_sampler_without_nvml_reports_no_clocks(fake_gpu):
    fake_gpu(clocks=[1965], bits=0, fail_init=True)
    with bench.ClockSampler(0) as c:
        pass
    s = c.summary()
    assert s["sm_mhz"] is None and s["sm_max_mhz"] is None and s["reasons"] == []
    assert "NVML" in s["error"]


def _rank_main(rank, world, port, path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(1.25 + rank, "cpu")  # each rank's own time
        with open(f"{path}.{rank}", "w") as f:
            f.write(repr(got))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_max_over_ranks_gloo(tmp_path):
    world = 2
    path = str(tmp_path / "t")
    mp.start_processes(_rank_main, args=(world, _free_port(), path), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        assert float(open(f"{path}.{r}").read()) == 2.25  # every rank gets the slowest time
    assert bench.max_over_ranks(0.5, "cpu") == 0.5  # no process group: the value itself


def test_timeline_summary_on_hand_made_stamps():
    # two layers, stages (a, b, c); stage c records nothing (a merge that launches nothing)
    stages = ("a", "b", "c")
    tr = np.zeros((2, 3, 4, 3), dtype=np.int64)

    def layer(l, t0):
        # stage a: CTAs 0-1 start t0, wait returns t0+1000, end t0+3000 / t0+3500
        tr[l, 0, 0] = (t0, t0 + 1000, t0 + 3000)
        tr[l, 0, 1] = (t0, t0 + 1100, t0 + 3500)
        # stage b: wait returns 500 ns after a's last end, ends 4000 ns after that end
        tr[l, 1, 0] = (t0 + 500, t0 + 4000, t0 + 7500)
        tr[l, 1, 2] = (t0 + 600, t0 + 4100, t0 + 6000)
        return t0 + 7500

    end0 = layer(0, 10_000)
    layer(1, end0 + 200)  # layer 1's first stage waits 200 ns + 1000 ns after layer 0's end
    s = bench.timeline_summary(tr, stages)
    assert s["critical_us"] == pytest.approx({"a": 3.7, "b": 4.0})
    assert s["wait_us"] == pytest.approx({"a": 1.2, "b": 0.5})
    assert s["span_us"] == pytest.approx({"a": 2.5, "b": 3.5})
    assert s["layer_step_us"] == pytest.approx(7.7)


def test_peak_lookup_burst_sustained_and_fallback(tmp_path, monkeypatch):
    """The roofline denominators: the measured file's burst and sustained bf16
    figures and its copy bandwidth; the stated fallback figures when the file,
    or one key of it, is absent."""
    import json
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (6650.0, "fallback")
    assert bench.measured_bf16_peak() == (1590.0, "fallback")
    assert bench.measured_bf16_peak(sustained=True) == (1400.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6500.5,
                                                              "bf16_tflops": 1650.0}))
    assert bench.measured_peaks() == (6500.5, "measured")
    assert bench.measured_bf16_peak() == (1650.0, "measured")
    assert bench.measured_bf16_peak(sustained=True) == (1400.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6500.5,
                                                              "bf16_tflops": 1650.0,
                                                              "bf16_tflops_sustained": 1390.0}))
    assert bench.measured_bf16_peak(sustained=True) == (1390.0, "measured")
