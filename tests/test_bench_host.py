"""Host logic of ``bench.py``'s extra legs on the CPU: the backward leg run with a stand-in library
and stand-in CUDA events (every launch "takes" 1 ms), checking the call sequence and the arithmetic
of its JSON object. No kernel runs here; the GPU runs of the bench exercise the real library."""
import os
import sys
import types

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


class _Event:
    clock = 0.0

    def __init__(self, enable_timing=True):
        self.t = None

    def record(self, stream=None):
        _Event.clock += 1.0  # ms: a launch's start and end events are 1 ms apart
        self.t = _Event.clock

    def elapsed_time(self, other):
        return other.t - self.t


def test_backward_leg_reports_rate_and_roofline(monkeypatch):
    import bench

    calls = []
    fake = types.SimpleNamespace(
        attn_fwd=lambda *a, **kw: calls.append("fwd"),
        attn_bwd=lambda *a, **kw: calls.append("bwd"),
        device_status=lambda stream=None: 0,
    )
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **kw: None)
    args = types.SimpleNamespace(steps=2000, warmup=3)
    ranks = bench.Ranks(1, torch.device("cpu"))
    w = bench.PREFILL
    q = torch.zeros((1, 1, 1, 1), dtype=torch.bfloat16)  # shapes only matter to the real library
    flushes = []
    out = bench.backward_leg(fake, args, ranks, torch.device("cpu"), None, lambda: flushes.append(1), q, q, q, q,
                             torch.zeros((1, 1, 1)), world=1)
    assert calls == ["fwd"] + ["bwd"] * (3 + 20)  # forward once, warm-up, then 20 timed launches
    assert len(flushes) == 3 + 20  # L2 flushed before every launch
    assert out["steps"] == 20 and out["device_status"] == 0
    flops = 5 * w.flops() // 2
    assert out["flops_per_launch"] == flops
    # each timed launch spans 1 ms between its events in the stand-in clock
    assert abs(out["us_per_launch"] - 1000.0) < 1e-9
    assert abs(out["value"] - flops / 1e-3 / 1e12) < 1e-6
    assert abs(out["roofline"]["frac"] - out["roofline"]["achieved"] / out["roofline"]["peak"]) < 1e-12
    assert out["roofline"]["bound"] == "tensor"
    # traffic comes from the committed capture when its source hash matches the kernel's source
    assert out["roofline"]["traffic"] == bench.read_traffic("bwd_kernel", w.name)


def test_whole_job_rate_scales_with_ranks_for_the_backward_leg(monkeypatch):
    import bench

    fake = types.SimpleNamespace(attn_fwd=lambda *a, **kw: None, attn_bwd=lambda *a, **kw: None,
                                 device_status=lambda stream=None: 0)
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **kw: None)
    ranks = bench.Ranks(1, torch.device("cpu"))
    q = torch.zeros((1, 1, 1, 1), dtype=torch.bfloat16)
    args = types.SimpleNamespace(steps=5, warmup=3)
    one = bench.backward_leg(fake, args, ranks, torch.device("cpu"), None, lambda: None, q, q, q, q,
                             torch.zeros((1, 1, 1)), world=1)
    two = bench.backward_leg(fake, args, ranks, torch.device("cpu"), None, lambda: None, q, q, q, q,
                             torch.zeros((1, 1, 1)), world=2)
    assert one["steps"] == 5 and abs(two["value"] - 2 * one["value"]) < 1e-9


def test_config_entry_reports_rate_roofline_and_baseline():
    import bench
    from causal_attention_attn_b200 import inputs

    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    w = inputs.CHUNKED_PREFILL
    base = {"value": 0.05, "unit": "TFLOP/s", "cores": 4, "kind": "oracle", "sample": "all"}
    e = bench.config_entry(w, 1e-3, 2, peaks, "measured", base)
    assert abs(e["value"] - 2 * w.flops() / 1e-3 / 1e12) < 1e-9  # two ranks, 1 ms each
    assert abs(e["roofline"]["achieved"] - w.flops() / 1e-3 / 1e12) < 1e-9
    assert abs(e["roofline"]["frac"] - e["roofline"]["achieved"] / 1000.0) < 1e-12
    assert e["roofline"]["bound"] == "tensor" and e["us_per_launch"] == 1000.0
    assert abs(e["vs_oracle"] - e["value"] / 0.05) < 1e-9
    d = bench.config_entry(inputs.DECODE_GQA, 1e-3, 1, peaks, "measured")
    assert d["roofline"]["bound"] == "hbm" and d["unit"] == "GB/s"
    assert abs(d["roofline"]["frac"] - inputs.DECODE_GQA.io_bytes() / 1e-3 / 1e9 / 5000.0) < 1e-12


def test_clock_summary_separates_samples_under_load():
    import bench

    lines = ["0, 1965, 1965, 120.5, 0x0, Not Active, Not Active, Not Active, Not Active",
             "0, 1700, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active",
             "0, 1650, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active",
             "0, 1600, 1965, 980.0, 0x4, Not Active, Not Active, Not Active, Active"]
    s = bench.summarise_clock_lines(lines, 300.0)
    assert s["samples"] == 4 and s["samples_under_load"] == 3
    assert s["sm_mhz_under_load"] == 1650.0 and s["sm_mhz"] == 1675.0
    assert s["reasons"] == ["sw_power_cap"] and s["sm_max_mhz"] == 1965.0
