"""bench.py's JSON line, assembled on the CPU with a stand-in for the device.

The kernels, streams and CUDA events are replaced by no-op doubles, so this
checks only the host-side plumbing of the bench: which keys the line carries,
the L2 policy per workload and the e2e byte counts.  It measures nothing and
says nothing about parity (the GPU tests do that).
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import pytest
import torch

import bench


class _Event:
    clock = 0.0

    def __init__(self, enable_timing=True):
        self.t = None

    def record(self, stream=None):
        _Event.clock += 0.1
        self.t = _Event.clock

    def elapsed_time(self, other):
        return other.t - self.t


class _Step:
    """The attributes bench.run_ours reads from GpuStep, on the CPU; append and attend do nothing."""

    def __init__(self, w, device, fused=True, cascade=True, fp8=False, plan=True):
        def t(a, dtype):
            return torch.from_numpy(np.ascontiguousarray(a).astype(dtype))
        self.w = w
        self.q, self.k_new, self.v_new = (t(x.view(np.int16), np.int16) for x in (w.q, w.k_new, w.v_new))
        self.block_tables, self.context_lens = t(w.block_tables, np.int32), t(w.context_lens, np.int32)
        self.query_start, self.slot_mapping = t(w.query_start, np.int32), t(w.slot_mapping, np.int32)
        self.out = torch.empty_like(self.q)
        self.status = torch.zeros(1, dtype=torch.int32)
        self.decode = w.is_decode
        self.fused = self.decode and fused
        self.fp8 = fp8
        self.cascade = False
        self.plan = None
        self.launches = 1 if self.fused else bench.step_launches(w)
        self.inputs = ["q", "k_new", "v_new", "block_tables", "context_lens"]
        if not self.fused:
            self.inputs.append("slot_mapping")
        if not self.decode:
            self.inputs.append("query_start")

    def append(self):
        pass

    def attend(self):
        pass


class _Stream:
    def wait_event(self, ev):
        pass


@pytest.fixture
def fake_device(monkeypatch):
    import contextlib
    monkeypatch.setattr(bench, "dist_setup", lambda n: (0, 1, 0))
    monkeypatch.setattr(bench, "GpuStep", _Step)
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: _Stream())
    monkeypatch.setattr(torch.cuda, "Stream", lambda *a, **k: _Stream())
    monkeypatch.setattr(torch.cuda, "stream", lambda s: contextlib.nullcontext())
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(bench, "FLUSH_BYTES", 1 << 20)


def _line(capsys, workload, **kw):
    args = argparse.Namespace(gpus=1, steps=4, warmup=3, workload=workload, impl="ours", cpu_seconds=0.2,
                              reference_seconds=1.0, no_cpu_baseline=True, kv_dtype="bf16", graph=False,
                              cascade=False, separate_append=False, no_plan=False, no_sub_records=True, no_calibrate=True,
                              sub_cpu_seconds=0.1)
    for k, v in kw.items():
        setattr(args, k, v)
    bench.run_ours(args, (6530.3, 1626.0, 1399.0, "measured"))
    out = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(out) == 1
    return json.loads(out[0])


def test_headline_line_carries_every_key(fake_device, capsys):
    d = _line(capsys, 3)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 4 and d["warmup"] == 3 and d["scaling"] == "weak"
    assert d["config"]["workload"] == "llama3.3-70b-layer-decode-b128"
    assert d["config"]["l2"].startswith("no flush") and "l2_warm" not in d
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6530.3
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-3)
    assert 0 < r["intensity_flop_per_byte"] < r["ridge_flop_per_byte"]
    # e2e copies q, k_new, v_new, the tables and the lengths in, and out back
    assert d["e2e"]["h2d_bytes_per_step"] == 2 * 1024 * 1024 + 2 * 128 * 8 * 128 * 2 + 128 * 512 * 4 + 128 * 4
    assert d["e2e"]["d2h_bytes_per_step"] == 2 * 1024 * 1024
    assert d["gpu_launches"] == 4 and d["cpu_baseline"] is None


def test_small_workload_runs_with_l2_flushed_and_times_the_oracle(fake_device, capsys):
    d = _line(capsys, 1, no_cpu_baseline=False)
    assert d["config"]["l2"].startswith("flushed")
    assert d["l2_warm"]["unit"] == "GB/s" and d["l2_warm"]["ms_per_step"] > 0
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["unit"] == "GB/s" and cpu["value"] > 0 and cpu["cores"] >= 1


def test_default_run_carries_the_other_workloads_as_sub_records(fake_device, capsys):
    d = _line(capsys, 3, no_sub_records=False)
    subs = d["workloads"]
    assert set(subs) == {"grpo-shared-prefix", "grpo-shared-prefix-cascade", "grpo-long-prefix",
                         "grpo-long-prefix-cascade", "mixed-chunk-decode", "llama3.3-70b-layer-decode-b128-fp8"}
    for key, sub in subs.items():
        for k in ("value", "unit", "ms_per_step", "dtype", "config", "roofline", "e2e", "gpu_launches", "clocks"):
            assert k in sub, (key, k)
        assert sub["roofline"]["frac"] == pytest.approx(sub["roofline"]["achieved"] / sub["roofline"]["peak"],
                                                        rel=1e-3)
    assert subs["grpo-shared-prefix"]["config"]["l2"].startswith("flushed")
    assert subs["mixed-chunk-decode"]["roofline_tensor"]["unit"] == "TFLOP/s"
    assert "overlap_bound" in subs["mixed-chunk-decode"]
    assert subs["llama3.3-70b-layer-decode-b128-fp8"]["dtype"].startswith("fp8")
