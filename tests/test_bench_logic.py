"""The measurement code of bench.py that runs on the host: work counts, the traffic record and
the reference arm's sampling.  CPU only."""
from __future__ import annotations

import argparse
import json
import os
import shutil

import numpy as np
import pytest

import bench
import oracle as O
from muon_newton_schulz_07_b200 import inputs as I


@pytest.mark.parametrize("name", ["single256", "gpt2s", "d24", "l38b"])
def test_flop_counts_match_the_oracle_definition(name):
    wl = I.WORKLOADS[name]
    fl = bench.flops_by_kind(wl.shapes, 5)
    assert sum(fl.values()) == sum(O.ns_flops(r, c, 5) for r, c in wl.shapes)
    m, n = 1536, 6144
    one = bench.flops_by_kind([(m, n)], 1)
    assert one == {"gram": m * m * n, "poly": m ** 3, "update": 2 * m * m * n}


def test_byte_counts_per_element():
    shapes = [(3, 5), (7, 2)]
    n = 3 * 5 + 7 * 2
    # bf16 storage: G, M in, M1 out, bf16 X0 out; W in, bf16 X_k in, W out
    assert bench.bytes_by_kind(shapes, 2) == {"momentum_norm": 8 * n, "write": 6 * n}
    # fp32 storage: the same tensors at 4 bytes, X stays bf16
    assert bench.bytes_by_kind(shapes, 4) == {"momentum_norm": 14 * n, "write": 10 * n}


def test_traffic_record_is_used_only_for_the_captured_source(tmp_path, monkeypatch):
    import hashlib

    # a record of a capture, and the kernel source it was taken from
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    src = root / "csrc" / "kernel.cu"
    src.parent.mkdir(parents=True)
    src.write_text("// the captured kernel\n")
    rec = {"kernel": "k", "source": "csrc/kernel.cu",
           "source_sha256_16": hashlib.sha256(src.read_bytes()).hexdigest()[:16],
           "dram_bytes_read": 600.0, "dram_bytes_write": 400.0, "scale_to_workload": {"d24": 3.0}}
    (root / "profiles" / "traffic_update_d24.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.measured_traffic("update", "d24") == 3000.0
    assert bench.measured_traffic("update", "gpt2s") is None  # no capture for that workload
    assert bench.measured_traffic("gram", "d24") is None      # no record for that kernel
    # a changed kernel source invalidates the record
    src.write_text("// a different kernel\n")
    assert bench.measured_traffic("update", "d24") is None


def test_reference_arm_times_every_shape_even_on_short_runs(monkeypatch, capsys):
    calls = []

    def fake_step(W, G, M, hp):
        calls.append(W.shape)
        return W, M, W

    monkeypatch.setattr(O, "muon_step", fake_step)
    args = argparse.Namespace(workload="d24", steps=1, warmup=1, ns_steps=5, gpus=1, reference_budget_s=150.0)
    bench.run_reference(args, rank=0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    shapes = sorted(set(I.WORKLOADS["d24"].shapes))
    assert sorted(set(calls)) == shapes           # every distinct shape was stepped
    # the line reports the requested steps, and separately how many single-matrix timings it took
    assert line["steps"] == 1 and line["impl"] == "reference"
    assert line["timed"]["count"] >= len(shapes) and line["ms_per_step_is_estimate"] is True
    assert sorted(line["timed"]["per_shape_median_s"]) == sorted(f"{r}x{c}" for r, c in shapes)
    assert line["value"] > 0 and np.isfinite(line["value"])
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_is_silent_on_other_ranks(capsys):
    args = argparse.Namespace(workload="d24", steps=1, warmup=1, ns_steps=5, gpus=2, reference_budget_s=1.0)
    bench.run_reference(args, rank=1)
    assert capsys.readouterr().out == ""


def test_kernel_table_uses_the_burst_peak_for_the_headline():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    shapes = [(1536, 1536)] * 4
    k = 5
    fl = bench.flops_by_kind(shapes, k)
    # every Update launch takes 1 ms, the other kernels less
    prof = {"momentum_norm": (0.1 * 2, 2), "gram": (0.2 * 2 * k, 2 * k), "poly": (0.1 * 2 * k, 2 * k),
            "update": (1.0 * 2 * k, 2 * k), "write": (0.0, 0), "sgemm_ref": (0.0, 0), "ns_small": (0.0, 0)}
    kern, roof, ns, targets = bench.kernel_table(prof, shapes, k, 2, 2, peaks, "measured", "d24")
    upd = fl["update"] / k / 1e-3 / 1e12
    assert roof["kernel"].endswith("(update)") and abs(roof["achieved"] - upd) < 1e-9
    assert abs(roof["frac"] - upd / 1600.0) < 1e-12 and abs(roof["frac_sustained"] - upd / 1400.0) < 1e-12
    assert abs(kern["gram"]["frac_of_burst_peak"] - kern["gram"]["tflops"] / 1600.0) < 1e-12
    assert "write" not in kern
    assert set(targets) == {"ns_frac_of_burst_peak", "momentum_norm_frac_of_hbm"}
    assert targets["momentum_norm_frac_of_hbm"]["met"] == (kern["momentum_norm"]["frac_of_hbm"] >= 0.80)


def test_ns_schedule_is_read_from_the_traced_kernels():
    import bench
    assert bench.ns_schedule_taken({"momentum_norm": {}, "ns_fused": {}}).startswith("single launch")
    assert bench.ns_schedule_taken({"momentum_norm": {}, "ns_small": {}}).startswith("small-matrix")
    assert bench.ns_schedule_taken({"momentum_norm": {}, "gram": {}, "poly": {}, "update": {}}).startswith("staged")
