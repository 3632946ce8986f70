"""The benchmark's algorithmic byte model (CPU only)."""

import numpy as np
import pytest

import bench
from linear_attention_recurrent_deltalog_b200 import deltalog as dlb


def test_step_bytes_uniform_phases_gdn_L16():
    # per head-step: read 65,536 (S_b) + 776 (q,k,v bf16, alpha, beta) + 4 (fill)
    # + 772 f (log entries: u fp32, k bf16, g); write 512 (o) + 4 (fill) +
    # 772 (append) or, for the fused merge at f = L-1, 65,536 (merged S_b).
    cfg = dlb.Config("gdn", 16, 32, 128, 128, 16, "bf16", fused_merge=True)
    fills = np.arange(16)
    rd, wr = bench.step_bytes(cfg, fills, fused=True)
    per = (rd + wr) / (16 * 32)
    assert per == pytest.approx(65536 + 776 + 4 + 772 * 7.5 + 516 + (15 * 772 + 65536) / 16)
    assert per == pytest.approx(77441.75)
    # unfused: no base write in the step
    rd2, wr2 = bench.step_bytes(cfg, fills, fused=False)
    assert rd2 == rd and wr2 == 16 * 32 * (516 + 772)


def test_step_bytes_int8_base():
    # the int8 base reads 16,384 codes + 512 B of row scales per head instead
    # of 65,536 B, and the fused merge writes the same 16,896 B
    cfg = dlb.Config("gdn", 16, 32, 128, 128, 16, "bf16", fused_merge=True, base="q8")
    fills = np.arange(16)
    rd, wr = bench.step_bytes(cfg, fills, fused=True)
    per = (rd + wr) / (16 * 32)
    assert per == pytest.approx(16896 + 776 + 4 + 772 * 7.5 + 516 + (15 * 772 + 16896) / 16)
    mr, mw = bench.merge_bytes(cfg, np.array([16, 3]))
    assert mr == 2 * 32 * 4 + 32 * (16896 + 16 * 772) and mw == 32 * (16896 + 4)


def test_eager_and_merge_bytes():
    cfg = dlb.Config("gdn", 2, 32, 128, 128, 16, "bf16")
    rd, wr = bench.eager_bytes(cfg)
    assert rd == 64 * (65536 + 776) and wr == 64 * (65536 + 512)
    # separate merge: every fill read; full heads read S_b + L entries, write S_b + fill
    mr, mw = bench.merge_bytes(cfg, np.array([16, 3]))
    assert mr == 2 * 32 * 4 + 32 * (65536 + 16 * 772)
    assert mw == 32 * (65536 + 4)


def test_reference_arm_prints_the_contract_line():
    # The reference arm (the fp64 oracle on the host cores) runs without a GPU.
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "3"], capture_output=True, text=True,
                         timeout=600, check=True).stdout.strip().splitlines()
    line = json.loads(out[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["steps"] == 2 and line["warmup"] == 3 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["nproc"] >= 1 and "cpu_model" in line["cpu_baseline"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["metric"] == bench.METRIC and line["unit"] == "tokens/s"


def test_single_core_oracle_sample():
    # the single-core figure of the CPU baseline: the oracle with one thread
    w = bench.wl.WORKLOADS["gdn_tiny"]
    r = bench.oracle_single_core(w, target_s=0.05)
    assert r["cores"] == 1 and r["value"] > 0 and "sequences" in r["sample"]


def test_traffic_records_match_the_sources():
    # the committed full-size ncu records of the headline step and of the
    # eager step are keyed by the hash of the sources they describe; the
    # bench line reports them (roofline.traffic, the measured write
    # reduction) only while that hash matches
    import types
    step = bench.traffic_record("dl_step_kernel", workload="gdn_serving", B=512, L=16,
                                merge="fused", base="f32")
    eager = bench.traffic_record("dl_eager_kernel", workload="gdn_serving", B=512)
    assert step is not None and eager is not None
    assert step["kernel_hash"] == bench.kernel_hash("dl_step_kernel")
    assert len(step["launches"]) >= 3
    assert step["bytes_per_launch"] == int(sum(x["dram_read"] + x["dram_write"]
                                               for x in step["launches"]) / len(step["launches"]))
    w = types.SimpleNamespace(name="gdn_serving", B=512)
    args = types.SimpleNamespace(steps=1, merge="fused")
    line = bench.write_bytes_line(w, args, dl_write_total=170_000 * 512,
                                  eager_write=2_113_536 * 512, step_rec=step)
    m = line["measured"]
    assert m is not None and m["measured_reduction"] > 10.0
    # another workload has no record
    assert bench.traffic_record("dl_step_kernel", workload="gdn_serving", B=64) is None


def test_traffic_record_of_changed_sources_is_not_reported(monkeypatch):
    monkeypatch.setattr(bench, "kernel_hash", lambda kernel="dl_step_kernel": "0" * 16)
    assert bench.traffic_record("dl_step_kernel", workload="gdn_serving", B=512, L=16,
                                merge="fused", base="f32") is None


def test_stream_hold_without_the_spin_helper(monkeypatch):
    # the hold before a timed region is skipped, not fatal, without torch's helper
    import torch
    monkeypatch.delattr(torch.cuda, "_sleep", raising=False)
    bench.hold_stream()
