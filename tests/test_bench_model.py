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


def test_eager_and_merge_bytes():
    cfg = dlb.Config("gdn", 2, 32, 128, 128, 16, "bf16")
    rd, wr = bench.eager_bytes(cfg)
    assert rd == 64 * (65536 + 776) and wr == 64 * (65536 + 512)
    # separate merge: every fill read; full heads read S_b + L entries, write S_b + fill
    mr, mw = bench.merge_bytes(cfg, np.array([16, 3]))
    assert mr == 2 * 32 * 4 + 32 * (65536 + 16 * 772)
    assert mw == 32 * (65536 + 4)
