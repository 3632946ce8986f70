"""GPU behaviour of the C ABI beyond numerics: the log-full contract, fill
bookkeeping, materialize leaving the state unchanged, reset, launch counts
and the device error word."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from linear_attention_recurrent_deltalog_b200 import deltalog as dlb
from linear_attention_recurrent_deltalog_b200 import workloads as wl
from tests.parity import step_to_device

pytestmark = pytest.mark.gpu


def _make(L=4, fused=False, B=3, H=2, variant="gdn"):
    cfg = dlb.Config(variant, B, H, 128, 128, L, "bf16", fused_merge=fused)
    st = dlb.DeltaLogState(cfg)
    return cfg, st


def test_log_full_is_reported_and_changes_nothing():
    cfg, st = _make(L=3)
    w = wl.WORKLOADS["gdn_qwen"].replace(B=3, H=2, L=3)
    S0 = torch.from_numpy(wl.initial_state(w)).cuda().reshape(-1)
    st.reset(S0, [0, 1, 2])
    o = torch.empty(cfg.heads * 128, device="cuda")
    s = step_to_device(wl.step_inputs(w, 0), "cuda")
    st.step(*s[:4], s[4], None, o)
    assert st.fill() == [1, 2, 3]
    before = st.materialize().clone()
    with pytest.raises(dlb.DeltaLogError) as e:
        st.step(*s[:4], s[4], None, o)
    assert e.value.status == dlb.DL_ERR_LOG_FULL
    assert st.fill() == [1, 2, 3]
    torch.testing.assert_close(st.materialize(), before, rtol=0, atol=0)
    st.merge(dlb.DL_MERGE_FULL)
    assert st.fill() == [1, 2, 0]
    after = st.materialize()
    torch.testing.assert_close(after, before, rtol=2e-6, atol=1e-7)
    st.merge(dlb.DL_MERGE_ALL)
    assert st.fill() == [0, 0, 0]
    torch.testing.assert_close(st.materialize(), before, rtol=2e-6, atol=1e-7)
    assert st.device_error() == (0, 0)
    st.close()


def test_fused_merge_never_fills_and_launch_counts():
    cfg, st = _make(L=2, fused=True)
    w = wl.WORKLOADS["gdn_qwen"].replace(B=3, H=2, L=2)
    st.reset(None, [0, 1, 0])
    o = torch.empty(cfg.heads * 128, device="cuda")
    n0 = dlb.dl_launch_count()
    for t in range(5):
        s = step_to_device(wl.step_inputs(w, t), "cuda")
        st.step(*s[:4], s[4], None, o)
        st.merge(dlb.DL_MERGE_FULL)  # never needed: no launch
    assert dlb.dl_launch_count() - n0 == 5
    assert max(st.fill()) < 2
    st.close()


def test_materialize_is_read_only_and_zero_state_reset():
    cfg, st = _make(L=8)
    w = wl.WORKLOADS["gdn_qwen"].replace(B=3, H=2, L=8)
    st.reset(None, None)
    z = st.materialize()
    assert torch.count_nonzero(z) == 0
    o = torch.empty(cfg.heads * 128, device="cuda")
    for t in range(3):
        s = step_to_device(wl.step_inputs(w, t), "cuda")
        st.step(*s[:4], s[4], None, o)
    a = st.materialize().clone()
    b = st.materialize()
    torch.testing.assert_close(a, b, rtol=0, atol=0)
    assert st.fill() == [3, 3, 3]
    st.close()


def test_python_binding_refuses_small_buffers_before_launch():
    cfg, st = _make(L=4)
    small = torch.empty(10, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        st.step(small, small, small, torch.empty(6, device="cuda"), torch.empty(6, device="cuda"))
    st.close()
