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


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("name", ["gdn_qwen", "kda", "rwkv6", "gdn2"])
def test_slot_admission_matches_oracle(name, fused):
    # Sequences 1 and 4 get new dense states mid-stream (different fill
    # phases), sequence 2 a zero state later; the others run on untouched.
    import types
    import oracle
    from tests.parity import OUT_TOL, STATE_TOL, host_to_device, step_bonus
    w = wl.WORKLOADS[name].replace(B=6, H=3, L=5, T=20, ragged=True)
    BH, dk, dv = w.heads, w.d_k, w.d_v
    cfg = dlb.Config(w.variant, w.B, w.H, dk, dv, w.L, w.in_dtype, fused_merge=fused)
    st = dlb.DeltaLogState(cfg)
    S0 = wl.initial_state(w)
    st.reset(torch.from_numpy(S0).cuda().reshape(-1), wl.fill_offsets(w).tolist())
    bonus = wl.rwkv6_bonus(w) if w.variant == "rwkv6" else None
    bonus_d = None if bonus is None else torch.from_numpy(bonus).cuda().reshape(-1)
    rec = w.variant == "rwkv6"
    S_or = S0.reshape(BH, dv, dk).astype(np.float64)
    if rec:
        S_or = S_or.transpose(0, 2, 1).copy()
    rng = np.random.default_rng(5)
    o = torch.empty(BH * dv, device="cuda")
    for t in range(w.T):
        if t in (7, 13):
            seqs = [1, 4] if t == 7 else [2]
            if t == 7:
                new = (rng.standard_normal((len(seqs), w.H, dv, dk)) * 0.05).astype(np.float32)
                st.load_seqs(seqs, torch.from_numpy(new).cuda().reshape(-1))
            else:
                new = np.zeros((len(seqs), w.H, dv, dk), np.float32)
                st.load_seqs(seqs)
            for i, b in enumerate(seqs):
                blk = new[i].astype(np.float64)
                S_or[b * w.H:(b + 1) * w.H] = blk.transpose(0, 2, 1) if rec else blk
            assert all(st.fill()[b] == 0 for b in seqs)
        s = wl.step_inputs(w, t)
        q, k, v = (host_to_device(s.device_array(n), "cuda").reshape(-1) for n in ("q", "k", "v"))
        dec = host_to_device(s.decay, "cuda").reshape(-1)
        beta = None if s.beta is None else host_to_device(s.beta, "cuda").reshape(-1)
        st.step(q, k, v, dec, beta, step_bonus(s, "cuda", bonus_d), o)
        if not fused:
            st.merge(dlb.DL_MERGE_FULL)
        flat = lambda x: None if x is None else x.reshape((BH,) + x.shape[2:])
        step = types.SimpleNamespace(q=flat(s.q)[:, None], k=flat(s.k)[:, None], v=flat(s.v)[:, None],
                                     decay=flat(s.decay)[:, None],
                                     beta=None if s.beta is None else flat(s.beta)[:, None],
                                     wgate=None if s.wgate is None else flat(s.wgate)[:, None])
        res = oracle.run_eager(w.variant, S_or, [step],
                               bonus=None if bonus is None else bonus[np.arange(BH) % w.H])
        S_or = res.S
        o_ref = res.outputs[0]
        o_gpu = o.view(BH, dv).cpu().numpy().astype(np.float64)
        assert np.max(np.abs(o_gpu - o_ref)) <= OUT_TOL * np.max(np.abs(o_ref))
    S_gpu = st.materialize().view(BH, dv, dk).cpu().numpy().astype(np.float64)
    S_ref = S_or.transpose(0, 2, 1) if rec else S_or
    assert np.max(np.abs(S_gpu - S_ref)) <= STATE_TOL * np.max(np.abs(S_ref))
    assert st.device_error() == (0, 0)
    st.close()


def test_bounded_wait_gives_up_and_reports():
    # A wait nothing completes: the kernel records a timeout (code 1) after
    # about a second and returns; the context stays usable afterwards.
    import time
    t0 = time.time()
    assert dlb.dl_selftest_wait_timeout() == 1
    assert time.time() - t0 < 30
    cfg, st = _make(L=4)
    st.reset(None, None)
    assert st.device_error() == (0, 0)
    o = torch.empty(cfg.heads * 128, device="cuda")
    w = wl.WORKLOADS["gdn_qwen"].replace(B=3, H=2, L=4)
    s = step_to_device(wl.step_inputs(w, 0), "cuda")
    st.step(*s[:4], s[4], None, o)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all()
    st.close()
