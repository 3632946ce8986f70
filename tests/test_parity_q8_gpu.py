"""GPU parity of the int8 base (per-window quantization) against the oracle.

The windowed oracle (``oracle.window_quant``) fixes what the path computes:
the eager recurrence with each head's state requantized to int8 (one scale
per value row) at every window end.  Checks:

* quantizing a loaded state (reset, slot admission) is integer work from
  identical fp32 inputs: codes and scales bit-identical to the oracle's;
* at every window end each new code is a correct rounding of the oracle's
  pre-quantization value to within the state tolerance (the GPU folds the
  log in fp32, so x may differ from the oracle's fp64 value by that much);
* with the oracle's codes written back after each window end (so every
  window starts from the same int8 base), outputs and materialized states
  meet the fp32 bars: output rel err <= 1e-3, state rel err <= 1e-4;
* run freely (no write-back) the path's quantization error against the
  unquantized fp64 recurrence matches the windowed oracle's.
"""

from __future__ import annotations

import types

import numpy as np
import pytest
import torch

import oracle
from linear_attention_recurrent_deltalog_b200 import deltalog as dlb
from linear_attention_recurrent_deltalog_b200 import workloads as wl
from tests.parity import (OUT_TOL, STATE_TOL, heads_covering_phases, host_to_device, run_parity_q8,
                          step_to_device)

pytestmark = pytest.mark.gpu


def _check(r, windows=True):
    assert r.reset_exact, "Q(S0) differs from the oracle's codes/scales"
    assert r.out_err <= OUT_TOL, f"output rel err {r.out_err:.3e}"
    assert r.state_err <= STATE_TOL, f"state rel err {r.state_err:.3e}"
    if windows:
        assert r.windows > 0
        assert r.code_excess <= 0, f"a code is off its rounding by {r.code_excess:.3e}"
        assert r.scale_excess <= 0, f"a scale is off by {r.scale_excess:.3e}"
        assert r.mismatch_frac <= 1e-2, f"{r.mismatch_frac:.2e} of codes differ"


@pytest.mark.parametrize("fused", [True, False])
def test_q8_tiny_all_heads(fused):
    # B=1, H=2, d=64, fp32 inputs, L=8, T=32: every head, four windows
    r = run_parity_q8(wl.WORKLOADS["gdn_tiny"], fused=fused)
    _check(r)


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("name", ["gdn_qwen", "kda", "rwkv6", "gdn2"])
def test_q8_workloads(name, fused):
    w = wl.WORKLOADS[name].replace(ragged=True)
    heads = heads_covering_phases(w, 24)
    r = run_parity_q8(w, T=2 * w.L + 7, heads=heads, fused=fused, snap_every=w.L // 2)
    _check(r)


def test_q8_serving_full_batch():
    # the benchmarked launch: B=512 H=32 d=128 L=16, ragged fills, fused
    # merge, one 128-row work item per head; more than two windows per sequence
    w = wl.WORKLOADS["gdn_serving"]
    heads = heads_covering_phases(w, 24)
    r = run_parity_q8(w, T=40, heads=heads, fused=True, snap_every=10, workers=None)
    _check(r)


@pytest.mark.parametrize("split", [1, 2, 4])
@pytest.mark.parametrize("variant,dk,dv,dtype", [
    ("gdn", 64, 128, "bf16"), ("kda", 128, 64, "f32"), ("rwkv6", 64, 64, "f32"),
    ("gdn", 128, 128, "f32"), ("kda", 64, 64, "bf16"), ("rwkv6", 128, 128, "bf16"),
    ("gdn2", 64, 128, "bf16"), ("gdn2", 128, 128, "f32"),
])
def test_q8_shapes_dtypes_splits(variant, dk, dv, dtype, split):
    if dv // split < 64:
        pytest.skip("int8 work items hold at least 64 rows (32 per warp, two warps)")
    base = {"gdn": "gdn_qwen", "kda": "kda", "rwkv6": "rwkv6", "gdn2": "gdn2"}[variant]
    w = wl.WORKLOADS[base].replace(B=6, H=3, d_k=dk, d_v=dv, in_dtype=dtype, L=5, ragged=True,
                                   seed=31 + split)
    for fused in (True, False):
        r = run_parity_q8(w, T=13, fused=fused, split=split, snap_every=3)
        _check(r)


@pytest.mark.parametrize("dk", [64, 128])
def test_q8_large_batch_merge(dk):
    # more than 4096 sequences merging at once: the TMEM merge reads each
    # head's fill from the device instead of the launch's list (d_k = 64
    # runs its MMAs with N = 64 over 64 TMEM columns)
    w = wl.WORKLOADS["gdn_qwen"].replace(B=4200, H=1, d_k=dk, d_v=128, L=2, ragged=False, seed=47)
    _check(run_parity_q8(w, T=5, heads=wl.sample_heads(w, 24), fused=False, snap_every=2))
    w = wl.WORKLOADS["kda"].replace(B=4200, H=1, d_k=dk, d_v=128, L=3, ragged=False, seed=48)
    _check(run_parity_q8(w, T=7, heads=wl.sample_heads(w, 24), fused=False, merge_all_at=(4,),
                         snap_every=3))


def test_q8_long_vector_log():
    # L = 64 with a vector decay: the merge takes the per-warp fold (the
    # two-stage TMEM pipeline would not fit in shared memory)
    w = wl.WORKLOADS["kda"].replace(B=3, H=2, L=64, ragged=True, seed=49)
    _check(run_parity_q8(w, T=70, fused=False, snap_every=10))
    _check(run_parity_q8(w, T=70, fused=True, snap_every=10))


def test_q8_forced_merges():
    # merges of every non-empty log mid-window end those windows early
    w = wl.WORKLOADS["gdn_qwen"].replace(B=8, H=4, L=6, ragged=True, seed=41)
    r = run_parity_q8(w, T=20, fused=False, merge_all_at=(3, 4, 11), snap_every=2)
    _check(r)
    r = run_parity_q8(w, T=20, fused=True, merge_all_at=(5, 12), snap_every=2)
    _check(r)


@pytest.mark.parametrize("name", ["gdn_qwen", "kda"])
def test_q8_kla(name):
    w = wl.WORKLOADS[name].replace(B=8, H=4, L=6, ragged=True, kla_eps=1e-6, seed=43)
    r = run_parity_q8(w, T=16, fused=True, snap_every=4)
    _check(r)


def test_q8_reset_edge_rows():
    # zero rows, rows below 2^-120 (stored as zero), one huge entry, exact ties
    B, H, d = 2, 2, 64
    cfg = dlb.Config("gdn", B, H, d, d, 4, "f32", base="q8")
    rng = np.random.default_rng(3)
    S = (rng.standard_normal((B * H, d, d)) * 0.02).astype(np.float32)
    S[0, 0] = 0.0
    S[0, 1] = 1e-37
    S[1, 2, 5] = 1e30
    S[2, 3] = np.float32(127.0) * (np.arange(d) % 7 - 3) / 6.0
    S[3, 4] = np.linspace(-127.0, 127.0, d).astype(np.float32)
    S[3, 4, ::2] = np.round(S[3, 4, ::2]) + 0.5
    st = dlb.DeltaLogState(cfg)
    st.reset(torch.from_numpy(S).cuda().reshape(-1))
    codes, scales = oracle.quantize_rows(S)
    assert np.array_equal(st.base_codes().cpu().numpy(), codes)
    assert np.array_equal(st.base_scales().cpu().numpy(), scales)
    M = st.materialize().view(B * H, d, d).cpu().numpy().astype(np.float64)
    assert np.array_equal(M, oracle.dequantize_rows(codes, scales))
    st.reset(None)
    assert torch.count_nonzero(st.base_codes_raw()) == 0 and torch.count_nonzero(st.base_scales()) == 0
    st.close()


def test_q8_slot_admission_quantizes_exactly():
    w = wl.WORKLOADS["gdn_qwen"].replace(B=6, H=3, L=5, ragged=True, seed=45)
    BH, d = w.heads, w.d_k
    cfg = dlb.Config("gdn", w.B, w.H, d, d, w.L, w.in_dtype, fused_merge=True, base="q8")
    st = dlb.DeltaLogState(cfg)
    S0 = wl.initial_state(w)
    st.reset(torch.from_numpy(S0).cuda().reshape(-1), wl.fill_offsets(w).tolist())
    o = torch.empty(BH * d, device="cuda")
    for t in range(3):
        s = step_to_device(wl.step_inputs(w, t), "cuda")
        st.step(*s[:4], s[4], None, o)
    before = st.base_codes().clone()
    new = (np.random.default_rng(5).standard_normal((2, w.H, d, d)) * 0.05).astype(np.float32)
    st.load_seqs([1, 4], torch.from_numpy(new).cuda().reshape(-1))
    codes, scales = oracle.quantize_rows(new.reshape(2 * w.H, d, d))
    got = st.base_codes().view(w.B, w.H, d, d)
    assert np.array_equal(got[[1, 4]].cpu().numpy().reshape(2 * w.H, d, d), codes)
    assert np.array_equal(st.base_scales().view(w.B, w.H, d)[[1, 4]].cpu().numpy().reshape(2 * w.H, d),
                          scales)
    keep = [0, 2, 3, 5]
    assert torch.equal(got[keep], before.view(w.B, w.H, d, d)[keep])
    assert [st.fill()[b] for b in (1, 4)] == [0, 0]
    st.load_seqs([2])
    assert torch.count_nonzero(st.base_codes().view(w.B, w.H, d, d)[2]) == 0
    assert st.device_error() == (0, 0)
    st.close()


def test_q8_free_run_error_matches_oracle():
    # no write-back: the GPU and the oracle each run their own quantized
    # trajectory; against the unquantized fp64 recurrence both carry the same
    # quantization error
    w = wl.WORKLOADS["gdn_qwen"].replace(B=16, H=4, L=8, ragged=True, seed=47)
    T = 48
    BH, d = w.heads, w.d_k
    cfg = dlb.Config("gdn", w.B, w.H, d, d, w.L, w.in_dtype, fused_merge=True, base="q8")
    st = dlb.DeltaLogState(cfg)
    S0 = wl.initial_state(w)
    fill0 = wl.fill_offsets(w)
    st.reset(torch.from_numpy(S0).cuda().reshape(-1), fill0.tolist())
    o = torch.empty(BH * d, device="cuda")
    outs, steps = [], []
    for t in range(T):
        s = wl.step_inputs(w, t)
        q, k, v, dec, beta = step_to_device(s, "cuda")
        st.step(q, k, v, dec, beta, None, o)
        outs.append(o.view(BH, d).cpu().numpy().astype(np.float64))
        flat = lambda x: None if x is None else x.reshape((BH,) + x.shape[2:])[:, None]
        steps.append(types.SimpleNamespace(q=flat(s.q), k=flat(s.k), v=flat(s.v), decay=flat(s.decay),
                                           beta=flat(s.beta)))
    exact = oracle.run_eager("gdn", S0.reshape(BH, d, d).astype(np.float64), steps)
    windowed = oracle.run_windowed("gdn", S0.reshape(BH, d, d), steps, w.L, fill0, w.H)
    ref = np.stack(exact.outputs[8:])
    e_gpu = np.sqrt(np.mean((np.stack(outs[8:]) - ref) ** 2))
    e_orc = np.sqrt(np.mean((np.stack(windowed.outputs[8:]) - ref) ** 2))
    assert e_orc > 0
    assert 0.8 <= e_gpu / e_orc <= 1.25, (e_gpu, e_orc)
    # and the two quantized trajectories stay within a few quantization steps
    d_go = np.max(np.abs(np.stack(outs) - np.stack(windowed.outputs)))
    assert d_go <= 8 * np.max(np.abs(np.stack(windowed.outputs) - np.stack(exact.outputs))) + 1e-6
    st.close()


@pytest.mark.parametrize("L", [4, 32, 64])
def test_q8_serving_L_sweep(L):
    # B=512 with ragged fills: every sequence ends at least two windows at its
    # own phase, separate and fused merge
    w = wl.WORKLOADS["gdn_serving"].replace(L=L)
    heads = heads_covering_phases(w, 16)
    for fused in (True, False):
        r = run_parity_q8(w, T=2 * L + 5, heads=heads, fused=fused, snap_every=max(L // 2, 4),
                          workers=None)
        _check(r)
