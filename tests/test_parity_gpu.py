"""GPU parity: the CUDA paths through the C ABI against the fp64 oracle.

Tolerances (fp32 state and arithmetic): max |dS| / max |S| <= 1e-4 at every
64th step and at T, and output relative error <= 1e-3 at every step.  The
five workloads run at their full batch sizes in the launch configuration
the benchmark times; the oracle checks a seeded sample of heads (every
fill phase included for ragged batches), since heads are independent.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from linear_attention_recurrent_deltalog_b200 import workloads as wl
from tests.parity import OUT_TOL, STATE_TOL, heads_covering_phases, run_parity

pytestmark = pytest.mark.gpu


def _check(res, arms=None):
    for arm, r in res.items():
        if arms is not None and arm not in arms:
            continue
        assert r.state_err <= STATE_TOL, f"{arm}: state rel err {r.state_err:.3e}"
        assert r.out_err <= OUT_TOL, f"{arm}: output rel err {r.out_err:.3e}"


def test_gdn_tiny_all_heads():
    # B=1, H=2, d=64, fp32 inputs, T=32, L=8: every head, every step
    res = run_parity(wl.WORKLOADS["gdn_tiny"], snap_every=8, workers=0)
    _check(res)


@pytest.mark.parametrize("name", ["gdn_qwen", "kda", "rwkv6"])
def test_full_workload(name):
    w = wl.WORKLOADS[name]
    heads = wl.sample_heads(w, 48)
    res = run_parity(w, heads=heads)
    _check(res)


def test_serving_L16_full_length():
    # B=512, H=32, d=128, ragged fills, T=1024: the benchmarked configuration
    w = wl.WORKLOADS["gdn_serving"]
    heads = heads_covering_phases(w, 24)
    res = run_parity(w, heads=heads, snap_every=256)
    _check(res)


@pytest.mark.parametrize("L", [4, 8, 32, 64])
def test_serving_L_sweep(L):
    # every sequence passes at least two merges at its own phase
    w = wl.WORKLOADS["gdn_serving"].replace(L=L)
    heads = heads_covering_phases(w, 16)
    res = run_parity(w, T=2 * L + 9, heads=heads, snap_every=max(L, 8), arms=("log", "fused"))
    _check(res)


@pytest.mark.parametrize("variant,dk,dv,dtype", [
    ("gdn", 64, 128, "bf16"), ("gdn", 128, 64, "f32"), ("kda", 64, 128, "f32"),
    ("kda", 128, 64, "bf16"), ("rwkv6", 128, 128, "bf16"), ("rwkv6", 64, 128, "f32"),
    ("gdn", 128, 128, "f32"), ("kda", 64, 64, "bf16"),
])
def test_shapes_and_dtypes(variant, dk, dv, dtype):
    base = {"gdn": "gdn_qwen", "kda": "kda", "rwkv6": "rwkv6"}[variant]
    w = wl.WORKLOADS[base].replace(B=5, H=3, d_k=dk, d_v=dv, in_dtype=dtype, L=6, T=29,
                                   ragged=True)
    for split in (1, dv // 32):
        _check(run_parity(w, snap_every=7, workers=0, split=split))


@pytest.mark.parametrize("split", [1, 2, 4])
@pytest.mark.parametrize("name", ["gdn_qwen", "kda", "rwkv6"])
def test_step_split(name, split):
    # a head cut into 1, 2 or 4 work items
    w = wl.WORKLOADS[name]
    if w.d_v // split < 32:
        pytest.skip("d_v / split < 32 is not built")
    w = w.replace(B=6, H=5, L=8, T=27, ragged=True)
    _check(run_parity(w, snap_every=9, workers=0, split=split, arms=("log", "fused")))


@pytest.mark.parametrize("L", [1, 2, 64])
def test_extreme_log_lengths(L):
    # L = 1 merges after every step; L = 64 is the largest log
    for name in ("gdn_qwen", "kda", "rwkv6"):
        w = wl.WORKLOADS[name].replace(B=3, H=4, L=L, T=max(3 * L, 12) + 1, ragged=True)
        for split in (1, w.d_v // 32):
            _check(run_parity(w, snap_every=max(L, 4), workers=0, split=split))


def test_forced_merges_mid_log():
    # DL_MERGE_ALL folds partial logs; results must not change
    w = wl.WORKLOADS["kda"].replace(B=4, H=3, L=16, T=40, ragged=True)
    res = run_parity(w, snap_every=5, merge_all_at=(3, 7, 20, 21), workers=0,
                     arms=("log", "fused"))
    _check(res)
    w = wl.WORKLOADS["rwkv6"].replace(B=4, H=3, L=16, T=40, ragged=True)
    _check(run_parity(w, snap_every=5, merge_all_at=(1, 17), workers=0, arms=("log", "fused")))


@pytest.mark.parametrize("B", [4200, 16400])
def test_large_batch_fallbacks(B):
    # More than 4096 sequences merging at once: the merge reads the device fills
    # (unsplit launch); more than 16384 sequences: the step reads the device
    # fills instead of the launch argument.
    w = wl.WORKLOADS["gdn_qwen"].replace(B=B, H=1, d_k=64, d_v=64, L=2, T=5, ragged=False)
    _check(run_parity(w, heads=wl.sample_heads(w, 32), snap_every=2, workers=0))
    w = wl.WORKLOADS["kda"].replace(B=B, H=1, d_k=64, d_v=128, L=3, T=7, ragged=True)
    _check(run_parity(w, heads=wl.sample_heads(w, 32), snap_every=3, workers=0,
                      arms=("log", "fused")))


@pytest.mark.parametrize("name", ["gdn_qwen", "kda"])
def test_kla_step_size(name):
    # beta = eta / (|k|^2 + eps) formed in the kernels, unnormalised keys
    w = wl.WORKLOADS[name].replace(B=6, H=5, L=8, T=27, ragged=True, kla_eps=1e-6)
    _check(run_parity(w, snap_every=9, workers=0))
    w = wl.WORKLOADS[name].replace(kla_eps=1e-3)
    _check(run_parity(w, T=40, heads=wl.sample_heads(w, 24), arms=("fused", "eager")))


# ---------------------------------------------------------------- GDN-2

def test_gdn2_full_workload():
    # B=128 H=32 d=128 L=16: erase and write gates per channel, every step
    w = wl.WORKLOADS["gdn2"]
    _check(run_parity(w, heads=wl.sample_heads(w, 48)))


@pytest.mark.parametrize("split", [1, 2, 4])
@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, "bf16"), (64, 128, "f32"), (128, 64, "bf16"),
                                         (64, 64, "f32")])
def test_gdn2_shapes_splits(dk, dv, dtype, split):
    if dv // split < 32:
        pytest.skip("d_v / split < 32 is not built")
    w = wl.WORKLOADS["gdn2"].replace(B=5, H=3, d_k=dk, d_v=dv, in_dtype=dtype, L=6, T=29,
                                     ragged=True)
    _check(run_parity(w, snap_every=7, workers=0, split=split))


def test_gdn2_log_lengths_and_forced_merges():
    for L in (1, 2, 64):
        w = wl.WORKLOADS["gdn2"].replace(B=3, H=4, L=L, T=max(3 * L, 12) + 1, ragged=True)
        _check(run_parity(w, snap_every=max(L, 4), workers=0))
    w = wl.WORKLOADS["gdn2"].replace(B=4, H=3, L=16, T=40, ragged=True)
    _check(run_parity(w, snap_every=5, merge_all_at=(3, 7, 20, 21), workers=0,
                      arms=("log", "fused")))
