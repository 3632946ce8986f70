"""The seeded input generator (CPU only): determinism, rounding, shapes."""

from __future__ import annotations

import numpy as np
import torch

from linear_attention_recurrent_deltalog_b200 import workloads as wl


def test_bf16_rounding_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    # include exact ties: values in [1, 2) whose low 16 bits are 0x8000
    mant = rng.integers(0, 128, 1000).astype(np.uint32) << np.uint32(16)
    ties = (mant | np.uint32(0x3F800000) | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties, np.array([0.0, -0.0, 1.0, -1.0], np.float32)])
    ours = wl.bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    np.testing.assert_array_equal(wl.bf16_to_f32(ours),
                                  torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_steps_are_deterministic_and_independent():
    w = wl.WORKLOADS["gdn_qwen"].replace(B=3, H=2)
    a = wl.step_inputs(w, 5)
    b = wl.step_inputs(w, 5)
    c = wl.step_inputs(w, 6)
    for f in ("q", "k", "v", "decay", "beta"):
        np.testing.assert_array_equal(getattr(a, f), getattr(b, f))
        assert not np.array_equal(getattr(a, f), getattr(c, f))


def test_shapes_dtypes_and_ranges():
    for name, w in wl.WORKLOADS.items():
        w = w.replace(B=min(w.B, 4), H=min(w.H, 3))
        s = wl.step_inputs(w, 0)
        assert s.q.shape == (w.B, w.H, w.d_k) and s.k.shape == (w.B, w.H, w.d_k)
        assert s.v.shape == (w.B, w.H, w.d_v)
        assert s.q.dtype == np.float32
        if w.variant == wl.RWKV6:
            assert s.beta is None and s.decay.shape == (w.B, w.H, w.d_k)
            assert np.all((s.decay > 0) & (s.decay < 1))
        else:
            bshape = (w.B, w.H, w.d_k) if w.variant == wl.GDN2 else (w.B, w.H)
            assert s.beta.shape == bshape
            assert np.all((s.beta > 0) & (s.beta < 1))
            # q and k are unit vectors up to input rounding
            tol = 1e-2 if w.in_dtype == "bf16" else 1e-6
            np.testing.assert_allclose(np.linalg.norm(s.k.astype(np.float64), axis=-1), 1, atol=tol)
            np.testing.assert_allclose(np.linalg.norm(s.q.astype(np.float64), axis=-1), 1, atol=tol)
        if w.variant in (wl.KDA, wl.GDN2):
            assert s.decay.shape == (w.B, w.H, w.d_k)
            assert np.all((s.decay >= 0.8) & (s.decay <= 1.0))
        if w.variant == wl.GDN2:
            assert s.wgate.shape == (w.B, w.H, w.d_v)
            assert np.all((s.wgate > 0) & (s.wgate < 1))
        else:
            assert s.wgate is None
        if w.variant == wl.GDN:
            assert s.decay.shape == (w.B, w.H)
            assert np.all((s.decay > 0.5) & (s.decay <= 1.0))
        if w.in_dtype == "bf16":
            for f in ("q", "k", "v"):
                x = getattr(s, f)
                np.testing.assert_array_equal(wl.round_bf16(x), x)
                assert s.device_array(f).dtype == np.uint16


def test_initial_state_fill_and_bonus():
    w = wl.WORKLOADS["gdn_serving"].replace(B=64, L=16)
    S0 = wl.initial_state(w.replace(B=8))
    assert S0.shape == (8, w.H, 128, 128) and S0.dtype == np.float32
    assert abs(float(S0.std()) - 0.01) < 1e-3
    f = wl.fill_offsets(w)
    assert f.shape == (64,) and f.min() >= 0 and f.max() <= 15
    assert len(set(f.tolist())) > 8
    assert np.all(wl.fill_offsets(wl.WORKLOADS["gdn_qwen"]) == 0)
    u = wl.rwkv6_bonus(wl.WORKLOADS["rwkv6"])
    assert u.shape == (64, 64) and abs(float(u.std()) - 0.5) < 0.05


def test_sample_heads():
    w = wl.WORKLOADS["gdn_serving"]
    h = wl.sample_heads(w, 50)
    assert len(h) == 50 and len(set(h.tolist())) == 50 and h.max() < w.heads
    np.testing.assert_array_equal(h, wl.sample_heads(w, 50))


def test_kla_workload_keeps_key_norms():
    w = wl.WORKLOADS["gdn_qwen"].replace(B=4, H=3, kla_eps=1e-6)
    s = wl.step_inputs(w, 0)
    n = np.linalg.norm(s.k.astype(np.float64), axis=-1)
    assert n.std() > 0.02  # not normalised: the KLA step size sees the norms
    assert abs(n.mean() - 1.0) < 0.2
