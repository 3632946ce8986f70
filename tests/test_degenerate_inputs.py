"""The degenerate-input edits: inside the input contract, and what the fp64
oracle makes of them matches the closed forms the limiting cases have."""

from __future__ import annotations

import numpy as np
import pytest

import oracle
from linear_attention_recurrent_deltalog_b200 import workloads as wl
from tests.degenerate_inputs import KINDS, TINY_DECAY, compose, make_edit

BASES = {"gdn": "gdn_qwen", "kda": "kda", "rwkv6": "rwkv6", "gdn2": "gdn2"}
VARIANTS = sorted(BASES)


def _w(variant):
    return wl.WORKLOADS[BASES[variant]].replace(B=2, H=2, d_k=64, d_v=64, L=4, T=7, seed=5)


def _run(w, edit, T=None):
    T = w.T if T is None else T
    steps = [edit(wl.step_inputs(w, t)) for t in range(T)]
    S0 = wl.initial_state(w).reshape(w.heads, w.d_v, w.d_k).astype(np.float64)
    if w.variant == wl.RWKV6:
        S0 = S0.transpose(0, 2, 1)
    bonus = None
    if w.variant == wl.RWKV6:
        bonus = wl.rwkv6_bonus(w)[np.arange(w.heads) % w.H]
    return steps, S0, oracle.run_eager(w.variant, S0, steps, bonus=bonus)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("variant", VARIANTS)
def test_edits_stay_inside_the_input_contract(variant, kind):
    w = _w(variant).replace(in_dtype="bf16")
    edit = make_edit(w, kind)
    for t in range(7):
        s0 = wl.step_inputs(w, t)
        s = edit(s0)
        for name in ("q", "k", "v", "decay", "beta", "wgate"):
            x, x0 = getattr(s, name), getattr(s0, name)
            assert (x is None) == (x0 is None)
            if x is None:
                continue
            assert x.dtype == np.float32 and x.shape == x0.shape, name
            if name in ("q", "k", "v"):  # bf16-exact: the bit patterns round-trip
                assert np.array_equal(wl.bf16_bits(x).astype(np.uint32) << 16,
                                      x.view(np.uint32)), name
        assert np.all(s.decay > 0) and np.all(s.decay <= 1)
        for g in (s.beta, s.wgate):
            if g is not None:
                assert np.all(g >= 0) and np.all(g <= 1)


@pytest.mark.parametrize("variant", VARIANTS)
def test_no_decay_and_no_write_keep_the_initial_state(variant):
    w = _w(variant)
    steps, S0, ref = _run(w, compose(make_edit(w, "no_decay"), make_edit(w, "no_write")))
    assert np.array_equal(ref.S, S0)
    for s, o in zip(steps, ref.outputs):
        q = s.q.reshape(w.heads, -1).astype(np.float64)
        want = (np.einsum("nck,nc->nk", S0, q) if variant == "rwkv6"
                else np.einsum("njc,nc->nj", S0, q))
        np.testing.assert_allclose(o, want, rtol=0, atol=1e-15)


@pytest.mark.parametrize("variant", VARIANTS)
def test_zero_query_gives_zero_outputs(variant):
    w = _w(variant)
    _, _, ref = _run(w, make_edit(w, "zero_query"))
    assert all(not o.any() for o in ref.outputs)


@pytest.mark.parametrize("variant", VARIANTS)
def test_vanishing_decay_keeps_only_the_last_write(variant):
    # decay 1e-30: the state after step T is the last write alone, up to
    # terms ~1e-30 times the previous state
    w = _w(variant)
    steps, _, ref = _run(w, make_edit(w, "vanishing_decay"))
    s = steps[-1]
    N = w.heads
    k = s.k.reshape(N, -1).astype(np.float64)
    v = s.v.reshape(N, -1).astype(np.float64)
    if variant == "rwkv6":
        want = np.einsum("nc,nj->ncj", k, v)
    elif variant == "gdn2":
        wg = s.wgate.reshape(N, -1).astype(np.float64)
        want = np.einsum("nj,nc->njc", wg * v, k)
    else:
        beta = s.beta.reshape(N, 1).astype(np.float64)
        want = np.einsum("nj,nc->njc", beta * v, k)
    scale = np.max(np.abs(want))
    assert np.max(np.abs(ref.S - want)) <= 1e-25 * scale
    assert float(TINY_DECAY) == pytest.approx(1e-30, rel=1e-7)


def test_mixed_extremes_gdn_splits_heads():
    # GDN: even heads forget everything each step, odd heads never decay
    w = _w("gdn")
    steps, S0, ref = _run(w, make_edit(w, "mixed_extremes"))
    s = steps[-1]
    assert np.all(s.decay[:, 0::2] == TINY_DECAY) and np.all(s.decay[:, 1::2] == 1.0)
    k = s.k.reshape(w.heads, -1).astype(np.float64)
    v = s.v.reshape(w.heads, -1).astype(np.float64)
    beta = s.beta.reshape(w.heads, 1).astype(np.float64)
    even = np.arange(w.heads) % w.H % 2 == 0
    want = np.einsum("nj,nc->njc", beta * v, k)[even]
    assert np.max(np.abs(ref.S[even] - want)) <= 1e-25 * np.max(np.abs(want))


def test_repeated_key_reuses_step_zero_keys():
    w = _w("kda")
    edit = make_edit(w, "repeated_key")
    k0 = wl.step_inputs(w, 0).k
    for t in (0, 3, 6):
        assert np.array_equal(edit(wl.step_inputs(w, t)).k, k0)


def test_wipe_then_recover_hits_only_its_steps():
    w = _w("gdn")
    edit = make_edit(w, "wipe_then_recover")
    for t in range(12):
        s0 = wl.step_inputs(w, t)
        s = edit(s0)
        if t % 5 == 2:
            assert np.all(s.decay == TINY_DECAY)
        else:
            assert np.array_equal(s.decay, s0.decay)
