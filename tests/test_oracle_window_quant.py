"""Pins of the per-window quantization oracle (CPU only).

Every pin fixes the oracle against something other than itself: hand-worked
rounding of rows whose products are exact, exact round trips on the int8
grid, the rounding error bound, and step-by-step readouts of states built so
that the output shows exactly when a window ended.  Planted mistakes (wrong
rounding, wrong scale axis, wrong precision, wrong window timing, wrong
orientation) each fail at least one pin: the mistakes are planted in copies
of the oracle, never in the CUDA path.
"""

from __future__ import annotations

import types

import numpy as np
import pytest

import oracle
from oracle import window_quant as wq_mod


def _steps(qs, ks, vs, alphas, betas):
    """Per-step namespaces shaped [B=1, H=1, ...]."""
    out = []
    for q, k, v, a, b in zip(qs, ks, vs, alphas, betas):
        out.append(types.SimpleNamespace(
            q=np.asarray(q, float)[None, None], k=np.asarray(k, float)[None, None],
            v=np.asarray(v, float)[None, None], decay=np.asarray(a, float)[None, None],
            beta=None if b is None else np.asarray(b, float)[None, None]))
    return out


# ---------------------------------------------------------------- pins

def pin_hand_rows(wq):
    # amax 127 -> inv = 1 and amax 254 -> inv = 0.5 exactly, so every
    # product is exact and only the rounding rule decides: half to even.
    X = np.array([[127.0, 63.5, -0.5, 1.5, 2.5, -2.5, 0.49, 100.2],
                  [254.0, 3.0, 5.0, -7.0, 1.0, -1.0, 0.0, 0.75],
                  [0.0] * 8,
                  [-127.0, 0.5, -1.5, 3.5, 126.5, -126.5, 0.51, -0.51]])
    codes, scales = wq.quantize_rows(X)
    assert codes.dtype == np.int8 and scales.dtype == np.float32
    assert codes.tolist() == [[127, 64, 0, 2, 2, -2, 0, 100],
                              [127, 2, 2, -4, 0, 0, 0, 0],
                              [0] * 8,
                              [-127, 0, -2, 4, 126, -126, 1, -1]]
    assert scales.tolist() == [1.0, 2.0, 0.0, 1.0]
    deq = wq.dequantize_rows(codes, scales)
    assert deq[1].tolist() == [254.0, 4.0, 4.0, -8.0, 0.0, 0.0, 0.0, 0.0]


def pin_decision_in_fp32(wq):
    # inv = fl32(127/3); x is the fp32 value whose fp32 product with inv is
    # exactly 10.5 (so it rounds to 10), while the fp64 product is above 10.5.
    x = np.array([0x3E7DFBF8], dtype=np.uint32).view(np.float32)[0]
    codes, _ = wq.quantize_rows(np.array([[3.0, float(x)]]))
    assert codes.tolist() == [[127, 10]]


def pin_per_row_scale(wq):
    rng = np.random.default_rng(11)
    X = rng.standard_normal((2, 6, 16)) * np.array([1e-3, 0.1, 1.0, 10.0, 3e2, 0.5])[None, :, None]
    codes, scales = wq.quantize_rows(X)
    assert scales.shape == (2, 6)
    assert np.all(np.max(np.abs(codes.astype(int)), axis=-1) == 127)
    amax = np.max(np.abs(X.astype(np.float32)), axis=-1)
    assert np.array_equal(scales, (amax / np.float32(127)).astype(np.float32))


def pin_roundtrip_exact(wq):
    rng = np.random.default_rng(12)
    codes = rng.integers(-127, 128, size=(3, 8, 32)).astype(np.int8)
    codes[:, :, 0] = 127
    codes[:, ::2, 0] = -127
    for e in (-7, 0, 5):
        X = codes.astype(np.float64) * 2.0 ** e
        c2, s2 = wq.quantize_rows(X)
        assert np.array_equal(c2, codes)
        assert np.all(s2 == np.float32(2.0 ** e))


def pin_error_bound(wq):
    rng = np.random.default_rng(13)
    X = rng.standard_normal((4, 16, 64)) * 0.05
    codes, scales = wq.quantize_rows(X)
    deq = wq.dequantize_rows(codes, scales)
    err = np.abs(deq - X)
    assert np.all(err <= scales[..., None].astype(np.float64) * (0.5 + 1e-5) + 1e-12)
    assert np.all(np.abs(codes.astype(int)) <= 127)


def _timing_case(L, fill0, T, merge_all_after=()):
    """GDN, d = 4, alpha = beta = 1: step t writes column t mod 2 (k = e_c)
    with a value off the int8 grid and reads the other column (q = e_other),
    written the step before.  Column 3 holds 127 in every row, so each row's
    scale is exactly 1 and quantizing rounds the values to integers: o_t shows
    whether a window ended after step t - 1."""
    d = 4
    S0 = np.zeros((1, d, d))
    S0[0, :, 3] = 127.0
    vals = [np.array([0.3, 1.5, 2.5, -0.7]) + 10.0 * t for t in range(T)]
    qs, ks = [], []
    for t in range(T):
        c = t % 2
        ks.append(np.eye(d)[c])
        qs.append(np.eye(d)[1 - c])
    steps = _steps(qs, ks, vals, [1.0] * T, [1.0] * T)
    return S0, steps, vals


def _expected_timing(vals, ends, T):
    out = [np.zeros(4)]
    for t in range(1, T):
        v = vals[t - 1]
        out.append(np.rint(v) if t in ends else v)  # scale 1: the grid is the integers
    return out


def _check_timing(wq, L, fill0, T, merge_all_after, ends):
    S0, steps, vals = _timing_case(L, fill0, T, merge_all_after)
    res = wq.run_windowed("gdn", S0, steps, L, fill0, H=1, merge_all_after=merge_all_after)
    exp = _expected_timing(vals, set(ends), T)
    for t in range(T):
        assert np.array_equal(res.outputs[t][0], exp[t]), (L, fill0, t)
    assert [e.step for e in res.ends] == list(ends)


def pin_window_timing(wq):
    # fill0 = 1, L = 3: windows end after steps 2, 5, 8
    _check_timing(wq, 3, [1], 10, (), [2, 5, 8])
    # L = 1: a window ends after every step
    _check_timing(wq, 1, [0], 5, (), [1, 2, 3, 4, 5])


def pin_forced_merge_timing(wq):
    # a merge of every non-empty log after step 4 ends that window early
    _check_timing(wq, 3, [1], 10, (4,), [2, 4, 7, 10])


def pin_initial_quantization(wq):
    # beta = 0, alpha = 1 and a window that never ends: the state stays the
    # quantized S0, exactly
    rng = np.random.default_rng(14)
    S0 = rng.standard_normal((2, 8, 8))
    T = 3
    steps = [types.SimpleNamespace(q=rng.standard_normal((1, 2, 8)), k=rng.standard_normal((1, 2, 8)),
                                   v=rng.standard_normal((1, 2, 8)), decay=np.ones((1, 2)),
                                   beta=np.zeros((1, 2))) for _ in range(T)]
    res = wq.run_windowed("gdn", S0, steps, 64, [0], H=2)
    codes, scales = wq.quantize_rows(S0)
    assert np.array_equal(res.S, wq.dequantize_rows(codes, scales))
    assert np.array_equal(res.start_codes, codes)


def pin_rwkv6_orientation(wq):
    # RWKV6's state (d_k x d_v in the recurrence) is quantized along its value
    # rows: columns of the recurrence's matrix share a scale.
    S = np.array([[[1.0, 3.0], [0.25, 0.5]]])     # [1, d_k, d_v]
    res = wq.run_windowed("rwkv6", S, [], 4, [0], H=1)
    inv0 = np.float32(127.0) / np.float32(1.0)
    inv1 = np.float32(127.0) / np.float32(3.0)
    s0 = np.float32(1.0) / np.float32(127.0)
    s1 = np.float32(3.0) / np.float32(127.0)
    c = [[127, int(np.rint(np.float32(0.25) * inv0))], [127, int(np.rint(np.float32(0.5) * inv1))]]
    assert res.start_codes[0].tolist() == c
    exp = np.array([[np.float32(127) * s0, np.float32(127) * s1],
                    [np.float32(c[0][1]) * s0, np.float32(c[1][1]) * s1]], np.float64)
    assert np.array_equal(res.S[0], exp)


def pin_long_window_is_eager(wq):
    # no window end inside the run: outputs are the eager recurrence started
    # from the dequantized base (the log is high precision)
    rng = np.random.default_rng(15)
    N, d, T = 3, 8, 6
    S0 = rng.standard_normal((N, d, d)) * 0.1
    kk = rng.standard_normal((T, 1, N, d))
    kk /= np.linalg.norm(kk, axis=-1, keepdims=True)
    steps = [types.SimpleNamespace(q=kk[t], k=np.roll(kk[t], 1, axis=-1), v=rng.standard_normal((1, N, d)),
                                   decay=rng.uniform(0.9, 1.0, (1, N)), beta=rng.uniform(0, 1, (1, N)))
             for t in range(T)]
    res = wq.run_windowed("gdn", S0, steps, 32, [0], H=N)
    codes, scales = wq.quantize_rows(S0)
    ref = oracle.run_eager("gdn", wq.dequantize_rows(codes, scales), steps)
    for a, b in zip(res.outputs, ref.outputs):
        assert np.array_equal(a, b)
    assert res.ends == []


def pin_row_inverse_hand(wq):
    # inv_j = 127 / amax_j in fp32 (amax over |x|), exact on these rows;
    # zero rows and rows below 2^-120 give 0, a row at exactly 2^-120 is live
    X = np.array([[127.0, -3.0, 5.0],
                  [-254.0, 3.0, 0.0],
                  [1.0, -0.5, 0.25],
                  [0.0, 0.0, 0.0],
                  [2.0 ** -121, -(2.0 ** -122), 0.0],
                  [2.0 ** -120, 0.0, 0.0]])
    inv = wq.row_inverse(X)
    assert inv.dtype == np.float32 and inv.shape == (6,)
    assert inv[:4].tolist() == [1.0, 0.5, 127.0, 0.0]
    assert inv[4] == 0.0
    assert inv[5] == np.float32(127.0 * 2.0 ** 120)  # exact: 127 * 2^120 is an fp32 value


def pin_row_inverse_fp32(wq):
    # 127/3 rounded once to fp32 has the bits 0x42295555 (binary expansion
    # 101010.0101..., cut at 24 significant bits, next bit 0); the product with
    # the element of pin_decision_in_fp32 is then exactly 10.5 in fp32
    x = np.array([0x3E7DFBF8], dtype=np.uint32).view(np.float32)[0]
    inv = wq.row_inverse(np.array([[3.0, float(x)], [-3.0, 1.0]]))
    assert inv.dtype == np.float32
    assert inv.view(np.uint32).tolist() == [0x42295555, 0x42295555]
    assert np.float32(x) * inv[0] == np.float32(10.5)


def pin_row_inverse_drives_codes(wq):
    # the quantizer's codes are rint(fl32(x * inv)) clipped to +-127 with the
    # same inv, on random rows of many magnitudes (ties the inverse to the
    # hand-pinned codes above)
    rng = np.random.default_rng(16)
    X = rng.standard_normal((3, 12, 32)) * (10.0 ** rng.uniform(-6, 6, (3, 12, 1)))
    X[0, 0] = 0.0
    codes, _ = wq.quantize_rows(X)
    inv = wq.row_inverse(X)
    prod = (X.astype(np.float32) * inv[..., None]).astype(np.float32)
    assert np.array_equal(codes.astype(np.int64), np.clip(np.rint(prod), -127, 127).astype(np.int64))


WQ_PINS = [pin_hand_rows, pin_decision_in_fp32, pin_per_row_scale, pin_roundtrip_exact,
           pin_error_bound, pin_window_timing, pin_forced_merge_timing, pin_initial_quantization,
           pin_rwkv6_orientation, pin_long_window_is_eager, pin_row_inverse_hand,
           pin_row_inverse_fp32, pin_row_inverse_drives_codes]


@pytest.mark.parametrize("pin", WQ_PINS, ids=lambda p: p.__name__)
def test_window_quant_pin(pin):
    pin(wq_mod)


# ------------------------------------------------------------- mutants

def _quantizer(round_fn=np.rint, axis="row", qmax=127.0, fp32=True):
    def q(X):
        x = np.asarray(X).astype(np.float32 if fp32 else np.float64)
        if axis == "row":
            amax = np.max(np.abs(x), axis=-1, keepdims=True)
        elif axis == "col":
            amax = np.max(np.abs(x), axis=-2, keepdims=True)
        else:
            amax = np.max(np.abs(x), axis=(-1, -2), keepdims=True)
        safe = np.where(amax > 0, amax, 1.0).astype(x.dtype)
        inv = (x.dtype.type(qmax) / safe).astype(x.dtype)
        codes = np.clip(round_fn((x * inv).astype(x.dtype)), -127, 127)
        codes = np.where(amax > 0, codes, 0).astype(np.int8)
        sc = np.where(amax > 0, amax / x.dtype.type(qmax), 0).astype(np.float32)
        sc = np.broadcast_to(sc, x.shape)
        if axis == "row":
            return codes, sc[..., 0].copy()
        # a scale per column (or per matrix) cannot be expressed per row:
        # hand back the row-wise view of the value each element used
        return codes, sc[..., 0].copy() if axis == "row" else np.ascontiguousarray(sc[..., 0])
    return q


def _half_away(x):
    return np.sign(x) * np.floor(np.abs(x) + 0.5)


def _windowed_mutant(kind):
    """A copy of run_windowed with one timing or orientation mistake."""
    base = wq_mod.run_windowed

    def run(variant, S0, steps, L, fill0, H, heads=None, bonus=None, merge_all_after=(),
            snapshot_at=(), kla_eps=None):
        if kind == "never":
            res = base(variant, S0, steps, 10 ** 9, fill0, H, heads, bonus, (), snapshot_at, kla_eps)
            return res
        if kind == "late":
            return base(variant, S0, steps, L + 1, fill0, H, heads, bonus, merge_all_after,
                        snapshot_at, kla_eps)
        if kind == "early":
            # ends a window one step before the log fills
            f0 = [min(int(f) + 1, L - 1) if L > 1 else 0 for f in fill0]
            return base(variant, S0, steps, L, f0, H, heads, bonus, merge_all_after, snapshot_at, kla_eps)
        if kind == "no_forced":
            return base(variant, S0, steps, L, fill0, H, heads, bonus, (), snapshot_at, kla_eps)
        if kind == "no_initial":
            orig = wq_mod.requantize
            calls = {"n": 0}

            def req(S, rec):
                calls["n"] += 1
                if calls["n"] == 1:
                    pre = np.swapaxes(S, -1, -2) if rec else np.asarray(S, np.float64)
                    c, s = wq_mod.quantize_rows(pre)
                    return np.asarray(S, np.float64).copy(), c, s, pre.copy()
                return orig(S, rec)
            wq_mod.requantize = req
            try:
                return base(variant, S0, steps, L, fill0, H, heads, bonus, merge_all_after,
                            snapshot_at, kla_eps)
            finally:
                wq_mod.requantize = orig
        if kind == "key_rows":
            orig = wq_mod._to_rows
            wq_mod._to_rows = lambda S, rec: S
            try:
                return base(variant, S0, steps, L, fill0, H, heads, bonus, merge_all_after,
                            snapshot_at, kla_eps)
            finally:
                wq_mod._to_rows = orig
        raise ValueError(kind)
    return run


Q_MUTANTS = {
    "floor_rounding": _quantizer(round_fn=np.floor),
    "half_away_from_zero": _quantizer(round_fn=_half_away),
    "scale_128": _quantizer(qmax=128.0),
    "decision_in_fp64": _quantizer(fp32=False),
    "scale_per_key_column": _quantizer(axis="col"),
    "scale_per_matrix": _quantizer(axis="all"),
}
def _inverse(qmax=127.0, fp32=True, cutoff="ge", absval=True):
    """A copy of row_inverse with one planted mistake."""
    def inv(X):
        x = np.asarray(X).astype(np.float32 if fp32 else np.float64)
        amax = np.max(np.abs(x) if absval else x, axis=-1)
        tiny = wq_mod.TINY_AMAX
        live = {"ge": amax >= tiny, "gt": amax > tiny, "none": amax > 0}[cutoff]
        safe = np.where(live, amax, 1.0).astype(x.dtype)
        return np.where(live, x.dtype.type(qmax) / safe, 0.0).astype(x.dtype)
    return inv


INV_MUTANTS = {
    "inverse_128": _inverse(qmax=128.0),
    "inverse_in_fp64": _inverse(fp32=False),
    "inverse_no_tiny_cutoff": _inverse(cutoff="none"),
    "inverse_strict_cutoff": _inverse(cutoff="gt"),
    "inverse_signed_max": _inverse(absval=False),
}
W_MUTANTS = ["never", "late", "early", "no_forced", "no_initial", "key_rows"]


@pytest.mark.parametrize("name", sorted(Q_MUTANTS) + sorted(INV_MUTANTS)
                         + ["window_" + k for k in W_MUTANTS])
def test_window_quant_mutant_is_caught(name, monkeypatch):
    if name.startswith("window_"):
        mutant = _windowed_mutant(name[len("window_"):])
        impl = types.SimpleNamespace(quantize_rows=wq_mod.quantize_rows,
                                     dequantize_rows=wq_mod.dequantize_rows, run_windowed=mutant,
                                     row_inverse=wq_mod.row_inverse)
    elif name in INV_MUTANTS:
        impl = types.SimpleNamespace(quantize_rows=wq_mod.quantize_rows,
                                     dequantize_rows=wq_mod.dequantize_rows,
                                     run_windowed=wq_mod.run_windowed, row_inverse=INV_MUTANTS[name])
    else:
        monkeypatch.setattr(wq_mod, "quantize_rows", Q_MUTANTS[name])
        impl = types.SimpleNamespace(quantize_rows=wq_mod.quantize_rows,
                                     dequantize_rows=wq_mod.dequantize_rows,
                                     run_windowed=wq_mod.run_windowed, row_inverse=wq_mod.row_inverse)
    failed = []
    for pin in WQ_PINS:
        try:
            pin(impl)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name} passed every pin"
