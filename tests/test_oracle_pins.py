"""Pins for the fp64 oracle (CPU only).

The pages print no worked example, so the oracle is pinned by facts that
hold independently of it:

* exact hand-derived examples (d = 2, rational inputs, derivations in the
  comments), for each recurrence;
* closed forms: beta = 0 is pure decay; RWKV6 with k = 0 is pure decay; RWKV6
  with w = 1, u = 0 is a plain sum of outer products;
* invariants: exact retrieval S k_i = v_i after alpha = beta = 1 writes with
  orthonormal keys; the Frobenius norm never grows when v = 0, |k| = 1,
  beta in [0, 1], alpha <= 1;
* a special case that reduces to another routine: KDA with a constant decay
  vector is GDN (the Gated DeltaNet-2 abstract describes KDA as GDN with a
  decay per key channel);
* brute force: DeltaLog's log form in exact rationals (tests/logform_exact.py)
  equals the oracle for several L and fill offsets, and L = 1 (merge after
  every step) as well.

Each pin is a function of an ``impl`` namespace holding the three step
functions, so ``test_oracle_mutants.py`` can run the same pins against copies
of the oracle with a planted mistake and show that every such mistake fails
at least one of them.
"""

from __future__ import annotations

import types
from fractions import Fraction as F

import numpy as np
import pytest

import oracle
from oracle import recurrence as rec
from tests.logform_exact import ExactDeltaLog

REAL = types.SimpleNamespace(gdn_step=rec.gdn_step, kda_step=rec.kda_step,
                             rwkv6_step=rec.rwkv6_step, gdn2_step=rec.gdn2_step)


def _fa(rows):
    return np.array([[float(x) for x in r] for r in rows], dtype=np.float64)


def _v(xs):
    return np.array([float(x) for x in xs], dtype=np.float64)


# ------------------------------------------------------------- hand examples

def pin_gdn_hand(impl):
    # S0 = [[1,2],[3,4]] (rows: value index, cols: key channel)
    # k = (3/5, 4/5), q = (1, -1), v = (2, 1), alpha = 1/2, beta = 1/2.
    # I - beta k k^T = [[41/50, -12/50], [-12/50, 34/50]]
    # S0 (I - beta k k^T) = [[17/50, 56/50], [3/2, 2]];  times alpha:
    #   [[17/100, 56/100], [3/4, 1]];   beta v k^T = [[3/5, 4/5], [3/10, 2/5]]
    # S1 = [[77/100, 136/100], [21/20, 7/5]],  o1 = S1 q = (-59/100, -7/20).
    # Step 2: k = (1, 0), q = (0, 1), v = (0, 1), alpha = 1, beta = 1:
    # S1 (I - k k^T) = [[0, 136/100], [0, 7/5]],  + v k^T = [[0,0],[1,0]]
    # S2 = [[0, 34/25], [1, 7/5]],  o2 = (34/25, 7/5);  note S2 k = v.
    S = _fa([[1, 2], [3, 4]])[None]
    S1, o1 = impl.gdn_step(S, _v([1, -1])[None], _v([F(3, 5), F(4, 5)])[None], _v([2, 1])[None], _v([F(1, 2)]), _v([F(1, 2)]))
    np.testing.assert_allclose(S1[0], _fa([[F(77, 100), F(136, 100)], [F(21, 20), F(7, 5)]]),
                               rtol=0, atol=1e-15)
    np.testing.assert_allclose(o1[0], _v([F(-59, 100), F(-7, 20)]), rtol=0, atol=1e-15)
    S2, o2 = impl.gdn_step(S1, _v([0, 1])[None], _v([1, 0])[None], _v([0, 1])[None],
                           _v([1]), _v([1]))
    np.testing.assert_allclose(S2[0], _fa([[0, F(34, 25)], [1, F(7, 5)]]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(o2[0], _v([F(34, 25), F(7, 5)]), rtol=0, atol=1e-15)


def pin_kda_hand(impl):
    # Same S0, k, q, v, beta as pin_gdn_hand; alpha = (1/2, 1/4) per key channel.
    # S0 Diag(alpha) = [[1/2, 1/2], [3/2, 1]]
    # times (I - beta k k^T): [[29/100, 22/100], [99/100, 32/100]]
    # plus beta v k^T:        S1 = [[89/100, 102/100], [129/100, 72/100]]
    # o1 = S1 (1, -1) = (-13/100, 57/100).
    # (Check by the delta form: P = S0 Diag(alpha), P k = (7/10, 17/10),
    #  u = beta (v - P k) = (13/20, -7/20), S1 = P + u k^T -- same matrix.)
    S = _fa([[1, 2], [3, 4]])[None]
    S1, o1 = impl.kda_step(S, _v([1, -1])[None], _v([F(3, 5), F(4, 5)])[None],
                           _v([2, 1])[None], _v([F(1, 2), F(1, 4)])[None], _v([F(1, 2)]))
    np.testing.assert_allclose(S1[0], _fa([[F(89, 100), F(102, 100)], [F(129, 100), F(72, 100)]]),
                               rtol=0, atol=1e-15)
    np.testing.assert_allclose(o1[0], _v([F(-13, 100), F(57, 100)]), rtol=0, atol=1e-15)


def pin_rwkv6_hand(impl):
    # Recurrence orientation (rows: key channel c, cols: value index j).
    # S0 = [[1,2],[3,4]], r = (1,2), k = (1,-1), v = (3,1), w = (1/2, 1/3), u = (2, 1/2).
    # k v^T = [[3,1],[-3,-1]],  diag(u) k v^T = [[6,2],[-3/2,-1/2]]
    # o1 = r^T (S0 + diag(u) k v^T) = r^T [[7,4],[3/2,7/2]] = (10, 11)
    # S1 = diag(w) S0 + k v^T = [[1/2,1],[1,4/3]] + [[3,1],[-3,-1]] = [[7/2, 2], [-2, 1/3]]
    S = _fa([[1, 2], [3, 4]])[None]
    S1, o1 = impl.rwkv6_step(S, _v([1, 2])[None], _v([1, -1])[None], _v([3, 1])[None],
                             _v([F(1, 2), F(1, 3)])[None], _v([2, F(1, 2)])[None])
    np.testing.assert_allclose(o1[0], _v([10, 11]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(S1[0], _fa([[F(7, 2), 2], [-2, F(1, 3)]]), rtol=0, atol=1e-15)


def pin_gdn2_hand(impl):
    # GDN-2, same S0, k, q, v as pin_kda_hand; alpha = (1/2, 1/4), erase gate
    # b = (1/2, 1/4), write gate w = (1, 1/2).
    # P = S0 Diag(alpha) = [[1/2, 1/2], [3/2, 1]];  b o k = (3/10, 1/5)
    # P (b o k) = (1/4, 13/20);  w o v = (2, 1/2);  u = w o v - P (b o k) = (7/4, -3/20)
    # S1 = P + u k^T = [[31/20, 19/10], [141/100, 22/25]],  o1 = S1 (1, -1) = (-7/20, 53/100).
    # (Check by the projection form: P (I - (b o k) k^T) = [[7/20, 3/10], [111/100, 12/25]],
    #  plus (w o v) k^T = [[6/5, 8/5], [3/10, 2/5]] -- same matrix.)
    S = _fa([[1, 2], [3, 4]])[None]
    S1, o1 = impl.gdn2_step(S, _v([1, -1])[None], _v([F(3, 5), F(4, 5)])[None], _v([2, 1])[None],
                            _v([F(1, 2), F(1, 4)])[None], _v([F(1, 2), F(1, 4)])[None],
                            _v([1, F(1, 2)])[None])
    np.testing.assert_allclose(S1[0], _fa([[F(31, 20), F(19, 10)], [F(141, 100), F(22, 25)]]),
                               rtol=0, atol=1e-15)
    np.testing.assert_allclose(o1[0], _v([F(-7, 20), F(53, 100)]), rtol=0, atol=1e-15)


# ------------------------------------------------------------- closed forms

def _unit(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def pin_beta_zero_is_pure_decay(impl):
    rng = np.random.default_rng(11)
    N, d, T = 3, 8, 5
    S0 = rng.standard_normal((N, d, d))
    # GDN: S_t = (prod alpha) S0 and o_t = S_t q_t
    S, prod = S0.copy(), np.ones(N)
    for _ in range(T):
        a = rng.uniform(0.5, 1.0, N)
        q = _unit(rng, N, d)
        S, o = impl.gdn_step(S, q, _unit(rng, N, d), rng.standard_normal((N, d)), a, np.zeros(N))
        prod *= a
        np.testing.assert_allclose(S, prod[:, None, None] * S0, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(o, np.einsum("nij,nj->ni", prod[:, None, None] * S0, q),
                                   rtol=1e-12, atol=1e-13)
    # KDA: S_t = S0 Diag(prod alpha)
    S, prod = S0.copy(), np.ones((N, d))
    for _ in range(T):
        a = rng.uniform(0.5, 1.0, (N, d))
        S, _ = impl.kda_step(S, _unit(rng, N, d), _unit(rng, N, d), rng.standard_normal((N, d)),
                             a, np.zeros(N))
        prod *= a
        np.testing.assert_allclose(S, S0 * prod[:, None, :], rtol=1e-13, atol=1e-14)


def pin_rwkv6_zero_keys_is_pure_decay(impl):
    rng = np.random.default_rng(12)
    N, d, T = 3, 8, 5
    S0 = rng.standard_normal((N, d, d))
    S, prod = S0.copy(), np.ones((N, d))
    u = rng.standard_normal((N, d))
    for _ in range(T):
        w = rng.uniform(0.3, 1.0, (N, d))
        r = rng.standard_normal((N, d))
        S_prev = S
        S, o = impl.rwkv6_step(S, r, np.zeros((N, d)), rng.standard_normal((N, d)), w, u)
        np.testing.assert_allclose(o, np.einsum("nc,ncj->nj", r, S_prev), rtol=1e-12, atol=1e-13)
        prod *= w
        np.testing.assert_allclose(S, prod[:, :, None] * S0, rtol=1e-13, atol=1e-14)


def pin_rwkv6_unit_decay_sums_outer_products(impl):
    rng = np.random.default_rng(13)
    N, dk, dv, T = 2, 6, 5, 6
    S0 = rng.standard_normal((N, dk, dv))
    S, acc = S0.copy(), S0.copy()
    for _ in range(T):
        r, k = rng.standard_normal((N, dk)), rng.standard_normal((N, dk))
        v = rng.standard_normal((N, dv))
        S_prev = acc.copy()
        S, o = impl.rwkv6_step(S, r, k, v, np.ones((N, dk)), np.zeros((N, dk)))
        acc = acc + k[:, :, None] * v[:, None, :]
        np.testing.assert_allclose(o, np.einsum("nc,ncj->nj", r, S_prev), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S, acc, rtol=1e-12, atol=1e-12)


def pin_exact_retrieval(impl):
    # alpha = 1, beta = 1, orthonormal keys: after writing (k_i, v_i), i = 1..n,
    # S_n k_i = v_i for every i, from any S0.
    rng = np.random.default_rng(14)
    N, d, n = 2, 8, 5
    S0 = rng.standard_normal((N, d, d))
    Q = np.stack([np.linalg.qr(rng.standard_normal((d, d)))[0] for _ in range(N)])  # columns orthonormal
    V = rng.standard_normal((N, n, d))
    for which in ("gdn", "kda"):
        S = S0.copy()
        for i in range(n):
            k = Q[:, :, i]
            q = _unit(rng, N, d)
            if which == "gdn":
                S, _ = impl.gdn_step(S, q, k, V[:, i], np.ones(N), np.ones(N))
            else:
                S, _ = impl.kda_step(S, q, k, V[:, i], np.ones((N, d)), np.ones(N))
        for i in range(n):
            np.testing.assert_allclose(np.einsum("nij,nj->ni", S, Q[:, :, i]), V[:, i],
                                       rtol=1e-11, atol=1e-11)


def pin_non_expansive_without_writes(impl):
    # v = 0, |k| = 1, beta in [0,1], alpha <= 1: (I - beta k k^T) is a
    # contraction and the write term vanishes, so |S|_F never grows; a
    # strictly positive beta with generic keys strictly shrinks it.
    rng = np.random.default_rng(15)
    N, d, T = 4, 8, 20
    for which in ("gdn", "kda"):
        S = rng.standard_normal((N, d, d))
        norm = np.linalg.norm(S, axis=(1, 2))
        first = norm.copy()
        for _ in range(T):
            k, q = _unit(rng, N, d), _unit(rng, N, d)
            beta = rng.uniform(0.1, 1.0, N)
            if which == "gdn":
                S, _ = impl.gdn_step(S, q, k, np.zeros((N, d)), rng.uniform(0.9, 1.0, N), beta)
            else:
                S, _ = impl.kda_step(S, q, k, np.zeros((N, d)), rng.uniform(0.9, 1.0, (N, d)), beta)
            new = np.linalg.norm(S, axis=(1, 2))
            assert np.all(new <= norm * (1 + 1e-12))
            norm = new
        assert np.all(norm < first * 0.99)


def pin_kda_constant_decay_is_gdn(impl):
    rng = np.random.default_rng(16)
    N, d, T = 3, 8, 6
    S_g = S_k = rng.standard_normal((N, d, d))
    for _ in range(T):
        q, k = _unit(rng, N, d), _unit(rng, N, d)
        v = rng.standard_normal((N, d))
        a, b = rng.uniform(0.8, 1.0, N), rng.uniform(0, 1, N)
        S_g, o_g = impl.gdn_step(S_g, q, k, v, a, b)
        S_k, o_k = impl.kda_step(S_k, q, k, v, np.repeat(a[:, None], d, axis=1), b)
        np.testing.assert_allclose(S_k, S_g, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(o_k, o_g, rtol=1e-12, atol=1e-13)


def pin_gdn2_equal_gates_is_kda(impl):
    # both gates the same scalar beta: GDN-2 is KDA (Gated DeltaNet-2 abstract)
    rng = np.random.default_rng(17)
    N, d, T = 3, 8, 6
    S_2 = S_k = rng.standard_normal((N, d, d))
    for _ in range(T):
        q, k = _unit(rng, N, d), _unit(rng, N, d)
        v = rng.standard_normal((N, d))
        a, b = rng.uniform(0.8, 1.0, (N, d)), rng.uniform(0, 1, N)
        gate = np.repeat(b[:, None], d, axis=1)
        S_2, o_2 = impl.gdn2_step(S_2, q, k, v, a, gate, gate)
        S_k, o_k = impl.kda_step(S_k, q, k, v, a, b)
        np.testing.assert_allclose(S_2, S_k, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(o_2, o_k, rtol=1e-12, atol=1e-13)


def pin_gdn2_open_erase_retrieves_gated_value(impl):
    # b = 1 and |k| = 1: the erase removes exactly what the decayed state
    # returns for k, so S_t k = w o v whatever S_{t-1} and alpha are
    rng = np.random.default_rng(18)
    N, dk, dv = 4, 6, 5
    S = rng.standard_normal((N, dv, dk))
    k = _unit(rng, N, dk)
    v, w = rng.standard_normal((N, dv)), rng.uniform(0, 1, (N, dv))
    S1, _ = impl.gdn2_step(S, _unit(rng, N, dk), k, v, rng.uniform(0.5, 1.0, (N, dk)),
                           np.ones((N, dk)), w)
    np.testing.assert_allclose(np.einsum("nvk,nk->nv", S1, k), w * v, rtol=1e-12, atol=1e-12)


def pin_gdn2_closed_gates_is_pure_decay(impl):
    # b = 0 and w = 0: no erase, no write, S_t = S_{t-1} Diag(alpha)
    rng = np.random.default_rng(19)
    N, dk, dv = 3, 5, 4
    S = rng.standard_normal((N, dv, dk))
    a = rng.uniform(0.5, 1.0, (N, dk))
    S1, o1 = impl.gdn2_step(S, _unit(rng, N, dk), _unit(rng, N, dk), rng.standard_normal((N, dv)),
                            a, np.zeros((N, dk)), np.zeros((N, dv)))
    np.testing.assert_allclose(S1, S * a[:, None, :], rtol=1e-14, atol=0)


# ------------------------------------------------- exact log form vs oracle

def _rat(rng, shape, den=8, lo=-8, hi=8):
    """Small random rationals (exact in binary floating point: den = 2^m)."""
    return np.vectorize(lambda n: F(int(n), den), otypes=[object])(rng.integers(lo, hi + 1, size=shape))


def _run_exact_vs_oracle(impl, variant, L, fill0, T, d=3, seed=0, merge_every_full=True):
    rng = np.random.default_rng(100 + seed)
    S0 = _rat(rng, (d, d))
    bonus = list(_rat(rng, (d,))) if variant == "rwkv6" else None
    dl = ExactDeltaLog(variant, S0.tolist(), L, fill0=fill0, bonus=bonus)
    # oracle orientation: RWKV6 uses d_k x d_v (transpose of the log form's)
    S_or = np.array(S0, dtype=np.float64)[None]
    if variant == "rwkv6":
        S_or = S_or.transpose(0, 2, 1).copy()
    for t in range(T):
        q = _rat(rng, (d,))
        k = _rat(rng, (d,))
        v = _rat(rng, (d,))
        if variant == "gdn":
            dec = F(int(rng.integers(5, 9)), 8)
        else:
            dec = list(np.vectorize(lambda n: F(int(n), 8), otypes=[object])(rng.integers(5, 9, size=d)))
        if variant == "gdn2":
            beta = list(_rat(rng, (d,), lo=0, hi=8))      # erase gate per key channel
            wgate = list(_rat(rng, (d,), lo=0, hi=8))     # write gate per value row
        else:
            beta = F(int(rng.integers(0, 9)), 8)
            wgate = None
        if dl.fill == L:
            dl.merge()
        o_ex = dl.step(list(q), list(k), list(v), dec, beta, wgate)
        f64 = lambda x: np.array(x, dtype=np.float64)[None]
        if variant == "gdn":
            S_or, o_or = impl.gdn_step(S_or, f64(q), f64(k), f64(v), np.array([float(dec)]),
                                       np.array([float(beta)]))
        elif variant == "kda":
            S_or, o_or = impl.kda_step(S_or, f64(q), f64(k), f64(v), f64(dec), np.array([float(beta)]))
        elif variant == "gdn2":
            S_or, o_or = impl.gdn2_step(S_or, f64(q), f64(k), f64(v), f64(dec), f64(beta), f64(wgate))
        else:
            S_or, o_or = impl.rwkv6_step(S_or, f64(q), f64(k), f64(v), f64(dec), f64(bonus))
        np.testing.assert_allclose(o_or[0], np.array(o_ex, dtype=np.float64), rtol=1e-12, atol=1e-12)
        dense = np.array(dl.dense(), dtype=np.float64)
        S_cmp = S_or[0].T if variant == "rwkv6" else S_or[0]
        np.testing.assert_allclose(S_cmp, dense, rtol=1e-12, atol=1e-12)


def pin_log_form_equals_oracle(impl):
    for variant in ("gdn", "kda", "rwkv6", "gdn2"):
        for (L, fill0, T) in ((4, 0, 9), (3, 2, 8), (1, 0, 4)):
            _run_exact_vs_oracle(impl, variant, L, fill0, T, seed=L * 10 + fill0)


PINS = [pin_gdn_hand, pin_kda_hand, pin_rwkv6_hand, pin_beta_zero_is_pure_decay,
        pin_rwkv6_zero_keys_is_pure_decay, pin_rwkv6_unit_decay_sums_outer_products,
        pin_exact_retrieval, pin_non_expansive_without_writes, pin_kda_constant_decay_is_gdn,
        pin_gdn2_hand, pin_gdn2_equal_gates_is_kda, pin_gdn2_open_erase_retrieves_gated_value,
        pin_gdn2_closed_gates_is_pure_decay, pin_log_form_equals_oracle]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(REAL)


def test_exact_log_form_merge_is_lossless():
    # merging (L = 1 .. 4) never changes the dense state, exactly
    rng = np.random.default_rng(7)
    for variant in ("gdn", "kda", "rwkv6"):
        d = 3
        S0 = _rat(rng, (d, d)).tolist()
        dl = ExactDeltaLog(variant, S0, L=4, bonus=list(_rat(rng, (d,))))
        for t in range(3):
            dec = F(3, 4) if variant == "gdn" else [F(3, 4), F(1, 2), F(7, 8)]
            dl.step(list(_rat(rng, (d,))), list(_rat(rng, (d,))), list(_rat(rng, (d,))), dec, F(1, 2))
        before = dl.dense()
        dl.merge()
        assert dl.fill == 0 and dl.dense() == before


def test_run_eager_matches_stepwise():
    # run_eager is the plain loop over the step functions with head selection
    rng = np.random.default_rng(3)
    B, H, d, T = 2, 3, 4, 4

    class St:
        pass

    steps = []
    for _ in range(T):
        s = St()
        s.q, s.k = rng.standard_normal((B, H, d)), rng.standard_normal((B, H, d))
        s.v = rng.standard_normal((B, H, d))
        s.decay, s.beta = rng.uniform(0.8, 1, (B, H)), rng.uniform(0, 1, (B, H))
        steps.append(s)
    S0 = rng.standard_normal((B * H, d, d))
    heads = np.array([1, 4])
    res = oracle.run_eager("gdn", S0[heads], steps, heads=heads, snapshot_at=[2])
    S = S0[heads]
    for n, s in enumerate(steps, 1):
        S, o = rec.gdn_step(S, s.q.reshape(-1, d)[heads], s.k.reshape(-1, d)[heads],
                            s.v.reshape(-1, d)[heads], s.decay.reshape(-1)[heads],
                            s.beta.reshape(-1)[heads])
        np.testing.assert_array_equal(res.outputs[n - 1], o)
        if n == 2:
            np.testing.assert_array_equal(res.states[2], S)
    np.testing.assert_array_equal(res.S, S)


# ------------------------------------------------------------- KLA step size

def test_kla_beta_hand_example():
    # k = (1, 2): |k|^2 = 5, so beta = eta / (5 + eps); eta = 1/2, eps = 1/4
    # gives beta = (1/2) / (21/4) = 2/21.
    b = rec.kla_beta(np.array([0.5]), np.array([[1.0, 2.0]]), 0.25)
    assert b[0] == pytest.approx(2.0 / 21.0, rel=1e-15)


def test_kla_write_is_a_kaczmarz_projection():
    # alpha = 1, eta = 1, eps = 0: beta |k|^2 = 1, so after each write the
    # state maps k_t exactly to v_t whatever the key's norm (GDN and KDA).
    rng = np.random.default_rng(21)
    N, d = 3, 8
    for which in ("gdn", "kda"):
        S = rng.standard_normal((N, d, d))
        for _ in range(6):
            k = rng.standard_normal((N, d)) * rng.uniform(0.2, 3.0, (N, 1))
            v = rng.standard_normal((N, d))
            beta = rec.kla_beta(np.ones(N), k, 0.0)
            if which == "gdn":
                S, _ = rec.gdn_step(S, rng.standard_normal((N, d)), k, v, np.ones(N), beta)
            else:
                S, _ = rec.kda_step(S, rng.standard_normal((N, d)), k, v, np.ones((N, d)), beta)
            np.testing.assert_allclose(np.einsum("nij,nj->ni", S, k), v, rtol=1e-11, atol=1e-11)


def test_run_eager_kla_uses_key_norms():
    rng = np.random.default_rng(22)
    B, H, d, T = 1, 2, 4, 3

    class St:
        pass

    steps = []
    for _ in range(T):
        s = St()
        s.q, s.k = rng.standard_normal((B, H, d)), rng.standard_normal((B, H, d))
        s.v = rng.standard_normal((B, H, d))
        s.decay, s.beta = rng.uniform(0.8, 1, (B, H)), rng.uniform(0, 1, (B, H))
        steps.append(s)
    S0 = rng.standard_normal((B * H, d, d))
    res = oracle.run_eager("gdn", S0, steps, kla_eps=1e-3)
    S = S0
    for s in steps:
        k = s.k.reshape(-1, d)
        beta = s.beta.reshape(-1) / (np.sum(k * k, axis=1) + 1e-3)
        S, o = rec.gdn_step(S, s.q.reshape(-1, d), k, s.v.reshape(-1, d), s.decay.reshape(-1), beta)
    np.testing.assert_allclose(res.S, S, rtol=1e-13, atol=1e-13)
