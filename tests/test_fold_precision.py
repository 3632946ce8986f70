"""The precision budget of the int8 step's direct GDN fold, on the CPU.

That fold (GDN with bf16 keys) forms U Kt as (U Diag(fac)) K on bf16
tensor-core MMAs: each decayed log value x = u * fac enters as the bf16 pair
hi = bf16(x), lo = bf16(x - hi), the stored bf16 keys enter exactly, the
products are exact and the sums run in fp32.  This test emulates that
arithmetic with numpy (bf16 as round-to-nearest-even on the top 16 bits of
fp32) and checks it against fp64 at the state tolerance's scale: the split
carries 16 significant bits, so the fold's error stays near 2^-17 of the
correction, far inside the 1e-4 bar the GPU parity tests hold the merged
state to.  It touches neither the oracle nor the CUDA path.
"""

import numpy as np

STATE_TOL = 1e-4


def bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 (ties to even) -> fp32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return r.astype(np.uint32).view(np.float32)


def direct_fold(u: np.ndarray, fac: np.ndarray, k_bf16: np.ndarray) -> np.ndarray:
    """u [rows, n], fac [n], k_bf16 [n, d] (already bf16) -> U Diag(fac) K as the fold forms it."""
    x = (u.astype(np.float32) * fac.astype(np.float32)).astype(np.float32)
    hi = bf16(x)
    lo = bf16((x - hi).astype(np.float32))
    k = k_bf16.astype(np.float32)
    # exact products, fp32 sums (one accumulation order; the MMA's differs only by fp32 rounding)
    return (hi @ k).astype(np.float32) + (lo @ k).astype(np.float32)


def test_bf16_round_trip():
    # bf16 keeps 7 explicit mantissa bits: spacing 2^-7 at 1
    x = np.array([1.0 + 2 ** -7, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5],
                 dtype=np.float32)
    y = bf16(x)
    assert y[0] == np.float32(1.0 + 2 ** -7)    # representable
    assert y[1] == 1.0                          # tie between mantissas 0 and 1: to even (0)
    assert y[2] == np.float32(1.0 + 2 ** -6)    # tie between mantissas 1 and 2: to even (2)
    assert y[3] == 1.0                          # below the tie
    assert y[4] == -2.5


def test_direct_fold_error_budget():
    rng = np.random.default_rng(7)
    rows, d = 128, 128
    for n in (1, 16, 64):
        u = rng.normal(0.0, 0.5, size=(rows, n))
        g = np.cumsum(np.log(rng.uniform(0.9, 1.0, size=n)))
        fac = np.exp(g[-1] - g)                                  # decays to the last entry
        k = rng.normal(0.0, 1.0, size=(n, d))
        k /= np.linalg.norm(k, axis=1, keepdims=True)
        k_b = bf16(k.astype(np.float32))                         # the log stores bf16 keys
        exact = (u * fac) @ k_b.astype(np.float64)
        got = direct_fold(u, fac, k_b).astype(np.float64)
        err = np.abs(got - exact).max() / np.abs(exact).max()
        assert err < 2e-5, (n, err)
        assert err < STATE_TOL / 5


def test_hi_alone_would_not_do():
    # the lo half is what the budget rests on: bf16(x) alone misses it by far
    rng = np.random.default_rng(8)
    u = rng.normal(0.0, 0.5, size=(128, 16))
    fac = np.ones(16)
    k_b = bf16(rng.normal(0.0, 0.3, size=(16, 128)).astype(np.float32))
    exact = u @ k_b.astype(np.float64)
    hi_only = bf16(u.astype(np.float32)).astype(np.float64) @ k_b.astype(np.float64)
    assert np.abs(hi_only - exact).max() / np.abs(exact).max() > STATE_TOL
