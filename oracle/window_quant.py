"""Per-window state quantization: the eager recurrence with a low-bit base.

TEST INFRASTRUCTURE: only tests, the smoke check and the benchmark's CPU
baseline call this module.  Nothing here is shared with the CUDA path.

What it computes ("LeapQuant" page, Abstract): the recurrent state is
quantized only once per window of tokens, at the window's end; inside a
window the outputs come from that fixed low-bit state plus the window's own
updates kept in high precision.  With DeltaLog's log as the high-precision
buffer, a window is the stretch between two merges of a sequence's log, so
the definition is:

    S <- deq(Q(S0)) at the start;
    every step: S, o_t <- the eager step (GDN / KDA / GDN-2 / RWKV6) on S;
    after a step that ends the sequence's window: S <- deq(Q(S)).

A window ends when the step's append fills the log (L entries, counting the
fill offset a sequence starts with), or when a merge of every non-empty log
is forced.  Between window ends the state evolves in fp64, exactly as the
eager oracle does: a low-bit base plus a high-precision log equals the eager
recurrence started from the dequantized base.

Readings (the pages give only "8-bit" and "per-window"):
  * Q is symmetric int8 with one scale per value row of the d_v x d_k state
    (row j = value index, the axis a base GEMV row reduces over is the key
    axis, so the scale factors out of each row's dot product):
        amax_j  = max_c |x_jc|
        inv_j   = 127 / amax_j
        code_jc = round-half-even(x_jc * inv_j), in [-127, 127]
        scale_j = amax_j / 127
    deq(code, scale)_jc = code_jc * scale_j.
  * The decision arithmetic is fp32 (the kernel's precision): x is first
    rounded to fp32, and inv, the product and scale are each one correctly
    rounded fp32 operation.  A row whose amax is below 2^-120 (where 127/amax
    could overflow fp32) is stored as zero codes with scale 0.
  * RWKV6's state is quantized in the library's orientation (d_v x d_k, the
    transpose of the recurrence's d_k x d_v), so rows are value indices for
    every variant.
  * The outlier "Compensator Tokens" and residual smoothing of the same
    abstract are not part of this definition.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Iterable, List, Optional, Sequence

import numpy as np

from .recurrence import gdn2_step, gdn_step, kda_step, kla_beta, rwkv6_step

TINY_AMAX = np.float32(2.0 ** -120)


def quantize_rows(X):
    """Q: rows of X (last axis = key index) -> (codes int8, scales fp32).

    X [..., d_v, d_k] (any float dtype); codes [..., d_v, d_k], scales
    [..., d_v].  See the module docstring for the arithmetic.
    """
    x = np.asarray(X).astype(np.float32)
    amax = np.max(np.abs(x), axis=-1)
    live = amax >= TINY_AMAX
    safe = np.where(live, amax, np.float32(1.0)).astype(np.float32)
    inv = (np.float32(127.0) / safe).astype(np.float32)
    prod = (x * inv[..., None]).astype(np.float32)
    codes = np.clip(np.rint(prod), -127, 127)
    codes = np.where(live[..., None], codes, 0).astype(np.int8)
    scales = np.where(live, (amax / np.float32(127.0)).astype(np.float32),
                      np.float32(0.0)).astype(np.float32)
    return codes, scales


def row_inverse(X):
    """The fp32 inv_j = 127 / amax_j Q uses for each row (0 for zero rows)."""
    x = np.asarray(X).astype(np.float32)
    amax = np.max(np.abs(x), axis=-1)
    live = amax >= TINY_AMAX
    safe = np.where(live, amax, np.float32(1.0)).astype(np.float32)
    return np.where(live, np.float32(127.0) / safe, np.float32(0.0)).astype(np.float32)


def dequantize_rows(codes, scales):
    """deq: code * scale, one fp32 product per element, returned as fp64."""
    c = np.asarray(codes).astype(np.float32)
    s = np.asarray(scales).astype(np.float32)
    return (c * s[..., None]).astype(np.float32).astype(np.float64)


def _to_rows(S, rec):
    """Recurrence orientation -> library orientation (rows = value index)."""
    return np.swapaxes(S, -1, -2) if rec else S


def requantize(S, rec):
    """deq(Q(S)) for states in the recurrence's orientation; also returns
    (codes, scales, pre) in the library orientation, pre = the fp64 values
    that were quantized."""
    pre = _to_rows(np.asarray(S, dtype=np.float64), rec)
    codes, scales = quantize_rows(pre)
    deq = dequantize_rows(codes, scales)
    return _to_rows(deq, rec).copy(), codes, scales, pre.copy()


@dataclasses.dataclass
class WindowEnd:
    step: int                 # 1-based step after which the window ended
    heads: np.ndarray         # selected-head indices (into the N heads run)
    codes: np.ndarray         # int8 [n, d_v, d_k] (library orientation)
    scales: np.ndarray        # fp32 [n, d_v]
    pre: np.ndarray           # fp64 [n, d_v, d_k], the values quantized


@dataclasses.dataclass
class WindowedResult:
    S: np.ndarray                     # final state (fp64, recurrence orientation)
    outputs: List[np.ndarray]         # o_t per step, fp64 [N, d_v]
    ends: List[WindowEnd]             # every window end, in order
    start_codes: np.ndarray           # Q(S0): int8 [N, d_v, d_k]
    start_scales: np.ndarray          # fp32 [N, d_v]
    states: Dict[int, np.ndarray]     # step -> state snapshot (if requested)


def _select(x, heads):
    x = np.asarray(x)
    flat = x.reshape((-1,) + x.shape[2:])
    return flat if heads is None else flat[heads]


def run_windowed(variant: str, S0, steps: Iterable, L: int, fill0, H: int,
                 heads: Optional[Sequence[int]] = None, bonus=None,
                 merge_all_after: Sequence[int] = (), snapshot_at: Sequence[int] = (),
                 kla_eps: Optional[float] = None) -> WindowedResult:
    """The eager recurrence with the state requantized at every window end.

    ``S0`` [N, ...] in the recurrence's orientation for the selected heads
    (RWKV6: d_k x d_v); ``steps`` and ``heads`` as in ``run_eager``; ``H``:
    heads per sequence, so selected flat head n belongs to sequence
    heads[n] // H.  ``fill0``: per-sequence log entries at the start (one int
    per sequence of the batch).  ``merge_all_after``: 1-based step counts
    after which every non-empty log is merged (and so its window ends).
    """
    rec = variant == "rwkv6"
    S0 = np.asarray(S0, dtype=np.float64)
    N = S0.shape[0]
    flat_heads = np.arange(N) if heads is None else np.asarray(heads)
    seq = flat_heads // H
    fill = np.asarray(fill0, dtype=np.int64)[seq].copy()
    S, c0, s0, _ = requantize(S0, rec)
    outs: List[np.ndarray] = []
    ends: List[WindowEnd] = []
    snaps: Dict[int, np.ndarray] = {}
    forced = set(int(x) for x in merge_all_after)
    want = set(int(x) for x in snapshot_at)
    for n, st in enumerate(steps, start=1):
        q = _select(st.q, heads)
        k = _select(st.k, heads)
        v = _select(st.v, heads)
        dec = _select(st.decay, heads)
        beta = None if st.beta is None else _select(st.beta, heads)
        if kla_eps is not None and variant in ("gdn", "kda"):
            beta = kla_beta(beta, k, kla_eps)
        if variant == "gdn":
            S, o = gdn_step(S, q, k, v, dec, beta)
        elif variant == "kda":
            S, o = kda_step(S, q, k, v, dec, beta)
        elif variant == "gdn2":
            S, o = gdn2_step(S, q, k, v, dec, beta, _select(st.wgate, heads))
        elif variant == "rwkv6":
            S, o = rwkv6_step(S, q, k, v, dec, bonus)
        else:
            raise ValueError(f"unknown variant {variant!r}")
        outs.append(o)
        fill += 1
        done = fill == L
        if n in forced:
            done = fill > 0
        idx = np.nonzero(done)[0]
        if idx.size:
            deq, codes, scales, pre = requantize(S[idx], rec)
            S[idx] = deq
            fill[idx] = 0
            ends.append(WindowEnd(n, idx, codes, scales, pre))
        if n in want:
            snaps[n] = S.copy()
    return WindowedResult(S, outs, ends, c0, s0, snaps)
