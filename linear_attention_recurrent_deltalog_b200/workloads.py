"""Seeded synthetic decode workloads for DeltaLog.

This module only draws random numbers and rounds them to the element type a
kernel receives.  It holds none of the recurrence's arithmetic, so it serves
both the fp64 oracle and the CUDA path without coupling them.

The five workloads follow the decode settings named for DeltaLog ("DeltaLog:
Deferred Materialization of Recurrent States for Linear Attention Decoding",
Abstract: GDN, KDA and RWKV6 decoding with batched per-head recurrent states).
The pages print no sizes, so the sizes below are the synthetic stand-ins this
library is measured on:

  gdn_tiny      GDN   B=1   H=2  d=64  T=32   L=8   fp32 inputs
  gdn_qwen      GDN   B=64  H=32 d=128 T=256  L=16  bf16 q/k/v
  kda           KDA   B=128 H=32 d=128 T=256  L=16  bf16 q/k/v, per-channel decay
  gdn2          GDN-2 B=128 H=32 d=128 T=256  L=16  as kda, plus per-channel erase
                                                    and write gates
  rwkv6         RWKV6 B=256 H=64 d=64  T=512  L=32  bf16 r/k/v, u-bonus per head
  gdn_serving   GDN   B=512 H=32 d=128 T=1024 L in {4,8,16,32,64}, ragged fills

Draw recipe (fixed, so any single step can be regenerated on its own):
  * step t uses numpy ``Generator(PCG64(SeedSequence([seed, 1, t])))`` and
    draws, in order, q (or r), k, v, decay, beta, each shaped [B, H, .] in
    C order (beta is not drawn for RWKV6; with the KLA step size the beta
    draw is the gate eta and q, k are scaled by 1/sqrt(d_k), not normalised;
    GDN-2 draws the erase gate b = sigmoid(N(0,1)) [B, H, d_k] in beta's
    place and then the write gate w = sigmoid(N(0,1)) [B, H, d_v]);
  * the initial state S0 uses ``SeedSequence([seed, 0, 0])``: fp32 N(0, 1)
    scaled by 0.01 (the "N(0, 0.01)" of the configs read as a standard
    deviation), shaped [B, H, d_v, d_k];
  * ragged fill offsets use ``SeedSequence([seed, 0, 1])``: integers
    U{0..L-1} per sequence;
  * the RWKV6 bonus u uses ``SeedSequence([seed, 0, 2])``: N(0, 0.5) of
    shape [H, d_k], fixed for the run.
Gaussians are drawn in float64, L2 normalisation (q, k of GDN/KDA) is done in
float64 with no epsilon, values are rounded to fp32 by round-to-nearest-even
and, for bf16 inputs, from fp32 to bf16 by round-to-nearest-even.
"""

from __future__ import annotations

import dataclasses
from typing import Iterator, Optional

import numpy as np

GDN = "gdn"
KDA = "kda"
RWKV6 = "rwkv6"
GDN2 = "gdn2"
VARIANTS = (GDN, KDA, RWKV6, GDN2)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode workload: sizes, dtypes and the seed."""

    name: str
    variant: str
    B: int
    H: int
    d_k: int
    d_v: int
    T: int
    L: int
    in_dtype: str  # "f32" or "bf16": type of q/r, k and v as the kernel sees them
    seed: int
    ragged: bool = False  # sequences start at fill offsets U{0..L-1}
    alpha_kind: str = "softplus"  # GDN scalar decay recipe: "uniform" or "softplus"
    s0_std: float = 0.01
    # KLA (Kaczmarz step size): q and k are scaled by 1/sqrt(d_k) instead of
    # L2-normalised, and the beta draw is the gate eta; None: plain GDN/KDA.
    kla_eps: Optional[float] = None

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def decay_is_vector(self) -> bool:
        return self.variant in (KDA, RWKV6, GDN2)

    @property
    def heads(self) -> int:
        return self.B * self.H


WORKLOADS = {
    "gdn_tiny": Workload("gdn_tiny", GDN, 1, 2, 64, 64, 32, 8, "f32", 1,
                         alpha_kind="uniform"),
    "gdn_qwen": Workload("gdn_qwen", GDN, 64, 32, 128, 128, 256, 16, "bf16", 2),
    "kda": Workload("kda", KDA, 128, 32, 128, 128, 256, 16, "bf16", 3),
    "rwkv6": Workload("rwkv6", RWKV6, 256, 64, 64, 64, 512, 32, "bf16", 4),
    "gdn2": Workload("gdn2", GDN2, 128, 32, 128, 128, 256, 16, "bf16", 6),
    "gdn_serving": Workload("gdn_serving", GDN, 512, 32, 128, 128, 1024, 16,
                            "bf16", 5, ragged=True),
}
SERVING_L_SWEEP = (4, 8, 16, 32, 64)


# ----------------------------------------------------------------- rounding

def round_f32(x: np.ndarray) -> np.ndarray:
    """float64 -> float32, round-to-nearest-even (numpy's cast)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def bf16_bits(x32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round-to-nearest-even.

    Finite inputs only (the generators never produce inf/nan).
    """
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> the exactly equal fp32 values."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_bf16(x32: np.ndarray) -> np.ndarray:
    """fp32 -> fp32 values that are exactly bf16-representable (RNE)."""
    return bf16_to_f32(bf16_bits(x32))


# ----------------------------------------------------------------- step data

@dataclasses.dataclass
class StepInputs:
    """One decode step's inputs, exact values as fp32 host arrays.

    ``q`` holds r for RWKV6.  For bf16 workloads every value of q/k/v is
    exactly bf16-representable; ``device_bits`` gives the bit patterns.
    ``decay`` is [B,H] (GDN alpha) or [B,H,d_k] (KDA and GDN-2 alpha, RWKV6
    w); ``beta`` is [B,H], the GDN-2 erase gate [B,H,d_k], or None (RWKV6);
    ``wgate`` is the GDN-2 write gate [B,H,d_v], None otherwise.
    """

    t: int
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    decay: np.ndarray
    beta: Optional[np.ndarray]
    in_dtype: str
    wgate: Optional[np.ndarray] = None

    def device_array(self, name: str) -> np.ndarray:
        """q/k/v as the kernel reads them: uint16 bf16 bits or fp32."""
        x = getattr(self, name)
        return bf16_bits(x) if self.in_dtype == "bf16" else x


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _to_in_dtype(x64: np.ndarray, in_dtype: str) -> np.ndarray:
    x32 = round_f32(x64)
    return round_bf16(x32) if in_dtype == "bf16" else x32


def _l2norm(x64: np.ndarray) -> np.ndarray:
    return x64 / np.sqrt(np.sum(x64 * x64, axis=-1, keepdims=True))


def step_inputs(w: Workload, t: int, B: Optional[int] = None) -> StepInputs:
    """Inputs of decode step ``t`` (0-based).

    ``B`` may restrict the draw to the first B sequences only when the caller
    knows it wants a prefix; the values of a prefix differ from the full draw
    (the draw shape changes), so tests always generate the full batch.
    """
    B = w.B if B is None else B
    H, dk, dv = w.H, w.d_k, w.d_v
    g = _rng(w.seed, 1, t)
    if w.variant == RWKV6:
        r = g.standard_normal((B, H, dk))
        k = g.standard_normal((B, H, dk))
        v = g.standard_normal((B, H, dv))
        wdec = np.exp(-np.exp(g.normal(-1.0, 0.5, size=(B, H, dk))))
        return StepInputs(t, _to_in_dtype(r, w.in_dtype), _to_in_dtype(k, w.in_dtype),
                          _to_in_dtype(v, w.in_dtype), round_f32(wdec), None, w.in_dtype)
    if w.kla_eps is None:
        q = _l2norm(g.standard_normal((B, H, dk)))
        k = _l2norm(g.standard_normal((B, H, dk)))
    else:
        q = g.standard_normal((B, H, dk)) / np.sqrt(dk)
        k = g.standard_normal((B, H, dk)) / np.sqrt(dk)
    v = g.standard_normal((B, H, dv))
    if w.variant == GDN:
        if w.alpha_kind == "uniform":
            alpha = g.uniform(0.90, 1.00, size=(B, H))
        else:
            x = g.standard_normal((B, H))
            alpha = np.exp(-np.logaddexp(0.0, x) * 0.1)  # exp(-softplus(x) * 0.1)
    else:  # KDA, GDN-2: per-key-channel decay
        alpha = g.uniform(0.80, 1.00, size=(B, H, dk))
    if w.variant == GDN2:
        bgate = 1.0 / (1.0 + np.exp(-g.standard_normal((B, H, dk))))
        wgate = 1.0 / (1.0 + np.exp(-g.standard_normal((B, H, dv))))
        return StepInputs(t, _to_in_dtype(q, w.in_dtype), _to_in_dtype(k, w.in_dtype),
                          _to_in_dtype(v, w.in_dtype), round_f32(alpha), round_f32(bgate),
                          w.in_dtype, round_f32(wgate))
    beta = 1.0 / (1.0 + np.exp(-g.standard_normal((B, H))))
    return StepInputs(t, _to_in_dtype(q, w.in_dtype), _to_in_dtype(k, w.in_dtype),
                      _to_in_dtype(v, w.in_dtype), round_f32(alpha), round_f32(beta),
                      w.in_dtype)


def iter_steps(w: Workload, T: Optional[int] = None, start: int = 0) -> Iterator[StepInputs]:
    T = w.T if T is None else T
    for t in range(start, start + T):
        yield step_inputs(w, t)


def initial_state(w: Workload) -> np.ndarray:
    """S0 as fp32 [B, H, d_v, d_k] (for RWKV6 this is the transpose of the
    d_k x d_v matrix of its recurrence; the draw itself is the same)."""
    g = _rng(w.seed, 0, 0)
    s = g.standard_normal((w.B, w.H, w.d_v, w.d_k), dtype=np.float32)
    return (s * np.float32(w.s0_std)).astype(np.float32)


def fill_offsets(w: Workload) -> np.ndarray:
    """Per-sequence initial log fill (int32 [B]); zeros unless ragged."""
    if not w.ragged:
        return np.zeros(w.B, dtype=np.int32)
    g = _rng(w.seed, 0, 1)
    return g.integers(0, w.L, size=w.B).astype(np.int32)


def rwkv6_bonus(w: Workload) -> np.ndarray:
    """The fixed per-head RWKV6 bonus u, fp32 [H, d_k]."""
    g = _rng(w.seed, 0, 2)
    return round_f32(g.normal(0.0, 0.5, size=(w.H, w.d_k)))


def sample_heads(w: Workload, n: int, seed: int = 0) -> np.ndarray:
    """A seeded sample of flat head indices (b*H + h), sorted, without
    replacement; used where a check covers a subset of a large batch."""
    n = min(n, w.heads)
    g = _rng(w.seed, 0, 3 + seed)
    return np.sort(g.choice(w.heads, size=n, replace=False)).astype(np.int64)


# ----------------------------------------------------------------- prefetch

def _step_job(args):
    w, t = args
    return step_inputs(w, t)


class StepStream:
    """Yields step_inputs(w, t) for t in [start, start + T) in order,
    drawing ahead in a pool of worker processes started with ``spawn`` (safe
    after CUDA is initialised in the parent).  ``workers=0`` draws inline."""

    def __init__(self, w: Workload, T: Optional[int] = None, start: int = 0,
                 workers: Optional[int] = None, ahead: int = 0):
        import os
        self.w = w
        self.T = w.T if T is None else T
        self.start = start
        if workers is None:
            workers = min(16, max(0, (os.cpu_count() or 1) - 1))
        self.workers = workers if self.T > 4 else 0
        self.ahead = ahead or 2 * max(1, self.workers)

    def __iter__(self) -> Iterator[StepInputs]:
        if self.workers <= 0:
            yield from iter_steps(self.w, self.T, self.start)
            return
        import collections
        import concurrent.futures as cf
        import multiprocessing as mp
        ctx = mp.get_context("spawn")
        with cf.ProcessPoolExecutor(max_workers=self.workers, mp_context=ctx) as ex:
            pending = collections.deque()
            nxt = self.start
            end = self.start + self.T
            while nxt < end and len(pending) < self.ahead:
                pending.append(ex.submit(_step_job, (self.w, nxt)))
                nxt += 1
            while pending:
                s = pending.popleft().result()
                if nxt < end:
                    pending.append(ex.submit(_step_job, (self.w, nxt)))
                    nxt += 1
                yield s
