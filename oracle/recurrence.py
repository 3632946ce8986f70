"""Eager fp64 recurrences: the definition DeltaLog must reproduce.

TEST INFRASTRUCTURE: only tests, the smoke check and the benchmark's CPU
baseline call this module.  Nothing here is shared with the CUDA path.

Every function works on a stack of N independent heads and follows the
recurrence exactly as written, forming the matrices the formula names
(no algebraic shortcuts, no blocking, no reordering):

* GDN (gated delta rule; "DeltaLog" page, Abstract names GDN; the gated
  decay plus delta-rule residual write is the GDN description on the KLA
  abstract of the same pages):
      S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
      o_t = S_t q_t,
  with S of shape d_v x d_k, alpha_t and beta_t scalars per head.

* KDA (the same delta rule with channel-wise decay; the Gated DeltaNet-2
  abstract credits KDA with a decay per key channel, which makes its
  forgetting finer than GDN's one scalar):
      S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
      o_t = S_t q_t,
  alpha_t a vector over the d_k key channels.  The decay acts on the key
  axis before the delta read, so a constant alpha vector gives GDN exactly.

* RWKV6 (diagonal decay, plain writes, bonus readout):
      S_t = diag(w_t) S_{t-1} + k_t v_t^T,
      o_t = r_t^T (S_{t-1} + diag(u) k_t v_t^T),
  with S of shape d_k x d_v (this orientation is the recurrence's own; the
  library stores the transpose), w_t a d_k vector, u a fixed d_k vector per
  head.  The readout uses the state before the update.

* GDN-2 (Gated DeltaNet-2 abstract: a channel-wise erase gate b_t on the
  key side and a channel-wise write gate w_t on the value side replace the
  delta rule's single beta; it reduces to KDA when both gates are the same
  scalar):
      S_t = S_{t-1} Diag(alpha_t) (I - (b_t o k_t) k_t^T) + (w_t o v_t) k_t^T,
      o_t = S_t q_t,
  alpha_t and b_t vectors over the d_k key channels, w_t over the d_v value
  rows.  The erase reads the decayed state through the gated key b_t o k_t
  and removes it along k_t, so every step stays a rank-1 update in k_t.

* KLA (Kaczmarz step size; "Kaczmarz Linear Attention" abstract): the GDN
  (or KDA) recurrence with beta_t formed from a gate eta_t and the key norm,
      beta_t = eta_t / (|k_t|_2^2 + eps),
  so the write is a Kaczmarz projection: with alpha_t = 1 and eta_t = 1,
  eps = 0, the updated state maps k_t exactly to v_t whatever |k_t| is.

Outputs are float64.  Inputs are widened exactly from whatever the kernel
received (fp32 or bf16 values), so input rounding is not counted as error.
"""

from __future__ import annotations

import dataclasses
from typing import Iterable, List, Optional, Sequence

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def gdn_step(S, q, k, v, alpha, beta):
    """One GDN step for N heads.

    S [N, d_v, d_k]; q, k [N, d_k]; v [N, d_v]; alpha, beta [N].
    Returns (S_t, o_t) with o_t [N, d_v].
    """
    S, q, k, v = _f64(S), _f64(q), _f64(k), _f64(v)
    alpha, beta = _f64(alpha), _f64(beta)
    dk = k.shape[-1]
    eye = np.eye(dk)[None, :, :]
    kkT = k[:, :, None] * k[:, None, :]                      # k k^T  [N, dk, dk]
    proj = eye - beta[:, None, None] * kkT                    # I - beta k k^T
    write = beta[:, None, None] * (v[:, :, None] * k[:, None, :])  # beta v k^T
    S_new = alpha[:, None, None] * (S @ proj) + write
    o = (S_new @ q[:, :, None])[:, :, 0]
    return S_new, o


def kda_step(S, q, k, v, alpha, beta):
    """One KDA step for N heads.

    S [N, d_v, d_k]; q, k [N, d_k]; v [N, d_v]; alpha [N, d_k]; beta [N].
    """
    S, q, k, v = _f64(S), _f64(q), _f64(k), _f64(v)
    alpha, beta = _f64(alpha), _f64(beta)
    dk = k.shape[-1]
    eye = np.eye(dk)[None, :, :]
    diag_alpha = alpha[:, :, None] * eye                      # Diag(alpha) [N, dk, dk]
    kkT = k[:, :, None] * k[:, None, :]
    proj = eye - beta[:, None, None] * kkT
    write = beta[:, None, None] * (v[:, :, None] * k[:, None, :])
    S_new = (S @ diag_alpha) @ proj + write
    o = (S_new @ q[:, :, None])[:, :, 0]
    return S_new, o


def gdn2_step(S, q, k, v, alpha, b, w):
    """One GDN-2 step for N heads.

    S [N, d_v, d_k]; q, k [N, d_k]; v [N, d_v]; alpha, b [N, d_k] (decay and
    erase gate per key channel); w [N, d_v] (write gate per value row).
    """
    S, q, k, v = _f64(S), _f64(q), _f64(k), _f64(v)
    alpha, b, w = _f64(alpha), _f64(b), _f64(w)
    dk = k.shape[-1]
    eye = np.eye(dk)[None, :, :]
    diag_alpha = alpha[:, :, None] * eye                      # Diag(alpha)
    erase = eye - (b * k)[:, :, None] * k[:, None, :]         # I - (b o k) k^T
    write = (w * v)[:, :, None] * k[:, None, :]               # (w o v) k^T
    S_new = (S @ diag_alpha) @ erase + write
    o = (S_new @ q[:, :, None])[:, :, 0]
    return S_new, o


def rwkv6_step(S, r, k, v, w, u):
    """One RWKV6 step for N heads.

    S [N, d_k, d_v] (the recurrence's orientation); r, k, w, u [N, d_k];
    v [N, d_v].  Returns (S_t, o_t), o_t = r^T (S_{t-1} + diag(u) k v^T).
    """
    S, r, k, v = _f64(S), _f64(r), _f64(k), _f64(v)
    w, u = _f64(w), _f64(u)
    dk = k.shape[-1]
    eye = np.eye(dk)[None, :, :]
    kvT = k[:, :, None] * v[:, None, :]                       # k v^T  [N, dk, dv]
    bonus = (u[:, :, None] * eye) @ kvT                       # diag(u) k v^T
    o = (r[:, None, :] @ (S + bonus))[:, 0, :]
    S_new = (w[:, :, None] * eye) @ S + kvT                   # diag(w) S + k v^T
    return S_new, o


def kla_beta(eta, k, eps):
    """KLA step size beta_t = eta_t / (|k_t|_2^2 + eps) for N heads.

    eta [N]; k [N, d_k]; eps a scalar.
    """
    eta, k = _f64(eta), _f64(k)
    return eta / (np.sum(k * k, axis=-1) + float(eps))


@dataclasses.dataclass
class EagerResult:
    S: np.ndarray                 # final state, float64, recurrence orientation
    outputs: List[np.ndarray]     # o_t for each step (float64 [N, d_v])
    states: dict                  # step index -> state snapshot (if requested)


def _select(x, heads):
    """[B, H, ...] -> [N, ...] for the chosen flat head indices."""
    x = np.asarray(x)
    flat = x.reshape((-1,) + x.shape[2:])
    return flat if heads is None else flat[heads]


def run_eager(variant: str, S0, steps: Iterable, heads: Optional[Sequence[int]] = None,
              bonus=None, snapshot_at: Sequence[int] = (), kla_eps: Optional[float] = None
              ) -> EagerResult:
    """Run the eager recurrence over ``steps``.

    ``S0``: float array [N, ...] in the recurrence's orientation for the
    selected heads.  ``steps``: objects with fields q (r for RWKV6), k, v,
    decay and beta (GDN-2: the erase gate b), and for GDN-2 wgate, each shaped
    [B, H, ...]; ``heads`` picks N flat
    (b*H + h) heads from them (all heads when None).  ``bonus``: RWKV6 u per
    selected head [N, d_k].  ``snapshot_at``: 1-based step counts after which
    a copy of the state is kept.  ``kla_eps`` (GDN/KDA): when given, each
    step's beta field holds the KLA gate eta_t and beta_t = kla_beta(eta_t,
    k_t, kla_eps).
    """
    S = _f64(S0).copy()
    outs: List[np.ndarray] = []
    snaps = {}
    want = set(int(s) for s in snapshot_at)
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
        if n in want:
            snaps[n] = S.copy()
    return EagerResult(S, outs, snaps)
