"""Degenerate decode-step inputs (test infrastructure).

Each kind rewrites the seeded inputs of a workload's steps into a limiting
case of the recurrences that stays inside the library's input contract
(decays in (0, 1], gates in [0, 1], q/k/v exact in the input dtype):

  no_decay          every decay 1: the log-decays stay 0
  vanishing_decay   every decay 1e-30: each step all but erases the state,
                    and the cumulative log-decay falls by ~69 per step
  wipe_then_recover decay 1e-30 on every fifth step (t = 2 mod 5), the drawn
                    decays otherwise: log-decay jumps inside one log
  mixed_extremes    GDN: decay 1e-30 on even heads, 1 on odd heads; vector
                    variants: the first half of the key channels 1e-30, the
                    second half 1
  no_write          GDN/KDA beta 0; GDN-2 erase and write gates 0; RWKV6
                    zero keys (its write is k v^T)
  zero_key          k_t = 0
  zero_query        q_t (r_t) = 0: every output is exactly 0
  zero_value        v_t = 0: the delta rule only erases
  repeated_key      k_t = k_0 at every step: every log entry shares one key

The values are built in fp32 (and are bf16-exact), so the kernels and the
oracle receive identical numbers.  Nothing here computes the recurrence.
"""

from __future__ import annotations

import dataclasses

import numpy as np

from linear_attention_recurrent_deltalog_b200 import workloads as wl

TINY_DECAY = np.float32(1e-30)

KINDS = ("no_decay", "vanishing_decay", "wipe_then_recover", "mixed_extremes", "no_write",
         "zero_key", "zero_query", "zero_value", "repeated_key")


def make_edit(w: wl.Workload, kind: str):
    """A function StepInputs -> StepInputs applying ``kind`` to every step."""
    if kind not in KINDS:
        raise ValueError(f"unknown kind {kind!r}")
    k0 = wl.step_inputs(w, 0).k.copy() if kind == "repeated_key" else None

    def edit(s: wl.StepInputs) -> wl.StepInputs:
        rep = {}
        dec = np.array(s.decay, dtype=np.float32, copy=True)
        if kind == "no_decay":
            rep["decay"] = np.ones_like(dec)
        elif kind == "vanishing_decay":
            rep["decay"] = np.full_like(dec, TINY_DECAY)
        elif kind == "wipe_then_recover":
            if s.t % 5 == 2:
                rep["decay"] = np.full_like(dec, TINY_DECAY)
        elif kind == "mixed_extremes":
            if dec.ndim == 2:  # [B, H]: scalar decay per head
                dec[:, 0::2] = TINY_DECAY
                dec[:, 1::2] = 1.0
            else:              # [B, H, d_k]: per key channel
                half = dec.shape[-1] // 2
                dec[..., :half] = TINY_DECAY
                dec[..., half:] = 1.0
            rep["decay"] = dec
        elif kind == "no_write":
            if w.variant == wl.RWKV6:
                rep["k"] = np.zeros_like(s.k)
            else:
                rep["beta"] = np.zeros_like(s.beta)
                if w.variant == wl.GDN2:
                    rep["wgate"] = np.zeros_like(s.wgate)
        elif kind == "zero_key":
            rep["k"] = np.zeros_like(s.k)
        elif kind == "zero_query":
            rep["q"] = np.zeros_like(s.q)
        elif kind == "zero_value":
            rep["v"] = np.zeros_like(s.v)
        elif kind == "repeated_key":
            rep["k"] = k0.copy()
        return dataclasses.replace(s, **rep)

    return edit


def compose(*edits):
    def edit(s):
        for e in edits:
            s = e(s)
        return s
    return edit
