"""Planted mistakes in the oracle must fail at least one pin (CPU only).

Each mutant is a copy of one oracle step function with one plausible
mistake: a dropped term, a flipped sign, an operand on the wrong side, the
wrong state in the readout, a decay on the wrong axis.  The mistakes are
planted here, in copies of the oracle, never in the CUDA path.
"""

from __future__ import annotations

import types

import numpy as np
import pytest

from oracle import recurrence as rec
from tests import test_oracle_pins as pins


def _eye(d):
    return np.eye(d)[None]


# ---- GDN mutants ---------------------------------------------------------

def gdn_no_beta_on_write(S, q, k, v, alpha, beta):
    proj = _eye(k.shape[-1]) - beta[:, None, None] * (k[:, :, None] * k[:, None, :])
    S_new = alpha[:, None, None] * (S @ proj) + v[:, :, None] * k[:, None, :]
    return S_new, (S_new @ q[:, :, None])[:, :, 0]


def gdn_plus_projection(S, q, k, v, alpha, beta):
    proj = _eye(k.shape[-1]) + beta[:, None, None] * (k[:, :, None] * k[:, None, :])
    S_new = alpha[:, None, None] * (S @ proj) + beta[:, None, None] * (v[:, :, None] * k[:, None, :])
    return S_new, (S_new @ q[:, :, None])[:, :, 0]


def gdn_projection_on_left(S, q, k, v, alpha, beta):
    proj = _eye(k.shape[-1]) - beta[:, None, None] * (k[:, :, None] * k[:, None, :])
    S_new = alpha[:, None, None] * (proj @ S) + beta[:, None, None] * (v[:, :, None] * k[:, None, :])
    return S_new, (S_new @ q[:, :, None])[:, :, 0]


def gdn_readout_before_update(S, q, k, v, alpha, beta):
    S_new, _ = rec.gdn_step(S, q, k, v, alpha, beta)
    return S_new, (np.asarray(S) @ q[:, :, None])[:, :, 0]


def gdn_decay_on_everything(S, q, k, v, alpha, beta):
    proj = _eye(k.shape[-1]) - beta[:, None, None] * (k[:, :, None] * k[:, None, :])
    S_new = alpha[:, None, None] * (S @ proj + beta[:, None, None] * (v[:, :, None] * k[:, None, :]))
    return S_new, (S_new @ q[:, :, None])[:, :, 0]


def gdn_readout_with_k(S, q, k, v, alpha, beta):
    S_new, _ = rec.gdn_step(S, q, k, v, alpha, beta)
    return S_new, (S_new @ k[:, :, None])[:, :, 0]


def gdn_write_transposed(S, q, k, v, alpha, beta):
    proj = _eye(k.shape[-1]) - beta[:, None, None] * (k[:, :, None] * k[:, None, :])
    S_new = alpha[:, None, None] * (S @ proj) + beta[:, None, None] * (k[:, :, None] * v[:, None, :])
    return S_new, (S_new @ q[:, :, None])[:, :, 0]


# ---- KDA mutants ---------------------------------------------------------

def kda_decay_after_projection(S, q, k, v, alpha, beta):
    d = k.shape[-1]
    proj = _eye(d) - beta[:, None, None] * (k[:, :, None] * k[:, None, :])
    S_new = (S @ proj) @ (alpha[:, :, None] * _eye(d)) + beta[:, None, None] * (v[:, :, None] * k[:, None, :])
    return S_new, (S_new @ q[:, :, None])[:, :, 0]


def kda_decay_on_value_axis(S, q, k, v, alpha, beta):
    d = k.shape[-1]
    proj = _eye(d) - beta[:, None, None] * (k[:, :, None] * k[:, None, :])
    S_new = ((alpha[:, :, None] * _eye(d)) @ S) @ proj + beta[:, None, None] * (v[:, :, None] * k[:, None, :])
    return S_new, (S_new @ q[:, :, None])[:, :, 0]


def kda_scalar_mean_decay(S, q, k, v, alpha, beta):
    return rec.gdn_step(S, q, k, v, np.asarray(alpha).mean(axis=1), beta)


# ---- RWKV6 mutants -------------------------------------------------------

def rwkv6_readout_after_update(S, r, k, v, w, u):
    S_new, _ = rec.rwkv6_step(S, r, k, v, w, u)
    bonus = (u * k)[:, :, None] * v[:, None, :]
    return S_new, (r[:, None, :] @ (S_new + bonus))[:, 0, :]


def rwkv6_no_bonus(S, r, k, v, w, u):
    return rec.rwkv6_step(S, r, k, v, w, np.zeros_like(np.asarray(u)))


def rwkv6_decay_on_value_axis(S, r, k, v, w, u):
    _, o = rec.rwkv6_step(S, r, k, v, w, u)
    d = k.shape[-1]
    S_new = np.asarray(S) @ (np.asarray(w)[:, :, None] * _eye(d)) + k[:, :, None] * v[:, None, :]
    return S_new, o


def rwkv6_bonus_without_u(S, r, k, v, w, u):
    return rec.rwkv6_step(S, r, k, v, w, np.ones_like(np.asarray(u)))


def rwkv6_write_not_decayed_order(S, r, k, v, w, u):
    # decays the new write too: diag(w) (S + k v^T)
    _, o = rec.rwkv6_step(S, r, k, v, w, u)
    S_new = np.asarray(w)[:, :, None] * (np.asarray(S) + k[:, :, None] * v[:, None, :])
    return S_new, o


# ---- GDN-2 mutants -------------------------------------------------------

def _gdn2_parts(S, k, alpha):
    d = k.shape[-1]
    return _eye(d), np.asarray(S) @ (np.asarray(alpha)[:, :, None] * _eye(d))


def gdn2_erase_transposed(S, q, k, v, alpha, b, w):
    # the other placement of the gate: S' (I - k (b o k)^T)
    eye, P = _gdn2_parts(S, k, alpha)
    S_new = P @ (eye - k[:, :, None] * (b * k)[:, None, :]) + (w * v)[:, :, None] * k[:, None, :]
    return S_new, (S_new @ q[:, :, None])[:, :, 0]


def gdn2_erase_ungated(S, q, k, v, alpha, b, w):
    eye, P = _gdn2_parts(S, k, alpha)
    S_new = P @ (eye - k[:, :, None] * k[:, None, :]) + (w * v)[:, :, None] * k[:, None, :]
    return S_new, (S_new @ q[:, :, None])[:, :, 0]


def gdn2_write_ungated(S, q, k, v, alpha, b, w):
    eye, P = _gdn2_parts(S, k, alpha)
    S_new = P @ (eye - (b * k)[:, :, None] * k[:, None, :]) + v[:, :, None] * k[:, None, :]
    return S_new, (S_new @ q[:, :, None])[:, :, 0]


def gdn2_decay_after_erase(S, q, k, v, alpha, b, w):
    eye, _ = _gdn2_parts(S, k, alpha)
    S_new = (np.asarray(S) @ (eye - (b * k)[:, :, None] * k[:, None, :])) @ \
        (np.asarray(alpha)[:, :, None] * eye) + (w * v)[:, :, None] * k[:, None, :]
    return S_new, (S_new @ q[:, :, None])[:, :, 0]


def gdn2_readout_before_update(S, q, k, v, alpha, b, w):
    S_new, _ = rec.gdn2_step(S, q, k, v, alpha, b, w)
    return S_new, (np.asarray(S) @ q[:, :, None])[:, :, 0]


MUTANTS = {
    "gdn_no_beta_on_write": ("gdn_step", gdn_no_beta_on_write),
    "gdn_plus_projection": ("gdn_step", gdn_plus_projection),
    "gdn_projection_on_left": ("gdn_step", gdn_projection_on_left),
    "gdn_readout_before_update": ("gdn_step", gdn_readout_before_update),
    "gdn_decay_on_everything": ("gdn_step", gdn_decay_on_everything),
    "gdn_readout_with_k": ("gdn_step", gdn_readout_with_k),
    "gdn_write_transposed": ("gdn_step", gdn_write_transposed),
    "kda_decay_after_projection": ("kda_step", kda_decay_after_projection),
    "kda_decay_on_value_axis": ("kda_step", kda_decay_on_value_axis),
    "kda_scalar_mean_decay": ("kda_step", kda_scalar_mean_decay),
    "rwkv6_readout_after_update": ("rwkv6_step", rwkv6_readout_after_update),
    "rwkv6_no_bonus": ("rwkv6_step", rwkv6_no_bonus),
    "rwkv6_decay_on_value_axis": ("rwkv6_step", rwkv6_decay_on_value_axis),
    "rwkv6_bonus_without_u": ("rwkv6_step", rwkv6_bonus_without_u),
    "rwkv6_write_not_decayed_order": ("rwkv6_step", rwkv6_write_not_decayed_order),
    "gdn2_erase_transposed": ("gdn2_step", gdn2_erase_transposed),
    "gdn2_erase_ungated": ("gdn2_step", gdn2_erase_ungated),
    "gdn2_write_ungated": ("gdn2_step", gdn2_write_ungated),
    "gdn2_decay_after_erase": ("gdn2_step", gdn2_decay_after_erase),
    "gdn2_readout_before_update": ("gdn2_step", gdn2_readout_before_update),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    slot, fn = MUTANTS[name]
    impl = types.SimpleNamespace(gdn_step=rec.gdn_step, kda_step=rec.kda_step,
                                 rwkv6_step=rec.rwkv6_step, gdn2_step=rec.gdn2_step)
    setattr(impl, slot, fn)
    failed = []
    for pin in pins.PINS:
        try:
            pin(impl)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name} passed every pin"
