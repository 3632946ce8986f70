"""GPU parity on degenerate inputs: limiting cases of the recurrences
(decay 1 or 1e-30, log-decay jumps inside a log, no writes, zero keys,
queries or values, one key repeated) for every variant, through the
DeltaLog step with separate and fused merges, the eager step and the int8
base, against the fp64 oracle at the usual tolerances (output rel err
<= 1e-3, state rel err <= 1e-4, int8 codes correct roundings)."""

from __future__ import annotations

import pytest

from linear_attention_recurrent_deltalog_b200 import workloads as wl
from tests.degenerate_inputs import KINDS, make_edit
from tests.parity import OUT_TOL, STATE_TOL, run_parity, run_parity_q8

pytestmark = pytest.mark.gpu

BASES = {"gdn": "gdn_qwen", "kda": "kda", "rwkv6": "rwkv6", "gdn2": "gdn2"}


def _small(variant: str, seed: int) -> wl.Workload:
    # 8 sequences x 4 heads, L = 6 with ragged fills over 20 steps: every
    # sequence merges two or three times at its own phase
    return wl.WORKLOADS[BASES[variant]].replace(B=8, H=4, L=6, T=20, ragged=True, seed=seed)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("variant", ["gdn", "kda", "rwkv6", "gdn2"])
def test_degenerate_inputs(variant, kind):
    w = _small(variant, 60 + KINDS.index(kind))
    res = run_parity(w, snap_every=3, workers=0, edit=make_edit(w, kind))
    for arm, r in res.items():
        assert r.state_err <= STATE_TOL, f"{arm}: state rel err {r.state_err:.3e}"
        assert r.out_err <= OUT_TOL, f"{arm}: output rel err {r.out_err:.3e}"
    if kind == "zero_query":
        for arm, r in res.items():
            assert all(not o.any() for o in r.outputs), f"{arm}: q = 0 must give o = 0"


@pytest.mark.parametrize("kind", ["vanishing_decay", "wipe_then_recover", "mixed_extremes",
                                  "no_write", "zero_value"])
@pytest.mark.parametrize("variant", ["gdn", "kda", "rwkv6", "gdn2"])
def test_degenerate_inputs_int8_base(variant, kind):
    w = _small(variant, 80 + KINDS.index(kind))
    for fused in (True, False):
        r = run_parity_q8(w, fused=fused, snap_every=3, edit=make_edit(w, kind))
        assert r.reset_exact
        assert r.windows > 0
        assert r.out_err <= OUT_TOL, f"output rel err {r.out_err:.3e}"
        assert r.state_err <= STATE_TOL, f"state rel err {r.state_err:.3e}"
        assert r.code_excess <= 0, f"a code is off its rounding by {r.code_excess:.3e}"
        assert r.scale_excess <= 0, f"a scale is off by {r.scale_excess:.3e}"
        assert r.mismatch_frac <= 1e-2, f"{r.mismatch_frac:.2e} of codes differ"
