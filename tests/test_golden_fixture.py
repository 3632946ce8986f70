"""The oracle still reproduces its frozen tiny-input fixture (CPU only)."""

import json
import os

import numpy as np

from oracle import recurrence as rec

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_tiny.json")


def test_oracle_matches_frozen_fixture():
    data = json.load(open(HERE))
    for c in data["cases"]:
        S = np.array(c["S0"])
        for st, o_ref in zip(c["steps"], c["outputs"]):
            a = {k: np.array(v) for k, v in st.items()}
            if c["variant"] == "gdn":
                S, o = rec.gdn_step(S, a["q"], a["k"], a["v"], a["decay"], a["beta"])
            elif c["variant"] == "kda":
                S, o = rec.kda_step(S, a["q"], a["k"], a["v"], a["decay"], a["beta"])
            else:
                S, o = rec.rwkv6_step(S, a["q"], a["k"], a["v"], a["decay"], a["u"])
            np.testing.assert_allclose(o, np.array(o_ref), rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(S, np.array(c["S_T"]), rtol=1e-13, atol=1e-13)
