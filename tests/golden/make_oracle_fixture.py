"""Writes tests/golden/oracle_tiny.json from the fp64 oracle alone.

The pages print no worked example for DeltaLog, so this fixture is not a
published value: it freezes the oracle's own output on tiny fixed inputs, so
that any later change to the oracle's arithmetic shows up as a fixture diff
that has to be justified.  Inputs are drawn here with numpy's default_rng
(fixed seed) and stored with the outputs; nothing else is called.

Run from the repository root:  python tests/golden/make_oracle_fixture.py
"""

import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
from oracle import recurrence as rec  # noqa: E402


def case(variant, seed, N=2, d=4, T=3):
    rng = np.random.default_rng(seed)
    S0 = rng.standard_normal((N, d, d)).round(3)
    steps = []
    S = S0.copy()
    outs = []
    for _ in range(T):
        q = rng.standard_normal((N, d)).round(3)
        k = rng.standard_normal((N, d)).round(3)
        v = rng.standard_normal((N, d)).round(3)
        if variant == "gdn":
            dec = rng.uniform(0.8, 1.0, N).round(3)
        else:
            dec = rng.uniform(0.5, 1.0, (N, d)).round(3)
        beta = rng.uniform(0.0, 1.0, N).round(3)
        u = rng.standard_normal((N, d)).round(3)
        if variant == "gdn":
            S, o = rec.gdn_step(S, q, k, v, dec, beta)
        elif variant == "kda":
            S, o = rec.kda_step(S, q, k, v, dec, beta)
        else:
            S, o = rec.rwkv6_step(S, q, k, v, dec, u)
        steps.append(dict(q=q.tolist(), k=k.tolist(), v=v.tolist(), decay=dec.tolist(),
                          beta=beta.tolist(), u=u.tolist()))
        outs.append(o.tolist())
    return dict(variant=variant, S0=S0.tolist(), steps=steps, outputs=outs, S_T=S.tolist())


def main():
    data = dict(note="oracle self-fixture; not a published value",
                cases=[case("gdn", 1), case("kda", 2), case("rwkv6", 3)])
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json")
    with open(out, "w") as f:
        json.dump(data, f, indent=1)
    print("wrote", out)


if __name__ == "__main__":
    main()
