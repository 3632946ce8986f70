"""fp64 CPU oracle for DeltaLog decoding -- TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, eager definition of the recurrences DeltaLog
decodes (GDN, KDA, RWKV6, and GDN-2 with separate erase and write gates), written in float64 numpy, and of the same
recurrences with the state quantized to int8 once per window
(``window_quant``).  It is what the
GPU path must reproduce: DeltaLog's claim is that the model observes the same
dense state as eager decoding ("DeltaLog: Deferred Materialization of
Recurrent States for Linear Attention Decoding", Abstract), so the oracle is
the eager recurrence itself, with no log and no merge.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU
baseline and reference arm) may import it.  The library never does: it shares
no code with the CUDA path and imports nothing from it.

Parity is not pinned to printed values: the pages print no worked example.
The oracle is pinned instead by closed forms, exact rational hand examples,
invariants and an exact-arithmetic brute force of the log form (see
``tests/test_oracle_pins.py``).
"""

from .recurrence import (  # noqa: F401
    gdn_step, kda_step, gdn2_step, rwkv6_step, kla_beta, run_eager, EagerResult,
)
from .window_quant import (  # noqa: F401
    quantize_rows, dequantize_rows, row_inverse, run_windowed, WindowedResult, WindowEnd,
)
