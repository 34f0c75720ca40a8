"""CPU oracle of the ReplaySSM decode path -- TEST INFRASTRUCTURE, not the product.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import it. It shares no code with the CUDA library and imports nothing from it.

Pins: every function here is checked by ``tests/test_oracle_pins.py`` against what the
pages and the mathematics fix (two forms of the same recurrence, closed forms, special
cases that reduce to a library routine, the pages' printed ratios, the OCP e4m3 table
and torch's own e4m3 conversion), and ``tests/test_oracle_mutations.py`` plants
plausible mistakes in it to show that the pins catch them.
"""

from .replay_oracle import *  # noqa: F401,F403
from .replay_oracle import (  # noqa: F401
    ReplayBatch,
    ReplaySeq,
    decay_weights,
    dequantize_rows_e2m1,
    dequantize_rows_e4m3,
    e2m1_decode,
    e2m1_encode,
    e4m3_decode,
    e4m3_encode,
    eager_batch_step,
    eager_fp8_batch_step,
    eager_step,
    history_state,
    output_only,
    quantize_rows_e2m1,
    quantize_rows_e4m3,
    relative_error,
    route_flops,
    state_route,
)
