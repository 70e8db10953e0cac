"""CPU oracle for the DoRA factored-norm / fused-compose path.

Test infrastructure: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline legs of ``bench.py`` import it.  The product path never does.
Every function is pinned by ``tests/test_oracle_pins.py``; no function is
"parity unpinned".
"""

from .dora_oracle import (  # noqa: F401
    compose_backward,
    compose_backward_columns,
    compose_forward,
    dense_adapted_weight,
    linear_forward,
    magnitude_scale,
    norm_backward,
    row_norm,
    row_norm_rows,
)
