"""CPU oracle for the KDA hot path (float64, NumPy).

TEST INFRASTRUCTURE: imported only by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  The product path never calls it.

Parity status: every function here is pinned by CPU tests against values the
source pages print, closed forms, invariants or library routines (see
``tests/test_oracle_pins.py`` and ``tests/test_oracle_prologue.py``); the
chunkwise evaluator is pinned against the recurrence.
"""
from .kda_oracle import (  # noqa: F401
    L2_EPS,
    gate,
    kda_chunkwise,
    kda_chunkwise_backward,
    kda_decode_step,
    kda_recurrent,
    kda_recurrent_backward,
    l2_normalize,
    output_epilogue,
    prologue,
    short_conv,
    silu,
    state_from_abi,
    state_to_abi,
)
