"""fp64 CPU oracle for dynamic short convolutions -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path never calls it and shares no
code with it.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(no function is "parity unpinned"); the pages print no worked numeric example,
so the pins are closed forms, invariants, brute force and a hand-derived
integer example.
"""
from .oracle import (  # noqa: F401
    LOWRANK, HEADWISE, Problem, build, forward, backward_rows, param_grads,
    param_grad_entries, filters,
)
