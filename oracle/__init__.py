"""CPU oracle for the LoopVQ decode hot path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product never does.
"""
from .loopvq_oracle import *  # noqa: F401,F403
