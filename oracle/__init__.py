"""fp64 CPU oracle for the TurboQuant compressed-KV hot path.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package. The CUDA library never
calls it and shares no code with it: the two meet only at the seeded inputs in
``workloads`` and at the packed byte format, which each side implements on its
own.

See ``oracle.turboquant`` for the functions and the passages each one follows.
"""
from .turboquant import *  # noqa: F401,F403
