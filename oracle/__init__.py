"""CPU fp64 oracle for gated linear attention -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline / reference
legs may import this package.  The product path (the CUDA library and its binding) never
does, and it shares no code with it.
"""
from .oracle import (LIB_PATH, SRC_PATH, Oracle, backward, build, compile_lib,  # noqa: F401
                     forward, num_threads)
