"""CPU oracle for the quantized attention forward (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never imports, links or
calls it, and it shares no code with the CUDA sources.
"""

from .sage_oracle import *  # noqa: F401,F403
