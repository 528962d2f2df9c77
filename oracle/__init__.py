"""CPU oracle for the AWQ W4A16 g128 path — test infrastructure only.

Importable only from ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py``. The CUDA library never uses it.
"""
from .awq_oracle import *  # noqa: F401,F403
