"""fp64 CPU oracle of the GPTQ layer-wise quantizer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.
"""
from .gptq_oracle import *  # noqa: F401,F403
