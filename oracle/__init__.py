"""fp64 CPU oracle of the DV-SSQ layer -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does.
"""
from .dvssq_oracle import *  # noqa: F401,F403
from . import dvssq_oracle as core  # noqa: F401
