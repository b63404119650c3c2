"""CPU oracle for the SparsePR per-call sparse-attention path (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
legs of ``bench.py`` may import this package.  The CUDA path never does.
"""
from .sparsepr_oracle import *  # noqa: F401,F403
