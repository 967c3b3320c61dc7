"""Float64 CPU oracle of the EntmaxKV decode step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg import this package.  It shares no code with the CUDA library.
"""
from .entmax_kv import *  # noqa: F401,F403
from .entmax_kv import __all__  # noqa: F401
