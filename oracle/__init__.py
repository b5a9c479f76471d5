"""fp64 CPU oracle (test infrastructure only; see ``duo_oracle``).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The CUDA library never does.
"""
from .duo_oracle import *  # noqa: F401,F403
from .duo_oracle import __all__  # noqa: F401
