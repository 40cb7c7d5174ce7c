"""fp64 CPU oracle for the Multi-Scale Retention hot path (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may import this package.  The CUDA library never does, and this package
never imports the library.
"""

from .retention import *  # noqa: F401,F403
from .retention import __all__  # noqa: F401
