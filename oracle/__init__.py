"""CPU oracle for the DASH prefill path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
library never imports, links or calls anything here, and nothing here calls
the CUDA library.
"""
from .dash_oracle import *  # noqa: F401,F403
