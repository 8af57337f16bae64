"""CPU oracle for the PR-Sink hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  The GPU library never calls it and shares no code with it.

Everything is float64 numpy, written as the plain definitions the sources state; see
``oracle/prsink_oracle.py`` for the function list, the citations and the readings taken where
the sources are silent.
"""
from .prsink_oracle import *  # noqa: F401,F403
from .prsink_oracle import __all__  # noqa: F401
