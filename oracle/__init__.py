"""Plain float64 CPU oracle for the CSA/HCA hybrid attention forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library and never imports it.

See ``oracle/csa_oracle.py`` for the functions and the passages they follow.
"""
from .csa_oracle import *  # noqa: F401,F403
from .csa_oracle import __all__  # noqa: F401
