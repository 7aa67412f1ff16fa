"""fp64 CPU oracle for the FLARE++ mixer forward (test infrastructure only).

Imported by ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py``; never by the library.
"""
from .flare_oracle import *  # noqa: F401,F403
from .flare_oracle import __all__  # noqa: F401
