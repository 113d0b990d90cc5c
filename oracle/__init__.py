"""CPU oracle for the lightning indexer — test infrastructure only.

Imported by ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py``; never by the product path.
"""
from . import dsa_oracle  # noqa: F401
from .dsa_oracle import *  # noqa: F401,F403
