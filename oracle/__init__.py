"""CPU oracle for the SVDQuant W4A4 linear layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package. See ``oracle/svdquant.py``.
"""
from .svdquant import *  # noqa: F401,F403
