"""fp64 CPU oracle for bifocal-RoPE attention (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
reference arm of ``bench.py`` may import this package.
"""
from .bifocal_ref import *  # noqa: F401,F403
from .bifocal_ref import __all__  # noqa: F401
