"""Plain CPU oracle for the selected-token denoising step (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (the C-ABI library and its Python binding) never calls it.
"""
from .oracle import *  # noqa: F401,F403
