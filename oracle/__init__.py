"""CPU oracle (fp64) for hybrid compressed attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and ``--impl reference`` legs may import this package.  The CUDA library
never does, and this package imports nothing from the library.
"""
from . import csa, formats  # noqa: F401
