"""CPU oracle of the MXFP8 routed-experts MLP (test infrastructure only).

Plain numpy, float64, written from the definitions; see ``oracle.mx``.  Only
the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it.  The library itself never does, and the two share
no code.
"""
from . import mx  # noqa: F401
from . import routing  # noqa: F401
