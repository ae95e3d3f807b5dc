"""OrbitQuant reference oracle (TEST INFRASTRUCTURE ONLY).

A plain, slow, fp64 CPU restatement of what the OrbitQuant quantized linear
layer computes, written from the pages' description of the method.  Only the
test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
leg of ``bench.py`` may import it.  The product path (the C-ABI library and its
Python binding) never imports, links or executes anything in this package, and
this package never imports the product.

See ``oracle/orbitquant_oracle.py`` for the functions and their citations.
"""

from .orbitquant_oracle import *  # noqa: F401,F403
from .orbitquant_oracle import __all__  # noqa: F401
