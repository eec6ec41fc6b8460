"""CPU oracle for the KVQuant decode path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` may import this package.  The CUDA library never calls it and it
never calls the CUDA library; the two share no code.
"""
from .kvquant_oracle import *  # noqa: F401,F403
