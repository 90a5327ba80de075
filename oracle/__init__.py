"""fp64 CPU oracle of the MC-Sparse hot path -- test infrastructure only.

Importable only from the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py``.  It shares no code with the CUDA library.
"""
from . import mcs_oracle  # noqa: F401
