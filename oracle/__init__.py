"""fp64 CPU oracle of the KronQ per-sublayer quantization engine.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``, never by the product
path.  It shares no code with the CUDA library.  See ``kronq_oracle.py``.
"""
from .kronq_oracle import *  # noqa: F401,F403
from .kronq_oracle import diag_scale_of, rotation_row, side_key  # noqa: F401
