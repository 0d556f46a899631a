"""CPU oracle for the packed ternary-weight GEMV -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package. The product path (``packed_ternary_weight_b200``)
never imports it and shares no code with it.
"""
from .tern_oracle import *  # noqa: F401,F403
from .unpack import *  # noqa: F401,F403
from . import decode  # noqa: F401,E402  (the BitNet decode layer composition)
