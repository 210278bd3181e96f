"""CPU oracle for the SVDQuant W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline / reference
legs of `bench.py` may import this package.  The product path (the C-ABI
library and its Python binding) never imports, calls or links it.
"""
from .svdq_oracle import *  # noqa: F401,F403
from .svdq_oracle import __all__  # noqa: F401
