"""CPU oracle for the ISA forward pass: test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package. The CUDA library never uses it.
"""
from .isa_oracle import *  # noqa: F401,F403
from .isa_oracle import __all__  # noqa: F401
