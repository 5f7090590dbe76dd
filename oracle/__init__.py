"""CPU fp64 oracle for absorbed-MLA decode.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
its Python binding) imports, links or runs this package; only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s cpu-baseline leg do.
"""
from .mla_oracle import *  # noqa: F401,F403
