"""CPU oracle for the compressed linear layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never calls it and shares no code with it.
"""
from .cql_oracle import *  # noqa: F401,F403
