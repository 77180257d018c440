"""fp64 CPU oracle of NABLA-style block-sparse attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package; the product path never does.
"""
from .nabla import *  # noqa: F401,F403
from . import nabla  # noqa: F401
