"""fp64 CPU oracle of exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library never uses it and
shares no code with it. Every function cites the FlashAttention page passage
it follows; all of them are pinned by ``tests/test_oracle.py``.
"""
from . import attention  # noqa: F401
