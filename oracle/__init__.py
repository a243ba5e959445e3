"""Float64 CPU oracle for tiered decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import, call or execute anything in this package.  The product path (the CUDA
library and its Python binding) never does, and this package never imports the
product.  Every function here is pinned by CPU tests in ``tests/test_oracle_*.py``.
"""
from . import akv_oracle, lloyd_max  # noqa: F401
