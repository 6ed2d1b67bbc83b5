"""CPU oracle for PISA pyramid block-sparse attention (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its Python binding) never imports it and fails loudly when the CUDA extension
is missing.
"""
from .pisa_oracle import *  # noqa: F401,F403
