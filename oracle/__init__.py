"""CPU oracle for the W1.58A8 BitLinear path -- test infrastructure only.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA
library.
"""
from . import bitlinear  # noqa: F401
