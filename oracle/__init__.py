"""CPU oracle for the fused static-FP8 attention-input chain.

Test infrastructure: only the test suite, ``__graft_entry__.smoke`` and the
benchmark's CPU-baseline leg may import this package.  The product library
never does, and this package imports nothing from the product.
"""

from .oracle import *  # noqa: F401,F403
