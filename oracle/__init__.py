"""fp64 CPU oracle of the MoE layer with zero-computation experts.

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The product path never
imports it and has no CPU fallback.  See ``moe_oracle`` for the method and
the passages each function follows.
"""
from . import moe_oracle  # noqa: F401
