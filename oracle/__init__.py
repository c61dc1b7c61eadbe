"""CPU oracle for the fused MoE layer -- test infrastructure only.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  The CUDA library never does, and this package imports nothing
from the library.
"""
from . import moe_oracle  # noqa: F401
