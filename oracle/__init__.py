"""fp64 CPU oracle of the W4 g32 MoE layer.

TEST INFRASTRUCTURE ONLY: imported by the tests, the package smoke check and
the benchmark's CPU-baseline arm, never by the GPU library.
"""
from .moe_ref import *  # noqa: F401,F403
from .moe_ref import __all__  # noqa: F401
