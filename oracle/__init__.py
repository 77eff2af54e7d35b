"""fp64 CPU oracles of the W4 g32 MoE layer (moe_ref), of the same layer with
MXFP4 routed experts (mxfp4_ref, imported as oracle.mxfp4_ref) and of the
online-FP8 LM head (lmhead_ref, imported as oracle.lmhead_ref).

TEST INFRASTRUCTURE ONLY: imported by the tests, the package smoke check and
the benchmark's CPU-baseline arm, never by the GPU library.
"""
from .moe_ref import *  # noqa: F401,F403
from .moe_ref import __all__  # noqa: F401
