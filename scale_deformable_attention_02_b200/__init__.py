"""Multi-scale deformable attention (MSDeformAttn) core for NVIDIA B200.

The compute path is libmsda.so (hand-written sm_100a CUDA kernels behind the
C ABI in include/msda.h); this package is its thin Python binding, plus the
seeded synthetic workloads used by the tests and the benchmark.
"""
from ._lib import LIB_CHECKED_PATH, LIB_PATH, MSDA_BF16, MSDA_F32
from .api import (MsdaError, TilePlan, checked_library, last_violation, msda_backward,
                  msda_backward_fused, msda_backward_fused_tiled, msda_backward_tiled, msda_debug_row_traffic, msda_debug_sample_points,
                  msda_debug_tiled_stalls, msda_forward, msda_forward_fused, msda_forward_fused_tiled,
                  msda_forward_tiled, msda_level_start_index, msda_tile_plan,
                  msda_tile_plan_rebuild)

__all__ = [
    "LIB_CHECKED_PATH", "LIB_PATH", "MSDA_BF16", "MSDA_F32", "MsdaError", "TilePlan",
    "checked_library",
    "last_violation", "msda_backward", "msda_backward_fused", "msda_backward_fused_tiled",
    "msda_backward_tiled", "msda_debug_row_traffic",
    "msda_debug_sample_points", "msda_debug_tiled_stalls",
    "msda_forward", "msda_forward_fused", "msda_forward_fused_tiled", "msda_forward_tiled",
    "msda_level_start_index", "msda_tile_plan", "msda_tile_plan_rebuild",
]
