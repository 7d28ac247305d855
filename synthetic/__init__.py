"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This package holds only input generation: workload shapes, seeded Q/K/V draws and
the random static block masks that stand in for calibrated masks.  It contains
none of the attention, reordering or mask-construction arithmetic; both the CUDA
path and the FP64 oracle receive what it produces as plain inputs.
"""
from .workloads import (WORKLOADS, Workload, make_qk_calibration, make_qkv, mask_variants,
                        spatial_repetition_map, static_calibrated_mask)

__all__ = ["WORKLOADS", "Workload", "make_qkv", "make_qk_calibration", "static_calibrated_mask",
           "mask_variants", "spatial_repetition_map"]
