"""Seeded synthetic inputs shared by the oracle side and the CUDA side of the tests and the bench."""
from .inputs import (  # noqa: F401
    Workload, WORKLOADS, bf16_bits_from_f32, bf16_bits_to_f64, bf16_bits_to_f32,
    normal_bf16, make_raster_inputs, add_smooth_field,
)
