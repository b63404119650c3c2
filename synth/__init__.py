"""Seeded synthetic inputs shared by the tests, the bench and the smoke check."""
from .video import (WORKLOADS, Workload, bf16_bits_to_f32, f32_to_bf16_bits,  # noqa: F401
                    frame_index, generate, perturb, to_f64, to_torch, workload)
