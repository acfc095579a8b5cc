"""Seeded synthetic workloads for per-denoise-step block-diffusion attention.

This package only draws random numbers, rounds them to the storage dtype and
lays them out (prefix KV pool, page table, per-step block q/k/v and update
counts). It holds none of the attention arithmetic, so that the GPU path and the
oracle can both be fed from it without sharing any of the method's code.
"""

from .gen import (  # noqa: F401
    SPECS,
    Prefix,
    Spec,
    StepInputs,
    Workload,
    bf16_bits_from_f32,
    make_workload,
)
