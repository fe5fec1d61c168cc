"""Seeded synthetic inputs for the LoopVQ decode hot path.

This package only draws random inputs: looped K/V caches, queries,
per-element weights, k-means codebooks and page tables. It performs none of
the method's own arithmetic (no sub-vector encoding, no dequantisation, no
attention), so both the CUDA path and the CPU oracle can take their inputs
from it without sharing any of the computation under test.

The pages publish no workload beyond the model families (Ouro 1.4B/2.6B,
Huginn-3.5B) and the window sizes; the shapes below are synthetic stand-ins
with the shapes of those models' decode step.
"""

from .configs import SHAPES, Shape  # noqa: F401
from .generators import (  # noqa: F401
    block_tables,
    codebooks_for_layer,
    head_scales,
    key_outlier_mask,
    lloyd_kmeans,
    loop_group_kv,
    queries,
    weights,
    window_kv,
)
