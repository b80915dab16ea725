"""Seeded synthetic STCA workloads shared by the oracle tests, the GPU tests and the bench.

This package draws inputs only (history lengths, target counts, embeddings,
weights) and stores them in the element type a configuration names.  It holds
none of the method's arithmetic: no encoding, no attention, no fusion.
"""
from .workloads import (  # noqa: F401
    CONFIGS,
    TRAIN_BATCH,
    TrainingHistories,
    Workload,
    bf16_bits_to_f32,
    config_shapes,
    f32_to_bf16_bits,
    make_config_workload,
    make_training_histories,
    make_workload,
    round_to_bf16,
)
