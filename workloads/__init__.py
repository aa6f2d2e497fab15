"""Seeded synthetic inputs shared by the tests, the oracle checks and the bench.

This package only draws random numbers and lays them out; it holds none of the
method's arithmetic (no logits, softmax, weights, advantages or gradients).
"""
from .synth import CONFIGS, Batch, ConfigSpec, make_batch, spec_for

__all__ = ["CONFIGS", "Batch", "ConfigSpec", "make_batch", "spec_for"]
