"""Seeded synthetic inputs shared by the tests, the oracle checks and the bench.

This package only draws random numbers and lays them out; it holds none of the
method's arithmetic (no logits, softmax, weights, advantages or gradients).
"""
from .synth import (CONFIGS, Batch, ConfigSpec, dense_inputs, logprob_pair_inputs, make_batch, make_global_batch,
                    norm_inputs, spec_for)

__all__ = ["CONFIGS", "Batch", "ConfigSpec", "dense_inputs", "logprob_pair_inputs", "make_batch", "make_global_batch",
           "norm_inputs", "spec_for"]
