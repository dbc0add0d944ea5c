"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This package holds no arithmetic of the attention method itself: it only draws the
Q, K, V fields, rounds them to bf16 and lays them out as padded [B, H, Npad, D]
arrays with a per-sample valid length and the tokens' latent-grid positions, and
draws the QK-norm weights the producer step takes and the token features that
saliency pruning ranks.
"""
from .synth import (CONFIGS, Workload, bf16_bits_to_f32, f64_to_bf16_bits, make_custom, make_hidden,
                    make_norm_weights, make_workload)

__all__ = ["CONFIGS", "Workload", "make_workload", "make_custom", "make_hidden", "make_norm_weights",
           "bf16_bits_to_f32", "f64_to_bf16_bits"]
