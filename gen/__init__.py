"""Seeded synthetic input generators (no method arithmetic lives here)."""
from .inputs import (CONFIGS, CONFIG_ORDER, DEFAULT_SEED, Case, HSTUConfig, LayerWeights,
                     algorithmic_counts, make_case, round_bf16, round_fp16, stochastic_length,
                     to_dtype)

__all__ = ["CONFIGS", "CONFIG_ORDER", "DEFAULT_SEED", "Case", "HSTUConfig", "LayerWeights",
           "algorithmic_counts", "make_case", "round_bf16", "round_fp16", "stochastic_length", "to_dtype"]
