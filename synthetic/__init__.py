"""Seeded synthetic inputs shared by the oracle and the CUDA path.

This module only draws random numbers and lays them out: workload shapes,
per-tensor seeded normal draws, and the bf16 / FP8 E4M3 storage encoding of
inputs that are *given* in those formats.  It holds none of the method's arithmetic (no norm, no
attention, no time embedding, no Euler step), so the oracle and the CUDA
path can both use it without sharing any computation.
"""

from .configs import (CONFIGS, DRAFTS, PREFILLS, DraftShape, ExpertShape, PrefillShape, get_config,  # noqa: F401
                      get_draft_config, get_prefill_config)
from .gen import (  # noqa: F401
    bf16_bits_to_f32,
    e4m3_encode,
    f32_to_bf16_bits,
    draft_weight_names,
    make_draft,
    make_draft_weights,
    make_noise,
    make_prefill_weights,
    make_prefix_embeddings,
    make_prefix_kv,
    make_state,
    make_visual_tokens,
    make_weights,
    prefill_weight_names,
    round_to_bf16,
    weight_names,
)
