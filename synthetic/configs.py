"""Workload presets: the expert shapes and run settings the pages describe.

Sources (page titles):
  * "DM0.5: high-performance embodied VLA and OpenDM reading guide",
    sec. 5.1-5.3 (prefix KV cache reused by every denoise step, action expert
    suffix, flow matching with diffusion_steps=10) and sec. 7.3 (chunk size 50).
  * "Realtime-VLA FLASH", sec. 03 (verification taus such as 0.2 / 0.5,
    threshold delta, gripper switch fallback).
  * "VLA design space" slides (Pi-Zero 300M action expert, bf16, batch 1).

Names:
  tiny-fp32      2-layer width-256 expert in fp32, 64 prefix tokens, 8 actions.
  pi0-bf16       Pi0-class expert: 18 layers, width 1024, 8 q / 1 kv heads,
                 head_dim 256, GeGLU 4096, 816 prefix tokens (3 views x 256
                 + 48 text), 1 state token + 50 action tokens of dim 32.
  pi0-verify     FLASH verification on the pi0-bf16 expert, taus 0.2/0.5/0.8.
  pi0-fp8mlp     pi0-bf16 with FP8 E4M3 MLP weights and a 560-token prefix.
  pi0-concat     pi0-bf16 with Pi0's time conditioning: the time MLP reads the
                 action embedding concatenated with e(t).
  dm05-adarms    pi0-bf16 with DM0.5's per-layer time modulator (scale, shift
                 and gate of each norm's branch from c(t)).

Draft models ("Realtime-VLA FLASH" sec. 03.1: one Gemma block and a linear
action head, about 110M parameters, learnable action queries reading the
current image features in one forward pass):
  draft-tiny     width-256 block in fp32, 8 queries, 7-dim actions, 64
                 visual tokens.
  flash-draft    Gemma-2B-width block (width 2048, 8 q / 1 kv heads,
                 head_dim 256, GeGLU 16384: 110.1M block parameters), 50
                 queries of 32-dim actions over the 768 image tokens (3 views
                 x 256) of the pi0-bf16 observation, bf16.

VLM prefill (the prefix side of the suffix loop; "DM0.5 reading guide" sec.
5.1: the prefix is encoded once into a per-layer KV cache):
  gemma2b-prefill  Gemma-2B-class stack: 18 layers, width 2048, 8 q / 1 kv
                   heads, head_dim 256, GeGLU 16384, over 816 random
                   embedding tokens, writing the pi0-bf16 expert's cache.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Tuple


@dataclass(frozen=True)
class ExpertShape:
    name: str
    n_layers: int
    width: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    mlp_dim: int
    action_dim: int
    state_dim: int
    chunk_len: int          # H, actions per chunk
    prefix_len: int         # P, cached prefix tokens per layer
    n_steps: int = 10       # N Euler steps
    batch: int = 1          # B independent chunks
    dtype: str = "f32"      # storage/MMA type of matrices and prefix KV: "f32" | "bf16"
    mlp_dtype: str = "same"  # "same" | "fp8_e4m3"
    suffix_mask: str = "bidir"  # "bidir" | "pi0_block"
    # how the flow time enters the expert: "add" (c(t) added to the action
    # tokens), "concat" (Pi0: time MLP over [action embedding ; e(t)]),
    # "adarms" (DM0.5: a per-layer time modulator scaling, shifting and gating
    # each norm's branch)
    time_cond: str = "add"
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0
    weight_std: float = 0.02
    # verification settings (FLASH)
    taus: Tuple[float, ...] = (0.2, 0.5, 0.8)
    delta: float = 0.05
    gripper_dim: int = -1   # -1 = last action dim
    draft_std: float = 0.5
    seed: int = 0
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def suffix_len(self) -> int:
        """S = 1 state token + H action tokens."""
        return 1 + self.chunk_len

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def gripper(self) -> int:
        return self.gripper_dim if self.gripper_dim >= 0 else self.action_dim - 1

    def with_(self, **kw) -> "ExpertShape":
        return replace(self, **kw)

    def layer_params(self) -> int:
        w, f = self.width, self.mlp_dim
        per = w * (self.q_dim + 2 * self.kv_dim) + self.q_dim * w + 3 * w * f
        if self.time_cond == "adarms":
            per += 6 * w * w
        return self.n_layers * per


TINY_FP32 = ExpertShape(
    name="tiny-fp32", n_layers=2, width=256, n_q_heads=4, n_kv_heads=1, head_dim=64,
    mlp_dim=1024, action_dim=7, state_dim=8, chunk_len=8, prefix_len=64, dtype="f32",
    gripper_dim=6,
)

PI0_BF16 = ExpertShape(
    name="pi0-bf16", n_layers=18, width=1024, n_q_heads=8, n_kv_heads=1, head_dim=256,
    mlp_dim=4096, action_dim=32, state_dim=32, chunk_len=50, prefix_len=816, dtype="bf16",
    gripper_dim=31,
)

PI0_VERIFY = PI0_BF16.with_(name="pi0-verify")

PI0_FP8MLP = PI0_BF16.with_(name="pi0-fp8mlp", mlp_dtype="fp8_e4m3", prefix_len=560)

PI0_CONCAT = PI0_BF16.with_(name="pi0-concat", time_cond="concat")
DM05_ADARMS = PI0_BF16.with_(name="dm05-adarms", time_cond="adarms")

CONFIGS = {c.name: c for c in (TINY_FP32, PI0_BF16, PI0_VERIFY, PI0_FP8MLP, PI0_CONCAT, DM05_ADARMS)}


@dataclass(frozen=True)
class DraftShape:
    """A FLASH draft model: one Gemma block over [visual tokens ; action
    queries] and a linear action head on the query rows."""
    name: str
    width: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    mlp_dim: int
    n_queries: int          # H, rows of the candidate chunk
    action_dim: int         # A
    n_vis: int              # V, visual tokens of one observation
    batch: int = 1
    dtype: str = "f32"      # storage/MMA type of matrices and visual tokens
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0
    weight_std: float = 0.02
    seed: int = 0

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def with_(self, **kw) -> "DraftShape":
        return replace(self, **kw)

    def block_params(self) -> int:
        w, f = self.width, self.mlp_dim
        return w * (self.q_dim + 2 * self.kv_dim) + self.q_dim * w + 3 * w * f + 2 * w

    def params(self) -> int:
        return self.block_params() + self.n_queries * self.width + self.action_dim * (self.width + 1)


TINY_DRAFT = DraftShape(
    name="draft-tiny", width=256, n_q_heads=4, n_kv_heads=1, head_dim=64, mlp_dim=1024, n_queries=8,
    action_dim=7, n_vis=64, dtype="f32",
)

FLASH_DRAFT = DraftShape(
    name="flash-draft", width=2048, n_q_heads=8, n_kv_heads=1, head_dim=256, mlp_dim=16384, n_queries=50,
    action_dim=32, n_vis=768, dtype="bf16",
)

DRAFTS = {c.name: c for c in (TINY_DRAFT, FLASH_DRAFT)}


def get_draft_config(name: str, **overrides) -> DraftShape:
    cfg = DRAFTS[name]
    return cfg.with_(**overrides) if overrides else cfg


def get_config(name: str, **overrides) -> ExpertShape:
    cfg = CONFIGS[name]
    return cfg.with_(**overrides) if overrides else cfg


@dataclass(frozen=True)
class PrefillShape:
    """A Gemma-style VLM stack that turns prefix embeddings into the
    per-layer KV cache the action expert reads."""
    name: str
    n_layers: int
    width: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    mlp_dim: int
    n_tokens: int           # P, prefix tokens
    dtype: str = "bf16"
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0
    weight_std: float = 0.02
    seed: int = 0

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def with_(self, **kw) -> "PrefillShape":
        return replace(self, **kw)

    def layer_params(self) -> int:
        w, f = self.width, self.mlp_dim
        return w * (self.q_dim + 2 * self.kv_dim) + self.q_dim * w + 3 * w * f + 2 * w

    def flops(self) -> float:
        """Dense FLOPs of the prefill: every layer but the last in full
        (projections and attention), the last one's K/V projection only."""
        p, w, f = self.n_tokens, self.width, self.mlp_dim
        full = 2 * p * (w * (self.q_dim + 2 * self.kv_dim) + self.q_dim * w + 3 * w * f) + \
            4 * p * p * self.q_dim
        return (self.n_layers - 1) * full + 2 * p * w * 2 * self.kv_dim


GEMMA2B_PREFILL = PrefillShape(
    name="gemma2b-prefill", n_layers=18, width=2048, n_q_heads=8, n_kv_heads=1, head_dim=256, mlp_dim=16384,
    n_tokens=816,
)

PREFILLS = {c.name: c for c in (GEMMA2B_PREFILL,)}


def get_prefill_config(name: str, **overrides) -> PrefillShape:
    cfg = PREFILLS[name]
    return cfg.with_(**overrides) if overrides else cfg
