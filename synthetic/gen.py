"""Seeded tensor generation.

Every tensor has its own stream: ``numpy.random.PCG64`` seeded with
``SeedSequence([seed, crc32(tensor name)])``, drawn with ``standard_normal``
in float32 and scaled by the tensor's standard deviation.  Adding or
removing a tensor therefore never changes another tensor's values.

Distributions (the workloads' stand-ins for the pages' real checkpoints and
camera/robot data, which are not available):
  * every weight matrix, bias and norm gain ~ N(0, 0.02)
  * prefix KV cache ~ N(0, 1)
  * noise eps ~ N(0, 1), robot state ~ N(0, 1)
  * FLASH draft chunk ~ N(0, 0.5) with the gripper dim set to +-1 and 0 or 1
    sign switch at a seeded row

bf16 inputs are produced by round-to-nearest-even of the float32 draw; both
the oracle and the CUDA path receive the same rounded values.

In an FP8-MLP workload the gate/up/down matrices are *given* in FP8 E4M3
storage with one fp32 scale per output row (the pi0-fp8mlp workload):
the float32 draw of a row is divided by scale = max|row| / 448 and rounded to
the nearest E4M3 value (ties to even).  The codes and scales are the inputs;
what an E4M3 code means is decoded by each side on its own.
"""

from __future__ import annotations

import zlib
from typing import Dict, List, Tuple

import numpy as np

from .configs import DraftShape, ExpertShape, PrefillShape


def _rng(seed: int, name: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, zlib.crc32(name.encode())])))


def _normal(seed: int, name: str, shape, std: float) -> np.ndarray:
    a = _rng(seed, name).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


# ---------------------------------------------------------------------------
# bf16 storage format (IEEE binary32 with the low 16 bits dropped after
# round-to-nearest-even).  Used only to produce inputs that are given in bf16.
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even); return the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """float32 array holding the bf16-rounded values of ``a``."""
    return bf16_bits_to_f32(f32_to_bf16_bits(a))


E4M3_MAX = 448.0


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """E4M3 codes (uint8: sign, 4 exponent bits with bias 7, 3 mantissa bits;
    no infinities) of float32 values with |x| <= 448, rounded to the nearest
    representable value, ties to even (storage encoding of given inputs)."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x).astype(np.float64)
    # quantum of the binade holding a: 2^(e-3) for normals (e >= -6), 2^-9 below 2^-6
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    q = 2.0 ** (e - 3)
    v = np.minimum(np.rint(a / q) * q, E4M3_MAX)          # numpy rint: half to even
    sub = v < 2.0 ** -6
    ev = np.floor(np.log2(np.where(sub, 1.0, v)))           # exponent of the rounded value
    mant = np.where(sub, np.rint(v / 2.0 ** -9), np.rint((v / 2.0 ** ev - 1.0) * 8.0))
    expf = np.where(sub, 0, ev + 7)
    code = (np.signbit(x).astype(np.uint32) << 7) | (expf.astype(np.uint32) << 3) | mant.astype(np.uint32)
    return code.astype(np.uint8)


# ---------------------------------------------------------------------------
# weights
# ---------------------------------------------------------------------------

def weight_names(cfg: ExpertShape) -> List[Tuple[str, Tuple[int, ...]]]:
    """(name, shape) of every expert parameter, matrices as [out][in]."""
    w, a, sd, f = cfg.width, cfg.action_dim, cfg.state_dim, cfg.mlp_dim
    tin = 2 * w if cfg.time_cond == "concat" else w
    out = [
        ("state_proj.w", (w, sd)), ("state_proj.b", (w,)),
        ("action_in_proj.w", (w, a)), ("action_in_proj.b", (w,)),
        ("time_mlp_in.w", (w, tin)), ("time_mlp_in.b", (w,)),
        ("time_mlp_out.w", (w, w)), ("time_mlp_out.b", (w,)),
    ]
    adarms = cfg.time_cond == "adarms"
    for l in range(cfg.n_layers):
        p = f"layers.{l}."
        out += [] if adarms else [(p + "attn_norm.g", (w,))]
        out += [
            (p + "q_proj.w", (cfg.q_dim, w)),
            (p + "k_proj.w", (cfg.kv_dim, w)),
            (p + "v_proj.w", (cfg.kv_dim, w)),
            (p + "o_proj.w", (w, cfg.q_dim)),
        ]
        out += [(p + "time_mod.w", (6 * w, w)), (p + "time_mod.b", (6 * w,))] if adarms else \
            [(p + "mlp_norm.g", (w,))]
        out += [
            (p + "gate_proj.w", (f, w)),
            (p + "up_proj.w", (f, w)),
            (p + "down_proj.w", (w, f)),
        ]
        if cfg.mlp_dtype == "fp8_e4m3":
            out += [(p + "gate_proj.s", (f,)), (p + "up_proj.s", (f,)), (p + "down_proj.s", (w,))]
    out += [("final_norm.g", (w,)), ("action_out_proj.w", (a, w)), ("action_out_proj.b", (a,))]
    return out


def make_weights(cfg: ExpertShape, seed: int | None = None) -> Dict[str, np.ndarray]:
    """All expert parameters as float32 arrays.

    In a "bf16" workload every 2-D matrix holds bf16-representable values
    (it is stored and streamed as bf16); 1-D biases and gains stay float32.
    In an FP8-MLP workload gate/up/down are uint8 E4M3 codes, each with a
    float32 per-row scale under the name ending in ".s".
    """
    seed = cfg.seed if seed is None else seed
    fp8 = cfg.mlp_dtype == "fp8_e4m3"
    ws: Dict[str, np.ndarray] = {}
    for name, shape in weight_names(cfg):
        if fp8 and name.endswith("_proj.s"):
            continue   # written with its matrix below
        a = _normal(seed, name, shape, cfg.weight_std)
        if fp8 and name.split(".")[-2] in ("gate_proj", "up_proj", "down_proj"):
            amax = np.max(np.abs(a), axis=1)
            scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
            ws[name] = e4m3_encode(a / scale[:, None])
            ws[name[:-2] + ".s"] = scale
            continue
        if cfg.dtype == "bf16" and len(shape) == 2:
            a = round_to_bf16(a)
        ws[name] = a
    return ws


def make_prefix_kv(cfg: ExpertShape, batch: int | None = None, prefix_len: int | None = None,
                   seed: int | None = None) -> np.ndarray:
    """Prefix KV cache [L][2][B][P][Hkv][D] ~ N(0,1) (bf16 values in a bf16 workload)."""
    seed = cfg.seed if seed is None else seed
    b = cfg.batch if batch is None else batch
    p = cfg.prefix_len if prefix_len is None else prefix_len
    kv = _normal(seed, "prefix_kv", (cfg.n_layers, 2, b, p, cfg.n_kv_heads, cfg.head_dim), 1.0)
    if cfg.dtype == "bf16":
        kv = round_to_bf16(kv)
    return kv


def make_noise(cfg: ExpertShape, batch: int | None = None, seed: int | None = None,
               name: str = "noise") -> np.ndarray:
    """eps ~ N(0,1), [B][H][A] float32."""
    seed = cfg.seed if seed is None else seed
    b = cfg.batch if batch is None else batch
    return _normal(seed, name, (b, cfg.chunk_len, cfg.action_dim), 1.0)


def make_state(cfg: ExpertShape, batch: int | None = None, seed: int | None = None) -> np.ndarray:
    """Robot state ~ N(0,1), [B][Sd] float32."""
    seed = cfg.seed if seed is None else seed
    b = cfg.batch if batch is None else batch
    return _normal(seed, "state", (b, cfg.state_dim), 1.0)


def make_draft(cfg: ExpertShape, n_switch: int = 0, seed: int | None = None) -> np.ndarray:
    """FLASH candidate chunk D [H][A] ~ N(0, draft_std); gripper dim in {-1,+1}.

    ``n_switch`` = 0: the gripper keeps one seeded sign over the chunk.
    ``n_switch`` = 1: the sign flips once, at a seeded row r in [1, H).
    """
    seed = cfg.seed if seed is None else seed
    d = _normal(seed, "draft", (cfg.chunk_len, cfg.action_dim), cfg.draft_std)
    rng = _rng(seed, "draft_gripper")
    sign0 = np.float32(1.0 if rng.integers(0, 2) else -1.0)
    g = np.full(cfg.chunk_len, sign0, dtype=np.float32)
    if n_switch:
        r = int(rng.integers(1, cfg.chunk_len))
        g[r:] = -sign0
    d[:, cfg.gripper] = g
    return d


# ---------------------------------------------------------------------------
# FLASH draft model (one Gemma block + linear action head over learnable
# action queries and the image features)
# ---------------------------------------------------------------------------

def draft_weight_names(dcfg: DraftShape) -> List[Tuple[str, Tuple[int, ...]]]:
    """(name, shape) of every draft-model parameter, matrices as [out][in]."""
    w, f = dcfg.width, dcfg.mlp_dim
    return [
        ("action_queries", (dcfg.n_queries, w)),
        ("attn_norm.g", (w,)),
        ("q_proj.w", (dcfg.q_dim, w)),
        ("k_proj.w", (dcfg.kv_dim, w)),
        ("v_proj.w", (dcfg.kv_dim, w)),
        ("o_proj.w", (w, dcfg.q_dim)),
        ("mlp_norm.g", (w,)),
        ("gate_proj.w", (f, w)),
        ("up_proj.w", (f, w)),
        ("down_proj.w", (w, f)),
        ("action_head.w", (dcfg.action_dim, w)),
        ("action_head.b", (dcfg.action_dim,)),
    ]


def make_draft_weights(dcfg: DraftShape, seed: int | None = None) -> Dict[str, np.ndarray]:
    """Draft-model parameters as float32 arrays: matrices, gains and the head
    bias ~ N(0, 0.02); the action queries ~ N(0, 1) (the scale of the visual
    tokens they are read beside).  In a "bf16" draft every weight matrix holds
    bf16-representable values; the queries stay float32 (they seed the fp32
    residual stream)."""
    seed = dcfg.seed if seed is None else seed
    ws: Dict[str, np.ndarray] = {}
    for name, shape in draft_weight_names(dcfg):
        std = 1.0 if name == "action_queries" else dcfg.weight_std
        a = _normal(seed, "draft." + name, shape, std)
        if dcfg.dtype == "bf16" and len(shape) == 2 and name != "action_queries":
            a = round_to_bf16(a)
        ws[name] = a
    return ws


def make_visual_tokens(dcfg: DraftShape, batch: int | None = None, n_vis: int | None = None,
                       seed: int | None = None) -> np.ndarray:
    """Image features [B][V][w] ~ N(0,1) (bf16 values in a bf16 draft): the
    stand-in for the vision encoder's projected tokens of one observation."""
    seed = dcfg.seed if seed is None else seed
    b = dcfg.batch if batch is None else batch
    v = dcfg.n_vis if n_vis is None else n_vis
    x = _normal(seed, "visual_tokens", (b, v, dcfg.width), 1.0)
    if dcfg.dtype == "bf16":
        x = round_to_bf16(x)
    return x



# ---------------------------------------------------------------------------
# VLM prefill (Gemma-style stack over the prefix embeddings)
# ---------------------------------------------------------------------------

def prefill_weight_names(pcfg: PrefillShape, layers=None) -> List[Tuple[str, Tuple[int, ...]]]:
    """(name, shape) of the prefill stack's parameters (the expert's layer
    names), for all layers or the given ones."""
    w, f = pcfg.width, pcfg.mlp_dim
    out = []
    for l in (range(pcfg.n_layers) if layers is None else layers):
        p = f"layers.{l}."
        out += [
            (p + "attn_norm.g", (w,)),
            (p + "q_proj.w", (pcfg.q_dim, w)),
            (p + "k_proj.w", (pcfg.kv_dim, w)),
            (p + "v_proj.w", (pcfg.kv_dim, w)),
            (p + "o_proj.w", (w, pcfg.q_dim)),
            (p + "mlp_norm.g", (w,)),
            (p + "gate_proj.w", (f, w)),
            (p + "up_proj.w", (f, w)),
            (p + "down_proj.w", (w, f)),
        ]
    return out


def make_prefill_weights(pcfg: PrefillShape, layers=None, seed: int | None = None) -> Dict[str, np.ndarray]:
    """Prefill-stack parameters ~ N(0, 0.02) as float32 arrays (bf16 values in
    a bf16 stack), for all layers or the given ones (each tensor has its own
    stream, so a subset equals the same entries of the whole)."""
    seed = pcfg.seed if seed is None else seed
    ws: Dict[str, np.ndarray] = {}
    for name, shape in prefill_weight_names(pcfg, layers):
        a = _normal(seed, "vlm." + name, shape, pcfg.weight_std)
        if pcfg.dtype == "bf16" and len(shape) == 2:
            a = round_to_bf16(a)
        ws[name] = a
    return ws


def make_prefix_embeddings(pcfg: PrefillShape, n_tokens: int | None = None, seed: int | None = None) -> np.ndarray:
    """Prefix embeddings [P][w] ~ N(0,1) (bf16 values in a bf16 stack): the
    stand-in for the vision tokens and text embeddings of one observation."""
    seed = pcfg.seed if seed is None else seed
    p = pcfg.n_tokens if n_tokens is None else n_tokens
    x = _normal(seed, "prefix_embeddings", (p, pcfg.width), 1.0)
    if pcfg.dtype == "bf16":
        x = round_to_bf16(x)
    return x
