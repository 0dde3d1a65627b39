"""Oracle: the VLM prefill that writes the action expert's prefix KV cache,
and prefill followed by the denoising loop, fp64 on the CPU.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this module.
It shares no code with the product package; its elementary operations are
the ones of ``oracle.expert``.

Passages followed (page titles and sections):
  [DM0.5]  "DM0.5: high-performance embodied VLA and OpenDM reading guide"
           sec. 5.1 (the prefix -- images, text, state -- is encoded once
           into a per-layer KV cache that every denoising step reads),
           sec. 5.2 (the suffix reads that cache), sec. 6.2 (prefix
           attention), sec. 6.5 (one captured graph per request).
  [RTVLA]  "Running VLAs at Real-time Speed" (the prefix pass is the VLM
           forward over the observation's tokens; tens of layers).

Readings where the pages are silent (the plainest one in each case):
  R15 prefill stack: Gemma layers of the expert's form (RMSNorm with gain
      1+g, q/k/v without bias, RoPE at positions 0..P-1, softmax attention
      in which every prefix token sees every prefix token, o_proj +
      residual, GeGLU (tanh) MLP + residual).  Layer l's keys (after RoPE)
      and values are the expert's cached prefix of layer l, so the stack has
      as many layers as the expert and the same kv heads and head_dim.  The
      last layer's attention output and MLP feed nothing and are not
      computed.
Pins (tests/test_oracle_prefill_pins.py): the zero-first-layer closed form,
token permutation equivariance without RoPE, the single-token closed form,
an independent PyTorch statement, and prefill + denoise = denoise on the
prefill's cache.  prefill_kv with random weights: parity unpinned by the
pages (no worked example); pinned only through those.
"""

from __future__ import annotations

from typing import Callable, Dict

import numpy as np

from .expert import F64, attention, denoise, gelu_tanh, linear, rms_norm, rope, to_f64


def prefill_kv(layer_weights: Callable[[int], Dict[str, np.ndarray]], pcfg, emb: np.ndarray) -> np.ndarray:
    """Prefix KV cache [L][2][1][P][Hkv][D] of one observation from its
    embeddings emb [P][w] (reading R15).  layer_weights(l) gives layer l's
    parameters under the names "layers.l.*" (fetched one layer at a time,
    so that a large stack need not be held in fp64 at once)."""
    h = np.asarray(emb, dtype=F64)
    p_len = h.shape[0]
    hq, hkv, d = pcfg.n_q_heads, pcfg.n_kv_heads, pcfg.head_dim
    positions = np.arange(p_len)
    visible = np.ones((p_len, p_len), dtype=bool)
    kv = np.zeros((pcfg.n_layers, 2, 1, p_len, hkv, d), dtype=F64)
    for l in range(pcfg.n_layers):
        W = to_f64(layer_weights(l))
        p = f"layers.{l}."
        u = rms_norm(h, W[p + "attn_norm.g"], pcfg.rms_eps)
        k = rope(linear(u, W[p + "k_proj.w"]).reshape(p_len, hkv, d), positions, pcfg.rope_theta)
        v = linear(u, W[p + "v_proj.w"]).reshape(p_len, hkv, d)
        kv[l, 0, 0] = k
        kv[l, 1, 0] = v
        if l == pcfg.n_layers - 1:
            break
        q = rope(linear(u, W[p + "q_proj.w"]).reshape(p_len, hq, d), positions, pcfg.rope_theta)
        o = attention(q, k, v, visible).reshape(p_len, hq * d)
        h = h + linear(o, W[p + "o_proj.w"])
        u = rms_norm(h, W[p + "mlp_norm.g"], pcfg.rms_eps)
        m = gelu_tanh(linear(u, W[p + "gate_proj.w"])) * linear(u, W[p + "up_proj.w"])
        h = h + linear(m, W[p + "down_proj.w"])
    return kv


def prefill_denoise(layer_weights: Callable[[int], Dict[str, np.ndarray]], pcfg, W_exp: Dict[str, np.ndarray],
                    cfg, emb: np.ndarray, noise: np.ndarray, state: np.ndarray, n_steps: int) -> np.ndarray:
    """Action chunk [1][H][A]: the prefill writes the cache, then the expert
    denoises from noise [1][H][A] with state [1][Sd] ([DM0.5] 5.1-5.3)."""
    kv = prefill_kv(layer_weights, pcfg, emb)
    return denoise(to_f64(W_exp), cfg, noise, state, kv, n_steps)
