"""Oracle: the FLASH draft model and one FLASH round, fp64 on the CPU.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this module.
It shares no code with the product package; its elementary operations are
the ones of ``oracle.expert``.

Passages followed (page titles and sections):
  [FLASH]  "Realtime-VLA FLASH: speculative inference for diffusion VLAs"
           sec. 03.1 (draft action generation: the draft model is a single
           Gemma block plus a linear action head, about 110M parameters; on
           the fast path the VLM prefill is skipped and the current image
           features go to the draft model, whose learnable action queries
           read the visual context and emit the whole candidate chunk in one
           forward pass), sec. 03.2 (multi-step parallel verification; zero
           accepted length -> full path), sec. 03.3 (a gripper switch in the
           candidate chunk forces the full path even when the distances pass).
  [DM0.5]  "DM0.5: high-performance embodied VLA and OpenDM reading guide"
           sec. 5.2 (the Gemma-style block: RMSNorm, grouped-query attention,
           gated MLP), sec. 5.3 (the full path: Euler denoising).

Readings where the pages are silent (the plainest one in each case):
  R13 draft block: the block is the expert's own layer type (Gemma RMSNorm
      with gain 1+g, q/k/v projections without bias, RoPE at positions
      0..V+H-1 of the sequence [visual tokens ; action queries], softmax
      attention in which every row sees every row, o_proj added to the
      residual, GeGLU (tanh) MLP added to the residual).  The action head is
      a linear map with bias applied to the query rows straight after the
      block (no norm in between: the page names only the block and the
      head).  The visual rows' own outputs feed nothing; one block means
      their keys and values depend on the visual tokens alone.
  R14 FLASH round: one noise sample eps per round serves both the
      verification (interpolation at every tau) and, on fallback, as the
      starting point x_1 of the full path's Euler integration.  The full path
      reuses the cached prefix (the observation's VLM prefill is outside the
      suffix loop).  On acceptance the returned chunk is the draft; the
      accepted length says how much of it the caller may execute.
Pins (tests/test_oracle_draft_pins.py): the zero-block closed form (all
block matrices zero -> head applied to the queries), invariance to the order
of the visual tokens without RoPE, equivariance in the query order without
RoPE, an independent PyTorch statement, and every branch of the round.
draft_forward with random weights: parity unpinned by the pages (they print
no worked example); pinned only through those closed forms, symmetries and
the independent statement.
"""

from __future__ import annotations

from typing import Dict, Sequence, Tuple

import numpy as np

from .expert import (F64, attention, denoise, fallback, gelu_tanh, linear, rms_norm, rope, to_f64,
                     verify)


def draft_block(W: Dict[str, np.ndarray], dcfg, x: np.ndarray) -> np.ndarray:
    """One Gemma block over the whole sequence x [n][w] (reading R13)."""
    n = x.shape[0]
    hq, hkv, d = dcfg.n_q_heads, dcfg.n_kv_heads, dcfg.head_dim
    positions = np.arange(n)
    visible = np.ones((n, n), dtype=bool)
    u = rms_norm(x, W["attn_norm.g"], dcfg.rms_eps)
    q = rope(linear(u, W["q_proj.w"]).reshape(n, hq, d), positions, dcfg.rope_theta)
    k = rope(linear(u, W["k_proj.w"]).reshape(n, hkv, d), positions, dcfg.rope_theta)
    v = linear(u, W["v_proj.w"]).reshape(n, hkv, d)
    o = attention(q, k, v, visible).reshape(n, hq * d)
    h = x + linear(o, W["o_proj.w"])
    u = rms_norm(h, W["mlp_norm.g"], dcfg.rms_eps)
    m = gelu_tanh(linear(u, W["gate_proj.w"])) * linear(u, W["up_proj.w"])
    return h + linear(m, W["down_proj.w"])


def draft_forward(W: Dict[str, np.ndarray], dcfg, vis: np.ndarray) -> np.ndarray:
    """Candidate chunk [H][A] from the image features vis [V][w] of one
    observation ([FLASH] 03.1): the learnable action queries are appended to
    the visual tokens, the block runs once, and the action head reads the
    query rows."""
    W = to_f64(W)
    vis = np.asarray(vis, dtype=F64)
    queries = W["action_queries"]
    h = draft_block(W, dcfg, np.concatenate([vis, queries], axis=0))
    return linear(h[vis.shape[0]:], W["action_head.w"], W["action_head.b"])


def draft_forward_batch(W: Dict[str, np.ndarray], dcfg, vis: np.ndarray) -> np.ndarray:
    """[B][H][A] for vis [B][V][w]; batch elements are independent."""
    return np.stack([draft_forward(W, dcfg, vis[b]) for b in range(vis.shape[0])])


def flash_round(W_exp: Dict[str, np.ndarray], cfg, W_draft: Dict[str, np.ndarray], dcfg, vis: np.ndarray,
                prefix_kv: np.ndarray, state: np.ndarray, eps: np.ndarray, taus: Sequence[float], delta: float,
                gripper_dim: int, n_steps: int) -> Tuple[np.ndarray, int, int, bool, np.ndarray]:
    """One round of the dual-path runtime ([FLASH] 03; reading R14).

    vis [V][w]; prefix_kv [L][2][1][P][Hkv][D]; state [Sd]; eps [H][A].
    Returns (chunk [H][A], accepted length, flags, took the full path, draft).
    """
    W_exp = to_f64(W_exp)
    draft = draft_forward(W_draft, dcfg, vis)
    n_acc, flags, _ = verify(W_exp, cfg, draft, eps, state, prefix_kv, taus, delta, gripper_dim)
    if fallback(flags):
        chunk = denoise(W_exp, cfg, np.asarray(eps, F64)[None], np.asarray(state, F64)[None], prefix_kv,
                        n_steps)[0]
        return chunk, n_acc, flags, True, draft
    return draft, n_acc, flags, False, draft
