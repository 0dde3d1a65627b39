"""Pins of the oracle's VLM prefill ("DM0.5 reading guide" sec. 5.1: the
prefix is encoded once into a per-layer KV cache) against closed forms,
symmetry and an independent PyTorch statement.

A slip in the prefill oracle -- a residual dropped between layers, keys
stored before RoPE, a mask that hides part of the prefix, a softmax without
its denominator, layer l's cache taken from the wrong layer's input -- fails
one of these.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import expert as O
from oracle import prefill as OP
from synthetic import get_config, get_prefill_config, make_noise, make_prefill_weights, make_prefix_embeddings, \
    make_state, make_weights
from tests import torch_restatement as TR

MATRICES = ("q_proj.w", "k_proj.w", "v_proj.w", "o_proj.w", "gate_proj.w", "up_proj.w", "down_proj.w")


def small(**kw):
    base = dict(n_layers=3, width=256, n_q_heads=4, n_kv_heads=1, head_dim=64, mlp_dim=512, n_tokens=24,
                dtype="f32")
    base.update(kw)
    return get_prefill_config("gemma2b-prefill", **base)


def provider(W):
    return lambda l: {k: v for k, v in W.items() if k.startswith(f"layers.{l}.")}


def _rope_ref(x, theta):
    pos = torch.arange(x.shape[0])
    return TR.rope_complex(torch.tensor(x)[None], pos, theta)[0].numpy()


def test_zero_first_layer_passes_the_embeddings_to_the_second():
    """Layer 0 with all matrices 0 adds nothing, so layer 1's cache is its
    projection of RMSNorm_1(emb); layer 0's own cache is all zero."""
    pc = small(n_layers=2)
    W = O.to_f64(make_prefill_weights(pc))
    for m in MATRICES:
        W["layers.0." + m][:] = 0.0
    emb = make_prefix_embeddings(pc).astype(np.float64)
    kv = OP.prefill_kv(provider(W), pc, emb)
    assert np.all(kv[0] == 0.0)
    u = F.rms_norm(torch.tensor(emb), (pc.width,), weight=1.0 + torch.tensor(W["layers.1.attn_norm.g"]),
                   eps=pc.rms_eps).numpy()
    k = (u @ W["layers.1.k_proj.w"].T).reshape(pc.n_tokens, 1, pc.head_dim)
    v = (u @ W["layers.1.v_proj.w"].T).reshape(pc.n_tokens, 1, pc.head_dim)
    np.testing.assert_allclose(kv[1, 0, 0], _rope_ref(k, pc.rope_theta), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(kv[1, 1, 0], v, rtol=1e-12, atol=1e-13)


def test_single_token_attends_to_itself_only():
    """One prefix token: the softmax over a single key is 1, so every q head
    reads the token's own value, and layer 1 sees emb + W_o [v; ...; v] + MLP."""
    pc = small(n_layers=2, n_tokens=1, rope_theta=0.0)
    W = O.to_f64(make_prefill_weights(pc, seed=2))
    emb = make_prefix_embeddings(pc, seed=2).astype(np.float64)
    kv = OP.prefill_kv(provider(W), pc, emb)
    v0 = kv[0, 1, 0, 0, 0]
    h = emb + np.tile(v0, pc.n_q_heads) @ W["layers.0.o_proj.w"].T
    u = O.rms_norm(h, W["layers.0.mlp_norm.g"], pc.rms_eps)
    h = h + (O.gelu_tanh(u @ W["layers.0.gate_proj.w"].T) * (u @ W["layers.0.up_proj.w"].T)) @ \
        W["layers.0.down_proj.w"].T
    u1 = O.rms_norm(h, W["layers.1.attn_norm.g"], pc.rms_eps)
    np.testing.assert_allclose(kv[1, 1, 0, :, 0], u1 @ W["layers.1.v_proj.w"].T, rtol=1e-11, atol=1e-12)


def test_token_order_permutes_the_cache_without_rope():
    pc = small(rope_theta=0.0)
    W = make_prefill_weights(pc, seed=3)
    emb = make_prefix_embeddings(pc, seed=3)
    perm = np.random.default_rng(0).permutation(pc.n_tokens)
    a = OP.prefill_kv(provider(W), pc, emb[perm])
    b = OP.prefill_kv(provider(W), pc, emb)
    np.testing.assert_allclose(a, b[:, :, :, perm], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("theta,hkv", [(10000.0, 1), (0.0, 1), (10000.0, 2)])
def test_prefill_matches_independent_torch_statement(theta, hkv):
    pc = small(rope_theta=theta, n_kv_heads=hkv)
    W = make_prefill_weights(pc, seed=4)
    emb = make_prefix_embeddings(pc, seed=4)
    np.testing.assert_allclose(OP.prefill_kv(provider(W), pc, emb), TR.prefill_kv(W, pc, emb),
                               rtol=1e-10, atol=1e-12)


def test_prefill_then_denoise_is_denoise_on_the_prefilled_cache():
    cfg = get_config("tiny-fp32")
    pc = small(n_layers=cfg.n_layers, n_tokens=cfg.prefix_len, n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim)
    W = make_prefill_weights(pc, seed=5)
    We = O.to_f64(make_weights(cfg))
    emb = make_prefix_embeddings(pc, seed=5)
    noise, state = make_noise(cfg), make_state(cfg)
    got = OP.prefill_denoise(provider(W), pc, We, cfg, emb, noise, state, 3)
    kv = OP.prefill_kv(provider(W), pc, emb)
    np.testing.assert_array_equal(got, O.denoise(We, cfg, noise, state, kv, 3))
