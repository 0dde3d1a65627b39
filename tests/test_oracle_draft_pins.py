"""Pins of the oracle's FLASH draft model and round ("Realtime-VLA FLASH"
sec. 03.1-03.3) against closed forms, symmetries and an independent
PyTorch statement.

A slip in the draft oracle -- a dropped residual, the head applied to the
wrong rows, the queries placed before the visual tokens, a transposed
projection, a mask that hides part of the sequence -- fails one of these.
"""

import numpy as np
import pytest

from oracle import draft as OD
from oracle import expert as O
from synthetic import (get_config, get_draft_config, make_draft_weights, make_noise, make_prefix_kv,
                       make_state, make_visual_tokens, make_weights)
from tests import torch_restatement as TR

BLOCK_MATRICES = ("q_proj.w", "k_proj.w", "v_proj.w", "o_proj.w", "gate_proj.w", "up_proj.w", "down_proj.w")


def tiny_draft(**kw):
    return get_draft_config("draft-tiny", **kw)


def test_zero_block_is_the_head_on_the_queries():
    """All block matrices 0: attention and MLP add 0 to the residual, so the
    chunk is the action head applied to the queries, whatever the image."""
    d = tiny_draft()
    W = O.to_f64(make_draft_weights(d))
    for k in BLOCK_MATRICES:
        W[k][:] = 0.0
    vis = make_visual_tokens(d)[0]
    got = OD.draft_forward(W, d, vis)
    expect = W["action_queries"] @ W["action_head.w"].T + W["action_head.b"]
    np.testing.assert_allclose(got, expect, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(OD.draft_forward(W, d, 3.0 * vis), expect, rtol=1e-13, atol=1e-14)


def test_chunk_depends_on_the_image():
    d = tiny_draft()
    W = make_draft_weights(d)
    a = OD.draft_forward(W, d, make_visual_tokens(d, seed=1)[0])
    b = OD.draft_forward(W, d, make_visual_tokens(d, seed=2)[0])
    assert np.max(np.abs(a - b)) > 1e-4


def test_visual_token_order_is_irrelevant_without_rope():
    """Without positions, attention is a function of the set of keys: any
    permutation of the visual tokens leaves the chunk unchanged."""
    d = tiny_draft(rope_theta=0.0)
    W = make_draft_weights(d, seed=5)
    vis = make_visual_tokens(d, seed=5)[0]
    perm = np.random.default_rng(0).permutation(vis.shape[0])
    np.testing.assert_allclose(OD.draft_forward(W, d, vis[perm]), OD.draft_forward(W, d, vis),
                               rtol=1e-10, atol=1e-12)


def test_query_order_permutes_the_chunk_rows_without_rope():
    d = tiny_draft(rope_theta=0.0)
    W = make_draft_weights(d, seed=6)
    vis = make_visual_tokens(d, seed=6)[0]
    perm = np.random.default_rng(1).permutation(d.n_queries)
    Wp = dict(W)
    Wp["action_queries"] = W["action_queries"][perm]
    np.testing.assert_allclose(OD.draft_forward(Wp, d, vis), OD.draft_forward(W, d, vis)[perm],
                               rtol=1e-10, atol=1e-12)


def test_rope_makes_the_visual_order_matter():
    d = tiny_draft()
    W = make_draft_weights(d, seed=7)
    vis = make_visual_tokens(d, seed=7)[0]
    a = OD.draft_forward(W, d, vis[::-1].copy())
    b = OD.draft_forward(W, d, vis)
    assert np.max(np.abs(a - b)) > 1e-6


@pytest.mark.parametrize("theta,hkv,batch", [(10000.0, 1, 2), (0.0, 1, 1), (10000.0, 2, 1)])
def test_draft_matches_independent_torch_statement(theta, hkv, batch):
    d = tiny_draft(rope_theta=theta, n_kv_heads=hkv)
    W = make_draft_weights(d, seed=8)
    vis = make_visual_tokens(d, batch=batch, seed=8)
    ref = TR.draft(W, d, vis)
    got = OD.draft_forward_batch(W, d, vis)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)


def test_batch_elements_are_independent():
    d = tiny_draft()
    W = make_draft_weights(d)
    vis = make_visual_tokens(d, batch=3, seed=9)
    both = OD.draft_forward_batch(W, d, vis)
    np.testing.assert_array_equal(both[2], OD.draft_forward(W, d, vis[2]))


# ---------------------------------------------------------------------------
# one FLASH round: draft -> verify -> accept or fall back
# ---------------------------------------------------------------------------

def _round_setup(gripper_pattern):
    """A zero-block draft whose gripper output is the sign pattern given
    (the head's gripper row reads query feature 0, which is set to it)."""
    cfg = get_config("tiny-fp32")
    d = tiny_draft()
    We = O.to_f64(make_weights(cfg))
    Wd = O.to_f64(make_draft_weights(d))
    for k in BLOCK_MATRICES:
        Wd[k][:] = 0.0
    g = cfg.gripper
    Wd["action_head.w"][g] = 0.0
    Wd["action_head.w"][g, 0] = 1.0
    Wd["action_head.b"][g] = 0.0
    Wd["action_queries"][:, 0] = np.asarray(gripper_pattern, dtype=np.float64)
    vis = make_visual_tokens(d)[0]
    kv = make_prefix_kv(cfg)
    state = make_state(cfg)[0]
    eps = make_noise(cfg)[0]
    return cfg, d, We, Wd, vis, kv, state, eps


def test_round_accepts_the_draft_when_every_distance_passes():
    cfg, d, We, Wd, vis, kv, state, eps = _round_setup([1.0] * 8)
    chunk, n_acc, flags, full, draft = OD.flash_round(We, cfg, Wd, d, vis, kv, state, eps, (0.2, 0.5, 0.8),
                                                      np.inf, cfg.gripper, 4)
    assert (n_acc, flags, full) == (cfg.chunk_len, 0, False)
    np.testing.assert_array_equal(chunk, draft)
    np.testing.assert_allclose(draft, Wd["action_queries"] @ Wd["action_head.w"].T + Wd["action_head.b"],
                               rtol=1e-13, atol=1e-14)


def test_round_falls_back_on_zero_accepted_length():
    cfg, d, We, Wd, vis, kv, state, eps = _round_setup([1.0] * 8)
    chunk, n_acc, flags, full, _ = OD.flash_round(We, cfg, Wd, d, vis, kv, state, eps, (0.2, 0.5), 0.0,
                                                  cfg.gripper, 4)
    assert (n_acc, flags, full) == (0, O.FLAG_ZERO_ACCEPT, True)
    np.testing.assert_array_equal(chunk, O.denoise(We, cfg, eps[None], state[None], kv, 4)[0])


def test_round_falls_back_on_a_gripper_switch_even_when_distances_pass():
    cfg, d, We, Wd, vis, kv, state, eps = _round_setup([1.0, 1.0, 1.0, -1.0, -1.0, -1.0, -1.0, -1.0])
    chunk, n_acc, flags, full, _ = OD.flash_round(We, cfg, Wd, d, vis, kv, state, eps, (0.5,), np.inf,
                                                  cfg.gripper, 3)
    assert n_acc == cfg.chunk_len and full
    assert flags == O.FLAG_SWITCH | O.FLAG_SWITCH_IN_PREFIX
    np.testing.assert_array_equal(chunk, O.denoise(We, cfg, eps[None], state[None], kv, 3)[0])
