"""GPU parity of the FLASH draft model and round ("Realtime-VLA FLASH" sec.
03.1-03.3) against the oracle, through the C ABI.

Tolerances as for the expert: fp32 max-abs <= 1e-4; bf16 (tensor-core
inputs rounded to bf16, fp32 accumulation) relative L2 <= 1e-2 and
max-abs <= 3e-2.  Accepted lengths and flags are compared exactly.
"""

import os

import numpy as np
import pytest

from oracle import draft as OD
from oracle import expert as O
from synthetic import (get_config, get_draft_config, make_draft_weights, make_noise, make_state,
                       make_visual_tokens)
from tests.helpers import bf16_tolerance_ok, build_expert, rel_l2

pytestmark = pytest.mark.gpu

BLOCK_MATRICES = ("q_proj.w", "k_proj.w", "v_proj.w", "o_proj.w", "gate_proj.w", "up_proj.w", "down_proj.w")

# a bf16 draft small enough for the oracle, on the tensor-core path: width
# 512, 2 q / 1 kv heads of 256, GeGLU 2048, 50 queries
SMALL_BF16 = dict(width=512, n_q_heads=2, n_kv_heads=1, head_dim=256, mlp_dim=2048, n_queries=50, action_dim=32,
                  n_vis=100, dtype="bf16")


def _draft(dcfg, weights=None, batch=1, n_vis=None, max_vis=None):
    from flow_matching_action_dm0_b200 import DraftModel
    weights = make_draft_weights(dcfg) if weights is None else weights
    n_vis = dcfg.n_vis if n_vis is None else n_vis
    vis = make_visual_tokens(dcfg, batch=batch, n_vis=n_vis)
    dm = DraftModel(dcfg, max_vis=max_vis or n_vis, max_batch=batch)
    dm.load(weights)
    got = dm.forward(vis)
    s, bits = dm.status()
    assert s == 0 and bits == 0
    assert dm.kernels_per_call(n_vis, batch) > 0
    path = dm.path
    dm.close()
    ref = OD.draft_forward_batch(weights, dcfg, vis)
    return got, ref, path


@pytest.mark.parametrize("batch,n_vis", [(1, 64), (2, 37), (1, 1)])
def test_fp32_draft_matches_oracle(cuda_ok, batch, n_vis):
    dcfg = get_draft_config("draft-tiny")
    got, ref, path = _draft(dcfg, batch=batch, n_vis=n_vis)
    assert path == "simt"
    assert np.max(np.abs(got - ref)) <= 1e-4, np.max(np.abs(got - ref))


def test_fp32_draft_without_rope_and_two_kv_heads(cuda_ok):
    dcfg = get_draft_config("draft-tiny", rope_theta=0.0, n_kv_heads=2)
    got, ref, _ = _draft(dcfg)
    assert np.max(np.abs(got - ref)) <= 1e-4


@pytest.mark.parametrize("batch,n_vis", [(1, 100), (2, 64), (3, 130), (1, 1)])
def test_bf16_draft_tensor_cores_match_oracle(cuda_ok, batch, n_vis):
    dcfg = get_draft_config("flash-draft", **SMALL_BF16)
    got, ref, path = _draft(dcfg, batch=batch, n_vis=n_vis)
    assert path == "tcgen05"
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


def test_bf16_draft_simt_path_matches_oracle(cuda_ok, monkeypatch):
    monkeypatch.setenv("RTV_PATH", "simt")
    dcfg = get_draft_config("flash-draft", **SMALL_BF16)
    got, ref, path = _draft(dcfg, n_vis=70)
    assert path == "simt"
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


def test_flash_draft_full_size_matches_oracle(cuda_ok):
    """The 110M-parameter block over the 768 image tokens, as timed."""
    dcfg = get_draft_config("flash-draft")
    got, ref, path = _draft(dcfg)
    assert path == "tcgen05"
    err_rel, err_abs = rel_l2(got, ref), float(np.max(np.abs(got - ref)))
    print(f"flash-draft rel_l2={err_rel:.3e} max_abs={err_abs:.3e}")
    assert err_rel <= 1e-2 and err_abs <= 3e-2


def test_draft_zero_block_is_the_head_on_the_queries(cuda_ok):
    dcfg = get_draft_config("flash-draft", **SMALL_BF16)
    W = make_draft_weights(dcfg)
    for k in BLOCK_MATRICES:
        W[k] = np.zeros_like(W[k])
    got, ref, _ = _draft(dcfg, weights=W)
    expect = W["action_queries"].astype(np.float64) @ W["action_head.w"].T.astype(np.float64) + W["action_head.b"]
    np.testing.assert_allclose(ref[0], expect, rtol=1e-12, atol=1e-12)
    assert np.max(np.abs(got[0] - expect)) <= 1e-3


def test_draft_refuses_shapes_beyond_its_maxima(cuda_ok):
    from flow_matching_action_dm0_b200 import DraftModel, RtvError
    dcfg = get_draft_config("draft-tiny")
    dm = DraftModel(dcfg, max_vis=32, max_batch=1)
    with pytest.raises(RtvError):
        dm.forward(make_visual_tokens(dcfg, n_vis=16))   # not loaded yet
    dm.load(make_draft_weights(dcfg))
    with pytest.raises(RtvError):
        dm.forward(make_visual_tokens(dcfg, n_vis=33))
    with pytest.raises(RtvError):
        dm.forward(make_visual_tokens(dcfg, batch=2, n_vis=16))
    dm.close()


# ---------------------------------------------------------------------------
# rounds
# ---------------------------------------------------------------------------

def _round_inputs(dcfg, cfg, gripper_pattern):
    """Zero-block draft whose gripper output is the given sign pattern."""
    W = make_draft_weights(dcfg)
    for k in BLOCK_MATRICES:
        W[k] = np.zeros_like(W[k])
    g = cfg.gripper
    W["action_head.w"] = W["action_head.w"].copy()
    W["action_head.w"][g] = 0.0
    W["action_head.w"][g, 0] = 1.0
    W["action_head.b"] = W["action_head.b"].copy()
    W["action_head.b"][g] = 0.0
    W["action_queries"] = W["action_queries"].copy()
    W["action_queries"][:, 0] = np.asarray(gripper_pattern, dtype=np.float32)
    return W


@pytest.mark.parametrize("case", ["accept", "zero", "switch", "random"])
def test_round_matches_oracle(cuda_ok, case):
    from flow_matching_action_dm0_b200 import DraftModel, flash_round
    cfg = get_config("tiny-fp32")
    dcfg = get_draft_config("draft-tiny")
    H = cfg.chunk_len
    pattern = [1.0] * H if case != "switch" else [1.0] * 3 + [-1.0] * (H - 3)
    Wd = make_draft_weights(dcfg) if case == "random" else _round_inputs(dcfg, cfg, pattern)
    delta = {"accept": np.inf, "zero": 0.0, "switch": np.inf, "random": 0.5}[case]
    n_steps = 4
    ex, We, kv = build_expert(cfg, batch=1)
    dm = DraftModel(dcfg, max_batch=1)
    dm.load(Wd)
    vis = make_visual_tokens(dcfg)[0]
    eps, state = make_noise(cfg)[0], make_state(cfg)[0]
    taus = (0.2, 0.5, 0.8)
    r = flash_round(ex, dm, vis, eps, state, taus, delta, cfg.gripper, n_steps)
    chunk, n_acc, flags, full, draft = OD.flash_round(We, cfg, Wd, dcfg, vis, kv, state, eps, taus, delta,
                                                      cfg.gripper, n_steps)
    assert (r.accepted_len, r.flags, r.used_full) == (n_acc, flags, full)
    assert np.max(np.abs(r.chunk - chunk)) <= 1e-4
    if case == "accept":
        assert (n_acc, flags, full) == (H, 0, False)
    elif case == "zero":
        assert full and flags == O.FLAG_ZERO_ACCEPT
    elif case == "switch":
        assert full and flags & O.FLAG_SWITCH
    dm.close()
    ex.close()


def test_full_size_round_is_consistent(cuda_ok):
    """pi0-bf16 expert + flash-draft: the verdict follows the rule and the
    chunk is the one of the branch taken (the draft, or the denoised chunk
    from the same noise)."""
    from flow_matching_action_dm0_b200 import DraftModel, flash_round
    cfg = get_config("pi0-bf16")
    dcfg = get_draft_config("flash-draft")
    ex, _, _ = build_expert(cfg, batch=1)
    dm = DraftModel(dcfg, max_batch=1)
    dm.load(make_draft_weights(dcfg))
    vis = make_visual_tokens(dcfg)
    eps, state = make_noise(cfg)[0], make_state(cfg)[0]
    draft = dm.forward(vis)[0]
    for delta in (0.0, 1e6):
        r = flash_round(ex, dm, vis[0], eps, state, cfg.taus, delta, cfg.gripper, 10)
        acc, flags, _ = ex.verify(draft, eps, state, cfg.taus, delta, cfg.gripper)
        assert (r.accepted_len, r.flags) == (acc, flags)
        assert r.used_full == bool(flags & (O.FLAG_ZERO_ACCEPT | O.FLAG_SWITCH))
        if r.used_full:
            # the denoised chunk from the same noise (fp32 sums in arrival order: equal to rounding)
            expect = ex.denoise(eps[None], state[None], 10)[0]
            assert rel_l2(r.chunk, expect) <= 1e-5
        else:
            np.testing.assert_array_equal(r.chunk, draft)
    s, bits = dm.status()
    assert s == 0 and bits == 0
    dm.close()
    ex.close()
