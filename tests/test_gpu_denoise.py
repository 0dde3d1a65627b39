"""GPU parity of rtv_denoise against the oracle (C ABI through the binding).

Tolerances are the ones fixed for this path: final-action max-abs error
<= 1e-4 for the fp32 expert; relative L2 <= 1e-2 and max-abs <= 3e-2 for the
bf16 expert.
"""

import os

import numpy as np
import pytest

from oracle import expert as O
from synthetic import get_config, make_noise, make_prefix_kv, make_state, make_weights
from tests.helpers import bf16_tolerance_ok, build_expert, rel_l2

pytestmark = pytest.mark.gpu


def run_denoise(cfg, n_steps=10, batch=1, weights=None, kv=None, seed=0, prefix_len=None):
    ex, weights, kv = build_expert(cfg, weights=weights, kv=kv, batch=batch, prefix_len=prefix_len)
    noise = make_noise(cfg, batch=batch, seed=seed)
    state = make_state(cfg, batch=batch, seed=seed)
    got = ex.denoise(noise, state, n_steps)
    s, bits = ex.status()
    assert s == 0 and bits == 0
    path = ex.path
    ex.close()
    ref = O.denoise(O.to_f64(weights), cfg, noise, state, kv, n_steps)
    return got, ref, path


@pytest.mark.parametrize("variant", [
    {}, {"suffix_mask": "pi0_block"}, {"rope_theta": 0.0}, {"n_kv_heads": 2},
])
def test_tiny_fp32_denoise_matches_oracle(cuda_ok, variant):
    cfg = get_config("tiny-fp32", **variant)
    got, ref, _ = run_denoise(cfg)
    assert np.max(np.abs(got - ref)) <= 1e-4


def test_tiny_fp32_batch_and_ragged_prefix(cuda_ok):
    cfg = get_config("tiny-fp32")
    # batch 3 with a prefix shorter than the config's (ragged, not a multiple of 16)
    got, ref, _ = run_denoise(cfg, batch=3, prefix_len=37, n_steps=4)
    assert np.max(np.abs(got - ref)) <= 1e-4


def test_tiny_fp32_single_prefix_token_and_one_step(cuda_ok):
    cfg = get_config("tiny-fp32")
    got, ref, _ = run_denoise(cfg, prefix_len=1, n_steps=1)
    assert np.max(np.abs(got - ref)) <= 1e-4


def test_constant_velocity_expert_lands_on_noise_minus_bias(cuda_ok):
    """Zero action_out weights: v == b for any input, so the chunk is eps - b."""
    for name in ("tiny-fp32", "pi0-bf16"):
        cfg = get_config(name) if name == "tiny-fp32" else get_config(name, n_layers=2)
        w = make_weights(cfg)
        w["action_out_proj.w"] = np.zeros_like(w["action_out_proj.w"])
        got, _, _ = run_denoise(cfg, weights=w, n_steps=10)
        noise = make_noise(cfg)
        expect = noise.astype(np.float64) - w["action_out_proj.b"].astype(np.float64)
        assert np.max(np.abs(got - expect)) <= 1e-5 * max(1.0, np.max(np.abs(expect)))


def test_pi0_two_layer_bf16_denoise_matches_oracle(cuda_ok):
    cfg = get_config("pi0-bf16", n_layers=2, prefix_len=100)
    got, ref, _ = run_denoise(cfg, n_steps=3)
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


@pytest.mark.parametrize("prefix_len", [37, 64, 960, 961])
def test_pi0_bf16_prefix_tiling_edges(cuda_ok, prefix_len):
    """Prefix lengths at the attention's 64-key tile edges: one partial tile,
    one full tile, the most tiles the tensor-core attention takes (15 prefix
    tiles + the suffix tile), and one key more (the warp-MMA attention)."""
    cfg = get_config("pi0-bf16", n_layers=1, prefix_len=prefix_len)
    got, ref, _ = run_denoise(cfg, n_steps=2)
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


@pytest.mark.parametrize("variant", [
    {"suffix_mask": "pi0_block"}, {"n_kv_heads": 2}, {"n_kv_heads": 8}, {"rope_theta": 0.0},
])
def test_pi0_bf16_attention_variants(cuda_ok, variant):
    """Mask, grouped and ungrouped KV heads (8 KV heads: no head pair shares
    one, so the warp-MMA attention runs), no RoPE."""
    cfg = get_config("pi0-bf16", n_layers=2, prefix_len=200, **variant)
    got, ref, _ = run_denoise(cfg, n_steps=2)
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


def test_warp_mma_attention_matches_oracle(cuda_ok, monkeypatch):
    """The warp-MMA attention kernel, selected explicitly, on the full prefix."""
    monkeypatch.setenv("RTV_ATTN", "mma")
    cfg = get_config("pi0-bf16", n_layers=2)
    got, ref, _ = run_denoise(cfg, n_steps=3)
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


def test_pi0_full_bf16_denoise_matches_oracle(cuda_ok):
    """The full 18-layer, 816-prefix, 10-step chunk, compared element by element."""
    cfg = get_config("pi0-bf16")
    got, ref, path = run_denoise(cfg, n_steps=10)
    err_rel, err_abs = rel_l2(got, ref), float(np.max(np.abs(got - ref)))
    print(f"pi0-bf16 path={path} rel_l2={err_rel:.3e} max_abs={err_abs:.3e}")
    assert err_rel <= 1e-2 and err_abs <= 3e-2


def test_pi0_bf16_batch_two_matches_oracle(cuda_ok):
    cfg = get_config("pi0-bf16", n_layers=3)
    got, ref, _ = run_denoise(cfg, batch=2, n_steps=2)
    assert bf16_tolerance_ok(got, ref)


@pytest.mark.parametrize("batch", [3, 4, 5])
def test_pi0_bf16_small_batches_token_tiling(cuda_ok, batch):
    """153, 204 and 255 token rows: each projection picks its own token tiling
    (1-4 tiles, the last one ragged) with its split; over the 816-token prefix
    the attention grid (14 key tiles x 4 head pairs x batch) exceeds the SM
    count, so it takes the compact two-CTAs-per-SM layout."""
    cfg = get_config("pi0-bf16", n_layers=2)
    got, ref, path = run_denoise(cfg, batch=batch, n_steps=2)
    assert path == "tcgen05"
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


def test_pi0_bf16_batch_sixteen_token_tiles(cuda_ok):
    """16 chunks = 816 token rows: four token tiles of the projections (the
    MMA N is at most 256), sixteen suffix groups in the attention."""
    cfg = get_config("pi0-bf16", n_layers=2, prefix_len=200)
    got, ref, path = run_denoise(cfg, batch=16, n_steps=2)
    assert path == "tcgen05"
    assert bf16_tolerance_ok(got, ref), (rel_l2(got, ref), np.max(np.abs(got - ref)))


@pytest.mark.parametrize("path", ["layered", "default"])
def test_repeat_calls_agree(cuda_ok, monkeypatch, path):
    """The layered kernels reduce split-K partial sums in a fixed rank order:
    repeated calls are bit-for-bit equal.  The resident kernel adds them in
    L2 in the order they arrive: repeated calls agree to fp32 rounding."""
    if path == "layered":
        monkeypatch.setenv("RTV_PATH", "layered")
    cfg = get_config("pi0-bf16", n_layers=2)
    ex, _, _ = build_expert(cfg)
    noise, state = make_noise(cfg), make_state(cfg)
    a = ex.denoise(noise, state, 5)
    b = ex.denoise(noise, state, 5)
    ex.close()
    if path == "layered":
        np.testing.assert_array_equal(a, b)
    else:
        assert rel_l2(b, a) <= 1e-5, rel_l2(b, a)


def test_simt_path_on_bf16_expert_matches_oracle(cuda_ok, monkeypatch):
    monkeypatch.setenv("RTV_PATH", "simt")
    cfg = get_config("pi0-bf16", n_layers=2, prefix_len=64)
    got, ref, path = run_denoise(cfg, n_steps=2)
    assert path == "simt"
    assert rel_l2(got, ref) <= 1e-4


def test_call_order_and_shape_errors(cuda_ok):
    from flow_matching_action_dm0_b200 import ActionExpert, RtvError
    cfg = get_config("tiny-fp32")
    ex = ActionExpert(cfg)
    with pytest.raises(RtvError) as e:
        ex.denoise(make_noise(cfg), make_state(cfg), 10)
    assert e.value.status == 3   # RTV_ERR_STATE
    ex.load(make_weights(cfg))
    with pytest.raises(RtvError) as e:
        ex.set_prefix_kv(make_prefix_kv(cfg, prefix_len=cfg.prefix_len + 1))
    assert e.value.status == 2   # RTV_ERR_SHAPE
    ex.set_prefix_kv(make_prefix_kv(cfg))
    with pytest.raises(RtvError) as e:
        ex.denoise(make_noise(cfg), make_state(cfg), 0)
    assert e.value.status == 2
    ex.close()
