"""GPU parity of the VLM prefill ("DM0.5 reading guide" sec. 5.1: the
prefix is encoded once into a per-layer KV cache) and of prefill + denoising
captured as one graph (sec. 6.5), against the oracle, through the C ABI.

bf16 tolerances as for the expert: relative L2 <= 1e-2, max-abs <= 3e-2 on
the action chunk that the prefilled cache produces.
"""

import numpy as np
import pytest

from oracle import expert as O
from oracle import prefill as OP
from synthetic import (f32_to_bf16_bits, get_config, get_prefill_config, make_noise, make_prefill_weights,
                       make_prefix_embeddings, make_state, make_weights)
from tests.helpers import rel_l2

pytestmark = pytest.mark.gpu


def stack_weights_bits(pc):
    """All stack parameters, matrices as bf16 bits, generated one layer at a
    time (the Gemma-2B-class stack is 4 GB in bf16)."""
    out = {}
    for l in range(pc.n_layers):
        for k, v in make_prefill_weights(pc, layers=[l]).items():
            out[k] = f32_to_bf16_bits(v) if v.ndim == 2 else v
    return out


def provider(pc):
    return lambda l: make_prefill_weights(pc, layers=[l])


def _run(cfg, pc, n_steps, n_tokens=None):
    from flow_matching_action_dm0_b200 import ActionExpert, PrefillStack
    n_tokens = pc.n_tokens if n_tokens is None else n_tokens
    We = make_weights(cfg)
    ex = ActionExpert(cfg, max_batch=1, max_taus=4, max_prefix_len=max(n_tokens, cfg.prefix_len))
    ex.load(We)
    pf = PrefillStack(pc, max_tokens=n_tokens)
    pf.load(stack_weights_bits(pc))
    emb = make_prefix_embeddings(pc, n_tokens=n_tokens)
    noise, state = make_noise(cfg), make_state(cfg)
    got = pf.denoise(ex, emb, noise[0], state[0], n_steps)
    s, bits = pf.status()
    assert s == 0 and bits == 0
    s, bits = ex.status()
    assert s == 0 and bits == 0
    assert pf.kernels_per_call(n_tokens, n_steps) > 0
    return ex, pf, We, emb, noise, state, got


def _expert_and_stack(n_layers, width, n_q_heads, mlp_dim, n_tokens):
    cfg = get_config("pi0-bf16", n_layers=n_layers, prefix_len=n_tokens)
    pc = get_prefill_config("gemma2b-prefill", n_layers=n_layers, width=width, n_q_heads=n_q_heads,
                            mlp_dim=mlp_dim, n_tokens=n_tokens)
    return cfg, pc


@pytest.mark.parametrize("n_tokens", [150, 64, 37, 1])
def test_prefill_denoise_matches_oracle_small(cuda_ok, n_tokens):
    """Two layers, width 512: ragged query groups (150 = 2 x 64 + 22), one
    exact group, one partial group, a single token."""
    cfg, pc = _expert_and_stack(2, 512, 2, 2048, n_tokens)
    ex, pf, We, emb, noise, state, got = _run(cfg, pc, 3)
    ref = OP.prefill_denoise(provider(pc), pc, We, cfg, emb, noise, state, 3)[0]
    assert rel_l2(got, ref) <= 1e-2 and np.max(np.abs(got - ref)) <= 3e-2, (rel_l2(got, ref),
                                                                          np.max(np.abs(got - ref)))
    # the installed prefix serves the expert's own calls: prefill alone then
    # rtv_denoise gives the same chunk as the one-graph call
    pf.kv(ex, emb)
    again = ex.denoise(noise, state, 3)[0]
    assert rel_l2(again, got) <= 1e-5, rel_l2(again, got)
    pf.close()
    ex.close()


def test_prefill_full_width_two_layers_matches_oracle(cuda_ok):
    """The Gemma-2B-class layer (width 2048, GeGLU 16384) over all 816
    tokens, two layers."""
    cfg, pc = _expert_and_stack(2, 2048, 8, 16384, 816)
    ex, pf, We, emb, noise, state, got = _run(cfg, pc, 2)
    ref = OP.prefill_denoise(provider(pc), pc, We, cfg, emb, noise, state, 2)[0]
    err_rel, err_abs = rel_l2(got, ref), float(np.max(np.abs(got - ref)))
    print(f"prefill 2-layer full width rel_l2={err_rel:.3e} max_abs={err_abs:.3e}")
    assert err_rel <= 1e-2 and err_abs <= 3e-2
    pf.close()
    ex.close()


def test_prefill_plus_chunk_full_size_matches_oracle(cuda_ok):
    """The whole configuration: 18-layer Gemma-2B-class prefill over 816
    tokens, then the pi0-bf16 10-step chunk, as one graph."""
    cfg = get_config("pi0-bf16")
    pc = get_prefill_config("gemma2b-prefill")
    ex, pf, We, emb, noise, state, got = _run(cfg, pc, 10)
    assert np.all(np.isfinite(got))
    ref = OP.prefill_denoise(provider(pc), pc, We, cfg, emb, noise, state, 10)[0]
    err_rel, err_abs = rel_l2(got, ref), float(np.max(np.abs(got - ref)))
    print(f"prefill+chunk full size rel_l2={err_rel:.3e} max_abs={err_abs:.3e}")
    assert err_rel <= 1e-2 and err_abs <= 3e-2
    pf.close()
    ex.close()


def test_prefill_refuses_mismatched_expert_and_sizes(cuda_ok):
    from flow_matching_action_dm0_b200 import ActionExpert, PrefillStack, RtvError
    cfg, pc = _expert_and_stack(2, 512, 2, 2048, 100)
    ex = ActionExpert(cfg.with_(n_layers=3), max_batch=1, max_prefix_len=100)
    ex.load(make_weights(cfg.with_(n_layers=3)))
    pf = PrefillStack(pc, max_tokens=100)
    emb = make_prefix_embeddings(pc, n_tokens=100)
    with pytest.raises(RtvError):
        pf.kv(ex, emb)                      # not loaded
    pf.load(stack_weights_bits(pc))
    with pytest.raises(RtvError):
        pf.kv(ex, emb)                      # 3-layer expert, 2-layer stack
    ex.close()
    ex = ActionExpert(cfg, max_batch=1, max_prefix_len=100)
    ex.load(make_weights(cfg))
    with pytest.raises(RtvError):
        pf.kv(ex, make_prefix_embeddings(pc, n_tokens=101))   # beyond max_tokens
    pf.close()
    ex.close()
    with pytest.raises(RtvError):
        PrefillStack(pc.with_(dtype="f32"))
