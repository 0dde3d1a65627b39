"""Host-side checks that need no GPU: the seeded generators' per-tensor
streams, and the binding's argument marshalling (dtype codes, bf16 bits,
shapes) for the C ABI."""

import ctypes as C

import numpy as np
import pytest

from flow_matching_action_dm0_b200 import _lib as L
from flow_matching_action_dm0_b200.expert import make_config, make_tensors, to_dtype_bits
from synthetic import (get_config, get_draft_config, get_prefill_config, make_draft_weights, make_prefill_weights,
                       make_weights, round_to_bf16)


def test_a_layer_subset_equals_the_same_entries_of_the_whole_stack():
    pc = get_prefill_config("gemma2b-prefill", n_layers=3, width=128, n_q_heads=2, head_dim=64, mlp_dim=256,
                            n_tokens=8)
    whole = make_prefill_weights(pc)
    part = make_prefill_weights(pc, layers=[1])
    assert set(part) == {k for k in whole if k.startswith("layers.1.")}
    for k, v in part.items():
        np.testing.assert_array_equal(v, whole[k])


def test_bf16_workloads_hold_bf16_values_and_fp32_queries():
    d = make_draft_weights(get_draft_config("flash-draft", width=128, n_q_heads=2, head_dim=64, mlp_dim=256))
    for k, v in d.items():
        if v.ndim == 2 and k != "action_queries":
            np.testing.assert_array_equal(v, round_to_bf16(v))
    q = d["action_queries"]
    assert np.any(q != round_to_bf16(q))   # the queries keep their float32 draw


def test_make_tensors_marshals_dtypes_shapes_and_bf16_bits():
    w = make_weights(get_config("pi0-bf16", n_layers=1, width=128, mlp_dim=256, n_q_heads=2, head_dim=64,
                                action_dim=4, state_dim=3, chunk_len=5, prefix_len=8))
    tensors, keep = make_tensors(w, L.RTV_BF16)
    by_name = {t.name.decode(): t for t in tensors}
    assert set(by_name) == set(w)
    for name, a in w.items():
        t = by_name[name]
        assert t.ndim == a.ndim and tuple(t.shape[:t.ndim]) == a.shape and t.is_device == 0
        assert t.dtype == (L.RTV_BF16 if a.ndim == 2 else L.RTV_F32)
    # a bf16 matrix travels as the high halves of its float32 values
    k = "layers.0.q_proj.w"
    bits = next(x for x, n in zip(keep, w) if n == k)
    assert bits.dtype == np.uint16
    np.testing.assert_array_equal((bits.astype(np.uint32) << 16).view(np.float32), w[k])


def test_bf16_bits_refuse_values_that_are_not_bf16():
    with pytest.raises(ValueError):
        to_dtype_bits(np.array([1.0 + 2.0 ** -10], dtype=np.float32), L.RTV_BF16, "x")
    ok = to_dtype_bits(np.array([1.5], dtype=np.float32), L.RTV_BF16, "x")
    assert ok.dtype == np.uint16 and ok[0] == 0x3FC0
    same = np.array([1.0 + 2.0 ** -10], dtype=np.float32)
    assert to_dtype_bits(same, L.RTV_F32, "x") is same


def test_config_structs_match_the_header_field_order():
    cfg = make_config(get_config("dm05-adarms"))
    assert cfg.time_cond == L.RTV_TIME_ADARMS and cfg.dtype == L.RTV_BF16
    assert C.sizeof(L.rtv_expert_config) % 8 == 0
    names = [f[0] for f in L.rtv_expert_config._fields_]
    assert names[-1] == "time_cond" and names[-2] == "barrier_timeout_ns"
