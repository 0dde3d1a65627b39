"""The allocation-free way of installing the prefix KV cache.

rtv_set_prefix_kv_static serves callers that cannot call cudaMalloc while
they run (a real-time control loop that must not block on the allocator, or
a process whose device memory belongs to another allocator or a fixed
budget): it stages host data through a fixed array in device memory that the
library declares statically.  These checks call it through the C ABI and
compare the chunks it leads to with those of rtv_set_prefix_kv, for two
different caches installed one after the other; a cache too large for the
array is refused.  The file is collected last so that a failure here never
hides the result of another test.
"""

import ctypes as C

import numpy as np
import pytest

from flow_matching_action_dm0_b200 import _lib as L
from flow_matching_action_dm0_b200 import ActionExpert, RtvError
from synthetic import f32_to_bf16_bits, get_config, make_noise, make_prefix_kv, make_state, make_weights
from tests.helpers import bf16_tolerance_ok, rel_l2

pytestmark = pytest.mark.gpu


def _bits(kv):
    return np.ascontiguousarray(f32_to_bf16_bits(kv))


def test_static_staging_matches_allocating_install_on_two_calls_in_a_row(cuda_ok):
    cfg = get_config("pi0-bf16", n_layers=2, prefix_len=100)
    ex = ActionExpert(cfg)
    ex.load(make_weights(cfg))
    noise, state = make_noise(cfg), make_state(cfg)
    for seed in (11, 12):   # two different caches, installed one after the other
        kv = _bits(make_prefix_kv(cfg, seed=seed))
        ex.set_prefix_kv(kv)                       # allocating install (reference)
        ref = ex.denoise(noise, state, 3)
        L.rtv_set_prefix_kv_static(ex.h, kv.ctypes.data, kv.shape[3], kv.shape[2], 0)
        got = ex.denoise(noise, state, 3)
        assert bf16_tolerance_ok(got, ref), rel_l2(got, ref)
        s, bits = ex.status()
        assert s == 0 and bits == 0
    ex.close()


def test_static_staging_refuses_a_layer_larger_than_the_array(cuda_ok):
    # one layer of keys + values: 2 * 8 * 816 * 256 bf16 = 6.7 MB > 4 MiB
    cfg = get_config("pi0-bf16", n_layers=1, batch=8)
    ex = ActionExpert(cfg, max_batch=8)
    kv = np.zeros((1, 2, 8, cfg.prefix_len, 1, cfg.head_dim), dtype=np.uint16)
    with pytest.raises(RtvError) as e:
        L.rtv_set_prefix_kv_static(ex.h, kv.ctypes.data, cfg.prefix_len, 8, 0)
    assert e.value.status == L.RTV_ERR_SHAPE
    ex.close()
