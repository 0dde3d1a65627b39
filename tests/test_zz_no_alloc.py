"""The allocation-free way of installing the prefix KV cache.

rtv_set_prefix_kv_static serves callers that cannot call cudaMalloc while
they run (a real-time control loop that must not block on the allocator, or
a process whose device memory belongs to another allocator or a fixed
budget): it stages host data through a fixed array in device memory that the
library declares statically, and reads device data of its own GPU in place.

Each check installs a first cache A with the allocating rtv_set_prefix_kv,
then a second cache B with rtv_set_prefix_kv_static, and requires the chunk
to be bit-for-bit the chunk of a fresh context that installed B with
rtv_set_prefix_kv.  A static call that wrote nothing, or skipped a layer,
would leave (part of) A in place and fail.  Both contexts run the layered
kernel path, whose reductions have a fixed order, so equal caches give equal
bits.  The file is collected last so that a failure here never hides the
result of another test.
"""

import os

import numpy as np
import pytest

from flow_matching_action_dm0_b200 import _lib as L
from flow_matching_action_dm0_b200 import ActionExpert, RtvError
from synthetic import f32_to_bf16_bits, get_config, make_noise, make_prefix_kv, make_state, make_weights

pytestmark = pytest.mark.gpu


@pytest.fixture
def layered_path(monkeypatch):
    # contexts created while this is set take the layered kernels (fixed reduction order)
    monkeypatch.setenv("RTV_PATH", "layered")
    yield


def _cache(cfg, seed):
    kv = make_prefix_kv(cfg, seed=seed)
    return np.ascontiguousarray(f32_to_bf16_bits(kv) if cfg.dtype == "bf16" else kv.astype(np.float32))


def _static_install(ex, kv, where):
    import torch
    if where == "host":
        L.rtv_set_prefix_kv_static(ex.h, kv.ctypes.data, kv.shape[3], kv.shape[2], 0)
        torch.cuda.synchronize()
        return None
    dev = torch.from_numpy(kv.view(np.int16) if kv.dtype == np.uint16 else kv).to("cuda:0")
    torch.cuda.synchronize()
    L.rtv_set_prefix_kv_static(ex.h, dev.data_ptr(), kv.shape[3], kv.shape[2], 0)
    torch.cuda.synchronize()
    return dev


@pytest.mark.parametrize("shape", ["pi0-bf16", "tiny-fp32"])
@pytest.mark.parametrize("where", ["host", "device"])
def test_static_install_replaces_a_previous_cache_exactly(cuda_ok, layered_path, shape, where):
    cfg = get_config(shape, n_layers=2, prefix_len=100) if shape == "pi0-bf16" else get_config(shape)
    weights = make_weights(cfg)
    noise, state = make_noise(cfg), make_state(cfg)
    kv_a, kv_b = _cache(cfg, 11), _cache(cfg, 12)

    ref_ex = ActionExpert(cfg)
    ref_ex.load(weights)
    ref_ex.set_prefix_kv(kv_b)                  # allocating install of B
    ref = ref_ex.denoise(noise, state, 3)
    ref_ex.close()

    ex = ActionExpert(cfg)
    ex.load(weights)
    ex.set_prefix_kv(kv_a)                      # allocating install of A
    got_a = ex.denoise(noise, state, 3)
    assert not np.array_equal(got_a, ref)       # the two caches lead to different chunks
    keep = _static_install(ex, kv_b, where)     # static install of B over A
    got = ex.denoise(noise, state, 3)
    np.testing.assert_array_equal(got, ref)
    s, bits = ex.status()
    assert s == 0 and bits == 0
    del keep
    ex.close()


def test_static_install_twice_in_a_row_allocates_nothing(cuda_ok, layered_path):
    import torch
    cfg = get_config("pi0-bf16", n_layers=2, prefix_len=100)
    weights = make_weights(cfg)
    noise, state = make_noise(cfg), make_state(cfg)
    ex = ActionExpert(cfg)
    ex.load(weights)
    refs = {}
    for seed in (21, 22):
        kv = _cache(cfg, seed)
        r = ActionExpert(cfg)
        r.load(weights)
        r.set_prefix_kv(kv)
        refs[seed] = (kv, r.denoise(noise, state, 3))
        r.close()
    # the first static call on the device looks up (and may load) the staging array
    _static_install(ex, refs[21][0], "host")
    np.testing.assert_array_equal(ex.denoise(noise, state, 3), refs[21][1])
    free0, _ = torch.cuda.mem_get_info(0)
    _static_install(ex, refs[22][0], "host")
    free1, _ = torch.cuda.mem_get_info(0)
    assert free1 == free0
    np.testing.assert_array_equal(ex.denoise(noise, state, 3), refs[22][1])
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
