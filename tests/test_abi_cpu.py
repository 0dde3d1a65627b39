"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and refuses bad calls without touching a device."""

import ctypes as C
import os
import re

import pytest

from flow_matching_action_dm0_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "rtv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rtv_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = L.load_library()
    names = declared_functions()
    assert names, "no declarations parsed"
    assert set(names) == set(L.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_null_arguments_are_refused():
    lib = L.load_library()
    assert lib.rtv_create(None, 0, None) == L.RTV_ERR_ARG
    h = C.c_void_p()
    assert lib.rtv_create(None, 0, C.byref(h)) == L.RTV_ERR_ARG
    assert not h.value
    assert lib.rtv_load_expert(None, None, 0) == L.RTV_ERR_ARG
    assert lib.rtv_denoise(None, None, None, 10, None, None) == L.RTV_ERR_ARG
    assert lib.rtv_verify(None, None, None, None, None, 0, C.c_float(0.05), 0, None, None, None, None) == \
        L.RTV_ERR_ARG
    lib.rtv_destroy(None)
    assert lib.rtv_last_error(None) == b"null context"


def test_invalid_config_is_refused_before_device_use():
    lib = L.load_library()
    cfg = L.rtv_expert_config()
    cfg.n_layers = 0   # invalid
    h = C.c_void_p()
    assert lib.rtv_create(C.byref(cfg), 0, C.byref(h)) == L.RTV_ERR_ARG
    assert not h.value


@pytest.mark.parametrize("value", [3, -1])
def test_invalid_time_condition_is_refused_before_device_use(value):
    from synthetic import get_config
    from flow_matching_action_dm0_b200 import make_config
    cfg = make_config(get_config("tiny-fp32"))
    cfg.time_cond = value
    h = C.c_void_p()
    assert L.load_library().rtv_create(C.byref(cfg), 0, C.byref(h)) == L.RTV_ERR_ARG
    assert not h.value


def test_create_without_gpu_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    from synthetic import get_config
    from flow_matching_action_dm0_b200 import make_config
    cfg = make_config(get_config("tiny-fp32"))
    h = C.c_void_p()
    assert L.load_library().rtv_create(C.byref(cfg), 0, C.byref(h)) == L.RTV_ERR_CUDA
    assert not h.value


def test_draft_null_arguments_are_refused():
    lib = L.load_library()
    assert lib.rtv_draft_create(None, 0, None) == L.RTV_ERR_ARG
    d = C.c_void_p()
    assert lib.rtv_draft_create(None, 0, C.byref(d)) == L.RTV_ERR_ARG
    assert not d.value
    assert lib.rtv_draft_load(None, None, 0) == L.RTV_ERR_ARG
    assert lib.rtv_draft_forward(None, None, 1, 1, None, None) == L.RTV_ERR_ARG
    assert lib.rtv_flash_round(None, None, None, 1, None, None, None, 1, C.c_float(0.05), 0, 10, None, None, None,
                               None, None) == L.RTV_ERR_ARG
    assert lib.rtv_draft_kernel_count(None, 1, 1) == -1
    lib.rtv_draft_destroy(None)
    assert lib.rtv_draft_last_error(None) == b"null draft model"


@pytest.mark.parametrize("field,value", [("width", 200), ("n_queries", 0), ("n_queries", 65), ("n_kv_heads", 3),
                                         ("max_vis", 0), ("dtype", 2)])
def test_invalid_draft_config_is_refused_before_device_use(field, value):
    from synthetic import get_draft_config
    from flow_matching_action_dm0_b200 import make_draft_config
    cfg = make_draft_config(get_draft_config("draft-tiny"))
    setattr(cfg, field, value)
    d = C.c_void_p()
    assert L.load_library().rtv_draft_create(C.byref(cfg), 0, C.byref(d)) == L.RTV_ERR_ARG
    assert not d.value
