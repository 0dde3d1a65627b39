"""ctypes binding of ``librtv.so`` (argument marshalling only).

The function names match the C ABI in ``include/rtv.h``.  Every step of the
computation runs in the library's CUDA kernels; this module only converts
Python objects (numpy arrays, torch tensors, ints) into pointers and sizes.
If the shared library is missing the import fails loudly: there is no
fallback implementation.
"""

from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librtv.so")

RTV_OK, RTV_ERR_ARG, RTV_ERR_SHAPE, RTV_ERR_STATE, RTV_ERR_CUDA, RTV_ERR_OOM, RTV_ERR_TIMEOUT, \
    RTV_ERR_NUMERIC, RTV_ERR_UNSUPPORTED = range(9)
STATUS_NAMES = ["RTV_OK", "RTV_ERR_ARG", "RTV_ERR_SHAPE", "RTV_ERR_STATE", "RTV_ERR_CUDA", "RTV_ERR_OOM",
                "RTV_ERR_TIMEOUT", "RTV_ERR_NUMERIC", "RTV_ERR_UNSUPPORTED"]
RTV_F32, RTV_BF16, RTV_FP8_E4M3, RTV_SAME = 0, 1, 2, 3
RTV_MASK_BIDIR, RTV_MASK_PI0_BLOCK = 0, 1
RTV_TIME_ADD, RTV_TIME_CONCAT, RTV_TIME_ADARMS = 0, 1, 2
RTV_DEV_TIMEOUT, RTV_DEV_NUMERIC, RTV_DEV_BOUNDS = 1, 2, 4
RTV_FLAG_ZERO_ACCEPT, RTV_FLAG_SWITCH, RTV_FLAG_SWITCH_IN_PREFIX = 1, 2, 4

# Every symbol include/rtv.h declares (checked by the CPU test suite).
EXPORTS = ("rtv_create", "rtv_load_expert", "rtv_set_prefix_kv", "rtv_denoise", "rtv_verify",
           "rtv_device_status", "rtv_last_error", "rtv_path_name", "rtv_graph_kernel_count", "rtv_destroy",
           "rtv_set_prefix_kv_static", "rtv_draft_create", "rtv_draft_load", "rtv_draft_forward", "rtv_flash_round",
           "rtv_draft_device_status", "rtv_draft_last_error", "rtv_draft_path_name", "rtv_draft_kernel_count",
           "rtv_draft_destroy", "rtv_prefill_create", "rtv_prefill_load", "rtv_prefill_kv", "rtv_prefill_denoise",
           "rtv_prefill_device_status", "rtv_prefill_last_error", "rtv_prefill_kernel_count", "rtv_prefill_destroy")


class rtv_expert_config(C.Structure):
    _fields_ = [
        ("n_layers", C.c_int), ("width", C.c_int), ("n_q_heads", C.c_int), ("n_kv_heads", C.c_int),
        ("head_dim", C.c_int), ("mlp_dim", C.c_int), ("action_dim", C.c_int), ("state_dim", C.c_int),
        ("chunk_len", C.c_int), ("max_prefix_len", C.c_int), ("max_batch", C.c_int), ("max_taus", C.c_int),
        ("dtype", C.c_int), ("mlp_dtype", C.c_int), ("suffix_mask", C.c_int),
        ("rms_eps", C.c_float), ("rope_theta", C.c_float), ("barrier_timeout_ns", C.c_longlong),
        ("time_cond", C.c_int),
    ]


class rtv_draft_config(C.Structure):
    _fields_ = [
        ("width", C.c_int), ("n_q_heads", C.c_int), ("n_kv_heads", C.c_int), ("head_dim", C.c_int),
        ("mlp_dim", C.c_int), ("n_queries", C.c_int), ("action_dim", C.c_int), ("max_vis", C.c_int),
        ("max_batch", C.c_int), ("dtype", C.c_int), ("rms_eps", C.c_float), ("rope_theta", C.c_float),
        ("barrier_timeout_ns", C.c_longlong),
    ]


class rtv_prefill_config(C.Structure):
    _fields_ = [
        ("n_layers", C.c_int), ("width", C.c_int), ("n_q_heads", C.c_int), ("n_kv_heads", C.c_int),
        ("head_dim", C.c_int), ("mlp_dim", C.c_int), ("max_tokens", C.c_int), ("dtype", C.c_int),
        ("rms_eps", C.c_float), ("rope_theta", C.c_float), ("barrier_timeout_ns", C.c_longlong),
    ]


class rtv_tensor(C.Structure):
    _fields_ = [
        ("name", C.c_char_p), ("data", C.c_void_p), ("dtype", C.c_int), ("ndim", C.c_int),
        ("shape", C.c_longlong * 4), ("is_device", C.c_int),
    ]


class RtvError(RuntimeError):
    def __init__(self, status: int, msg: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else status}: {msg}")


_lib = None


def load_library(path: str = LIB_PATH):
    """Load librtv.so (once).  Raises ImportError when it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m flow_matching_action_dm0_b200.build`")
    lib = C.CDLL(path)
    P, I, F, U = C.c_void_p, C.c_int, C.c_float, C.POINTER(C.c_uint)
    lib.rtv_create.argtypes = [C.POINTER(rtv_expert_config), I, C.POINTER(P)]
    lib.rtv_load_expert.argtypes = [P, C.POINTER(rtv_tensor), I]
    lib.rtv_set_prefix_kv.argtypes = [P, P, I, I, P]
    lib.rtv_set_prefix_kv_static.argtypes = [P, P, I, I, P]
    lib.rtv_denoise.argtypes = [P, P, P, I, P, P]
    lib.rtv_verify.argtypes = [P, P, P, P, P, I, F, I, P, P, P, P]
    lib.rtv_device_status.argtypes = [P, U]
    lib.rtv_last_error.argtypes = [P]
    lib.rtv_last_error.restype = C.c_char_p
    lib.rtv_path_name.argtypes = [P]
    lib.rtv_path_name.restype = C.c_char_p
    lib.rtv_graph_kernel_count.argtypes = [P, I, I]
    lib.rtv_graph_kernel_count.restype = I
    lib.rtv_destroy.argtypes = [P]
    lib.rtv_destroy.restype = None
    lib.rtv_draft_create.argtypes = [C.POINTER(rtv_draft_config), I, C.POINTER(P)]
    lib.rtv_draft_load.argtypes = [P, C.POINTER(rtv_tensor), I]
    lib.rtv_draft_forward.argtypes = [P, P, I, I, P, P]
    lib.rtv_flash_round.argtypes = [P, P, P, I, P, P, P, I, F, I, I, P, P, P, P, P]
    lib.rtv_draft_device_status.argtypes = [P, U]
    lib.rtv_draft_last_error.argtypes = [P]
    lib.rtv_draft_last_error.restype = C.c_char_p
    lib.rtv_draft_path_name.argtypes = [P]
    lib.rtv_draft_path_name.restype = C.c_char_p
    lib.rtv_draft_kernel_count.argtypes = [P, I, I]
    lib.rtv_draft_kernel_count.restype = I
    lib.rtv_draft_destroy.argtypes = [P]
    lib.rtv_draft_destroy.restype = None
    lib.rtv_prefill_create.argtypes = [C.POINTER(rtv_prefill_config), I, C.POINTER(P)]
    lib.rtv_prefill_load.argtypes = [P, C.POINTER(rtv_tensor), I]
    lib.rtv_prefill_kv.argtypes = [P, P, P, I, P]
    lib.rtv_prefill_denoise.argtypes = [P, P, P, I, P, P, I, P, P]
    lib.rtv_prefill_device_status.argtypes = [P, U]
    lib.rtv_prefill_last_error.argtypes = [P]
    lib.rtv_prefill_last_error.restype = C.c_char_p
    lib.rtv_prefill_kernel_count.argtypes = [P, I, I]
    lib.rtv_prefill_kernel_count.restype = I
    lib.rtv_prefill_destroy.argtypes = [P]
    lib.rtv_prefill_destroy.restype = None
    for n in ("rtv_create", "rtv_load_expert", "rtv_set_prefix_kv", "rtv_set_prefix_kv_static", "rtv_denoise",
              "rtv_verify", "rtv_device_status", "rtv_draft_create", "rtv_draft_load", "rtv_draft_forward",
              "rtv_flash_round", "rtv_draft_device_status", "rtv_prefill_create", "rtv_prefill_load",
              "rtv_prefill_kv", "rtv_prefill_denoise", "rtv_prefill_device_status"):
        getattr(lib, n).restype = I
    _lib = lib
    return lib


# thin same-name wrappers ---------------------------------------------------

def rtv_create(cfg: rtv_expert_config, device: int = 0):
    lib = load_library()
    h = C.c_void_p()
    s = lib.rtv_create(C.byref(cfg), int(device), C.byref(h))
    if s != RTV_OK:
        raise RtvError(s, "rtv_create failed")
    return h


def _check(h, s):
    if s != RTV_OK:
        raise RtvError(s, load_library().rtv_last_error(h).decode())
    return s


def rtv_load_expert(h, tensors):
    arr = (rtv_tensor * len(tensors))(*tensors)
    return _check(h, load_library().rtv_load_expert(h, arr, len(tensors)))


def rtv_set_prefix_kv(h, kv_ptr: int, prefix_len: int, batch: int, stream: int = 0):
    return _check(h, load_library().rtv_set_prefix_kv(h, C.c_void_p(kv_ptr), prefix_len, batch, C.c_void_p(stream)))


def rtv_set_prefix_kv_static(h, kv_ptr: int, prefix_len: int, batch: int, stream: int = 0):
    """Like rtv_set_prefix_kv, staging host data through the library's static device array (no allocation)."""
    return _check(h, load_library().rtv_set_prefix_kv_static(h, C.c_void_p(kv_ptr), prefix_len, batch,
                                                             C.c_void_p(stream)))


def rtv_denoise(h, noise_ptr: int, state_ptr: int, n_steps: int, out_ptr: int, stream: int = 0):
    return _check(h, load_library().rtv_denoise(h, C.c_void_p(noise_ptr), C.c_void_p(state_ptr), n_steps,
                                                C.c_void_p(out_ptr), C.c_void_p(stream)))


def rtv_verify(h, draft_ptr, noise_ptr, state_ptr, taus_ptr, n_taus, delta, gripper_dim, acc_ptr, flags_ptr,
               dist_ptr, stream: int = 0):
    return _check(h, load_library().rtv_verify(
        h, C.c_void_p(draft_ptr), C.c_void_p(noise_ptr), C.c_void_p(state_ptr), C.c_void_p(taus_ptr), n_taus,
        C.c_float(delta), gripper_dim, C.c_void_p(acc_ptr), C.c_void_p(flags_ptr),
        C.c_void_p(dist_ptr or 0), C.c_void_p(stream)))


def rtv_device_status(h):
    bits = C.c_uint(0)
    s = load_library().rtv_device_status(h, C.byref(bits))
    return s, bits.value


def rtv_last_error(h) -> str:
    return load_library().rtv_last_error(h).decode()


def rtv_path_name(h) -> str:
    return load_library().rtv_path_name(h).decode()


def rtv_graph_kernel_count(h, n: int, is_verify: bool = False) -> int:
    return int(load_library().rtv_graph_kernel_count(h, int(n), int(bool(is_verify))))


def rtv_destroy(h):
    if h:
        load_library().rtv_destroy(h)


# draft model and FLASH round ------------------------------------------------

def rtv_draft_create(cfg: rtv_draft_config, device: int = 0):
    lib = load_library()
    h = C.c_void_p()
    s = lib.rtv_draft_create(C.byref(cfg), int(device), C.byref(h))
    if s != RTV_OK:
        raise RtvError(s, "rtv_draft_create failed")
    return h


def _dcheck(d, s):
    if s != RTV_OK:
        raise RtvError(s, load_library().rtv_draft_last_error(d).decode())
    return s


def rtv_draft_load(d, tensors):
    arr = (rtv_tensor * len(tensors))(*tensors)
    return _dcheck(d, load_library().rtv_draft_load(d, arr, len(tensors)))


def rtv_draft_forward(d, vis_ptr: int, n_vis: int, batch: int, out_ptr: int, stream: int = 0):
    return _dcheck(d, load_library().rtv_draft_forward(d, C.c_void_p(vis_ptr), int(n_vis), int(batch),
                                                       C.c_void_p(out_ptr), C.c_void_p(stream)))


def rtv_flash_round(h, d, vis_ptr, n_vis, noise_ptr, state_ptr, taus_ptr, n_taus, delta, gripper_dim, n_steps,
                    out_ptr, acc_ptr, flags_ptr, used_full_ptr, stream: int = 0):
    return _dcheck(d, load_library().rtv_flash_round(
        h, d, C.c_void_p(vis_ptr), int(n_vis), C.c_void_p(noise_ptr), C.c_void_p(state_ptr), C.c_void_p(taus_ptr),
        int(n_taus), C.c_float(delta), int(gripper_dim), int(n_steps), C.c_void_p(out_ptr), C.c_void_p(acc_ptr),
        C.c_void_p(flags_ptr), C.c_void_p(used_full_ptr), C.c_void_p(stream)))


def rtv_draft_device_status(d):
    bits = C.c_uint(0)
    s = load_library().rtv_draft_device_status(d, C.byref(bits))
    return s, bits.value


def rtv_draft_last_error(d) -> str:
    return load_library().rtv_draft_last_error(d).decode()


def rtv_draft_path_name(d) -> str:
    return load_library().rtv_draft_path_name(d).decode()


def rtv_draft_kernel_count(d, n_vis: int, batch: int) -> int:
    return int(load_library().rtv_draft_kernel_count(d, int(n_vis), int(batch)))


def rtv_draft_destroy(d):
    if d:
        load_library().rtv_draft_destroy(d)


# VLM prefill -------------------------------------------------------------------

def rtv_prefill_create(cfg: rtv_prefill_config, device: int = 0):
    lib = load_library()
    h = C.c_void_p()
    s = lib.rtv_prefill_create(C.byref(cfg), int(device), C.byref(h))
    if s != RTV_OK:
        raise RtvError(s, "rtv_prefill_create failed")
    return h


def _pcheck(p, s):
    if s != RTV_OK:
        raise RtvError(s, load_library().rtv_prefill_last_error(p).decode())
    return s


def rtv_prefill_load(p, tensors):
    arr = (rtv_tensor * len(tensors))(*tensors)
    return _pcheck(p, load_library().rtv_prefill_load(p, arr, len(tensors)))


def rtv_prefill_kv(p, h, emb_ptr: int, n_tokens: int, stream: int = 0):
    return _pcheck(p, load_library().rtv_prefill_kv(p, h, C.c_void_p(emb_ptr), int(n_tokens), C.c_void_p(stream)))


def rtv_prefill_denoise(p, h, emb_ptr: int, n_tokens: int, noise_ptr: int, state_ptr: int, n_steps: int,
                        out_ptr: int, stream: int = 0):
    return _pcheck(p, load_library().rtv_prefill_denoise(
        p, h, C.c_void_p(emb_ptr), int(n_tokens), C.c_void_p(noise_ptr), C.c_void_p(state_ptr), int(n_steps),
        C.c_void_p(out_ptr), C.c_void_p(stream)))


def rtv_prefill_device_status(p):
    bits = C.c_uint(0)
    s = load_library().rtv_prefill_device_status(p, C.byref(bits))
    return s, bits.value


def rtv_prefill_last_error(p) -> str:
    return load_library().rtv_prefill_last_error(p).decode()


def rtv_prefill_kernel_count(p, n_tokens: int, n_steps: int = 0) -> int:
    return int(load_library().rtv_prefill_kernel_count(p, int(n_tokens), int(n_steps)))


def rtv_prefill_destroy(p):
    if p:
        load_library().rtv_prefill_destroy(p)
