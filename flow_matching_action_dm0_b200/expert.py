"""Python-side handle of an rtv context (argument marshalling only).

    ex = ActionExpert(shape, device=0)       # rtv_create
    ex.load(weights)                         # rtv_load_expert
    ex.set_prefix_kv(kv)                     # rtv_set_prefix_kv
    chunk = ex.denoise(noise, state, 10)     # rtv_denoise
    acc, flags, dist = ex.verify(draft, eps, state, taus, delta, gripper_dim)   # rtv_verify

``shape`` is any object with the rtv_expert_config field names (n_layers,
width, n_q_heads, ...; dtype "f32"/"bf16").  Arrays may be numpy (host) or
torch tensors (host or CUDA); pointers are handed to the C ABI unchanged.
"""

from __future__ import annotations

import ctypes as C
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

from . import _lib as L

_DTYPES = {"f32": L.RTV_F32, "bf16": L.RTV_BF16, "fp8_e4m3": L.RTV_FP8_E4M3, "same": L.RTV_SAME}
_MASKS = {"bidir": L.RTV_MASK_BIDIR, "pi0_block": L.RTV_MASK_PI0_BLOCK}
_TIME = {"add": L.RTV_TIME_ADD, "concat": L.RTV_TIME_CONCAT, "adarms": L.RTV_TIME_ADARMS}


def make_config(shape, max_batch: Optional[int] = None, max_taus: int = 4,
                max_prefix_len: Optional[int] = None, barrier_timeout_ns: int = 0) -> L.rtv_expert_config:
    g = lambda n, d=None: getattr(shape, n, d)  # noqa: E731
    cfg = L.rtv_expert_config()
    for n in ("n_layers", "width", "n_q_heads", "n_kv_heads", "head_dim", "mlp_dim", "action_dim", "state_dim",
              "chunk_len"):
        setattr(cfg, n, int(g(n)))
    cfg.max_prefix_len = int(max_prefix_len or g("prefix_len"))
    cfg.max_batch = int(max_batch or g("batch", 1))
    cfg.max_taus = int(max_taus)
    cfg.dtype = _DTYPES[g("dtype", "f32")]
    cfg.mlp_dtype = _DTYPES[g("mlp_dtype", "same")]
    cfg.suffix_mask = _MASKS[g("suffix_mask", "bidir")]
    cfg.rms_eps = float(g("rms_eps", 1e-6))
    cfg.rope_theta = float(g("rope_theta", 10000.0))
    cfg.barrier_timeout_ns = int(barrier_timeout_ns)   # 0: the library's default limit
    cfg.time_cond = _TIME[g("time_cond", "add")]
    return cfg


def _ptr(a) -> Tuple[int, bool]:
    """(address, is_device) of a numpy array or torch tensor (must be contiguous)."""
    if isinstance(a, np.ndarray):
        if not a.flags.c_contiguous:
            raise ValueError("array must be C-contiguous")
        return a.ctypes.data, False
    if hasattr(a, "data_ptr"):
        if not a.is_contiguous():
            raise ValueError("tensor must be contiguous")
        return a.data_ptr(), bool(a.is_cuda)
    raise TypeError(f"unsupported array type {type(a)}")


def _stream(stream) -> int:
    if stream is None:
        try:
            import torch
            return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else 0
        except Exception:  # pragma: no cover
            return 0
    return int(getattr(stream, "cuda_stream", stream))


def _dtype_code(name: str, a, matrix_dtype: int, overrides) -> int:
    if overrides and name in overrides:
        return overrides[name]
    if hasattr(a, "dtype") and str(a.dtype) in ("torch.bfloat16",):
        return L.RTV_BF16
    if hasattr(a, "dtype") and str(a.dtype) in ("torch.float8_e4m3fn",):
        return L.RTV_FP8_E4M3
    if isinstance(a, np.ndarray) and a.dtype == np.uint16:
        return L.RTV_BF16
    if isinstance(a, np.ndarray) and a.dtype == np.uint8:
        return L.RTV_FP8_E4M3
    return matrix_dtype if len(a.shape) == 2 else L.RTV_F32


def to_dtype_bits(a, dtype_code: int, what: str):
    """numpy float32 values given in bf16 -> their uint16 bits (checked)."""
    if isinstance(a, np.ndarray) and dtype_code == L.RTV_BF16 and a.dtype == np.float32:
        bits = np.ascontiguousarray(a).view(np.uint32)
        if np.any(bits & np.uint32(0xFFFF)):
            raise ValueError(f"{what}: float32 values are not bf16-representable")
        return (bits >> np.uint32(16)).astype(np.uint16)
    return a


def make_tensors(weights: Dict[str, object], matrix_dtype: int, overrides: Optional[Dict[str, int]] = None):
    """rtv_tensor entries for a name -> array table, and the arrays they point
    into (keep them alive during the load call).  2-D arrays are given in
    matrix_dtype unless their own dtype or ``overrides`` says otherwise;
    float32 numpy values of a bf16 matrix are passed as their bf16 bits."""
    tensors, keep = [], []
    for name, a in weights.items():
        code = _dtype_code(name, a, matrix_dtype, overrides)
        a = to_dtype_bits(a, code, name)
        if isinstance(a, np.ndarray):
            a = np.ascontiguousarray(a)
        ptr, dev = _ptr(a)
        keep.append(a)
        t = L.rtv_tensor()
        t.name = name.encode()
        t.data = ptr
        t.dtype = code
        t.ndim = len(a.shape)
        for i, d in enumerate(a.shape):
            t.shape[i] = int(d)
        t.is_device = int(dev)
        tensors.append(t)
    return tensors, keep


class ActionExpert:
    def __init__(self, shape, device: int = 0, max_batch: Optional[int] = None, max_taus: int = 4,
                 max_prefix_len: Optional[int] = None, barrier_timeout_ns: int = 0):
        self.shape = shape
        self.cfg = make_config(shape, max_batch, max_taus, max_prefix_len, barrier_timeout_ns)
        self.device = device
        self.h = L.rtv_create(self.cfg, device)
        self._keep = []

    # ------------------------------------------------------------------
    def load(self, weights: Dict[str, object], mlp_dtype_codes: Optional[Dict[str, int]] = None):
        """weights: name -> array.  float32 numpy arrays are accepted for bf16
        matrices when their values are bf16-representable (passed as bits)."""
        tensors, keep = make_tensors(weights, self.cfg.dtype, mlp_dtype_codes)
        L.rtv_load_expert(self.h, tensors)
        del keep

    # ------------------------------------------------------------------
    def set_prefix_kv(self, kv, prefix_len: Optional[int] = None, batch: Optional[int] = None, stream=None):
        """kv [L][2][B][P][Hkv][D] in the config dtype (torch tensor, or numpy
        float32 / uint16 bf16 bits)."""
        kv = to_dtype_bits(kv, self.cfg.dtype, "prefix kv")
        b = int(batch if batch is not None else kv.shape[2])
        p = int(prefix_len if prefix_len is not None else kv.shape[3])
        ptr, _ = _ptr(kv)
        self._keep = [kv]
        L.rtv_set_prefix_kv(self.h, ptr, p, b, _stream(stream))

    def denoise(self, noise, state, n_steps: int, out=None, stream=None):
        """Action chunk [B][H][A] fp32.  noise/state/out: numpy or torch fp32."""
        if out is None:
            if isinstance(noise, np.ndarray):
                out = np.empty_like(noise, dtype=np.float32)
            else:
                out = noise.new_empty(noise.shape)
        pn, _ = _ptr(noise)
        ps, _ = _ptr(state)
        po, _ = _ptr(out)
        L.rtv_denoise(self.h, pn, ps, int(n_steps), po, _stream(stream))
        if isinstance(out, np.ndarray):
            self.synchronize(stream)
        return out

    def verify(self, draft, noise, state, taus: Sequence[float], delta: float, gripper_dim: int,
               want_dist: bool = True, stream=None):
        """(accepted length, flags, d[T][H] or None); runs on host buffers and
        waits for the result."""
        taus_h = np.ascontiguousarray(np.asarray(taus, dtype=np.float32))
        acc = np.zeros(1, dtype=np.int32)
        flags = np.zeros(1, dtype=np.uint32)
        h_len = self.cfg.chunk_len
        dist = np.zeros((len(taus_h), h_len), dtype=np.float32) if want_dist else None
        pd, _ = _ptr(draft)
        pe, _ = _ptr(noise)
        ps, _ = _ptr(state)
        L.rtv_verify(self.h, pd, pe, ps, taus_h.ctypes.data, len(taus_h), float(delta), int(gripper_dim),
                     acc.ctypes.data, flags.ctypes.data, dist.ctypes.data if dist is not None else 0,
                     _stream(stream))
        self.synchronize(stream)
        return int(acc[0]), int(flags[0]), dist

    # ------------------------------------------------------------------
    def synchronize(self, stream=None):
        try:
            import torch
            if torch.cuda.is_available():
                torch.cuda.synchronize(self.device)
        except Exception:  # pragma: no cover
            pass

    def status(self) -> Tuple[int, int]:
        return L.rtv_device_status(self.h)

    def kernels_per_call(self, n: int, verify: bool = False) -> int:
        return L.rtv_graph_kernel_count(self.h, n, verify)

    @property
    def path(self) -> str:
        return L.rtv_path_name(self.h)

    def close(self):
        if self.h:
            L.rtv_destroy(self.h)
            self.h = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass
