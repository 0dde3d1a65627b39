"""Python-side handle of a FLASH draft model and the dual-path round
(argument marshalling only; the computation runs in ``librtv.so``).

    dm = DraftModel(shape, device=0)          # rtv_draft_create
    dm.load(weights)                          # rtv_draft_load
    chunk = dm.forward(vis)                   # rtv_draft_forward, [B][H][A]
    r = flash_round(expert, dm, vis[0], eps, state, taus, delta, gripper_dim, n_steps)   # rtv_flash_round

``shape`` is any object with the rtv_draft_config field names (width,
n_q_heads, n_kv_heads, head_dim, mlp_dim, n_queries, action_dim; n_vis and
batch give the maxima unless passed; dtype "f32"/"bf16").
"""

from __future__ import annotations

from typing import Dict, NamedTuple, Optional, Sequence

import numpy as np

from . import _lib as L
from .expert import _DTYPES, ActionExpert, _ptr, _stream, make_tensors, to_dtype_bits


def make_draft_config(shape, max_vis: Optional[int] = None, max_batch: Optional[int] = None) -> L.rtv_draft_config:
    g = lambda n, d=None: getattr(shape, n, d)  # noqa: E731
    cfg = L.rtv_draft_config()
    for n in ("width", "n_q_heads", "n_kv_heads", "head_dim", "mlp_dim", "n_queries", "action_dim"):
        setattr(cfg, n, int(g(n)))
    cfg.max_vis = int(max_vis or g("n_vis"))
    cfg.max_batch = int(max_batch or g("batch", 1))
    cfg.dtype = _DTYPES[g("dtype", "f32")]
    cfg.rms_eps = float(g("rms_eps", 1e-6))
    cfg.rope_theta = float(g("rope_theta", 10000.0))
    cfg.barrier_timeout_ns = 0
    return cfg


class DraftModel:
    def __init__(self, shape, device: int = 0, max_vis: Optional[int] = None, max_batch: Optional[int] = None):
        self.shape = shape
        self.cfg = make_draft_config(shape, max_vis, max_batch)
        self.device = device
        self.h = L.rtv_draft_create(self.cfg, device)
        self._keep = []

    def load(self, weights: Dict[str, object]):
        """weights: name -> array (the action queries are always fp32)."""
        tensors, keep = make_tensors(weights, self.cfg.dtype, {"action_queries": L.RTV_F32})
        L.rtv_draft_load(self.h, tensors)
        del keep

    def forward(self, vis, out=None, stream=None):
        """Candidate chunks [B][H][A] fp32 for image features vis [B][V][w]
        (numpy float32 with bf16 values / uint16 bits, or a torch tensor)."""
        vis = to_dtype_bits(vis, self.cfg.dtype, "visual tokens")
        if isinstance(vis, np.ndarray):
            vis = np.ascontiguousarray(vis)
        b, v = int(vis.shape[0]), int(vis.shape[1])
        if out is None:
            if isinstance(vis, np.ndarray):
                out = np.empty((b, self.cfg.n_queries, self.cfg.action_dim), dtype=np.float32)
            else:
                import torch
                out = torch.empty((b, self.cfg.n_queries, self.cfg.action_dim), dtype=torch.float32,
                                  device=vis.device)
        pv, _ = _ptr(vis)
        po, _ = _ptr(out)
        self._keep = [vis]
        L.rtv_draft_forward(self.h, pv, v, b, po, _stream(stream))
        if isinstance(out, np.ndarray):
            self.synchronize()
        return out

    def synchronize(self):
        try:
            import torch
            if torch.cuda.is_available():
                torch.cuda.synchronize(self.device)
        except Exception:  # pragma: no cover
            pass

    def status(self):
        return L.rtv_draft_device_status(self.h)

    def kernels_per_call(self, n_vis: int, batch: int = 1) -> int:
        return L.rtv_draft_kernel_count(self.h, n_vis, batch)

    @property
    def path(self) -> str:
        return L.rtv_draft_path_name(self.h)

    def close(self):
        if self.h:
            L.rtv_draft_destroy(self.h)
            self.h = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass


class RoundResult(NamedTuple):
    chunk: object          # [H][A] fp32: the draft, or the denoised chunk
    accepted_len: int
    flags: int
    used_full: bool


def flash_round(expert: ActionExpert, draft: DraftModel, vis, noise, state, taus: Sequence[float], delta: float,
                gripper_dim: int, n_steps: int, out=None, stream=None) -> RoundResult:
    """One FLASH round (rtv_flash_round) for one observation: vis [V][w],
    noise [H][A], state [Sd]; returns once the chunk is in ``out``."""
    vis = to_dtype_bits(vis, draft.cfg.dtype, "visual tokens")
    if isinstance(vis, np.ndarray):
        vis = np.ascontiguousarray(vis)
    taus_h = np.ascontiguousarray(np.asarray(taus, dtype=np.float32))
    if out is None:
        shape = (expert.cfg.chunk_len, expert.cfg.action_dim)
        if isinstance(noise, np.ndarray):
            out = np.empty(shape, dtype=np.float32)
        else:
            out = noise.new_empty(shape)
    acc = np.zeros(1, dtype=np.int32)
    flags = np.zeros(1, dtype=np.uint32)
    full = np.zeros(1, dtype=np.int32)
    pv, _ = _ptr(vis)
    pn, _ = _ptr(noise)
    ps, _ = _ptr(state)
    po, _ = _ptr(out)
    L.rtv_flash_round(expert.h, draft.h, pv, int(vis.shape[0]), pn, ps, taus_h.ctypes.data, len(taus_h), float(delta),
                      int(gripper_dim), int(n_steps), po, acc.ctypes.data, flags.ctypes.data, full.ctypes.data,
                      _stream(stream))
    return RoundResult(out, int(acc[0]), int(flags[0]), bool(full[0]))
