"""Python-side handle of the VLM prefill stack (argument marshalling only;
the computation runs in ``librtv.so``).

    pf = PrefillStack(shape, device=0)                  # rtv_prefill_create
    pf.load(weights)                                     # rtv_prefill_load
    pf.kv(expert, emb)                                   # rtv_prefill_kv: installs the expert's prefix
    chunk = pf.denoise(expert, emb, noise, state, 10)    # rtv_prefill_denoise: prefill + denoise, one graph

``shape`` is any object with the rtv_prefill_config field names (n_layers,
width, n_q_heads, n_kv_heads, head_dim, mlp_dim; n_tokens gives the maximum
unless passed; dtype "bf16").
"""

from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from . import _lib as L
from .expert import _DTYPES, ActionExpert, _ptr, _stream, make_tensors, to_dtype_bits


def make_prefill_config(shape, max_tokens: Optional[int] = None) -> L.rtv_prefill_config:
    g = lambda n, d=None: getattr(shape, n, d)  # noqa: E731
    cfg = L.rtv_prefill_config()
    for n in ("n_layers", "width", "n_q_heads", "n_kv_heads", "head_dim", "mlp_dim"):
        setattr(cfg, n, int(g(n)))
    cfg.max_tokens = int(max_tokens or g("n_tokens"))
    cfg.dtype = _DTYPES[g("dtype", "bf16")]
    cfg.rms_eps = float(g("rms_eps", 1e-6))
    cfg.rope_theta = float(g("rope_theta", 10000.0))
    cfg.barrier_timeout_ns = 0
    return cfg


class PrefillStack:
    def __init__(self, shape, device: int = 0, max_tokens: Optional[int] = None):
        self.shape = shape
        self.cfg = make_prefill_config(shape, max_tokens)
        self.device = device
        self.h = L.rtv_prefill_create(self.cfg, device)
        self._keep = []

    def load(self, weights: Dict[str, object]):
        tensors, keep = make_tensors(weights, self.cfg.dtype)
        L.rtv_prefill_load(self.h, tensors)
        del keep

    def _emb(self, emb):
        emb = to_dtype_bits(emb, self.cfg.dtype, "prefix embeddings")
        if isinstance(emb, np.ndarray):
            emb = np.ascontiguousarray(emb)
        self._keep = [emb]
        return emb

    def kv(self, expert: ActionExpert, emb, stream=None):
        """Install the cache of emb [P][w] as the expert's prefix (batch 1)."""
        emb = self._emb(emb)
        pe, _ = _ptr(emb)
        L.rtv_prefill_kv(self.h, expert.h, pe, int(emb.shape[0]), _stream(stream))
        if isinstance(emb, np.ndarray):
            expert.synchronize()

    def denoise(self, expert: ActionExpert, emb, noise, state, n_steps: int, out=None, stream=None):
        """Prefill + denoising in one graph: chunk [H][A] from emb [P][w],
        noise [H][A], state [Sd]."""
        emb = self._emb(emb)
        if out is None:
            if isinstance(noise, np.ndarray):
                out = np.empty_like(noise, dtype=np.float32)
            else:
                out = noise.new_empty(noise.shape)
        pe, _ = _ptr(emb)
        pn, _ = _ptr(noise)
        ps, _ = _ptr(state)
        po, _ = _ptr(out)
        L.rtv_prefill_denoise(self.h, expert.h, pe, int(emb.shape[0]), pn, ps, int(n_steps), po, _stream(stream))
        if isinstance(out, np.ndarray):
            expert.synchronize()
        return out

    def status(self):
        return L.rtv_prefill_device_status(self.h)

    def kernels_per_call(self, n_tokens: int, n_steps: int = 0) -> int:
        return L.rtv_prefill_kernel_count(self.h, n_tokens, n_steps)

    def close(self):
        if self.h:
            L.rtv_prefill_destroy(self.h)
            self.h = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass
