"""Device buffers of an AQUA KV cache, allocated with PyTorch (memory only).

The cache owns its torch tensors and the aqua_cache descriptor that points at
them; all computation on the buffers happens in the CUDA library.
"""
from __future__ import annotations

import torch

from . import abi


class AquaCache:
    """Projected-key cache (dimension-major), value cache (token-major) and lengths.

    k_proj [B, Hkv, d_store, Tcap], v [B, Hkv, Tcap, d] (with dv_store: the
    first dv_store projected value dims, [B, Hkv, Tcap, dv_store]), len [B],
    n_abs [B]; with h2o=True also pos [B, Hkv, Tcap] (int32) and score
    [B, Hkv, Tcap] (f32).
    """

    def __init__(self, B: int, Hkv: int, Tcap: int, d: int = 128, d_store: int | None = None,
                 dtype: torch.dtype = torch.bfloat16, h2o: bool = False, device="cuda", dv_store: int | None = None):
        d_store = d if d_store is None else d_store
        if Tcap % 16:
            Tcap += 16 - Tcap % 16
        self.B, self.Hkv, self.d, self.d_store, self.Tcap, self.dtype = B, Hkv, d, d_store, Tcap, dtype
        self.dv_store = dv_store or 0
        self.k_proj = torch.zeros((B, Hkv, d_store, Tcap), dtype=dtype, device=device)
        self.v = torch.zeros((B, Hkv, Tcap, self.dv_store or d), dtype=dtype, device=device)
        self.len = torch.zeros((B,), dtype=torch.int32, device=device)
        self.n_abs = torch.zeros((B,), dtype=torch.int32, device=device)
        self.ctrl = torch.zeros((abi.AQUA_CTRL_WORDS,), dtype=torch.int32, device=device)
        self.pos = torch.zeros((B, Hkv, Tcap), dtype=torch.int32, device=device) if h2o else None
        self.score = torch.zeros((B, Hkv, Tcap), dtype=torch.float32, device=device) if h2o else None
        self.desc = abi.aqua_cache(
            self.k_proj.data_ptr(), self.v.data_ptr(), self.len.data_ptr(), self.n_abs.data_ptr(),
            self.pos.data_ptr() if h2o else None, self.score.data_ptr() if h2o else None,
            self.ctrl.data_ptr(), B, Hkv, d, d_store, Tcap, 0,
            abi.AQUA_BF16 if dtype == torch.bfloat16 else abi.AQUA_F32, self.dv_store)

    @property
    def max_len(self) -> int:
        return self.desc.max_len

    def reset(self) -> None:
        """Forget every token (lengths to zero); buffers keep their contents."""
        self.len.zero_()
        self.n_abs.zero_()
        self.desc.max_len = 0

    def snapshot(self) -> dict:
        """Device-to-host copy of every buffer and the host length bound (checkpoint)."""
        snap = {name: getattr(self, name).detach().cpu().clone()
                for name in ("k_proj", "v", "len", "n_abs", "pos", "score") if getattr(self, name) is not None}
        snap["max_len"] = self.desc.max_len
        return snap

    def restore(self, snap: dict) -> None:
        """Copy a snapshot back into this cache's buffers (same shapes)."""
        for name, t in snap.items():
            if name == "max_len":
                self.desc.max_len = int(t)
            else:
                getattr(self, name).copy_(t)
