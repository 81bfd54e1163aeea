"""Per-batch helper around the C ABI: owns the metadata block and scratch of one
jagged batch and allocates outputs with torch (device memory only).

Every computation happens in libmtfm's kernels; this class only sizes buffers
and forwards pointers.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import (Config, alloc_meta, attn_full_bwd, attn_full_fwd, attn_target_bwd, attn_target_fwd,
               bwd_workspace_bytes, pack, pack_check)


class HybridAttention:
    """Masked SiLU attention for one packed jagged batch (Full and Target layers)."""

    def __init__(self, cfg: Config, device: str = "cuda"):
        self.cfg = cfg
        self.device = torch.device(device)
        self.meta = alloc_meta(cfg, self.device)
        self._ws = {}

    # -- packing -------------------------------------------------------------
    def pack(self, lh, lr, lt, r_ts, t_exp, stream=None, check: bool = False):
        """Build offsets, per-row mask metadata and the work lists on the device."""
        pack(self.cfg, lh, lr, lt, r_ts, t_exp, self.meta, stream)
        if check:
            pack_check(self.meta, stream)

    # -- forward -------------------------------------------------------------
    def _fwd_out(self, rows: int, gln: bool):
        D = self.cfg.D
        y = torch.empty(rows, D, dtype=torch.float32, device=self.device)
        a = torch.empty(rows, D, dtype=torch.float32, device=self.device)
        stats = torch.empty(rows, 2, dtype=torch.float32, device=self.device) if gln else None
        return y, a, stats

    def full_fwd(self, q, k, v, u, gamma=None, beta=None, out=None, stream=None):
        y, a, stats = out if out is not None else self._fwd_out(self.cfg.total_tokens, gamma is not None)
        attn_full_fwd(self.cfg, self.meta, q, k, v, u, gamma, beta, y, a, stats, stream)
        return y, a, stats

    def target_fwd(self, q, k, v, u, gamma=None, beta=None, out=None, stream=None):
        y, a, stats = out if out is not None else self._fwd_out(self.cfg.total_t, gamma is not None)
        attn_target_fwd(self.cfg, self.meta, q, k, v, u, gamma, beta, y, a, stats, stream)
        return y, a, stats

    # -- backward ------------------------------------------------------------
    def workspace(self, target: bool) -> torch.Tensor:
        if target not in self._ws:
            n = bwd_workspace_bytes(self.cfg, target)
            self._ws[target] = torch.empty(n, dtype=torch.uint8, device=self.device)
        return self._ws[target]

    def _bwd(self, fn, rows, target, q, k, v, u, gamma, beta, a, stats, dy, stream):
        D, Dkv, N = self.cfg.D, self.cfg.Dkv, self.cfg.total_tokens
        f = dict(dtype=torch.float32, device=self.device)
        dq = torch.empty(rows, D, **f)
        du = torch.empty(rows, D, **f)
        dk = torch.empty(N, Dkv, **f)
        dv = torch.empty(N, Dkv, **f)
        dgamma = torch.empty(3, D, **f) if gamma is not None else None
        dbeta = torch.empty(3, D, **f) if gamma is not None else None
        fn(self.cfg, self.meta, q, k, v, u, gamma, beta, a, stats, dy, dq, dk, dv, du, dgamma, dbeta,
           self.workspace(target), stream)
        return {"dq": dq, "dk": dk, "dv": dv, "du": du, "dgamma": dgamma, "dbeta": dbeta}

    def full_bwd(self, q, k, v, u, gamma, beta, a, stats, dy, stream=None):
        return self._bwd(attn_full_bwd, self.cfg.total_tokens, False, q, k, v, u, gamma, beta, a,
                         stats, dy, stream)

    def target_bwd(self, q, k, v, u, gamma, beta, a, stats, dy, stream=None):
        return self._bwd(attn_target_bwd, self.cfg.total_t, True, q, k, v, u, gamma, beta, a, stats,
                         dy, stream)
