"""Python binding of libmtfm, the B200 (sm_100a) MTFM hybrid masked-attention library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/mtfm.h``.  PyTorch supplies
device memory and streams.  There is no fallback: if ``libmtfm.so`` is missing
this import fails; build it with ``python hybrid_masked_attention_b200/build.py``.

Function names mirror the C entry points:
    meta_bytes, max_items, pack, pack_check, meta_read,
    attn_full_fwd, attn_target_fwd, attn_full, attn_target, gate_fwd,
    attn_target_cached_fwd, attn_target_cached,
    bwd_workspace_bytes, attn_full_bwd, attn_target_bwd, attn_target_bwd_static,
    stack_workspace_bytes, layer_fwd, stack_fwd, v2_workspace_bytes, v2_target_layer_fwd,
    selftest_wait_timeout
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MTFM_LIBRARY may name another build of the same library (the bounds-checked
# libmtfm_debug_bounds.so); it changes which file is loaded, not what it runs.
LIB_PATH = os.environ.get("MTFM_LIBRARY") or os.path.join(_PKG, "libmtfm.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} not found; build it with "
        "`python hybrid_masked_attention_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

MTFM_OK = 0
STATUS_NAMES = {
    0: "MTFM_OK", 1: "MTFM_ERR_INVALID_ARG", 2: "MTFM_ERR_UNSORTED_TS", 3: "MTFM_ERR_UNSUPPORTED",
    4: "MTFM_ERR_WORKSPACE_TOO_SMALL", 5: "MTFM_ERR_CUDA", 6: "MTFM_ERR_TIMEOUT",
    7: "MTFM_ERR_BAD_LENGTHS", 8: "MTFM_ERR_BOUNDS",
}


class MtfmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.mtfm_status_string(status).decode()
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({msg})")


class CCfg(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("total_tokens", ctypes.c_int32),
                ("total_r", ctypes.c_int32), ("total_t", ctypes.c_int32),
                ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("v2_subtokens", ctypes.c_int32), ("alpha", ctypes.c_float),
                ("gln_eps", ctypes.c_float)]


@dataclass
class Config:
    """Problem description (mirrors ``mtfm_cfg``)."""
    batch: int
    total_tokens: int
    total_r: int
    total_t: int
    hq: int
    hkv: int
    head_dim: int
    v2_subtokens: int = 1
    alpha: float = 0.0      # <= 0: 1/sqrt(head_dim)
    gln_eps: float = 0.0    # <= 0: 1e-5

    def c(self) -> CCfg:
        return CCfg(self.batch, self.total_tokens, self.total_r, self.total_t, self.hq, self.hkv,
                    self.head_dim, self.v2_subtokens, self.alpha, self.gln_eps)

    @property
    def D(self) -> int:
        return self.hq * self.head_dim

    @property
    def Dkv(self) -> int:
        return self.hkv * self.head_dim

    @property
    def alpha_eff(self) -> float:
        return self.alpha if self.alpha > 0 else 1.0 / math.sqrt(self.head_dim)


class CLayerWeights(ctypes.Structure):
    _fields_ = [("rms_w", ctypes.c_void_p), ("w_in", ctypes.c_void_p), ("w_kv", ctypes.c_void_p),
                ("w_o", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("beta", ctypes.c_void_p)]


class CV2LayerWeights(ctypes.Structure):
    _fields_ = [("rms_w", ctypes.c_void_p), ("w_uq", ctypes.c_void_p * 4), ("w_kv", ctypes.c_void_p),
                ("w_o", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("beta", ctypes.c_void_p),
                ("rms_w2", ctypes.c_void_p), ("w_gate", ctypes.c_void_p * 4), ("w_up", ctypes.c_void_p * 4),
                ("w_down", ctypes.c_void_p * 4)]


_P = ctypes.c_void_p
_CP = ctypes.POINTER(CCfg)
_LWP = ctypes.POINTER(CLayerWeights)
_V2P = ctypes.POINTER(CV2LayerWeights)
_sigs = {
    "mtfm_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mtfm_meta_bytes": (ctypes.c_size_t, [_CP]),
    "mtfm_pack": (ctypes.c_int, [_CP, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "mtfm_pack_check": (ctypes.c_int, [_P, _P]),
    "mtfm_debug_bounds_build": (ctypes.c_int32, []),
    "mtfm_debug_site": (ctypes.c_int, [_P, _P, _P]),
    "mtfm_meta_read": (ctypes.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "mtfm_max_items": (ctypes.c_int32, [_CP, ctypes.c_int]),
    "mtfm_attn_full_fwd": (ctypes.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "mtfm_attn_target_fwd": (ctypes.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "mtfm_attn_full_fwd_bf16y": (ctypes.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "mtfm_attn_target_fwd_bf16y": (ctypes.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "mtfm_attn_full": (ctypes.c_int, [_CP, _P, _P, _P, _P, _P, _P]),
    "mtfm_attn_target": (ctypes.c_int, [_CP, _P, _P, _P, _P, _P, _P]),
    "mtfm_attn_target_cached_fwd": (ctypes.c_int, [_CP] + [_P] * 13),
    "mtfm_attn_target_cached": (ctypes.c_int, [_CP] + [_P] * 8),
    "mtfm_gate_fwd": (ctypes.c_int, [_CP, _P, ctypes.c_int, _P, _P, _P, _P, _P, _P, _P]),
    "mtfm_bwd_workspace_bytes": (ctypes.c_size_t, [_CP, ctypes.c_int]),
    "mtfm_attn_full_bwd": (ctypes.c_int, [_CP] + [_P] * 17 + [ctypes.c_size_t, _P]),
    "mtfm_attn_target_bwd": (ctypes.c_int, [_CP] + [_P] * 17 + [ctypes.c_size_t, _P]),
    "mtfm_attn_target_bwd_static": (ctypes.c_int, [_CP] + [_P] * 17),
    "mtfm_selftest_wait_timeout": (ctypes.c_int, [_P, ctypes.c_int64, _P]),
    "mtfm_v2_workspace_bytes": (ctypes.c_size_t, [_CP, ctypes.c_int32, ctypes.c_int32]),
    "mtfm_v2_target_layer_fwd": (ctypes.c_int, [_CP, _P, ctypes.c_int32, ctypes.c_int32, _V2P, _P, _P,
                                                ctypes.c_size_t, _P]),
    "mtfm_stack_workspace_bytes": (ctypes.c_size_t, [_CP, ctypes.c_int32]),
    "mtfm_layer_fwd": (ctypes.c_int, [_CP, _P, ctypes.c_int32, ctypes.c_int, _LWP, _P, _P, ctypes.c_size_t, _P]),
    "mtfm_stack_fwd": (ctypes.c_int, [_CP, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_char_p, _LWP, _P, _P,
                                      ctypes.c_size_t, _P]),
}
for _name, (_res, _args) in _sigs.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_sigs)


def _check(status: int, where: str):
    if status != MTFM_OK:
        raise MtfmError(status, where)


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor], dtype=None, shape=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr() if t.numel() else (t.data_ptr() or None)


def meta_bytes(cfg: Config) -> int:
    c = cfg.c()
    n = _lib.mtfm_meta_bytes(ctypes.byref(c))
    if n == 0:
        raise MtfmError(1, "mtfm_meta_bytes")
    return n


def max_items(cfg: Config, target: bool) -> int:
    """Capacity of the Full or Target work list of the metadata block."""
    c = cfg.c()
    n = _lib.mtfm_max_items(ctypes.byref(c), int(bool(target)))
    if n < 0:
        raise MtfmError(1, "mtfm_max_items")
    return n


def alloc_meta(cfg: Config, device="cuda") -> torch.Tensor:
    """A metadata block of the right size (torch's allocator aligns to >= 256 bytes)."""
    return torch.empty(meta_bytes(cfg), dtype=torch.uint8, device=device)


def pack(cfg: Config, lh, lr, lt, r_ts, t_exp, meta: torch.Tensor, stream=None):
    c = cfg.c()
    B = cfg.batch
    st = _lib.mtfm_pack(ctypes.byref(c),
                        _ptr(lh, torch.int32, (B,), "lh"), _ptr(lr, torch.int32, (B,), "lr"),
                        _ptr(lt, torch.int32, (B,), "lt"),
                        _ptr(r_ts, torch.int64, (cfg.total_r,), "r_ts"),
                        _ptr(t_exp, torch.int64, (cfg.total_t,), "t_exp"),
                        _ptr(meta, torch.uint8, None, "meta"), meta.numel(), _stream(stream))
    _check(st, "mtfm_pack")


def pack_check(meta: torch.Tensor, stream=None):
    _check(_lib.mtfm_pack_check(_ptr(meta, torch.uint8, None, "meta"), _stream(stream)), "mtfm_pack_check")


def debug_bounds_build() -> bool:
    """True when the loaded library is the bounds-checked build (-DMTFM_DEBUG_BOUNDS)."""
    return bool(_lib.mtfm_debug_bounds_build())


def debug_site(meta: torch.Tensor, stream=None) -> int:
    """Site (file id * 100000 + line) of the first failed check of the bounds-checked build, or 0."""
    site = ctypes.c_int32()
    _check(_lib.mtfm_debug_site(_ptr(meta, torch.uint8, None, "meta"), ctypes.byref(site), _stream(stream)),
           "mtfm_debug_site")
    return site.value


def meta_read(cfg: Config, meta: torch.Tensor, stream=None) -> dict:
    B, T = cfg.batch, cfg.total_tokens
    out = {"seq_off": np.zeros(B + 1, np.int32), "r_off": np.zeros(B + 1, np.int32),
           "t_off": np.zeros(B + 1, np.int32), "kv_end": np.zeros(max(T, 1), np.int32),
           "row_type": np.zeros(max(T, 1), np.uint8)}
    nf = ctypes.c_int32()
    nt = ctypes.c_int32()
    c = cfg.c()
    mf = max_items(cfg, False)
    mt = max_items(cfg, True)
    out["items_full"] = np.zeros((max(mf, 1), 4), np.int32)
    out["items_target"] = np.zeros((max(mt, 1), 4), np.int32)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    st = _lib.mtfm_meta_read(ctypes.byref(c), _ptr(meta, torch.uint8, None, "meta"), p(out["seq_off"]),
                             p(out["r_off"]), p(out["t_off"]), p(out["kv_end"]), p(out["row_type"]),
                             ctypes.byref(nf), ctypes.byref(nt), p(out["items_full"]),
                             p(out["items_target"]), _stream(stream))
    _check(st, "mtfm_meta_read")
    out["kv_end"] = out["kv_end"][:T]
    out["row_type"] = out["row_type"][:T]
    out["n_items_full"] = nf.value
    out["n_items_target"] = nt.value
    out["items_full"] = out["items_full"][:nf.value]
    out["items_target"] = out["items_target"][:nt.value]
    return out


def _fwd(fn, where, cfg, meta, q, k, v, u, gamma, beta, y, a, stats, stream, rows, y_dtype=torch.float32):
    c = cfg.c()
    D, Dkv, N = cfg.D, cfg.Dkv, cfg.total_tokens
    bf = torch.bfloat16
    st = fn(ctypes.byref(c), _ptr(meta, torch.uint8, None, "meta"),
            _ptr(q, bf, (rows, D), "q"), _ptr(k, bf, (N, Dkv), "k"), _ptr(v, bf, (N, Dkv), "v"),
            _ptr(u, bf, (rows, D), "u"),
            _ptr(gamma, torch.float32, (3, D), "gamma"), _ptr(beta, torch.float32, (3, D), "beta"),
            _ptr(y, y_dtype, (rows, D), "y"), _ptr(a, torch.float32, (rows, D), "a"),
            _ptr(stats, torch.float32, (rows, 2), "stats"), _stream(stream))
    _check(st, where)


def attn_full_fwd(cfg, meta, q, k, v, u, gamma, beta, y, a, stats, stream=None):
    """Full-Attention layer forward: writes y, a (and stats when gamma is given)."""
    _fwd(_lib.mtfm_attn_full_fwd, "mtfm_attn_full_fwd", cfg, meta, q, k, v, u, gamma, beta, y, a,
         stats, stream, cfg.total_tokens)


def attn_target_fwd(cfg, meta, q, k, v, u, gamma, beta, y, a, stats, stream=None):
    """Target-Attention layer forward (T rows only)."""
    _fwd(_lib.mtfm_attn_target_fwd, "mtfm_attn_target_fwd", cfg, meta, q, k, v, u, gamma, beta, y,
         a, stats, stream, cfg.total_t)


def attn_full_fwd_bf16y(cfg, meta, q, k, v, u, gamma, beta, y, a, stats, stream=None):
    """attn_full_fwd with y as bf16 (the fp32 value rounded to nearest)."""
    _fwd(_lib.mtfm_attn_full_fwd_bf16y, "mtfm_attn_full_fwd_bf16y", cfg, meta, q, k, v, u, gamma, beta, y, a,
         stats, stream, cfg.total_tokens, torch.bfloat16)


def attn_target_fwd_bf16y(cfg, meta, q, k, v, u, gamma, beta, y, a, stats, stream=None):
    """attn_target_fwd with y as bf16 (the fp32 value rounded to nearest)."""
    _fwd(_lib.mtfm_attn_target_fwd_bf16y, "mtfm_attn_target_fwd_bf16y", cfg, meta, q, k, v, u, gamma, beta, y,
         a, stats, stream, cfg.total_t, torch.bfloat16)


def _attn_only(fn, where, cfg, meta, q, k, v, a, stream, rows):
    c = cfg.c()
    D, Dkv, N = cfg.D, cfg.Dkv, cfg.total_tokens
    bf = torch.bfloat16
    st = fn(ctypes.byref(c), _ptr(meta, torch.uint8, None, "meta"), _ptr(q, bf, (rows, D), "q"),
            _ptr(k, bf, (N, Dkv), "k"), _ptr(v, bf, (N, Dkv), "v"),
            _ptr(a, torch.float32, (rows, D), "a"), _stream(stream))
    _check(st, where)


def attn_full(cfg, meta, q, k, v, a, stream=None):
    """Full-layer attention only (A, fp32)."""
    _attn_only(_lib.mtfm_attn_full, "mtfm_attn_full", cfg, meta, q, k, v, a, stream, cfg.total_tokens)


def attn_target(cfg, meta, q, k, v, a, stream=None):
    """Target-layer attention only (A of the T rows, fp32)."""
    _attn_only(_lib.mtfm_attn_target, "mtfm_attn_target", cfg, meta, q, k, v, a, stream, cfg.total_t)


def attn_target_cached_fwd(cfg, meta, q, k_prefix, v_prefix, k_cand, v_cand, u, gamma, beta, y, a, stats,
                           stream=None):
    """Target-Attention layer forward over a cached key/value prefix: k_prefix, v_prefix hold
    the H and R rows of every user [total_tokens - total_t, Dkv], k_cand, v_cand the T rows
    (the candidates) [total_t, Dkv]; everything else as attn_target_fwd."""
    c = cfg.c()
    D, Dkv, T = cfg.D, cfg.Dkv, cfg.total_t
    P = cfg.total_tokens - T
    bf, f32 = torch.bfloat16, torch.float32
    st = _lib.mtfm_attn_target_cached_fwd(
        ctypes.byref(c), _ptr(meta, torch.uint8, None, "meta"), _ptr(q, bf, (T, D), "q"),
        _ptr(k_prefix, bf, (P, Dkv), "k_prefix"), _ptr(v_prefix, bf, (P, Dkv), "v_prefix"),
        _ptr(k_cand, bf, (T, Dkv), "k_cand"), _ptr(v_cand, bf, (T, Dkv), "v_cand"),
        _ptr(u, bf, (T, D), "u"), _ptr(gamma, f32, (3, D), "gamma"), _ptr(beta, f32, (3, D), "beta"),
        _ptr(y, f32, (T, D), "y"), _ptr(a, f32, (T, D), "a"), _ptr(stats, f32, (T, 2), "stats"), _stream(stream))
    _check(st, "mtfm_attn_target_cached_fwd")


def attn_target_cached(cfg, meta, q, k_prefix, v_prefix, k_cand, v_cand, a, stream=None):
    """Target attention only over a cached key/value prefix (A of the T rows, fp32)."""
    c = cfg.c()
    D, Dkv, T = cfg.D, cfg.Dkv, cfg.total_t
    P = cfg.total_tokens - T
    bf = torch.bfloat16
    st = _lib.mtfm_attn_target_cached(
        ctypes.byref(c), _ptr(meta, torch.uint8, None, "meta"), _ptr(q, bf, (T, D), "q"),
        _ptr(k_prefix, bf, (P, Dkv), "k_prefix"), _ptr(v_prefix, bf, (P, Dkv), "v_prefix"),
        _ptr(k_cand, bf, (T, Dkv), "k_cand"), _ptr(v_cand, bf, (T, Dkv), "v_cand"),
        _ptr(a, torch.float32, (T, D), "a"), _stream(stream))
    _check(st, "mtfm_attn_target_cached")


def gate_fwd(cfg, meta, target: bool, a, u, gamma, beta, y, stats, stream=None):
    """Y = GLN(A) (*) U for the Full or Target layout."""
    c = cfg.c()
    rows = cfg.total_t if target else cfg.total_tokens
    D = cfg.D
    f32 = torch.float32
    st = _lib.mtfm_gate_fwd(ctypes.byref(c), _ptr(meta, torch.uint8, None, "meta"), int(bool(target)),
                            _ptr(a, f32, (rows, D), "a"), _ptr(u, torch.bfloat16, (rows, D), "u"),
                            _ptr(gamma, f32, (3, D), "gamma"), _ptr(beta, f32, (3, D), "beta"),
                            _ptr(y, f32, (rows, D), "y"), _ptr(stats, f32, (rows, 2), "stats"),
                            _stream(stream))
    _check(st, "mtfm_gate_fwd")


def bwd_workspace_bytes(cfg: Config, target: bool) -> int:
    c = cfg.c()
    n = _lib.mtfm_bwd_workspace_bytes(ctypes.byref(c), int(bool(target)))
    if n == 0:
        raise MtfmError(1, "mtfm_bwd_workspace_bytes")
    return n


def _bwd(fn, where, cfg, meta, q, k, v, u, gamma, beta, a, stats, dy, dq, dk, dv, du, dgamma,
         dbeta, ws, stream, rows):
    c = cfg.c()
    D, Dkv, N = cfg.D, cfg.Dkv, cfg.total_tokens
    bf, f32 = torch.bfloat16, torch.float32
    st = fn(ctypes.byref(c), _ptr(meta, torch.uint8, None, "meta"),
            _ptr(q, bf, (rows, D), "q"), _ptr(k, bf, (N, Dkv), "k"), _ptr(v, bf, (N, Dkv), "v"),
            _ptr(u, bf, (rows, D), "u"), _ptr(gamma, f32, (3, D), "gamma"),
            _ptr(beta, f32, (3, D), "beta"), _ptr(a, f32, (rows, D), "a"),
            _ptr(stats, f32, (rows, 2), "stats"), _ptr(dy, bf, (rows, D), "dy"),
            _ptr(dq, f32, (rows, D), "dq"), _ptr(dk, f32, (N, Dkv), "dk"),
            _ptr(dv, f32, (N, Dkv), "dv"), _ptr(du, f32, (rows, D), "du"),
            _ptr(dgamma, f32, (3, D), "dgamma"), _ptr(dbeta, f32, (3, D), "dbeta"),
            _ptr(ws, torch.uint8, None, "ws"), ws.numel(), _stream(stream))
    _check(st, where)


def attn_full_bwd(cfg, meta, q, k, v, u, gamma, beta, a, stats, dy, dq, dk, dv, du, dgamma, dbeta,
                  ws, stream=None):
    _bwd(_lib.mtfm_attn_full_bwd, "mtfm_attn_full_bwd", cfg, meta, q, k, v, u, gamma, beta, a,
         stats, dy, dq, dk, dv, du, dgamma, dbeta, ws, stream, cfg.total_tokens)


def attn_target_bwd(cfg, meta, q, k, v, u, gamma, beta, a, stats, dy, dq, dk, dv, du, dgamma,
                    dbeta, ws, stream=None):
    _bwd(_lib.mtfm_attn_target_bwd, "mtfm_attn_target_bwd", cfg, meta, q, k, v, u, gamma, beta, a,
         stats, dy, dq, dk, dv, du, dgamma, dbeta, ws, stream, cfg.total_t)


def attn_target_bwd_static(cfg, meta, q, k, v, u, gamma, beta, a, stats, dy, dq, dk, dv, du, dgamma,
                           dbeta, stream=None):
    """Target-layer backward without a caller scratch block: the library's fixed
    24 MiB device array is used instead (for callers that cannot allocate).
    Calls that may overlap on the GPU must be serialised by the caller."""
    c = cfg.c()
    D, Dkv, N, rows = cfg.D, cfg.Dkv, cfg.total_tokens, cfg.total_t
    bf, f32 = torch.bfloat16, torch.float32
    st = _lib.mtfm_attn_target_bwd_static(
        ctypes.byref(c), _ptr(meta, torch.uint8, None, "meta"),
        _ptr(q, bf, (rows, D), "q"), _ptr(k, bf, (N, Dkv), "k"), _ptr(v, bf, (N, Dkv), "v"),
        _ptr(u, bf, (rows, D), "u"), _ptr(gamma, f32, (3, D), "gamma"),
        _ptr(beta, f32, (3, D), "beta"), _ptr(a, f32, (rows, D), "a"),
        _ptr(stats, f32, (rows, 2), "stats"), _ptr(dy, bf, (rows, D), "dy"),
        _ptr(dq, f32, (rows, D), "dq"), _ptr(dk, f32, (N, Dkv), "dk"),
        _ptr(dv, f32, (N, Dkv), "dv"), _ptr(du, f32, (rows, D), "du"),
        _ptr(dgamma, f32, (3, D), "dgamma"), _ptr(dbeta, f32, (3, D), "dbeta"), _stream(stream))
    _check(st, "mtfm_attn_target_bwd_static")


# ---------------------------------------------------------------------------- backbone stack

@dataclass
class LayerWeights:
    """Device tensors of one backbone layer (see ``mtfm_layer_weights`` in mtfm.h).

    rms_w fp32 [d_model]; w_in bf16 [out, d_model]; w_kv bf16 [2*Dkv, d_model] for a
    Target layer (None for Full); w_o bf16 [d_model, D]; gamma, beta fp32 [3, D] or None.
    """
    kind: str
    rms_w: torch.Tensor
    w_in: torch.Tensor
    w_kv: Optional[torch.Tensor]
    w_o: torch.Tensor
    gamma: Optional[torch.Tensor] = None
    beta: Optional[torch.Tensor] = None


def _layer_struct(cfg: Config, d_model: int, w: LayerWeights) -> CLayerWeights:
    D, Dkv = cfg.D, cfg.Dkv
    target = w.kind == "T"
    out = 2 * D if target else 2 * D + 2 * Dkv
    if w.kind not in ("F", "T"):
        raise ValueError("layer kind must be 'F' or 'T'")
    if target != (w.w_kv is not None):
        raise ValueError("w_kv is required for a Target layer and must be None for a Full layer")
    return CLayerWeights(
        _ptr(w.rms_w, torch.float32, (d_model,), "rms_w"),
        _ptr(w.w_in, torch.bfloat16, (out, d_model), "w_in"),
        _ptr(w.w_kv, torch.bfloat16, (2 * Dkv, d_model), "w_kv"),
        _ptr(w.w_o, torch.bfloat16, (d_model, D), "w_o"),
        _ptr(w.gamma, torch.float32, (3, D), "gamma"),
        _ptr(w.beta, torch.float32, (3, D), "beta"))


def stack_workspace_bytes(cfg: Config, d_model: int) -> int:
    c = cfg.c()
    n = _lib.mtfm_stack_workspace_bytes(ctypes.byref(c), int(d_model))
    if n == 0:
        raise MtfmError(3, "mtfm_stack_workspace_bytes")
    return n


def layer_fwd(cfg: Config, meta: torch.Tensor, d_model: int, w: LayerWeights, x: torch.Tensor,
              ws: torch.Tensor, stream=None):
    """One backbone layer on X (fp32 [total_tokens, d_model], updated in place)."""
    c = cfg.c()
    lw = _layer_struct(cfg, d_model, w)
    _check(_lib.mtfm_layer_fwd(ctypes.byref(c), _ptr(meta, torch.uint8, name="meta"), int(d_model),
                               int(w.kind == "T"), ctypes.byref(lw),
                               _ptr(x, torch.float32, (cfg.total_tokens, d_model), "x"),
                               _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream)),
           "mtfm_layer_fwd")


def stack_fwd(cfg: Config, meta: torch.Tensor, d_model: int, layers, x: torch.Tensor, ws: torch.Tensor,
              stream=None):
    """Run ``layers`` (a list of LayerWeights) on X in place."""
    c = cfg.c()
    arr = (CLayerWeights * max(1, len(layers)))(*[_layer_struct(cfg, d_model, w) for w in layers])
    kinds = "".join(w.kind for w in layers).encode()
    _check(_lib.mtfm_stack_fwd(ctypes.byref(c), _ptr(meta, torch.uint8, name="meta"), int(d_model),
                               len(layers), kinds, arr,
                               _ptr(x, torch.float32, (cfg.total_tokens, d_model), "x"),
                               _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream)),
           "mtfm_stack_fwd")


# ---------------------------------------------------------------------------- V2 Target layer

@dataclass
class V2LayerWeights:
    """Device tensors of one V2 Target Scale-Up layer (``mtfm_v2_layer_weights``).

    rms_w, rms_w2 fp32 [d_model]; w_uq: 4 bf16 [2*D, d_model] (U rows, then Q rows), one per
    sub-token position; w_kv bf16 [2*Dkv, d_model]; w_o bf16 [d_model, D]; gamma, beta fp32
    [3, D] or None; w_gate, w_up: 4 bf16 [d_ff, d_model]; w_down: 4 bf16 [d_model, d_ff].
    """
    rms_w: torch.Tensor
    w_uq: list
    w_kv: torch.Tensor
    w_o: torch.Tensor
    gamma: Optional[torch.Tensor]
    beta: Optional[torch.Tensor]
    rms_w2: torch.Tensor
    w_gate: list
    w_up: list
    w_down: list


def v2_workspace_bytes(cfg: Config, d_model: int, d_ff: int) -> int:
    c = cfg.c()
    n = _lib.mtfm_v2_workspace_bytes(ctypes.byref(c), int(d_model), int(d_ff))
    if n == 0:
        raise MtfmError(3, "mtfm_v2_workspace_bytes")
    return n


def v2_target_layer_fwd(cfg: Config, meta: torch.Tensor, d_model: int, d_ff: int, w: V2LayerWeights,
                        x: torch.Tensor, ws: torch.Tensor, stream=None):
    """One V2 Target Scale-Up layer on X (fp32 [total_tokens, d_model], updated in place)."""
    D, Dkv = cfg.D, cfg.Dkv
    bf, f32 = torch.bfloat16, torch.float32
    if len(w.w_uq) != 4 or len(w.w_gate) != 4 or len(w.w_up) != 4 or len(w.w_down) != 4:
        raise ValueError("w_uq, w_gate, w_up, w_down need one tensor per sub-token position (4)")
    four = lambda ts, shape, name: (ctypes.c_void_p * 4)(*[_ptr(t, bf, shape, f"{name}[{k}]") for k, t in enumerate(ts)])
    lw = CV2LayerWeights(
        _ptr(w.rms_w, f32, (d_model,), "rms_w"), four(w.w_uq, (2 * D, d_model), "w_uq"),
        _ptr(w.w_kv, bf, (2 * Dkv, d_model), "w_kv"), _ptr(w.w_o, bf, (d_model, D), "w_o"),
        _ptr(w.gamma, f32, (3, D), "gamma"), _ptr(w.beta, f32, (3, D), "beta"),
        _ptr(w.rms_w2, f32, (d_model,), "rms_w2"), four(w.w_gate, (d_ff, d_model), "w_gate"),
        four(w.w_up, (d_ff, d_model), "w_up"), four(w.w_down, (d_model, d_ff), "w_down"))
    c = cfg.c()
    _check(_lib.mtfm_v2_target_layer_fwd(ctypes.byref(c), _ptr(meta, torch.uint8, name="meta"), int(d_model),
                                         int(d_ff), ctypes.byref(lw),
                                         _ptr(x, f32, (cfg.total_tokens, d_model), "x"),
                                         _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream)),
           "mtfm_v2_target_layer_fwd")


def selftest_wait_timeout(meta: torch.Tensor, limit_cycles: int = 2_000_000, stream=None):
    """Make one bounded wait run out on the GPU; the timeout is recorded in ``meta``
    (``pack_check`` then raises MtfmError with MTFM_ERR_TIMEOUT)."""
    _check(_lib.mtfm_selftest_wait_timeout(_ptr(meta, torch.uint8, name="meta"), int(limit_cycles),
                                           _stream(stream)), "mtfm_selftest_wait_timeout")

