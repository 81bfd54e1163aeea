"""Seeded synthetic workloads for the MTFM masked-attention path.

This module only draws inputs: jagged user lengths, R-token timestamps, T-token
exposure times and bf16 activations.  It holds none of the attention, mask or
normalisation arithmetic, so both the fp64 oracle (``oracle/``) and the CUDA
path (``hybrid_masked_attention_b200``) can consume the very same arrays
without sharing any of the method's code.

Workload shapes follow the pages:
  * user-level samples [H | R | T] with history lengths in the hundreds to
    thousands ("MTFM: Meituan unified recommendation foundation model ..."
    tech blog, section 3.3.1, and section 7.1 for the 400-2000 length range);
  * several exposure targets per user, spread over scenarios (same blog,
    section 4.1, user-level samples);
  * R tokens sorted by their action timestamps, T tokens carrying the
    exposure time of their request (same blog, section 3.1 and 3.2).
The proprietary logs the pages train on are not available; these seeded
draws stand in for them.

Every tensor gets its own numpy ``SeedSequence`` stream ``[seed, stream_id]``
so that adding a tensor never changes the values of the others.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

# Stream ids (one independent generator per drawn quantity).
S_LEN, S_TS, S_EXP, S_SCEN, S_Q, S_K, S_V, S_U, S_DY, S_GAMMA, S_BETA, S_W = range(12)


def rng_for(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(stream)]))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even); return the raw uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    out = ((u + rounding) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def normal_bf16(seed: int, stream: int, shape, std: float = 1.0) -> np.ndarray:
    """N(0, std^2) draws rounded to bf16; returns uint16 bit patterns."""
    g = rng_for(seed, stream)
    x = (g.standard_normal(size=shape) * std).astype(np.float32)
    return f32_to_bf16_bits(x)


@dataclass
class JaggedBatch:
    """Per-user lengths and timestamps of one jagged batch of user-level samples."""
    L_H: np.ndarray            # int32 [B]
    L_R: np.ndarray            # int32 [B]
    L_T: np.ndarray            # int32 [B]
    r_ts: np.ndarray           # int64 [sum L_R], sorted ascending within each user
    t_exp: np.ndarray          # int64 [sum L_T], exposure time of each T token
    scenario: np.ndarray       # int32 [sum L_T], scenario id (metadata only)
    v2_subtokens: int = 1      # 1: one token per target; 4: V2 target scale-up

    @property
    def B(self) -> int:
        return int(self.L_H.shape[0])

    @property
    def N(self) -> np.ndarray:
        return (self.L_H.astype(np.int64) + self.L_R + self.L_T)

    @property
    def total_tokens(self) -> int:
        return int(self.N.sum())

    @property
    def total_t(self) -> int:
        return int(self.L_T.sum())

    @property
    def total_r(self) -> int:
        return int(self.L_R.sum())


def _draw_times(seed, lens_r, lens_t_targets, v2):
    g_ts = rng_for(seed, S_TS)
    g_ex = rng_for(seed, S_EXP)
    g_sc = rng_for(seed, S_SCEN)
    r_parts, e_parts, s_parts = [], [], []
    for lr, nt in zip(lens_r, lens_t_targets):
        r_parts.append(np.sort(g_ts.integers(0, 1000, size=int(lr), dtype=np.int64)))
        e = g_ex.integers(0, 1000, size=int(nt), dtype=np.int64)
        s = g_sc.integers(0, 3, size=int(nt), dtype=np.int64).astype(np.int32)
        e_parts.append(np.repeat(e, v2))
        s_parts.append(np.repeat(s, v2))
    cat = lambda parts, dt: (np.concatenate(parts).astype(dt) if parts else np.zeros(0, dt))
    return cat(r_parts, np.int64), cat(e_parts, np.int64), cat(s_parts, np.int32)


def fixed_batch(L_H, L_R, L_T, seed: int, v2_subtokens: int = 1) -> JaggedBatch:
    """A batch with given per-user lengths; timestamps drawn uniformly in [0, 1000)."""
    L_H = np.asarray(L_H, dtype=np.int32)
    L_R = np.asarray(L_R, dtype=np.int32)
    L_T = np.asarray(L_T, dtype=np.int32)
    assert np.all(L_T % v2_subtokens == 0)
    r_ts, t_exp, scen = _draw_times(seed, L_R, L_T // v2_subtokens, v2_subtokens)
    return JaggedBatch(L_H, L_R, L_T, r_ts, t_exp, scen, v2_subtokens)


def tiny_batch(seed: int = 1000) -> JaggedBatch:
    """2 users of 32 H + 16 R + 8 T tokens."""
    return fixed_batch([32, 32], [16, 16], [8, 8], seed)


def pair_batch(B: int = 32, seed: int = 1001) -> JaggedBatch:
    """Production-shape jagged batch: L_H ~ U[256,1024], L_R ~ U[32,256], L_T ~ U[16,128]."""
    g = rng_for(seed, S_LEN)
    L_H = g.integers(256, 1025, size=B).astype(np.int32)
    L_R = g.integers(32, 257, size=B).astype(np.int32)
    L_T = g.integers(16, 129, size=B).astype(np.int32)
    return fixed_batch(L_H, L_R, L_T, seed)


def sweep_batch(N: int, v2: bool = False, total_tokens: int = 1 << 21, B: Optional[int] = None,
                seed: int = 1003) -> JaggedBatch:
    """Sequence-length sweep: every user has N tokens split H:R:T ~ 70:15:15.

    V1: L_H = round(0.7 N), L_R = round(0.15 N), L_T = N - L_H - L_R.
    V2: n_targets = round(0.15 N / 4) targets of 4 sub-tokens each; H absorbs the rounding.
    """
    if B is None:
        B = max(1, total_tokens // N)
    L_R = int(round(0.15 * N))
    if v2:
        nt = int(round(0.15 * N / 4))
        L_T = 4 * nt
        L_H = N - L_R - L_T
        sub = 4
    else:
        L_H = int(round(0.7 * N))
        L_T = N - L_H - L_R
        sub = 1
    return fixed_batch([L_H] * B, [L_R] * B, [L_T] * B, seed, v2_subtokens=sub)


@dataclass
class Heads:
    hq: int
    hkv: int
    dh: int

    @property
    def dq(self) -> int:
        return self.hq * self.dh

    @property
    def dkv(self) -> int:
        return self.hkv * self.dh


TINY_HEADS = Heads(2, 1, 32)
PAIR_HEADS = Heads(8, 2, 64)


@dataclass
class LayerInputs:
    """bf16 bit patterns (uint16) of one attention layer's inputs."""
    q: np.ndarray      # [rows_q, hq*dh]
    k: np.ndarray      # [sum N, hkv*dh]
    v: np.ndarray      # [sum N, hkv*dh]
    u: np.ndarray      # [rows_q, hq*dh]
    gamma: Optional[np.ndarray] = None   # float32 [3, hq*dh]
    beta: Optional[np.ndarray] = None    # float32 [3, hq*dh]
    dy: Optional[np.ndarray] = None      # bf16 bits [rows_q, hq*dh]


def layer_inputs(batch: JaggedBatch, heads: Heads, target: bool, seed: int,
                 gln: bool = True, with_dy: bool = False, random_affine: bool = True) -> LayerInputs:
    """Q, K, V, U ~ N(0,1) in bf16; GLN gamma/beta per token type (H, R, T).

    ``target`` selects the Target-Attention layout where Q and U exist only for T rows.
    """
    rows_q = batch.total_t if target else batch.total_tokens
    off = 50 if target else 0
    q = normal_bf16(seed, S_Q + off, (rows_q, heads.dq))
    k = normal_bf16(seed, S_K + off, (batch.total_tokens, heads.dkv))
    v = normal_bf16(seed, S_V + off, (batch.total_tokens, heads.dkv))
    u = normal_bf16(seed, S_U + off, (rows_q, heads.dq))
    gamma = beta = None
    if gln:
        if random_affine:
            gamma = (1.0 + 0.25 * rng_for(seed, S_GAMMA + off).standard_normal((3, heads.dq))).astype(np.float32)
            beta = (0.25 * rng_for(seed, S_BETA + off).standard_normal((3, heads.dq))).astype(np.float32)
        else:
            gamma = np.ones((3, heads.dq), np.float32)
            beta = np.zeros((3, heads.dq), np.float32)
    dy = normal_bf16(seed, S_DY + off, (rows_q, heads.dq)) if with_dy else None
    return LayerInputs(q, k, v, u, gamma, beta, dy)


# ----------------------------------------------------------------------------
# Backbone stack (4 blocks of one Full-Attention layer and three Target-Attention
# layers; page "美团推荐大模型 MTFM 深度硬核解析" §4.1-4.2): projection weights
# and the input token matrix.
# ----------------------------------------------------------------------------

STACK_KINDS = ("F", "T", "T", "T") * 4
S_X0, S_WIN, S_WKV, S_WO, S_RMS = 20, 21, 22, 23, 24


@dataclass
class LayerWeights:
    """One layer's parameters.  Projection matrices are bf16 bit patterns in the
    [out_features, in_features] layout; norms' parameters are float32."""
    kind: str                     # "F" (Full) or "T" (Target)
    rms_w: np.ndarray             # [d_model] RMSNorm weight
    w_in: np.ndarray              # F: W_uqkv [2*dq + 2*dkv, d_model]; T: W_uq [2*dq, d_model]
    w_kv: Optional[np.ndarray]    # T: W_kv [2*dkv, d_model]; F: None
    w_o: np.ndarray               # [d_model, dq]
    gamma: np.ndarray             # [3, dq] GLN affine rows (H, R, T)
    beta: np.ndarray              # [3, dq]


def stack_weights(heads: Heads, d_model: int, seed: int, kinds=STACK_KINDS, std: float = 0.02,
                  std_o: Optional[float] = None, random_norms: bool = False) -> list:
    """Weights ~ N(0, std) (std 0.02), output projections ~ N(0, std_o) with the
    depth-scaled std_o = 0.02 / sqrt(layers) (Meituan tech blog §5.1, depth-aware
    initialisation; its formula is garbled, the standard deviation is the reading).  Norm parameters are the identity
    (RMSNorm weight 1, GLN gamma 1 and beta 0) unless ``random_norms``."""
    if std_o is None:
        std_o = std / np.sqrt(len(kinds))
    dq, dkv = heads.dq, heads.dkv
    out = []
    for l, kind in enumerate(kinds):
        s = seed * 1000 + l
        if kind == "F":
            w_in = normal_bf16(s, S_WIN, (2 * dq + 2 * dkv, d_model), std)
            w_kv = None
        else:
            w_in = normal_bf16(s, S_WIN, (2 * dq, d_model), std)
            w_kv = normal_bf16(s, S_WKV, (2 * dkv, d_model), std)
        w_o = normal_bf16(s, S_WO, (d_model, dq), std_o)
        if random_norms:
            g = rng_for(s, S_RMS)
            rms_w = (1.0 + 0.25 * g.standard_normal(d_model)).astype(np.float32)
            gamma = (1.0 + 0.25 * g.standard_normal((3, dq))).astype(np.float32)
            beta = (0.25 * g.standard_normal((3, dq))).astype(np.float32)
        else:
            rms_w = np.ones(d_model, np.float32)
            gamma = np.ones((3, dq), np.float32)
            beta = np.zeros((3, dq), np.float32)
        out.append(LayerWeights(kind, rms_w, w_in, w_kv, w_o, gamma, beta))
    return out


def stack_input(batch: JaggedBatch, d_model: int, seed: int) -> np.ndarray:
    """Token matrix X0 [sum N, d_model] ~ N(0, 1), bf16 bit patterns."""
    return normal_bf16(seed, S_X0, (batch.total_tokens, d_model))


# ----------------------------------------------------------------------------
# V2 Target Scale-Up layer (Meituan tech blog §3.3.2): per-sub-token query-side
# projections and SwiGLU FFNs.
# ----------------------------------------------------------------------------

S_WUQ4, S_WG4, S_WU4, S_WD4, S_RMS2 = 30, 31, 32, 33, 34


@dataclass
class V2LayerWeights:
    """Weights of one V2 Target layer: bf16 bit patterns [out, in]; norms float32."""
    rms_w: np.ndarray              # [d_model] pre-norm of the attention block
    w_uq: list                     # 4 x [2*dq, d_model]: U then Q rows, one per sub-token position
    w_kv: np.ndarray               # [2*dkv, d_model]
    w_o: np.ndarray                # [d_model, dq]
    gamma: np.ndarray              # [3, dq]
    beta: np.ndarray               # [3, dq]
    rms_w2: np.ndarray             # [d_model] pre-norm of the FFN
    w_gate: list                   # 4 x [d_ff, d_model]
    w_up: list                     # 4 x [d_ff, d_model]
    w_down: list                   # 4 x [d_model, d_ff]


def v2_layer_weights(heads: Heads, d_model: int, d_ff: int, seed: int, std: float = 0.02,
                     std_o: float = 0.02, std_ffn: float = 0.02, random_norms: bool = True) -> V2LayerWeights:
    dq, dkv = heads.dq, heads.dkv
    w_uq = [normal_bf16(seed * 10 + s, S_WUQ4, (2 * dq, d_model), std) for s in range(4)]
    w_kv = normal_bf16(seed, S_WKV, (2 * dkv, d_model), std)
    w_o = normal_bf16(seed, S_WO, (d_model, dq), std_o)
    w_gate = [normal_bf16(seed * 10 + s, S_WG4, (d_ff, d_model), std_ffn) for s in range(4)]
    w_up = [normal_bf16(seed * 10 + s, S_WU4, (d_ff, d_model), std_ffn) for s in range(4)]
    w_down = [normal_bf16(seed * 10 + s, S_WD4, (d_model, d_ff), std_ffn) for s in range(4)]
    if random_norms:
        g = rng_for(seed, S_RMS2)
        rms_w = (1.0 + 0.25 * g.standard_normal(d_model)).astype(np.float32)
        rms_w2 = (1.0 + 0.25 * g.standard_normal(d_model)).astype(np.float32)
        gamma = (1.0 + 0.25 * g.standard_normal((3, dq))).astype(np.float32)
        beta = (0.25 * g.standard_normal((3, dq))).astype(np.float32)
    else:
        rms_w = np.ones(d_model, np.float32)
        rms_w2 = np.ones(d_model, np.float32)
        gamma = np.ones((3, dq), np.float32)
        beta = np.zeros((3, dq), np.float32)
    return V2LayerWeights(rms_w, w_uq, w_kv, w_o, gamma, beta, rms_w2, w_gate, w_up, w_down)
