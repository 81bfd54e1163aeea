"""fp64 CPU oracle for the MTFM hybrid masked-attention path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA product path
never calls it, and it shares no code with ``hybrid_masked_attention_b200``:
the only thing both sides use is the seeded input generator ``mtfm_synth``.

Everything here is the plain definition written out in float64 with numpy:
a dense N x N 0/1 mask built cell by cell from the visibility rules, dense
score matrices, explicit SiLU, a dense masked product and a textbook
LayerNorm.  No tiling, skipping or interval tricks.  Matrix products use
numpy's matmul as a library step.

Sources (web pages on MTFM, the Meituan multi-scenario ranking model):
  [DY] "美团推荐大模型 MTFM 深度硬核解析" (dingyadong.top post)
  [MT] "MTFM：美团统一推荐基座大模型在外卖多业务场景的落地实践" (Meituan tech
       blog, dujian.net mirror) -- authoritative where the pages disagree.

Readings taken where the pages are silent or disagree (each is a parameter or
stated below):
  * T rows see ALL H tokens ([MT] §3.2 "H visible to every token"; [DY] §8.2
    table row T1/T2 shows T->H all ones), not only H earlier than the exposure.
  * H rows see only H ([DY] §8.2 table rows H1..H3).
  * R is causal by index, self included ([DY] §8.2 table, R1/R2 rows).
  * A target sees an R token only when ts_R < exposure (strict) ([MT] §3.2).
  * phi_2 = SiLU(alpha * s) summed over visible keys and divided by N_u, the
    user's total token count; alpha defaults to 1/sqrt(head_dim).
  * GQA: query head h reads KV group g = h // r, r = Hq / Hkv.
  * GLN: LayerNorm over the whole concatenated row A = A^(1)||...||A^(H) with
    per-token-type gamma/beta (types H, R, T), biased variance, eps = 1e-5.
  * V2 target scale-up: the 4 sub-tokens of one target see each other and the
    target's shared prefix; other targets stay invisible.

Parity pins for every function live in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import numpy as np

ROW_H, ROW_R, ROW_T = 0, 1, 2
GLN_EPS = 1e-5


# ----------------------------------------------------------------------------
# Jagged layout
# ----------------------------------------------------------------------------

def offsets(lengths) -> np.ndarray:
    """Exclusive prefix offsets [B+1] of per-user lengths (jagged row-major layout)."""
    lengths = np.asarray(lengths, dtype=np.int64)
    out = np.zeros(lengths.shape[0] + 1, dtype=np.int64)
    out[1:] = np.cumsum(lengths)
    return out


def row_types(L_H: int, L_R: int, L_T: int) -> np.ndarray:
    """Token type of every row of one user's sequence X0 = (H; R; T) ([DY] §4.2, X0 row concat)."""
    return np.concatenate([np.full(L_H, ROW_H), np.full(L_R, ROW_R), np.full(L_T, ROW_T)]).astype(np.int64)


# ----------------------------------------------------------------------------
# Dynamic mask ([MT] §3.2; [DY] §4.1.1 and §8.2)
# ----------------------------------------------------------------------------

def dense_mask(L_H: int, L_R: int, L_T: int, r_ts, t_exp, v2_subtokens: int = 1) -> np.ndarray:
    """Dense visibility matrix M[i, j] (query row i may read key j) of one user.

    Built cell by cell from the rules:
      key H  : visible to every query.
      key R_b: visible to query R_a iff b <= a (causal, self included);
               visible to query T_t iff ts(R_b) < exposure(T_t);
               invisible to H queries.
      key T_s: visible only to T_s itself (V1) or to the sub-tokens of the
               same target (V2, v2_subtokens = 4); invisible to H and R.
    """
    N = L_H + L_R + L_T
    typ = row_types(L_H, L_R, L_T)
    M = np.zeros((N, N), dtype=bool)
    for i in range(N):
        for j in range(N):
            ti, tj = typ[i], typ[j]
            if tj == ROW_H:
                vis = True
            elif tj == ROW_R:
                b = j - L_H
                if ti == ROW_R:
                    vis = b <= i - L_H
                elif ti == ROW_T:
                    vis = bool(r_ts[b] < t_exp[i - L_H - L_R])
                else:
                    vis = False
            else:  # key is a T token
                if ti == ROW_T:
                    a, s = i - L_H - L_R, j - L_H - L_R
                    vis = (a // v2_subtokens) == (s // v2_subtokens)
                else:
                    vis = False
            M[i, j] = vis
    return M


def dense_mask_fast(L_H: int, L_R: int, L_T: int, r_ts, t_exp, v2_subtokens: int = 1) -> np.ndarray:
    """Same matrix as ``dense_mask`` built block by block (for large users); pinned against it in tests."""
    N = L_H + L_R + L_T
    M = np.zeros((N, N), dtype=bool)
    M[:, :L_H] = True
    M[L_H:L_H + L_R, L_H:L_H + L_R] = np.tril(np.ones((L_R, L_R), dtype=bool))
    r_ts = np.asarray(r_ts)
    t_exp = np.asarray(t_exp)
    if L_T and L_R:
        M[L_H + L_R:, L_H:L_H + L_R] = r_ts[None, :] < t_exp[:, None]
    tid = np.arange(L_T) // v2_subtokens
    M[L_H + L_R:, L_H + L_R:] = tid[:, None] == tid[None, :]
    return M


# ----------------------------------------------------------------------------
# phi_2 = pointwise SiLU, normalised by length
# ----------------------------------------------------------------------------

def silu(x):
    """SiLU(x) = x / (1 + exp(-x))."""
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def sigmoid(x):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def default_alpha(dh: int) -> float:
    return 1.0 / np.sqrt(dh)


def attention_user(q, k, v, M, hq: int, hkv: int, dh: int, alpha: float, n_norm: int):
    """A^(h) = (1/n_norm) * (M o SiLU(alpha * Q^(h) K^(g)T)) V^(g), heads concatenated.

    [DY] §4.1 attention equation (phi_2 applied to the masked scores, then times
    V) and §4.2 for the T-row slice; GQA group g = h // (hq/hkv) ([DY] §4.1).
    The page writes the mask inside phi_2, phi_2(Q K^T o M); since SiLU(0) = 0
    that equals M o SiLU(alpha Q K^T), the form used here.
    q: [nq, hq*dh], k, v: [N, hkv*dh], M: [nq, N] bool.  Returns [nq, hq*dh].
    """
    r = hq // hkv
    A = np.zeros((q.shape[0], hq * dh), dtype=np.float64)
    Mf = M.astype(np.float64)
    for h in range(hq):
        g = h // r
        qh = q[:, h * dh:(h + 1) * dh]
        kg = k[:, g * dh:(g + 1) * dh]
        vg = v[:, g * dh:(g + 1) * dh]
        S = qh @ kg.T
        P = Mf * silu(alpha * S)
        A[:, h * dh:(h + 1) * dh] = (P @ vg) / n_norm
    return A


# ----------------------------------------------------------------------------
# GLN gate ([DY] §4.1 "gated layer norm and residual"; [MT] §6.1 GLN kernel:
# one [G, D] parameter matrix indexed by each token's group id)
# ----------------------------------------------------------------------------

def gln(A, types, gamma, beta, eps: float = GLN_EPS):
    """Group LayerNorm: per-row LayerNorm, affine parameters picked by the row's token type.

    Returns (G, mean, rstd).  gamma/beta are [3, D] (rows H, R, T).
    """
    mean = A.mean(axis=1)
    var = ((A - mean[:, None]) ** 2).mean(axis=1)
    rstd = 1.0 / np.sqrt(var + eps)
    z = (A - mean[:, None]) * rstd[:, None]
    G = z * gamma[types] + beta[types]
    return G, mean, rstd


def gate(A, U, types, gamma, beta, eps: float = GLN_EPS):
    """Y = GLN(A) o U ([DY] §4.1).  With gamma None the gate is Y = A o U (no norm)."""
    if gamma is None:
        return A * U, None, None
    G, mean, rstd = gln(A, types, gamma, beta, eps)
    return G * U, mean, rstd


# ----------------------------------------------------------------------------
# Layers over a jagged batch
# ----------------------------------------------------------------------------

def _f64(x):
    if x is None:
        return None
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def _users(batch):
    so = offsets(batch.N)
    ro = offsets(batch.L_R)
    to = offsets(batch.L_T)
    for u in range(batch.B):
        LH, LR, LT = int(batch.L_H[u]), int(batch.L_R[u]), int(batch.L_T[u])
        yield u, LH, LR, LT, int(so[u]), int(ro[u]), int(to[u])


def user_mask(batch, u, fast=True):
    ro = offsets(batch.L_R)
    to = offsets(batch.L_T)
    LH, LR, LT = int(batch.L_H[u]), int(batch.L_R[u]), int(batch.L_T[u])
    r_ts = batch.r_ts[ro[u]:ro[u + 1]]
    t_exp = batch.t_exp[to[u]:to[u + 1]]
    f = dense_mask_fast if fast else dense_mask
    return f(LH, LR, LT, r_ts, t_exp, batch.v2_subtokens)


def full_fwd(batch, heads, inp, alpha=None, eps: float = GLN_EPS, users=None):
    """Full-Attention layer forward ([DY] §4.1): every token is a query.

    Returns dict with A [sum N, D], Y [sum N, D], mean/rstd [sum N] (None when no GLN).
    ``users`` restricts the computation to a subset (rows of other users stay NaN).
    """
    hq, hkv, dh = heads.hq, heads.hkv, heads.dh
    alpha = default_alpha(dh) if alpha is None else alpha
    q, k, v, U = _f64(inp.q), _f64(inp.k), _f64(inp.v), _f64(inp.u)
    gamma, beta = _f64(inp.gamma), _f64(inp.beta)
    T = batch.total_tokens
    A = np.full((T, hq * dh), np.nan)
    Y = np.full((T, hq * dh), np.nan)
    mean = np.full(T, np.nan)
    rstd = np.full(T, np.nan)
    for u, LH, LR, LT, s0, _, _ in _users(batch):
        if users is not None and u not in users:
            continue
        N = LH + LR + LT
        if N == 0:
            continue
        M = user_mask(batch, u)
        sl = slice(s0, s0 + N)
        A[sl] = attention_user(q[sl], k[sl], v[sl], M, hq, hkv, dh, alpha, N)
        y, m, r = gate(A[sl], U[sl], row_types(LH, LR, LT), gamma, beta, eps)
        Y[sl] = y
        if m is not None:
            mean[sl], rstd[sl] = m, r
    return {"A": A, "Y": Y, "mean": mean, "rstd": rstd}


def target_fwd(batch, heads, inp, alpha=None, eps: float = GLN_EPS, users=None):
    """Target-Attention layer forward ([DY] §4.2): only T rows are queries.

    Q, U, A, Y are [sum L_T, D]; K, V cover every row of each user.  The mask
    is the T-row slice M[L_H+L_R:] of the Full-layer mask.
    """
    hq, hkv, dh = heads.hq, heads.hkv, heads.dh
    alpha = default_alpha(dh) if alpha is None else alpha
    q, k, v, U = _f64(inp.q), _f64(inp.k), _f64(inp.v), _f64(inp.u)
    gamma, beta = _f64(inp.gamma), _f64(inp.beta)
    R = batch.total_t
    A = np.full((R, hq * dh), np.nan)
    Y = np.full((R, hq * dh), np.nan)
    mean = np.full(R, np.nan)
    rstd = np.full(R, np.nan)
    for u, LH, LR, LT, s0, _, t0 in _users(batch):
        if users is not None and u not in users:
            continue
        N = LH + LR + LT
        if LT == 0:
            continue
        M = user_mask(batch, u)[LH + LR:]
        ks = slice(s0, s0 + N)
        ts = slice(t0, t0 + LT)
        A[ts] = attention_user(q[ts], k[ks], v[ks], M, hq, hkv, dh, alpha, N)
        y, m, r = gate(A[ts], U[ts], np.full(LT, ROW_T), gamma, beta, eps)
        Y[ts] = y
        if m is not None:
            mean[ts], rstd[ts] = m, r
    return {"A": A, "Y": Y, "mean": mean, "rstd": rstd}


# ----------------------------------------------------------------------------
# Backward (chain rule written out; pinned by finite differences in tests)
# ----------------------------------------------------------------------------

def gate_bwd(A, U, types, gamma, beta, dY, eps: float = GLN_EPS):
    """Gradients of Y = GLN(A) o U.  Returns (dA, dU, dgamma[3,D], dbeta[3,D])."""
    if gamma is None:
        return dY * U, dY * A, None, None
    D = A.shape[1]
    mean = A.mean(axis=1)
    var = ((A - mean[:, None]) ** 2).mean(axis=1)
    rstd = 1.0 / np.sqrt(var + eps)
    z = (A - mean[:, None]) * rstd[:, None]
    G = z * gamma[types] + beta[types]
    dU = dY * G
    dG = dY * U
    dgamma = np.zeros_like(gamma)
    dbeta = np.zeros_like(beta)
    for t in range(gamma.shape[0]):
        sel = types == t
        dgamma[t] = (dG[sel] * z[sel]).sum(axis=0)
        dbeta[t] = dG[sel].sum(axis=0)
    dz = dG * gamma[types]
    dA = rstd[:, None] * (dz - dz.mean(axis=1, keepdims=True) - z * (dz * z).mean(axis=1, keepdims=True))
    assert dA.shape[1] == D
    return dA, dU, dgamma, dbeta


def attention_user_bwd(q, k, v, M, dA, hq, hkv, dh, alpha, n_norm):
    """Gradients of ``attention_user`` w.r.t. q, k, v given dA.

    With x = alpha * q.k, sigma = 1/(1+e^-x): d SiLU(x)/dx = sigma (1 + x (1 - sigma)).
    """
    r = hq // hkv
    Mf = M.astype(np.float64)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for h in range(hq):
        g = h // r
        hs = slice(h * dh, (h + 1) * dh)
        gs = slice(g * dh, (g + 1) * dh)
        X = alpha * (q[:, hs] @ k[:, gs].T)
        sg = sigmoid(X)
        P = Mf * X * sg / n_norm
        dAh = dA[:, hs]
        dv[:, gs] += P.T @ dAh
        dP = dAh @ v[:, gs].T
        dX = dP * Mf * sg * (1.0 + X * (1.0 - sg)) / n_norm
        dS = alpha * dX
        dq[:, hs] = dS @ k[:, gs]
        dk[:, gs] += dS.T @ q[:, hs]
    return dq, dk, dv


def full_bwd(batch, heads, inp, alpha=None, eps: float = GLN_EPS, users=None):
    """Backward of the Full-Attention layer: dQ, dK, dV, dU [rows, D] and dgamma, dbeta [3, D]."""
    hq, hkv, dh = heads.hq, heads.hkv, heads.dh
    alpha = default_alpha(dh) if alpha is None else alpha
    q, k, v, U, dY = _f64(inp.q), _f64(inp.k), _f64(inp.v), _f64(inp.u), _f64(inp.dy)
    gamma, beta = _f64(inp.gamma), _f64(inp.beta)
    dq = np.full_like(q, np.nan)
    dk = np.full_like(k, np.nan)
    dv = np.full_like(v, np.nan)
    dU = np.full_like(U, np.nan)
    dgamma = None if gamma is None else np.zeros_like(gamma)
    dbeta = None if gamma is None else np.zeros_like(beta)
    for u, LH, LR, LT, s0, _, _ in _users(batch):
        if users is not None and u not in users:
            continue
        N = LH + LR + LT
        if N == 0:
            continue
        sl = slice(s0, s0 + N)
        M = user_mask(batch, u)
        A = attention_user(q[sl], k[sl], v[sl], M, hq, hkv, dh, alpha, N)
        dA, du, dg, db = gate_bwd(A, U[sl], row_types(LH, LR, LT), gamma, beta, dY[sl], eps)
        dU[sl] = du
        if dg is not None:
            dgamma += dg
            dbeta += db
        dq[sl], dk[sl], dv[sl] = attention_user_bwd(q[sl], k[sl], v[sl], M, dA, hq, hkv, dh, alpha, N)
    return {"dq": dq, "dk": dk, "dv": dv, "du": dU, "dgamma": dgamma, "dbeta": dbeta}


def target_bwd(batch, heads, inp, alpha=None, eps: float = GLN_EPS, users=None):
    """Backward of the Target-Attention layer: dQ, dU for T rows; dK, dV for all rows."""
    hq, hkv, dh = heads.hq, heads.hkv, heads.dh
    alpha = default_alpha(dh) if alpha is None else alpha
    q, k, v, U, dY = _f64(inp.q), _f64(inp.k), _f64(inp.v), _f64(inp.u), _f64(inp.dy)
    gamma, beta = _f64(inp.gamma), _f64(inp.beta)
    dq = np.full_like(q, np.nan)
    dk = np.full_like(k, np.nan)
    dv = np.full_like(v, np.nan)
    dU = np.full_like(U, np.nan)
    dgamma = None if gamma is None else np.zeros_like(gamma)
    dbeta = None if gamma is None else np.zeros_like(beta)
    for u, LH, LR, LT, s0, _, t0 in _users(batch):
        if users is not None and u not in users:
            continue
        N = LH + LR + LT
        ks = slice(s0, s0 + N)
        ts = slice(t0, t0 + LT)
        if LT == 0:
            dk[ks] = 0.0
            dv[ks] = 0.0
            continue
        M = user_mask(batch, u)[LH + LR:]
        A = attention_user(q[ts], k[ks], v[ks], M, hq, hkv, dh, alpha, N)
        dA, du, dg, db = gate_bwd(A, U[ts], np.full(LT, ROW_T), gamma, beta, dY[ts], eps)
        dU[ts] = du
        if dg is not None:
            dgamma += dg
            dbeta += db
        dq[ts], dk[ks], dv[ks] = attention_user_bwd(q[ts], k[ks], v[ks], M, dA, hq, hkv, dh, alpha, N)
    return {"dq": dq, "dk": dk, "dv": dv, "du": dU, "dgamma": dgamma, "dbeta": dbeta}


# ----------------------------------------------------------------------------
# Backbone stack: layers of the form of [DY] §4.1 (Full) and §4.2 (Target),
# interleaved 1 Full : 3 Target ([DY] §4.1 block structure; [MT] §3.3).
# ----------------------------------------------------------------------------

RMS_EPS = 1e-6


def rmsnorm(X, w, eps: float = RMS_EPS):
    """Pre-norm X~ = X / sqrt(mean_j X_ij^2 + eps) * w, row by row.

    [DY] §4.2 projects a normalised X~ but does not say which norm; RMSNorm
    with eps = 1e-6 is the reading taken here.
    """
    X = np.asarray(X, dtype=np.float64)
    ms = (X * X).mean(axis=1, keepdims=True)
    return X / np.sqrt(ms + eps) * np.asarray(w, dtype=np.float64)


def t_row_index(batch) -> np.ndarray:
    """Global row of every T token, in the Target layout order (user by user)."""
    out = []
    for u, LH, LR, LT, s0, _, _ in _users(batch):
        out.append(np.arange(s0 + LH + LR, s0 + LH + LR + LT))
    return np.concatenate(out) if out else np.zeros(0, np.int64)


class _Proj:
    """Attention inputs handed to full_fwd / target_fwd (float64 arrays)."""

    def __init__(self, q, k, v, u, gamma, beta):
        self.q, self.k, self.v, self.u, self.gamma, self.beta = q, k, v, u, gamma, beta


def full_layer(batch, heads, X, lw, alpha=None):
    """X' = f2(GLN(A) o U) + X with U, Q, K, V = Split(SiLU(f1(RMSNorm(X)))) ([DY] §4.1).

    f1 = X~ W_in^T, W_in = [W_u; W_q; W_k; W_v] (heads contiguous inside each
    part); phi_1 = SiLU; f2 = Y W_o^T; no biases.  X: [sum N, d_model] float64.
    """
    dq, dkv = heads.dq, heads.dkv
    Xn = rmsnorm(X, lw.rms_w)
    Z = silu(Xn @ _f64(lw.w_in).T)
    U, Q, K, V = Z[:, :dq], Z[:, dq:2 * dq], Z[:, 2 * dq:2 * dq + dkv], Z[:, 2 * dq + dkv:]
    out = full_fwd(batch, heads, _Proj(Q, K, V, U, _f64(lw.gamma), _f64(lw.beta)), alpha)
    return X + out["Y"] @ _f64(lw.w_o).T


def target_layer(batch, heads, X, lw, alpha=None):
    """Target-Attention layer ([DY] §4.2): U_T, Q_T = Split(SiLU(X~_T W_uq^T)),
    K, V = Split(SiLU(X~ W_kv^T)); only T rows are updated,
    X'_T = f2(GLN(A_T) o U_T) + X_T, and the H / R rows pass through unchanged."""
    dq, dkv = heads.dq, heads.dkv
    Xn = rmsnorm(X, lw.rms_w)
    trow = t_row_index(batch)
    ZT = silu(Xn[trow] @ _f64(lw.w_in).T)
    Zkv = silu(Xn @ _f64(lw.w_kv).T)
    inp = _Proj(ZT[:, dq:], Zkv[:, :dkv], Zkv[:, dkv:], ZT[:, :dq], _f64(lw.gamma), _f64(lw.beta))
    out = target_fwd(batch, heads, inp, alpha)
    Xo = np.array(X, dtype=np.float64, copy=True)
    Xo[trow] = Xo[trow] + out["Y"] @ _f64(lw.w_o).T
    return Xo


def stack_fwd(batch, heads, weights, X0, alpha=None, record: bool = False):
    """Run the layers in order (kind "F" = Full, "T" = Target).  Returns X_L, or
    the list [X_0, ..., X_L] when ``record``."""
    X = _f64(X0)
    xs = [X]
    for lw in weights:
        X = (full_layer if lw.kind == "F" else target_layer)(batch, heads, X, lw, alpha)
        xs.append(X)
    return xs if record else X


# ----------------------------------------------------------------------------
# V2 Target Scale-Up layer (Meituan tech blog §3.3.2, items 2-4): every target is
# 4 sub-tokens; in a Target-Attention layer each sub-token position has its own
# query-side projection and its own SwiGLU FFN, and the sub-tokens of a target are
# crossed by a zero-parameter token mixing.
# ----------------------------------------------------------------------------

V2_SUB = 4


def v2_sub_index(batch) -> np.ndarray:
    """Sub-token position (0..3) of every T row, in the Target layout order: the
    position of the row among its user's T rows, modulo 4 (each target is 4
    consecutive T rows, item 1 of §3.3.2)."""
    out = []
    for u, LH, LR, LT, s0, _, _ in _users(batch):
        out.append(np.arange(LT) % V2_SUB)
    return np.concatenate(out) if out else np.zeros(0, np.int64)


def mix_tokens(Xt, n_sub: int = V2_SUB):
    """Zero-parameter token mixing of the sub-tokens of each target (§3.3.2 item 4,
    the mixing of RankMixer): every sub-token vector is cut into n_sub equal parts,
    and new sub-token h is the concatenation of part h of sub-tokens 0, 1, ...,
    n_sub - 1 of the same target.  Xt: [n_targets * n_sub, d], targets consecutive."""
    Xt = np.asarray(Xt, dtype=np.float64)
    n, d = Xt.shape
    assert n % n_sub == 0 and d % n_sub == 0
    parts = Xt.reshape(n // n_sub, n_sub, n_sub, d // n_sub)   # [target, sub-token j, part h, :]
    return parts.transpose(0, 2, 1, 3).reshape(n, d)           # [target, new sub-token h, j, :]


def swiglu(X, w_gate, w_up, w_down):
    """SwiGLU feed-forward network: (SiLU(X W_gate^T) * (X W_up^T)) W_down^T."""
    return (silu(X @ w_gate.T) * (X @ w_up.T)) @ w_down.T


def v2_target_layer(batch, heads, X, lw, alpha=None):
    """Target-Attention layer of the V2 Target Scale-Up (§3.3.2), on a batch whose
    targets are 4 sub-tokens (v2_subtokens = 4).  Readings taken where the page is
    brief: the attention block is the V1 Target layer (§4.2 of the dingyadong.top
    page) except that sub-token position s projects its [U Q] with its own matrix
    w_uq[s] (item 2: "different Q projection"; U comes from the same query-side
    projection); K, V come from the shared w_kv over all rows; the output
    projection w_o is shared.  Then the 4 sub-tokens of each target are mixed
    (item 4), and each sub-token position s applies its own pre-normed SwiGLU FFN
    with a residual (item 2):
        X_T <- X_T + f2(GLN(A_T) (*) U_T)              (attention, per-s U, Q)
        X_T <- Mix(X_T)                                (per target)
        X_T <- X_T + SwiGLU_s(RMSNorm(X_T) * rms_w2)   (per sub-token position s)
    H / R rows pass through unchanged.  lw: syn.V2LayerWeights."""
    assert batch.v2_subtokens == V2_SUB
    dq, dkv = heads.dq, heads.dkv
    Xn = rmsnorm(X, lw.rms_w)
    trow = t_row_index(batch)
    sub = v2_sub_index(batch)
    ZT = np.zeros((len(trow), 2 * dq))
    for s in range(V2_SUB):
        sel = sub == s
        ZT[sel] = silu(Xn[trow[sel]] @ _f64(lw.w_uq[s]).T)
    Zkv = silu(Xn @ _f64(lw.w_kv).T)
    inp = _Proj(ZT[:, dq:], Zkv[:, :dkv], Zkv[:, dkv:], ZT[:, :dq], _f64(lw.gamma), _f64(lw.beta))
    out = target_fwd(batch, heads, inp, alpha)
    XT = _f64(X)[trow] + out["Y"] @ _f64(lw.w_o).T
    XT = mix_tokens(XT)
    Xn2 = rmsnorm(XT, lw.rms_w2)
    F = np.zeros_like(XT)
    for s in range(V2_SUB):
        sel = sub == s
        F[sel] = swiglu(Xn2[sel], _f64(lw.w_gate[s]), _f64(lw.w_up[s]), _f64(lw.w_down[s]))
    Xo = np.array(X, dtype=np.float64, copy=True)
    Xo[trow] = XT + F
    return Xo
