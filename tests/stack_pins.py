"""Checks that pin the oracle's backbone stack (RMSNorm pre-norm, UQKV / UQ / KV
projections with SiLU, gate, output projection, residual; Full and Target layers
interleaved) to facts fixed outside the oracle itself:
  * library routines for the special cases they cover (torch's rms_norm),
  * closed forms (a constant row under RMSNorm),
  * scalar-loop brute force of a Full and a Target layer on tiny inputs,
  * structural facts of the layer equations on the pages ("美团推荐大模型 MTFM
    深度硬核解析" §4.1 and §4.2): a zero output projection or a zero U part
    leaves X unchanged; a Target layer passes the H / R rows through; T tokens
    never reach H / R rows or each other (V1); users are independent.
``test_oracle_stack.py`` runs them; ``test_oracle_mutations.py`` plants mistakes.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import mtfm_synth as syn
from oracle import mtfm_oracle as O

GQA_HEADS = syn.Heads(2, 1, 8)      # d_model 16, dq 16, dkv 8: r = 2
SQUARE_HEADS = syn.Heads(1, 1, 16)  # d_model == dq: a transposed W_o is visible
D_SMALL = 16


def _batch(seed=41):
    return syn.fixed_batch([5, 3], [4, 6], [3, 4], seed)


def _weights(heads, d, seed, kinds, std=0.3, std_o=0.3):
    return syn.stack_weights(heads, d, seed, kinds, std=std, std_o=std_o, random_norms=True)


def _x0(batch, d, seed):
    return syn.bf16_bits_to_f32(syn.stack_input(batch, d, seed)).astype(np.float64)


def _w(x):
    return syn.bf16_bits_to_f32(x).astype(np.float64) if x.dtype == np.uint16 else np.asarray(x, np.float64)


# ----------------------------------------------------------------------------- RMSNorm

def check_rmsnorm_library():
    g = np.random.default_rng(5)
    x = 3.0 * g.standard_normal((50, 37))
    w = g.standard_normal(37)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (37,), torch.from_numpy(w), eps=O.RMS_EPS)
    assert np.allclose(O.rmsnorm(x, w), ref.numpy(), rtol=1e-12, atol=1e-13)


def check_rmsnorm_constant_row():
    for c in (-3.0, 0.5, 1e-2):
        x = np.full((1, 24), c)
        got = O.rmsnorm(x, np.ones(24))
        assert np.allclose(got, c / math.sqrt(c * c + O.RMS_EPS), rtol=1e-14, atol=0)


# ----------------------------------------------------------------------------- brute force

def _brute_layer(batch, heads, X, lw):
    """One layer with scalar loops: row-wise RMSNorm, per-output dot products,
    SiLU, visible-key sums, GLN, gate, output projection, residual."""
    d = X.shape[1]
    hq, hkv, dh = heads.hq, heads.hkv, heads.dh
    dq, dkv, r = hq * dh, hkv * dh, hq // hkv
    alpha = 1.0 / math.sqrt(dh)
    w_in, w_o = _w(lw.w_in), _w(lw.w_o)
    w_kv = _w(lw.w_kv) if lw.w_kv is not None else None
    rms_w, gamma, beta = _w(lw.rms_w), _w(lw.gamma), _w(lw.beta)

    def silu(z):
        return z / (1.0 + math.exp(-z))

    def norm_row(i):
        ms = sum(X[i, j] * X[i, j] for j in range(d)) / d
        inv = 1.0 / math.sqrt(ms + 1e-6)
        return [X[i, j] * inv * rms_w[j] for j in range(d)]

    def proj(xn, W, o):
        return silu(sum(xn[j] * W[o, j] for j in range(d)))

    out = np.array(X, dtype=np.float64, copy=True)
    so = O.offsets(batch.N)
    ro = O.offsets(batch.L_R)
    to = O.offsets(batch.L_T)
    for u in range(batch.B):
        LH, LR, LT = int(batch.L_H[u]), int(batch.L_R[u]), int(batch.L_T[u])
        N = LH + LR + LT
        s0 = int(so[u])
        M = O.dense_mask(LH, LR, LT, batch.r_ts[ro[u]:ro[u + 1]], batch.t_exp[to[u]:to[u + 1]],
                         batch.v2_subtokens)
        xn = [norm_row(s0 + j) for j in range(N)]
        if lw.kind == "F":
            K = [[proj(xn[j], w_in, 2 * dq + c) for c in range(dkv)] for j in range(N)]
            V = [[proj(xn[j], w_in, 2 * dq + dkv + c) for c in range(dkv)] for j in range(N)]
            queries = range(N)
        else:
            K = [[proj(xn[j], w_kv, c) for c in range(dkv)] for j in range(N)]
            V = [[proj(xn[j], w_kv, dkv + c) for c in range(dkv)] for j in range(N)]
            queries = range(LH + LR, N)
        for i in queries:
            Ui = [proj(xn[i], w_in, c) for c in range(dq)]
            Qi = [proj(xn[i], w_in, dq + c) for c in range(dq)]
            A = [0.0] * dq
            for h in range(hq):
                g = h // r
                for j in range(N):
                    if not M[i, j]:
                        continue
                    s = sum(Qi[h * dh + c] * K[j][g * dh + c] for c in range(dh))
                    p = silu(alpha * s) / N
                    for c in range(dh):
                        A[h * dh + c] += p * V[j][g * dh + c]
            mean = sum(A) / dq
            var = sum((a - mean) ** 2 for a in A) / dq
            rstd = 1.0 / math.sqrt(var + 1e-5)
            t = 2 if (lw.kind == "T" or i >= LH + LR) else (0 if i < LH else 1)
            Y = [((A[c] - mean) * rstd * gamma[t, c] + beta[t, c]) * Ui[c] for c in range(dq)]
            for m in range(d):
                out[s0 + i, m] = X[s0 + i, m] + sum(Y[c] * w_o[m, c] for c in range(dq))
    return out


def check_stack_layers_bruteforce():
    b = _batch()
    for heads in (GQA_HEADS, SQUARE_HEADS):
        ws = _weights(heads, D_SMALL, 7, ("F", "T"))
        X = _x0(b, D_SMALL, 7)
        for lw in ws:
            want = _brute_layer(b, heads, X, lw)
            got = (O.full_layer if lw.kind == "F" else O.target_layer)(b, heads, X, lw)
            assert np.allclose(got, want, rtol=1e-10, atol=1e-12), lw.kind
            X = want


# ----------------------------------------------------------------------------- structure

def check_stack_zero_out_proj_is_identity():
    b = _batch()
    ws = _weights(GQA_HEADS, D_SMALL, 8, syn.STACK_KINDS)
    for lw in ws:
        lw.w_o = np.zeros_like(lw.w_o)
    X0 = _x0(b, D_SMALL, 8)
    assert np.array_equal(O.stack_fwd(b, GQA_HEADS, ws, X0), X0)


def check_stack_zero_u_is_identity():
    """U = SiLU(0) = 0 when its projection rows are zero, so the gate closes."""
    b = _batch()
    ws = _weights(GQA_HEADS, D_SMALL, 9, syn.STACK_KINDS)
    dq = GQA_HEADS.dq
    for lw in ws:
        lw.w_in = lw.w_in.copy()
        lw.w_in[:dq] = 0
    X0 = _x0(b, D_SMALL, 9)
    assert np.array_equal(O.stack_fwd(b, GQA_HEADS, ws, X0), X0)


def check_target_layer_shortcut_and_kinds():
    """Target layers leave H / R rows bit-identical; Full layers update them."""
    b = _batch()
    ws = _weights(GQA_HEADS, D_SMALL, 10, syn.STACK_KINDS)
    xs = O.stack_fwd(b, GQA_HEADS, ws, _x0(b, D_SMALL, 10), record=True)
    trow = O.t_row_index(b)
    hr = np.setdiff1d(np.arange(b.total_tokens), trow)
    types = np.concatenate([O.row_types(int(b.L_H[u]), int(b.L_R[u]), int(b.L_T[u])) for u in range(b.B)])
    assert len(trow) == b.total_t and np.all(types[trow] == O.ROW_T)
    for l, lw in enumerate(ws):
        same_hr = np.array_equal(xs[l + 1][hr], xs[l][hr])
        assert same_hr == (lw.kind == "T"), (l, lw.kind)
        assert not np.array_equal(xs[l + 1][trow], xs[l][trow])


def check_stack_locality():
    """Through all 16 layers: T inputs never reach H / R rows, and (V1) one T
    token never reaches another."""
    b = _batch()
    ws = _weights(GQA_HEADS, D_SMALL, 11, syn.STACK_KINDS)
    X0 = _x0(b, D_SMALL, 11)
    base = O.stack_fwd(b, GQA_HEADS, ws, X0)
    trow = O.t_row_index(b)
    hr = np.setdiff1d(np.arange(b.total_tokens), trow)
    X1 = X0.copy()
    X1[trow] += 0.5
    out = O.stack_fwd(b, GQA_HEADS, ws, X1)
    assert np.array_equal(out[hr], base[hr])
    assert not np.array_equal(out[trow], base[trow])
    X2 = X0.copy()
    X2[trow[1]] *= -1.0
    out = O.stack_fwd(b, GQA_HEADS, ws, X2)
    others = np.setdiff1d(np.arange(b.total_tokens), [trow[1]])
    assert np.array_equal(out[others], base[others])


def _subset(batch, users):
    ro, to = O.offsets(batch.L_R), O.offsets(batch.L_T)
    idx = np.asarray(users)
    return syn.JaggedBatch(batch.L_H[idx], batch.L_R[idx], batch.L_T[idx],
                           np.concatenate([batch.r_ts[ro[u]:ro[u + 1]] for u in users]),
                           np.concatenate([batch.t_exp[to[u]:to[u + 1]] for u in users]),
                           np.zeros(int(batch.L_T[idx].sum()), np.int32), batch.v2_subtokens)


def _rows(batch, users):
    so = O.offsets(batch.N)
    return np.concatenate([np.arange(so[u], so[u + 1]) for u in users])


def check_stack_users_independent_and_permutable():
    b = syn.fixed_batch([5, 3, 6], [4, 6, 2], [3, 4, 2], 43)
    ws = _weights(GQA_HEADS, D_SMALL, 12, syn.STACK_KINDS)
    X0 = _x0(b, D_SMALL, 12)
    base = O.stack_fwd(b, GQA_HEADS, ws, X0)
    for users in ([2, 0, 1], [1]):
        sub = _subset(b, users)
        rows = _rows(b, users)
        out = O.stack_fwd(sub, GQA_HEADS, ws, X0[rows])
        assert np.allclose(out, base[rows], rtol=1e-12, atol=1e-14), users


STACK_CHECKS = [
    check_rmsnorm_library,
    check_rmsnorm_constant_row,
    check_stack_layers_bruteforce,
    check_stack_zero_out_proj_is_identity,
    check_stack_zero_u_is_identity,
    check_target_layer_shortcut_and_kinds,
    check_stack_locality,
    check_stack_users_independent_and_permutable,
]
