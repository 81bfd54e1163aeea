"""Checks that pin the oracle's V2 Target Scale-Up layer (Meituan tech blog §3.3.2,
items 2-4: per-sub-token query-side projections and SwiGLU FFNs, zero-parameter
mixing of a target's 4 sub-tokens) to facts fixed outside the oracle itself:
  * the mixing written out index by index in scalar loops, and its algebra (a
    permutation of the entries, its own inverse when the parts are as many as the
    sub-tokens, linear);
  * SwiGLU in scalar loops, and its zero case;
  * the whole layer in scalar loops on a tiny batch (an independent loop nest);
  * structural facts: H / R rows pass through bit-identical; targets do not reach
    each other; with equal per-sub-token projections and a zero FFN the layer is
    the mixing of the V1 Target layer's T rows (the V1 layer is pinned itself).
``test_oracle_v2.py`` runs them; ``test_oracle_mutations.py`` plants mistakes.
"""
from __future__ import annotations

import math

import numpy as np

import mtfm_synth as syn
from oracle import mtfm_oracle as O

HEADS = syn.Heads(2, 1, 8)   # dq 16, dkv 8
D, DFF = 16, 8


def _batch(seed=61):
    # two users; targets of 4 sub-tokens (L_T multiple of 4), exposures shared per target
    return syn.fixed_batch([5, 3], [3, 4], [8, 4], seed, v2_subtokens=4)


def _w(x):
    return syn.bf16_bits_to_f32(x).astype(np.float64) if x.dtype == np.uint16 else np.asarray(x, np.float64)


def _weights(seed=7, std=0.3):
    return syn.v2_layer_weights(HEADS, D, DFF, seed, std=std, std_o=std, std_ffn=std)


def _x0(batch, seed=8):
    return syn.bf16_bits_to_f32(syn.stack_input(batch, D, seed)).astype(np.float64)


# ----------------------------------------------------------------------------- mixing

def check_mix_index_formula():
    """New sub-token h, columns [j d/4, (j+1) d/4) = part h of old sub-token j."""
    g = np.random.default_rng(3)
    X = g.standard_normal((8, 12))   # 2 targets x 4 sub-tokens, d = 12 (parts of 3)
    got = O.mix_tokens(X)
    q = 3
    for tgt in range(2):
        for h in range(4):
            for j in range(4):
                for c in range(q):
                    assert got[4 * tgt + h, j * q + c] == X[4 * tgt + j, h * q + c]


def check_mix_algebra():
    g = np.random.default_rng(4)
    X, Y = g.standard_normal((12, 8)), g.standard_normal((12, 8))
    M = O.mix_tokens(X)
    assert np.array_equal(np.sort(M.ravel()), np.sort(X.ravel()))          # a permutation
    assert np.array_equal(O.mix_tokens(M), X)                               # its own inverse
    assert np.allclose(O.mix_tokens(2.0 * X - 3.0 * Y), 2.0 * M - 3.0 * O.mix_tokens(Y), rtol=0, atol=1e-13)
    assert not np.array_equal(M, X)


# ----------------------------------------------------------------------------- SwiGLU

def check_swiglu_loops():
    g = np.random.default_rng(5)
    X = g.standard_normal((3, 5))
    wg, wu, wd = g.standard_normal((4, 5)), g.standard_normal((4, 5)), g.standard_normal((5, 4))
    got = O.swiglu(X, wg, wu, wd)
    for i in range(3):
        h = []
        for k in range(4):
            a = sum(X[i, j] * wg[k, j] for j in range(5))
            b = sum(X[i, j] * wu[k, j] for j in range(5))
            h.append(a / (1.0 + math.exp(-a)) * b)
        for o in range(5):
            assert abs(got[i, o] - sum(h[k] * wd[o, k] for k in range(4))) < 1e-12
    assert np.array_equal(O.swiglu(X, wg, np.zeros_like(wu), wd), np.zeros((3, 5)))


# ----------------------------------------------------------------------------- layer

def _brute_v2(batch, heads, X, lw):
    """The V2 Target layer with scalar loops (RMSNorm, per-sub-token [U Q], shared
    K / V, masked SiLU attention, GLN gate, output projection, residual, mixing,
    per-sub-token pre-normed SwiGLU with residual)."""
    d = X.shape[1]
    hq, hkv, dh = heads.hq, heads.hkv, heads.dh
    dq, dkv, r = hq * dh, hkv * dh, hq // hkv
    alpha = 1.0 / math.sqrt(dh)
    w_uq = [_w(x) for x in lw.w_uq]
    w_kv, w_o = _w(lw.w_kv), _w(lw.w_o)
    rms_w, rms_w2, gamma, beta = _w(lw.rms_w), _w(lw.rms_w2), _w(lw.gamma), _w(lw.beta)
    wg, wu, wd = [_w(x) for x in lw.w_gate], [_w(x) for x in lw.w_up], [_w(x) for x in lw.w_down]
    dff = wg[0].shape[0]

    def silu(z):
        return z / (1.0 + math.exp(-z))

    def norm(v, w):
        ms = sum(x * x for x in v) / len(v)
        inv = 1.0 / math.sqrt(ms + 1e-6)
        return [v[j] * inv * w[j] for j in range(len(v))]

    out = np.array(X, dtype=np.float64, copy=True)
    so, ro, to = O.offsets(batch.N), O.offsets(batch.L_R), O.offsets(batch.L_T)
    for u in range(batch.B):
        LH, LR, LT = int(batch.L_H[u]), int(batch.L_R[u]), int(batch.L_T[u])
        N, s0 = LH + LR + LT, int(so[u])
        M = O.dense_mask(LH, LR, LT, batch.r_ts[ro[u]:ro[u + 1]], batch.t_exp[to[u]:to[u + 1]], 4)
        xn = [norm(list(X[s0 + j]), rms_w) for j in range(N)]
        K = [[silu(sum(xn[j][c] * w_kv[o, c] for c in range(d))) for o in range(dkv)] for j in range(N)]
        V = [[silu(sum(xn[j][c] * w_kv[dkv + o, c] for c in range(d))) for o in range(dkv)] for j in range(N)]
        xt = []
        for t in range(LT):
            i = LH + LR + t
            W = w_uq[t % 4]
            Ui = [silu(sum(xn[i][c] * W[o, c] for c in range(d))) for o in range(dq)]
            Qi = [silu(sum(xn[i][c] * W[dq + o, c] for c in range(d))) for o in range(dq)]
            A = [0.0] * dq
            for h in range(hq):
                g = h // r
                for j in range(N):
                    if M[i, j]:
                        p = silu(alpha * sum(Qi[h * dh + c] * K[j][g * dh + c] for c in range(dh))) / N
                        for c in range(dh):
                            A[h * dh + c] += p * V[j][g * dh + c]
            mean = sum(A) / dq
            rstd = 1.0 / math.sqrt(sum((a - mean) ** 2 for a in A) / dq + 1e-5)
            Y = [((A[c] - mean) * rstd * gamma[2, c] + beta[2, c]) * Ui[c] for c in range(dq)]
            xt.append([X[s0 + i, o] + sum(Y[c] * w_o[o, c] for c in range(dq)) for o in range(d)])
        q = d // 4
        for tg in range(LT // 4):
            mixed = [[xt[4 * tg + j][h * q + c] for j in range(4) for c in range(q)] for h in range(4)]
            for h in range(4):
                x = mixed[h]
                xn2 = norm(x, rms_w2)
                hid = []
                for k in range(dff):
                    a = sum(xn2[c] * wg[h][k, c] for c in range(d))
                    b = sum(xn2[c] * wu[h][k, c] for c in range(d))
                    hid.append(silu(a) * b)
                row = s0 + LH + LR + 4 * tg + h
                for o in range(d):
                    out[row, o] = x[o] + sum(hid[k] * wd[h][o, k] for k in range(dff))
    return out


def check_v2_layer_brute_force():
    b, lw = _batch(), _weights()
    X0 = _x0(b)
    got = O.v2_target_layer(b, HEADS, X0, lw)
    ref = _brute_v2(b, HEADS, X0, lw)
    assert np.allclose(got, ref, rtol=1e-10, atol=1e-11), np.abs(got - ref).max()


def check_v2_hr_rows_untouched():
    b, lw = _batch(), _weights()
    X0 = _x0(b)
    got = O.v2_target_layer(b, HEADS, X0, lw)
    hr = np.setdiff1d(np.arange(b.total_tokens), O.t_row_index(b))
    assert np.array_equal(got[hr], X0[hr])
    assert not np.allclose(got[O.t_row_index(b)], X0[O.t_row_index(b)])


def check_v2_targets_independent():
    """Changing the rows of one target changes only that target's rows."""
    b, lw = _batch(), _weights()
    X0 = _x0(b)
    base = O.v2_target_layer(b, HEADS, X0, lw)
    trow = O.t_row_index(b)
    X1 = X0.copy()
    X1[trow[4:8]] += 0.5           # the second target of user 0
    got = O.v2_target_layer(b, HEADS, X1, lw)
    others = np.setdiff1d(np.arange(b.total_tokens), trow[4:8])
    assert np.array_equal(got[others], base[others])
    assert not np.allclose(got[trow[4:8]], base[trow[4:8]])


def check_v2_reduces_to_mixed_v1():
    """Equal per-sub-token projections and a zero FFN: the V1 Target layer's T rows, mixed."""
    b, lw = _batch(), _weights()
    lw.w_uq = [lw.w_uq[0]] * 4
    lw.w_down = [np.zeros_like(x) for x in lw.w_down]
    X0 = _x0(b)
    got = O.v2_target_layer(b, HEADS, X0, lw)
    v1w = syn.LayerWeights("T", lw.rms_w, lw.w_uq[0], lw.w_kv, lw.w_o, lw.gamma, lw.beta)
    v1 = O.target_layer(b, HEADS, X0, v1w)
    trow = O.t_row_index(b)
    assert np.allclose(got[trow], O.mix_tokens(v1[trow]), rtol=1e-12, atol=1e-13)


V2_CHECKS = [
    check_mix_index_formula,
    check_mix_algebra,
    check_swiglu_loops,
    check_v2_layer_brute_force,
    check_v2_hr_rows_untouched,
    check_v2_targets_independent,
    check_v2_reduces_to_mixed_v1,
]
