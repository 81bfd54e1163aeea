"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch each one.

A pin set that lets a dropped term, a wrong sign or index or a transposed operand
through is not a pin; every mutation below must make at least one check fail.
"""
import numpy as np
import pytest

import oracle_pins as P
import stack_pins as S
import v2_pins as V
from oracle import mtfm_oracle as O


def _mask_no_self_t(L_H, L_R, L_T, r_ts, t_exp, v2_subtokens=1):
    M = O.dense_mask_fast.__wrapped__(L_H, L_R, L_T, r_ts, t_exp, v2_subtokens)
    n = L_H + L_R
    M[n:, n:] = False
    return M


def _mask_fast_ties_visible(L_H, L_R, L_T, r_ts, t_exp, v2_subtokens=1):
    M = O.dense_mask_fast.__wrapped__(L_H, L_R, L_T, r_ts, t_exp, v2_subtokens)
    if L_T and L_R:
        M[L_H + L_R:, L_H:L_H + L_R] = np.asarray(r_ts)[None, :] <= np.asarray(t_exp)[:, None]
    return M


def _mask_cell_strict_causal(L_H, L_R, L_T, r_ts, t_exp, v2_subtokens=1):
    M = O.dense_mask.__wrapped__(L_H, L_R, L_T, r_ts, t_exp, v2_subtokens)
    for a in range(L_R):
        M[L_H + a, L_H + a] = False
    return M


def _mask_cell_t_sees_later_h_only(L_H, L_R, L_T, r_ts, t_exp, v2_subtokens=1):
    M = O.dense_mask.__wrapped__(L_H, L_R, L_T, r_ts, t_exp, v2_subtokens)
    M[:L_H, L_H:L_H + L_R] = True          # H rows wrongly see R
    return M


def _attn_norm_by_count(q, k, v, M, hq, hkv, dh, alpha, n_norm):
    r = hq // hkv
    A = np.zeros((q.shape[0], hq * dh))
    cnt = np.maximum(M.sum(axis=1, keepdims=True), 1)
    for h in range(hq):
        g = h // r
        S = q[:, h * dh:(h + 1) * dh] @ k[:, g * dh:(g + 1) * dh].T
        A[:, h * dh:(h + 1) * dh] = (M * O.silu(alpha * S)) @ v[:, g * dh:(g + 1) * dh] / cnt
    return A


def _attn_gqa_modulo(q, k, v, M, hq, hkv, dh, alpha, n_norm):
    A = np.zeros((q.shape[0], hq * dh))
    for h in range(hq):
        g = h % hkv
        S = q[:, h * dh:(h + 1) * dh] @ k[:, g * dh:(g + 1) * dh].T
        A[:, h * dh:(h + 1) * dh] = (M * O.silu(alpha * S)) @ v[:, g * dh:(g + 1) * dh] / n_norm
    return A


def _attn_no_alpha(q, k, v, M, hq, hkv, dh, alpha, n_norm):
    return O.attention_user.__wrapped__(q, k, v, M, hq, hkv, dh, 1.0, n_norm)


def _gln_unbiased(A, types, gamma, beta, eps=O.GLN_EPS):
    mean = A.mean(axis=1)
    var = A.var(axis=1, ddof=1)
    rstd = 1.0 / np.sqrt(var + eps)
    z = (A - mean[:, None]) * rstd[:, None]
    return z * gamma[types] + beta[types], mean, rstd


def _gln_first_group(A, types, gamma, beta, eps=O.GLN_EPS):
    return O.gln.__wrapped__(A, np.zeros_like(types), gamma, beta, eps)


def _bwd_sign(q, k, v, M, dA, hq, hkv, dh, alpha, n_norm):
    r = hq // hkv
    dq = np.zeros_like(q); dk = np.zeros_like(k); dv = np.zeros_like(v)
    for h in range(hq):
        g = h // r
        hs = slice(h * dh, (h + 1) * dh); gs = slice(g * dh, (g + 1) * dh)
        X = alpha * (q[:, hs] @ k[:, gs].T)
        sg = O.sigmoid(X)
        P_ = M * X * sg / n_norm
        dv[:, gs] += P_.T @ dA[:, hs]
        dP = dA[:, hs] @ v[:, gs].T
        dX = dP * M * sg * (1.0 - X * (1.0 - sg)) / n_norm        # wrong sign
        dq[:, hs] = alpha * dX @ k[:, gs]
        dk[:, gs] += alpha * dX.T @ q[:, hs]
    return dq, dk, dv


def _bwd_dk_transposed(q, k, v, M, dA, hq, hkv, dh, alpha, n_norm):
    dq, dk, dv = O.attention_user_bwd.__wrapped__(q, k, v, M, dA, hq, hkv, dh, alpha, n_norm)
    return dq, dk[::-1].copy(), dv


def _gate_bwd_no_mean_term(A, U, types, gamma, beta, dY, eps=O.GLN_EPS):
    dA, dU, dg, db = O.gate_bwd.__wrapped__(A, U, types, gamma, beta, dY, eps)
    if gamma is None:
        return dA, dU, dg, db
    mean = A.mean(axis=1)
    var = ((A - mean[:, None]) ** 2).mean(axis=1)
    rstd = 1.0 / np.sqrt(var + eps)
    dz = dY * U * gamma[types]
    return rstd[:, None] * dz, dU, dg, db


def _rms_no_sqrt(X, w, eps=O.RMS_EPS):
    X = np.asarray(X, dtype=np.float64)
    return X / ((X * X).mean(axis=1, keepdims=True) + eps) * w


def _rms_no_weight(X, w, eps=O.RMS_EPS):
    return O.rmsnorm.__wrapped__(X, np.ones_like(np.asarray(w, dtype=np.float64)), eps)


def _full_layer_variant(phi1=True, split_q_first=False, residual=True, gln=True, w_o_t=False):
    def layer(batch, heads, X, lw, alpha=None):
        dq, dkv = heads.dq, heads.dkv
        Xn = O.rmsnorm(X, lw.rms_w)
        Z = Xn @ O._f64(lw.w_in).T
        if phi1:
            Z = O.silu(Z)
        U, Q = Z[:, :dq], Z[:, dq:2 * dq]
        if split_q_first:
            U, Q = Q, U
        K, V = Z[:, 2 * dq:2 * dq + dkv], Z[:, 2 * dq + dkv:]
        g = O._f64(lw.gamma) if gln else None
        out = O.full_fwd(batch, heads, O._Proj(Q, K, V, U, g, O._f64(lw.beta)), alpha)
        Wo = O._f64(lw.w_o)
        upd = out["Y"] @ (Wo if w_o_t else Wo.T)
        return X + upd if residual else upd
    return layer


def _target_layer_kv_from_t_rows(batch, heads, X, lw, alpha=None):
    dq, dkv = heads.dq, heads.dkv
    Xn = O.rmsnorm(X, lw.rms_w)
    trow = O.t_row_index(batch)
    ZT = O.silu(Xn[trow] @ O._f64(lw.w_in).T)
    Xk = np.zeros_like(Xn)
    Xk[trow] = Xn[trow]                     # keys and values from T rows only
    Zkv = O.silu(Xk @ O._f64(lw.w_kv).T)
    inp = O._Proj(ZT[:, dq:], Zkv[:, :dkv], Zkv[:, dkv:], ZT[:, :dq], O._f64(lw.gamma), O._f64(lw.beta))
    out = O.target_fwd(batch, heads, inp, alpha)
    Xo = np.array(X, dtype=np.float64, copy=True)
    Xo[trow] = Xo[trow] + out["Y"] @ O._f64(lw.w_o).T
    return Xo


def _target_layer_updates_all_rows(batch, heads, X, lw, alpha=None):
    Xo = O.target_layer.__wrapped__(batch, heads, X, lw, alpha)
    return Xo + 1e-3 * O.rmsnorm(X, lw.rms_w)


def _t_rows_shifted(batch):
    return O.t_row_index.__wrapped__(batch) - 1


def _v2_sub_by_target(batch):
    return (np.arange(batch.total_t) // 4) % 4


def _mix_interleaved(Xt, n_sub=O.V2_SUB):
    n, d = Xt.shape
    parts = np.asarray(Xt, np.float64).reshape(n // n_sub, n_sub, d // n_sub, n_sub)  # strided parts
    return parts.transpose(0, 3, 1, 2).reshape(n, d)


def _swiglu_gate_up_swapped(X, w_gate, w_up, w_down):
    return (O.silu(X @ w_up.T) * (X @ w_gate.T)) @ w_down.T


def _v2_variant(ffn_residual=True, ffn_per_sub=True, ffn_norm=True):
    def layer(batch, heads, X, lw, alpha=None):
        lw2 = syn_copy(lw)
        if not ffn_per_sub:
            lw2.w_gate, lw2.w_up, lw2.w_down = [lw.w_gate[0]] * 4, [lw.w_up[0]] * 4, [lw.w_down[0]] * 4
        if not ffn_norm:
            lw2.rms_w2 = None
        Xo = O.v2_target_layer.__wrapped__(batch, heads, X, lw2, alpha) if ffn_norm else _v2_no_norm(batch, heads, X, lw2)
        if not ffn_residual:
            trow = O.t_row_index(batch)
            Xo[trow] = Xo[trow] - _mixed_attn(batch, heads, X, lw2)[trow]
        return Xo
    return layer


def syn_copy(lw):
    import copy
    return copy.copy(lw)


def _mixed_attn(batch, heads, X, lw):
    lw0 = syn_copy(lw)
    lw0.w_down = [np.zeros_like(x) for x in lw.w_down]
    return O.v2_target_layer.__wrapped__(batch, heads, X, lw0)


def _v2_no_norm(batch, heads, X, lw):
    orig = O.rmsnorm
    calls = []

    def rms(Xa, w, eps=O.RMS_EPS):
        calls.append(1)
        return orig(Xa, w, eps) if len(calls) == 1 else np.asarray(Xa, np.float64)
    O.rmsnorm = rms
    try:
        return O.v2_target_layer.__wrapped__(batch, heads, X, lw)
    finally:
        O.rmsnorm = orig


MUTATIONS = {
    "t_rows_do_not_see_self": ("dense_mask_fast", _mask_no_self_t),
    "tie_visible": ("dense_mask_fast", _mask_fast_ties_visible),
    "r_causal_excludes_self": ("dense_mask", _mask_cell_strict_causal),
    "h_rows_see_r": ("dense_mask", _mask_cell_t_sees_later_h_only),
    "normalise_by_visible_count": ("attention_user", _attn_norm_by_count),
    "gqa_modulo_mapping": ("attention_user", _attn_gqa_modulo),
    "alpha_dropped": ("attention_user", _attn_no_alpha),
    "silu_is_sigmoid": ("silu", lambda x: O.sigmoid(x)),
    "silu_sign": ("silu", lambda x: x / (1.0 + np.exp(x))),
    "gln_unbiased_var": ("gln", _gln_unbiased),
    "gln_single_group": ("gln", _gln_first_group),
    "bwd_wrong_sign": ("attention_user_bwd", _bwd_sign),
    "bwd_dk_rows_reversed": ("attention_user_bwd", _bwd_dk_transposed),
    "gate_bwd_dropped_mean_terms": ("gate_bwd", _gate_bwd_no_mean_term),
    "rmsnorm_no_sqrt": ("rmsnorm", _rms_no_sqrt),
    "rmsnorm_ignores_weight": ("rmsnorm", _rms_no_weight),
    "stack_phi1_dropped": ("full_layer", _full_layer_variant(phi1=False)),
    "stack_u_q_swapped": ("full_layer", _full_layer_variant(split_q_first=True)),
    "stack_residual_dropped": ("full_layer", _full_layer_variant(residual=False)),
    "stack_gate_without_gln": ("full_layer", _full_layer_variant(gln=False)),
    "stack_w_o_transposed": ("full_layer", _full_layer_variant(w_o_t=True)),
    "target_kv_from_t_rows": ("target_layer", _target_layer_kv_from_t_rows),
    "target_updates_hr_rows": ("target_layer", _target_layer_updates_all_rows),
    "t_rows_shifted": ("t_row_index", _t_rows_shifted),
    "v2_sub_by_target_index": ("v2_sub_index", _v2_sub_by_target),
    "v2_mix_identity": ("mix_tokens", lambda Xt, n_sub=4: np.asarray(Xt, np.float64)),
    "v2_mix_strided_parts": ("mix_tokens", _mix_interleaved),
    "v2_swiglu_gate_up_swapped": ("swiglu", _swiglu_gate_up_swapped),
    "v2_ffn_residual_dropped": ("v2_target_layer", _v2_variant(ffn_residual=False)),
    "v2_ffn_shared_weights": ("v2_target_layer", _v2_variant(ffn_per_sub=False)),
    "v2_ffn_prenorm_dropped": ("v2_target_layer", _v2_variant(ffn_norm=False)),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    orig = getattr(O, attr)
    if not hasattr(orig, "__wrapped__"):
        # allow the mutants to reach the original implementation
        def passthrough(*a, **kw):
            return orig(*a, **kw)
        passthrough.__wrapped__ = orig
    fn.__wrapped__ = orig
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for check in P.ALL_CHECKS + S.STACK_CHECKS + V.V2_CHECKS:
        try:
            check()
        except AssertionError:
            caught.append(check.__name__)
        except (ValueError, IndexError, FloatingPointError) as e:   # shape errors count as caught
            caught.append(check.__name__ + ":" + type(e).__name__)
    assert caught, f"mutation {name} passed every pin"
