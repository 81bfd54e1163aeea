"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch each one.

A pin set that lets a dropped term, a wrong sign or index or a transposed operand
through is not a pin; every mutation below must make at least one check fail.
"""
import numpy as np
import pytest

import oracle_pins as P
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
    for check in P.ALL_CHECKS:
        try:
            check()
        except AssertionError:
            caught.append(check.__name__)
        except (ValueError, IndexError, FloatingPointError) as e:   # shape errors count as caught
            caught.append(check.__name__ + ":" + type(e).__name__)
    assert caught, f"mutation {name} passed every pin"
