"""Checks that pin the fp64 oracle to facts fixed outside itself.

Each ``check_*`` raises AssertionError when the oracle disagrees with:
  * values printed on the pages (the 7-token mask table, tests/golden/),
  * closed forms and special cases that reduce to textbook or library routines,
  * brute force on tiny inputs written as independent scalar loops,
  * structural invariants that follow from the method's definition,
  * central finite differences (for the backward pass).
``test_oracle_pins.py`` runs them; ``test_oracle_mutations.py`` plants mistakes
in the oracle and checks that at least one of these checks catches each one.
"""
from __future__ import annotations

import math
import os

import numpy as np
import scipy.special
import torch

import mtfm_synth as syn
from oracle import mtfm_oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load_golden_mask():
    rows = []
    with open(os.path.join(GOLDEN, "mask_7token.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([int(x) for x in line.split()[1:]])
    return np.array(rows, dtype=bool)


# ----------------------------------------------------------------------------- mask

def check_mask_worked_example():
    """[DY] §8.2: 3 H, 2 R, 2 T, both exposures after every R action."""
    want = _load_golden_mask()
    got = O.dense_mask(3, 2, 2, np.array([100, 200]), np.array([900, 950]))
    assert got.shape == want.shape and np.array_equal(got, want), f"\n{got.astype(int)}\n!=\n{want.astype(int)}"


def check_mask_rules_counts():
    """Per-row visible-key counts fixed by the rules ([MT] §3.2), incl. timestamp ties."""
    rng = np.random.default_rng(7)
    for LH, LR, LT in [(4, 5, 3), (0, 3, 2), (3, 0, 2), (2, 3, 0), (1, 1, 1), (6, 7, 5)]:
        r_ts = np.sort(rng.integers(0, 10, LR))
        t_exp = rng.integers(0, 10, LT)
        if LR and LT:
            t_exp[0] = r_ts[LR // 2]          # a tie: must NOT be visible (strict <)
        M = O.dense_mask(LH, LR, LT, r_ts, t_exp)
        N = LH + LR + LT
        assert M.shape == (N, N)
        for i in range(LH):                   # H row: exactly the H block
            assert M[i].sum() == LH and M[i, :LH].all()
        for a in range(LR):                   # R row a: H + R_0..R_a
            i = LH + a
            assert M[i].sum() == LH + a + 1 and M[i, :LH + a + 1].all()
        for t in range(LT):                   # T row: H + {R: ts < exp} + itself
            i = LH + LR + t
            n_r = int((r_ts < t_exp[t]).sum())
            assert M[i].sum() == LH + n_r + 1
            assert M[i, i]
            assert not M[i, LH + LR:].sum() - 1   # no other T token
            for b in range(LR):
                assert M[i, LH + b] == (r_ts[b] < t_exp[t])
        # nobody but T sees T; H/R queries never see T keys
        assert not M[:LH + LR, LH + LR:].any()


def check_mask_fast_equals_cellwise():
    rng = np.random.default_rng(11)
    for _ in range(20):
        LH, LR = rng.integers(0, 6, 2)
        v2 = int(rng.choice([1, 4]))
        LT = int(rng.integers(0, 3)) * v2
        r_ts = np.sort(rng.integers(0, 8, LR))
        t_exp = np.repeat(rng.integers(0, 8, LT // v2), v2)
        a = O.dense_mask(LH, LR, LT, r_ts, t_exp, v2)
        b = O.dense_mask_fast(LH, LR, LT, r_ts, t_exp, v2)
        assert np.array_equal(a, b)


def check_mask_v2_siblings():
    """V2 target scale-up: 4 sub-tokens of a target see each other and share the prefix."""
    r_ts = np.array([1, 5, 9])
    t_exp = np.repeat(np.array([6, 2]), 4)
    M = O.dense_mask(2, 3, 8, r_ts, t_exp, 4)
    TT = M[5:, 5:]
    want = np.kron(np.eye(2, dtype=int), np.ones((4, 4), dtype=int)).astype(bool)
    assert np.array_equal(TT, want)
    assert M[5:9, :5].sum(axis=1).tolist() == [4] * 4     # 2 H + R with ts < 6 -> 2 R
    assert M[9:13, :5].sum(axis=1).tolist() == [3] * 4    # 2 H + R with ts < 2 -> 1 R


# ----------------------------------------------------------------------------- attention

def check_silu_library():
    x = np.linspace(-30, 30, 1001)
    assert np.allclose(O.silu(x), x * scipy.special.expit(x), rtol=1e-14, atol=1e-300)


def _brute_attention(q, k, v, M, hq, hkv, dh, alpha, n_norm):
    """Scalar loops: independent restatement used on tiny inputs only."""
    r = hq // hkv
    nq = q.shape[0]
    N = k.shape[0]
    out = np.zeros((nq, hq * dh))
    for i in range(nq):
        for h in range(hq):
            g = h // r
            for j in range(N):
                if not M[i, j]:
                    continue
                s = 0.0
                for c in range(dh):
                    s += q[i, h * dh + c] * k[j, g * dh + c]
                x = alpha * s
                w = x * (1.0 / (1.0 + math.exp(-x))) / n_norm
                for c in range(dh):
                    out[i, h * dh + c] += w * v[j, g * dh + c]
    return out


def check_attention_bruteforce():
    rng = np.random.default_rng(3)
    # the last case has r = 3 query heads per KV head (the 768-wide Hq 3 / Hkv 1 shape)
    for (LH, LR, LT, hq, hkv, dh) in [(3, 2, 2, 2, 1, 4), (2, 3, 3, 4, 2, 3), (0, 2, 1, 2, 2, 2), (2, 2, 3, 3, 1, 5)]:
        N = LH + LR + LT
        r_ts = np.sort(rng.integers(0, 10, LR))
        t_exp = rng.integers(0, 10, LT)
        M = O.dense_mask(LH, LR, LT, r_ts, t_exp)
        q = rng.standard_normal((N, hq * dh))
        k = rng.standard_normal((N, hkv * dh))
        v = rng.standard_normal((N, hkv * dh))
        alpha = 0.7
        a = O.attention_user(q, k, v, M, hq, hkv, dh, alpha, N)
        b = _brute_attention(q, k, v, M, hq, hkv, dh, alpha, N)
        assert np.allclose(a, b, rtol=1e-12, atol=1e-14), np.abs(a - b).max()


def check_attention_closed_form():
    """q_i = a e1, k_j = b e1  =>  A_i = SiLU(alpha a b) / N * sum_{j visible} v_j."""
    rng = np.random.default_rng(5)
    LH, LR, LT, hq, hkv, dh = 4, 3, 3, 2, 1, 5
    N = LH + LR + LT
    r_ts = np.array([1, 4, 8])
    t_exp = np.array([0, 5, 9])
    M = O.dense_mask(LH, LR, LT, r_ts, t_exp)
    a_, b_, alpha = 1.3, -0.8, 0.5
    q = np.zeros((N, hq * dh))
    q[:, 0] = a_
    q[:, dh] = a_
    k = np.zeros((N, hkv * dh))
    k[:, 0] = b_
    v = rng.standard_normal((N, hkv * dh))
    A = O.attention_user(q, k, v, M, hq, hkv, dh, alpha, N)
    x = alpha * a_ * b_
    w = x * scipy.special.expit(x) / N
    for i in range(N):
        want = w * v[M[i]].sum(axis=0)
        for h in range(hq):
            assert np.allclose(A[i, h * dh:(h + 1) * dh], want, rtol=1e-13, atol=1e-15)
    # Visible counts: with v = 1 the output equals SiLU(x)/N times the visible count.
    A1 = O.attention_user(q, k, np.ones_like(v), M, hq, hkv, dh, alpha, N)
    counts = np.array([LH] * LH + [LH + 1, LH + 2, LH + 3] + [LH + 0 + 1, LH + 2 + 1, LH + 3 + 1])
    assert np.allclose(A1[:, 0], w * counts, rtol=1e-13)


def check_attention_zero_keys():
    rng = np.random.default_rng(6)
    N = 9
    M = O.dense_mask(4, 3, 2, np.array([1, 2, 3]), np.array([2, 9]))
    q = rng.standard_normal((N, 8))
    A = O.attention_user(q, np.zeros((N, 4)), rng.standard_normal((N, 4)), M, 2, 1, 4, 0.5, N)
    assert np.all(A == 0.0)


def _small_batch(seed=21, v2=1):
    if v2 == 1:
        return syn.fixed_batch([5, 0, 3], [4, 3, 0], [3, 2, 2], seed)
    return syn.fixed_batch([5, 2], [4, 3], [8, 4], seed, v2_subtokens=4)


def check_target_equals_full_t_rows():
    """A Target layer equals the T rows of a Full layer fed the same weights ([DY] §4.2)."""
    for v2 in (1, 4):
        b = _small_batch(v2=v2)
        hd = syn.Heads(4, 2, 8)
        full = syn.layer_inputs(b, hd, target=False, seed=3)
        so = O.offsets(b.N)
        trows = np.concatenate([np.arange(so[u] + b.L_H[u] + b.L_R[u], so[u + 1]) for u in range(b.B)])
        tgt = syn.LayerInputs(full.q[trows], full.k, full.v, full.u[trows], full.gamma, full.beta)
        F = O.full_fwd(b, hd, full)
        T = O.target_fwd(b, hd, tgt)
        assert np.allclose(F["A"][trows], T["A"], rtol=1e-13, atol=1e-15)
        assert np.allclose(F["Y"][trows], T["Y"], rtol=1e-12, atol=1e-13)


def check_gqa_equals_repeated_mha():
    b = _small_batch()
    hd = syn.Heads(4, 2, 8)
    inp = syn.layer_inputs(b, hd, target=False, seed=4)
    k = syn.bf16_bits_to_f32(inp.k).astype(np.float64)
    v = syn.bf16_bits_to_f32(inp.v).astype(np.float64)
    r = hd.hq // hd.hkv
    rep = lambda x: np.concatenate([x[:, (h // r) * hd.dh:(h // r + 1) * hd.dh] for h in range(hd.hq)], axis=1)
    mha = syn.LayerInputs(inp.q, rep(k), rep(v), inp.u, inp.gamma, inp.beta)
    a = O.full_fwd(b, hd, inp)["Y"]
    m = O.full_fwd(b, syn.Heads(hd.hq, hd.hq, hd.dh), mha)["Y"]
    assert np.allclose(a, m, rtol=1e-13, atol=1e-13)


def check_permutation_equivariance():
    """Permuting the candidates of a user (rows and exposures together) permutes its outputs;
    permuting users permutes the jagged blocks."""
    b = syn.fixed_batch([4, 3], [3, 4], [4, 3], seed=31)
    hd = syn.Heads(2, 1, 8)
    inp = syn.layer_inputs(b, hd, target=False, seed=5)
    base = O.full_fwd(b, hd, inp)["Y"]
    so = O.offsets(b.N)
    to = O.offsets(b.L_T)
    perm_t = np.array([2, 0, 3, 1])
    rows = np.arange(b.total_tokens)
    t0 = so[0] + b.L_H[0] + b.L_R[0]
    rows[t0:t0 + 4] = t0 + perm_t
    b2 = syn.JaggedBatch(b.L_H, b.L_R, b.L_T, b.r_ts, b.t_exp.copy(), b.scenario)
    b2.t_exp[to[0]:to[0] + 4] = b.t_exp[to[0] + perm_t]
    inp2 = syn.LayerInputs(inp.q[rows], inp.k[rows], inp.v[rows], inp.u[rows], inp.gamma, inp.beta)
    got = O.full_fwd(b2, hd, inp2)["Y"]
    assert np.allclose(got, base[rows], rtol=1e-13, atol=1e-13)
    # swap the two users
    b3 = syn.JaggedBatch(b.L_H[::-1].copy(), b.L_R[::-1].copy(), b.L_T[::-1].copy(),
                         np.concatenate([b.r_ts[3:], b.r_ts[:3]]),
                         np.concatenate([b.t_exp[4:], b.t_exp[:4]]), b.scenario)
    urows = np.concatenate([np.arange(so[1], so[2]), np.arange(so[0], so[1])])
    inp3 = syn.LayerInputs(inp.q[urows], inp.k[urows], inp.v[urows], inp.u[urows], inp.gamma, inp.beta)
    got3 = O.full_fwd(b3, hd, inp3)["Y"]
    assert np.allclose(got3, base[urows], rtol=1e-13, atol=1e-13)


def check_locality():
    """Perturbing R/T inputs leaves H rows bit-identical; perturbing T leaves R rows; T_t' leaves T_t."""
    b = syn.fixed_batch([5], [4], [3], seed=41)
    hd = syn.Heads(2, 1, 8)
    inp = syn.layer_inputs(b, hd, target=False, seed=6)
    base = O.full_fwd(b, hd, inp)["A"]

    def pert(rows):
        k = inp.k.copy()
        v = inp.v.copy()
        q = inp.q.copy()
        k[rows] ^= 0x0040
        v[rows] ^= 0x0040
        q[rows] ^= 0x0040
        return O.full_fwd(b, hd, syn.LayerInputs(q, k, v, inp.u, inp.gamma, inp.beta))["A"]

    a = pert(np.arange(5, 12))          # all R and T
    assert np.array_equal(a[:5], base[:5])
    a = pert(np.arange(9, 12))          # all T
    assert np.array_equal(a[:9], base[:9])
    a = pert(np.array([10]))            # one target
    assert np.array_equal(a[[0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 11]], base[[0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 11]])
    assert not np.array_equal(a[10], base[10])


def check_gln_is_layernorm():
    """gamma = 1, beta = 0, U = 1: Y equals a plain LayerNorm (torch library routine, fp64)."""
    rng = np.random.default_rng(8)
    A = rng.standard_normal((7, 24)) * 3 + 1
    types = np.array([0, 1, 2, 2, 1, 0, 2])
    Y, _, _ = O.gate(A, np.ones_like(A), types, np.ones((3, 24)), np.zeros((3, 24)), 1e-5)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(A), (24,), eps=1e-5).numpy()
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
    # per-type affine: each row uses the gamma/beta row of its own type
    g = rng.standard_normal((3, 24))
    bt = rng.standard_normal((3, 24))
    U = rng.standard_normal((7, 24))
    Y2, _, _ = O.gate(A, U, types, g, bt, 1e-5)
    for i in range(7):
        want = torch.nn.functional.layer_norm(torch.from_numpy(A[i:i + 1]), (24,),
                                              weight=torch.from_numpy(g[types[i]]),
                                              bias=torch.from_numpy(bt[types[i]]), eps=1e-5).numpy()[0] * U[i]
        assert np.allclose(Y2[i], want, rtol=1e-12, atol=1e-12)
    Y3, m, r = O.gate(A, U, types, None, None)
    assert m is None and np.array_equal(Y3, A * U)


def check_target_rows_ignore_hr_queries():
    """A row's output depends on its own query and U only ([DY] §4.2: the Target layer
    drops the H/R queries): changing the Q and U rows of every H and R token leaves
    the T rows of a Full layer bit-identical, and those rows still equal the Target
    layer computed without any H/R query, while the H/R rows do change."""
    b = _small_batch()
    hd = syn.Heads(2, 1, 8)
    full = syn.layer_inputs(b, hd, target=False, seed=9)
    tr = O.t_row_index(b)
    hr = np.setdiff1d(np.arange(b.total_tokens), tr)
    base = O.full_fwd(b, hd, full)
    q, u = full.q.copy(), full.u.copy()
    q[hr] ^= 0x0041
    u[hr] ^= 0x0041
    pert = O.full_fwd(b, hd, syn.LayerInputs(q, full.k, full.v, u, full.gamma, full.beta))
    assert np.array_equal(pert["Y"][tr], base["Y"][tr])
    assert np.array_equal(pert["A"][tr], base["A"][tr])
    assert not np.allclose(pert["Y"][hr], base["Y"][hr])
    tgt = O.target_fwd(b, hd, syn.LayerInputs(full.q[tr], full.k, full.v, full.u[tr], full.gamma, full.beta))
    assert np.allclose(tgt["Y"], pert["Y"][tr], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- backward

def _loss_full(b, hd, q, k, v, U, gamma, beta, dY, target):
    inp = syn.LayerInputs(q, k, v, U, gamma, beta)
    f = O.target_fwd if target else O.full_fwd
    return float((f(b, hd, inp, alpha=0.6)["Y"] * dY).sum())


def check_backward_finite_differences():
    """Central differences (h = 1e-6) on every input element of a tiny layer, Full and Target."""
    rng = np.random.default_rng(12)
    b = syn.fixed_batch([3, 2], [2, 3], [2, 2], seed=55)
    hd = syn.Heads(2, 1, 3)
    for target in (False, True):
        rows_q = b.total_t if target else b.total_tokens
        q = rng.standard_normal((rows_q, hd.dq))
        k = rng.standard_normal((b.total_tokens, hd.dkv))
        v = rng.standard_normal((b.total_tokens, hd.dkv))
        U = rng.standard_normal((rows_q, hd.dq))
        gamma = 1 + 0.3 * rng.standard_normal((3, hd.dq))
        beta = 0.3 * rng.standard_normal((3, hd.dq))
        dY = rng.standard_normal((rows_q, hd.dq))
        inp = syn.LayerInputs(q, k, v, U, gamma, beta, dY)
        g = (O.target_bwd if target else O.full_bwd)(b, hd, inp, alpha=0.6)
        args = dict(q=q, k=k, v=v, U=U, gamma=gamma, beta=beta)
        names = dict(q="dq", k="dk", v="dv", U="du", gamma="dgamma", beta="dbeta")
        h = 1e-6
        for name, arr in args.items():
            flat = arr.reshape(-1)
            num = np.zeros_like(flat)
            for idx in range(flat.size):
                old = flat[idx]
                flat[idx] = old + h
                lp = _loss_full(b, hd, q, k, v, U, gamma, beta, dY, target)
                flat[idx] = old - h
                lm = _loss_full(b, hd, q, k, v, U, gamma, beta, dY, target)
                flat[idx] = old
                num[idx] = (lp - lm) / (2 * h)
            ana = g[names[name]].reshape(-1)
            err = np.abs(ana - num).max() / max(1e-12, np.abs(num).max())
            assert err < 1e-6, (target, name, err)


def check_dv_closed_form():
    """dV = P^T dA with P the masked, normalised SiLU weights (textbook linear-map gradient)."""
    rng = np.random.default_rng(14)
    LH, LR, LT = 3, 3, 2
    N = 8
    M = O.dense_mask(LH, LR, LT, np.array([1, 2, 3]), np.array([3, 0]))
    q = rng.standard_normal((N, 4))
    k = rng.standard_normal((N, 4))
    v = rng.standard_normal((N, 4))
    dA = rng.standard_normal((N, 4))
    _, _, dv = O.attention_user_bwd(q, k, v, M, dA, 1, 1, 4, 0.5, N)
    x = 0.5 * q @ k.T
    P = np.where(M, x * scipy.special.expit(x), 0.0) / N
    assert np.allclose(dv, P.T @ dA, rtol=1e-13, atol=1e-15)


ALL_CHECKS = [
    check_mask_worked_example,
    check_mask_rules_counts,
    check_mask_fast_equals_cellwise,
    check_mask_v2_siblings,
    check_silu_library,
    check_attention_bruteforce,
    check_attention_closed_form,
    check_attention_zero_keys,
    check_target_equals_full_t_rows,
    check_gqa_equals_repeated_mha,
    check_permutation_equivariance,
    check_locality,
    check_gln_is_layernorm,
    check_target_rows_ignore_hr_queries,
    check_backward_finite_differences,
    check_dv_closed_form,
]
