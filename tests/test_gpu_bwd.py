"""Full and Target backward on the GPU (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import mtfm_synth as syn
from gpu_cases import BATCHES, HEADS
from gpu_helpers import assert_close, packed, upload_layer
from oracle import mtfm_oracle as O

pytestmark = pytest.mark.gpu


def _run(batch, heads, target, gln, seed=17, users=None):
    inp = syn.layer_inputs(batch, heads, target=target, seed=seed, gln=gln, with_dy=True)
    s = packed(batch, heads)
    d = upload_layer(inp)
    fwd = s.target_fwd if target else s.full_fwd
    y, a, st = fwd(d["q"], d["k"], d["v"], d["u"], d["gamma"], d["beta"])
    bwd = s.target_bwd if target else s.full_bwd
    g = bwd(d["q"], d["k"], d["v"], d["u"], d["gamma"], d["beta"], a, st, d["dy"])
    torch.cuda.synchronize()
    ref = (O.target_bwd if target else O.full_bwd)(batch, heads, inp, users=users)
    return {k: (None if v is None else v.cpu().numpy()) for k, v in g.items()}, ref


def _rows(batch, users, target):
    so = O.offsets(batch.N)
    to = O.offsets(batch.L_T)
    qo = to if target else so
    q = np.concatenate([np.arange(qo[u], qo[u + 1]) for u in users]) if users else np.zeros(0, int)
    k = np.concatenate([np.arange(so[u], so[u + 1]) for u in users]) if users else np.zeros(0, int)
    return q, k


CASES = [("tiny", "tiny", True), ("tiny", "tiny", False), ("edge", "pair", True),
         ("edge", "r8", True), ("v2_n512", "pair", True), ("pair", "pair", True),
         ("pair", "dh128", False), ("edge", "dh256", True), ("tiny", "dh256", False),
         ("edge", "r1", True), ("edge", "r2", True), ("v2_n512", "r2", True),
         # head_dim 32 on the tcgen05 backward (64-byte swizzle): r = 2, 1, 4 (and 8 above)
         ("edge", "tiny", True), ("pair", "tiny", False), ("v2_n512", "dh32_r1", True),
         ("edge", "dh32_r4", True)]


@pytest.mark.parametrize("bname,hname,gln", CASES)
@pytest.mark.parametrize("target", [False, True], ids=["full", "target"])
def test_bwd_parity(bname, hname, gln, target, cuda_ok):
    b, hd = BATCHES[bname](), HEADS[hname]
    g, ref = _run(b, hd, target, gln)
    for name in ("dq", "dk", "dv", "du"):
        assert_close(g[name], ref[name], name)
    if gln:
        assert_close(g["dgamma"], ref["dgamma"], "dgamma")
        assert_close(g["dbeta"], ref["dbeta"], "dbeta")


@pytest.mark.parametrize("B", [96, 160])
@pytest.mark.parametrize("target", [False, True], ids=["full", "target"])
def test_bwd_training_shapes(B, target, cuda_ok):
    """Training-step shapes (production lengths, batch 96 and 160); oracle on a user sample."""
    b = syn.pair_batch(B, seed=1005)
    users = list(range(0, B, B // 12))
    g, ref = _run(b, HEADS["pair"], target, True, users=users)
    qr, kr = _rows(b, users, target)
    for name, rows in (("dq", qr), ("du", qr), ("dk", kr), ("dv", kr)):
        assert_close(g[name][rows], ref[name][rows], name)
