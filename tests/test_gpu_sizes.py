"""Parity at the full configuration sizes, on sampled users.

The GPU runs the whole batch (2^21 tokens for the length sweep, 96/160 users for the training
shapes, the 64-user stack batch size); the oracle recomputes a few sampled users from scratch
(users are independent, so their rows are exact checks of the full-size launch).  Rows of the
other users hold seeded device-side normals.
"""
import numpy as np
import pytest
import torch

import mtfm_synth as syn
from gpu_helpers import assert_close, bf16_tensor, config_for, upload_batch
from oracle import mtfm_oracle as O

pytestmark = pytest.mark.gpu


def _subset(batch, users):
    ro = O.offsets(batch.L_R)
    to = O.offsets(batch.L_T)
    r_ts = np.concatenate([batch.r_ts[ro[u]:ro[u + 1]] for u in users])
    t_exp = np.concatenate([batch.t_exp[to[u]:to[u + 1]] for u in users])
    idx = np.array(users)
    return syn.JaggedBatch(batch.L_H[idx], batch.L_R[idx], batch.L_T[idx], r_ts, t_exp,
                           np.zeros(len(t_exp), np.int32), batch.v2_subtokens)


def _rows(batch, users, target):
    so = O.offsets(batch.L_T if target else batch.N)
    return np.concatenate([np.arange(so[u], so[u + 1]) for u in users])


def _run(batch, heads, users, target, seed):
    from hybrid_masked_attention_b200.session import HybridAttention
    cfg = config_for(batch, heads)
    s = HybridAttention(cfg, "cuda")
    s.pack(*upload_batch(batch), check=True)
    sub = _subset(batch, users)
    inp = syn.layer_inputs(sub, heads, target=target, seed=seed)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    rows_q = batch.total_t if target else batch.total_tokens
    dev = {}
    for name, rows, width in (("q", rows_q, heads.dq), ("u", rows_q, heads.dq),
                              ("k", batch.total_tokens, heads.dkv), ("v", batch.total_tokens, heads.dkv)):
        dev[name] = torch.randn(rows, width, generator=gen, device="cuda").to(torch.bfloat16)
    rq = torch.from_numpy(_rows(batch, users, target)).cuda()
    rk = torch.from_numpy(_rows(batch, users, False)).cuda()
    dev["q"][rq] = bf16_tensor(inp.q)
    dev["u"][rq] = bf16_tensor(inp.u)
    dev["k"][rk] = bf16_tensor(inp.k)
    dev["v"][rk] = bf16_tensor(inp.v)
    g = torch.from_numpy(inp.gamma).cuda()
    b = torch.from_numpy(inp.beta).cuda()
    f = s.target_fwd if target else s.full_fwd
    y, a, _ = f(dev["q"], dev["k"], dev["v"], dev["u"], g, b)
    torch.cuda.synchronize()
    ref = (O.target_fwd if target else O.full_fwd)(sub, heads, inp)
    return a[rq].cpu().numpy(), y[rq].cpu().numpy(), ref


@pytest.mark.parametrize("N,v2", [(512, False), (2048, False), (8192, False), (512, True), (4096, True)])
@pytest.mark.parametrize("target", [False, True], ids=["full", "target"])
def test_sweep_full_size(N, v2, target, cuda_ok):
    batch = syn.sweep_batch(N, v2=v2, seed=1003)
    users = [0, batch.B // 2, batch.B - 1]
    a, y, ref = _run(batch, syn.PAIR_HEADS, users, target, seed=31)
    assert_close(a, ref["A"], "A")
    assert_close(y, ref["Y"], "Y")


@pytest.mark.parametrize("B", [64, 96, 160])
@pytest.mark.parametrize("target", [False, True], ids=["full", "target"])
def test_production_batches_full_size(B, target, cuda_ok):
    batch = syn.pair_batch(B, seed=1005)
    users = list(range(0, B, max(1, B // 6)))
    a, y, ref = _run(batch, syn.PAIR_HEADS, users, target, seed=37)
    assert_close(a, ref["A"], "A")
    assert_close(y, ref["Y"], "Y")
