"""Target attention over a cached key/value prefix (request-level inference with shared user
K/V) on the GPU, through the C ABI.  The result is by definition the Target layer on the
sequence [prefix; candidates] of each user, so it is checked against the fp64 oracle's
Target layer on that sequence, and against the GPU's own Target layer on the concatenated
layout."""
import numpy as np
import pytest
import torch

import hybrid_masked_attention_b200 as M
import mtfm_synth as syn
from gpu_cases import BATCHES, edge_batch
from gpu_helpers import assert_close, bf16_tensor, config_for, upload_batch, upload_layer
from oracle import mtfm_oracle as O

pytestmark = pytest.mark.gpu


def split_kv(batch: syn.JaggedBatch, kv_bits: np.ndarray):
    """Rows of a [sum N, Dkv] tensor split into the H and R rows of every user (in batch order)
    and the T rows (the layouts of the cache and of the candidates)."""
    pre, cand, so = [], [], 0
    for u in range(batch.B):
        p = int(batch.L_H[u]) + int(batch.L_R[u])
        n = p + int(batch.L_T[u])
        pre.append(kv_bits[so:so + p])
        cand.append(kv_bits[so + p:so + n])
        so += n
    dkv = kv_bits.shape[1]
    cat = lambda parts: np.concatenate(parts) if parts else np.zeros((0, dkv), kv_bits.dtype)
    return cat(pre), cat(cand)


def _run(batch, heads, gln=True, seed=111):
    inp = syn.layer_inputs(batch, heads, target=True, seed=seed, gln=gln)
    cfg = config_for(batch, heads)
    meta = M.alloc_meta(cfg)
    M.pack(cfg, *upload_batch(batch), meta)
    M.pack_check(meta)
    d = upload_layer(inp)
    kp, kc = split_kv(batch, inp.k)
    vp, vc = split_kv(batch, inp.v)
    kp, kc, vp, vc = (bf16_tensor(x) for x in (kp, kc, vp, vc))
    T, D = batch.total_t, heads.dq
    f32 = dict(dtype=torch.float32, device="cuda")
    y, a, st = torch.empty(T, D, **f32), torch.empty(T, D, **f32), torch.empty(T, 2, **f32)
    M.attn_target_cached_fwd(cfg, meta, d["q"], kp, vp, kc, vc, d["u"], d["gamma"], d["beta"], y, a, st)
    y2, a2, st2 = torch.empty(T, D, **f32), torch.empty(T, D, **f32), torch.empty(T, 2, **f32)
    M.attn_target_fwd(cfg, meta, d["q"], d["k"], d["v"], d["u"], d["gamma"], d["beta"], y2, a2, st2)
    torch.cuda.synchronize()
    M.pack_check(meta)
    return inp, (y, a, st), (y2, a2, st2)


CASES = [("pair", syn.PAIR_HEADS), ("edge", syn.PAIR_HEADS), ("v2_n512", syn.PAIR_HEADS),
         ("v1_n2048", syn.Heads(4, 2, 64)), ("pair", syn.Heads(2, 2, 64)),
         # head_dim 32 (64-byte swizzle) at r = 2, 1, 4
         ("tiny", syn.TINY_HEADS), ("pair", syn.Heads(2, 2, 32)), ("v2_n512", syn.Heads(4, 1, 32)),
         # r = 8 (16 T rows per sub-tile) at head_dim 32 and 64
         ("pair", syn.Heads(8, 1, 32)), ("edge", syn.Heads(8, 1, 64))]


@pytest.mark.parametrize("bname,heads", CASES, ids=[f"{b}-{h.hq}x{h.hkv}" for b, h in CASES])
def test_cached_prefix_matches_target_layer(bname, heads, cuda_ok):
    batch = BATCHES[bname]()
    inp, (y, a, st), (y2, a2, st2) = _run(batch, heads)
    ref = O.target_fwd(batch, heads, inp)
    assert_close(a.cpu().numpy(), ref["A"], "A")
    assert_close(y.cpu().numpy(), ref["Y"], "Y")
    if batch.total_t:
        assert_close(st[:, 0].cpu().numpy(), ref["mean"], "mean")
    # the same numbers as the Target layer on the concatenated layout, up to fp32 summation order
    torch.testing.assert_close(a, a2, rtol=1e-4, atol=1e-6)
    torch.testing.assert_close(y, y2, rtol=1e-3, atol=1e-4)


def test_cached_prefix_plain_gate_and_attention_only(cuda_ok):
    batch, heads = edge_batch(), syn.PAIR_HEADS
    inp = syn.layer_inputs(batch, heads, target=True, seed=5, gln=False)
    cfg = config_for(batch, heads)
    meta = M.alloc_meta(cfg)
    M.pack(cfg, *upload_batch(batch), meta)
    d = upload_layer(inp)
    kp, kc = (bf16_tensor(x) for x in split_kv(batch, inp.k))
    vp, vc = (bf16_tensor(x) for x in split_kv(batch, inp.v))
    T, D = batch.total_t, heads.dq
    a = torch.empty(T, D, device="cuda")
    M.attn_target_cached(cfg, meta, d["q"], kp, vp, kc, vc, a)
    y = torch.empty(T, D, device="cuda")
    a2 = torch.empty(T, D, device="cuda")
    M.attn_target_cached_fwd(cfg, meta, d["q"], kp, vp, kc, vc, d["u"], None, None, y, a2, None)
    torch.cuda.synchronize()
    M.pack_check(meta)
    ref = O.target_fwd(batch, heads, inp)
    assert_close(a.cpu().numpy(), ref["A"], "A")
    assert_close(y.cpu().numpy(), ref["Y"], "Y = A (*) U")


def test_cached_prefix_unsupported_shape(cuda_ok):
    batch, heads = BATCHES["tiny"](), syn.Heads(4, 1, 128)   # head_dim 128: no tensor-core Target kernel
    cfg = config_for(batch, heads)
    meta = M.alloc_meta(cfg)
    M.pack(cfg, *upload_batch(batch), meta)
    T, P, D, Dkv = batch.total_t, batch.total_tokens - batch.total_t, heads.dq, heads.dkv
    z = lambda r, c: torch.zeros(r, c, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(M.MtfmError):
        M.attn_target_cached(cfg, meta, z(T, D), z(P, Dkv), z(P, Dkv), z(T, Dkv), z(T, Dkv),
                             torch.empty(T, D, device="cuda"))
