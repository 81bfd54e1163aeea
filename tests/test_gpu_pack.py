"""mtfm_pack on the GPU against the oracle: offsets, row types and the mask, bit-exact."""
import numpy as np
import pytest
import torch

import mtfm_synth as syn
from gpu_cases import BATCHES, HEADS
from gpu_helpers import gpu_mask_rows, packed, upload_batch
from oracle import mtfm_oracle as O

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", sorted(BATCHES))
def test_pack_matches_oracle(name, cuda_ok):
    from hybrid_masked_attention_b200 import meta_read
    b = BATCHES[name]()
    s = packed(b, HEADS["tiny"])
    m = meta_read(s.cfg, s.meta)
    assert np.array_equal(m["seq_off"], O.offsets(b.N))
    assert np.array_equal(m["r_off"], O.offsets(b.L_R))
    assert np.array_equal(m["t_off"], O.offsets(b.L_T))
    types = np.concatenate([O.row_types(int(b.L_H[u]), int(b.L_R[u]), int(b.L_T[u])) for u in range(b.B)]) \
        if b.total_tokens else np.zeros(0, np.int64)
    assert np.array_equal(m["row_type"].astype(np.int64), types)
    for u in range(b.B):
        assert np.array_equal(gpu_mask_rows(m, b, u), O.user_mask(b, u)), f"user {u}"
    # work lists: every (user, tile) exactly once, bounds equal the rows' prefix ends
    nq_full = np.asarray(b.N)
    nq_tgt = np.asarray(b.L_T)
    for items, nq, tgt in ((m["items_full"], nq_full, False), (m["items_target"], nq_tgt, True)):
        want = {(u, t) for u in range(b.B) for t in range((int(nq[u]) + 127) // 128)}
        got = [(int(r[0]), int(r[1])) for r in items]
        assert len(got) == len(set(got)) and set(got) == want
        so = m["seq_off"]
        for (u, t, kmin, kmax) in items:
            pos0 = int(b.L_H[u] + b.L_R[u]) if tgt else 0
            rows = np.arange(t * 128, min((t + 1) * 128, int(nq[u]))) + pos0
            kv = m["kv_end"][so[u] + rows]
            assert kmin == kv.min() and kmax == kv.max()
    # longest users first
    if len(m["items_full"]):
        order = [int(r[0]) for r in m["items_full"]]
        firsts = list(dict.fromkeys(order))
        Ns = [int(b.N[u]) for u in firsts]
        assert Ns == sorted(Ns, reverse=True)


def test_pack_rejects_bad_lengths(cuda_ok):
    from hybrid_masked_attention_b200 import MtfmError, pack_check
    b = syn.fixed_batch([3, 4], [2, 2], [1, 2], seed=5)
    s = packed(b, HEADS["tiny"])
    lh, lr, lt, r_ts, t_exp = upload_batch(b)
    lh[0] += 1                                   # sums no longer match the totals
    s.pack(lh, lr, lt, r_ts, t_exp)
    with pytest.raises(MtfmError, match="BAD_LENGTHS"):
        pack_check(s.meta)
    lh, lr, lt, r_ts, t_exp = upload_batch(b)
    lt[1] = -1
    lt[0] = 4                                    # totals still match but a length is negative
    s.pack(lh, lr, lt, r_ts, t_exp)
    with pytest.raises(MtfmError, match="BAD_LENGTHS"):
        pack_check(s.meta)


def test_pack_rejects_unsorted_and_skips_work(cuda_ok):
    from hybrid_masked_attention_b200 import MtfmError, pack_check
    b = syn.fixed_batch([3, 4], [3, 2], [1, 2], seed=6)
    s = packed(b, HEADS["tiny"])
    lh, lr, lt, r_ts, t_exp = upload_batch(b)
    r_ts[0], r_ts[2] = 900, 100                  # user 0's R timestamps out of order
    s.pack(lh, lr, lt, r_ts, t_exp)
    with pytest.raises(MtfmError, match="UNSORTED"):
        pack_check(s.meta)
    # kernels reading a failed metadata block do nothing: outputs keep their sentinel
    from gpu_helpers import upload_layer
    inp = upload_layer(syn.layer_inputs(b, HEADS["tiny"], target=False, seed=1))
    D = HEADS["tiny"].dq
    y = torch.full((b.total_tokens, D), 7.0, device="cuda")
    a = torch.full((b.total_tokens, D), 7.0, device="cuda")
    st = torch.full((b.total_tokens, 2), 7.0, device="cuda")
    s.full_fwd(inp["q"], inp["k"], inp["v"], inp["u"], inp["gamma"], inp["beta"], out=(y, a, st))
    torch.cuda.synchronize()
    assert bool((y == 7.0).all()) and bool((a == 7.0).all())


def test_pack_empty_batch(cuda_ok):
    from hybrid_masked_attention_b200 import meta_read
    b = syn.fixed_batch([], [], [], seed=7)
    s = packed(b, HEADS["tiny"])
    m = meta_read(s.cfg, s.meta)
    assert m["n_items_full"] == 0 and m["n_items_target"] == 0
