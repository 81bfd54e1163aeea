"""V2 Target Scale-Up layer (Meituan tech blog §3.3.2: per-sub-token [U Q] projections
and SwiGLU FFNs, zero-parameter mixing of each target's 4 sub-tokens) on the GPU
through the C ABI, against the fp64 oracle, at the standard bar (rel-L2 <= 1e-2,
max-abs <= 2e-2 x RMS) on the T rows it updates; H / R rows must come back
bit-identical."""
import numpy as np
import pytest
import torch

import mtfm_synth as syn
from gpu_helpers import assert_close, bf16_tensor, close_report, config_for, f32_tensor, upload_batch
from oracle import mtfm_oracle as O

pytestmark = pytest.mark.gpu


def _device_weights(lw):
    import hybrid_masked_attention_b200 as M
    b4 = lambda xs: [bf16_tensor(x) for x in xs]
    return M.V2LayerWeights(f32_tensor(lw.rms_w), b4(lw.w_uq), bf16_tensor(lw.w_kv), bf16_tensor(lw.w_o),
                            f32_tensor(lw.gamma), f32_tensor(lw.beta), f32_tensor(lw.rms_w2), b4(lw.w_gate),
                            b4(lw.w_up), b4(lw.w_down))


def _run(batch, heads, d, dff, lw, X0):
    import hybrid_masked_attention_b200 as M
    cfg = config_for(batch, heads)
    meta = M.alloc_meta(cfg)
    M.pack(cfg, *upload_batch(batch), meta)
    M.pack_check(meta)
    ws = torch.empty(M.v2_workspace_bytes(cfg, d, dff), dtype=torch.uint8, device="cuda")
    x = torch.from_numpy(X0.astype(np.float32)).cuda()
    M.v2_target_layer_fwd(cfg, meta, d, dff, _device_weights(lw), x, ws)
    M.pack_check(meta)
    return x.cpu().numpy().astype(np.float64)


BATCHES = {
    "sweep_n512": lambda: syn.sweep_batch(512, v2=True, B=4, seed=1013),
    # ragged: users without targets, one target, a tile boundary inside the T rows
    "ragged": lambda: syn.fixed_batch([300, 17, 64, 5, 0], [40, 3, 0, 2, 0], [32, 0, 136, 4, 8], 1014, v2_subtokens=4),
}


@pytest.mark.parametrize("bname", sorted(BATCHES))
@pytest.mark.parametrize("heads", [syn.PAIR_HEADS, syn.Heads(4, 1, 64)], ids=["hq8_hkv2", "hq4_hkv1"])
def test_v2_layer_matches_oracle(bname, heads, cuda_ok):
    b, d, dff = BATCHES[bname](), 512, 1024
    lw = syn.v2_layer_weights(heads, d, dff, 81, std=0.05, std_o=0.02, std_ffn=0.03)
    X0 = syn.bf16_bits_to_f32(syn.stack_input(b, d, 81)).astype(np.float64)
    got = _run(b, heads, d, dff, lw, X0)
    ref = O.v2_target_layer(b, heads, X0, lw)
    trow = O.t_row_index(b)
    hr = np.setdiff1d(np.arange(b.total_tokens), trow)
    assert np.array_equal(got[hr], X0[hr]), "the V2 Target layer changed H/R rows"
    assert_close(got[trow], ref[trow], f"X' T rows ({bname})")
    # the layer moves the T rows far beyond the tolerance (the check is not automatic)
    rel, _, _ = close_report(X0[trow], ref[trow])
    assert rel > 0.1


def test_v2_rejects_v1_batches(cuda_ok):
    import hybrid_masked_attention_b200 as M
    b = syn.pair_batch(4, 1015)
    cfg = config_for(b, syn.PAIR_HEADS)
    assert M._lib.mtfm_v2_workspace_bytes(__import__("ctypes").byref(cfg.c()), 512, 1024) == 0
