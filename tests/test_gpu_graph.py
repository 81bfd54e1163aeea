"""The forward path captured in a CUDA graph and replayed: pack + Full layer + Target layer,
and the 16-layer stack.  Replays must give the eager results (the Full layer and the stack
bit for bit; the Target layer, whose partial sums land in A through TMA reduce-adds in any
order, to within fp32 summation order) and, for the pair step, the oracle's."""
import numpy as np
import pytest
import torch

import hybrid_masked_attention_b200 as M
import mtfm_synth as syn
from gpu_helpers import assert_close, bf16_tensor, config_for, f32_tensor, upload_batch, upload_layer
from oracle import mtfm_oracle as O

pytestmark = pytest.mark.gpu


def _pair_step_tensors(b, hd):
    cfg = config_for(b, hd)
    fi = syn.layer_inputs(b, hd, target=False, seed=11)
    ti = syn.layer_inputs(b, hd, target=True, seed=111)
    f32 = dict(dtype=torch.float32, device="cuda")
    N, T = b.total_tokens, b.total_t
    out = {"A_f": torch.empty(N, hd.dq, **f32), "Y_f": torch.empty(N, hd.dq, **f32), "S_f": torch.empty(N, 2, **f32),
           "A_t": torch.empty(T, hd.dq, **f32), "Y_t": torch.empty(T, hd.dq, **f32), "S_t": torch.empty(T, 2, **f32)}
    return cfg, fi, ti, upload_layer(fi), upload_layer(ti), out


def test_pair_step_graph_replay(cuda_ok):
    b, hd = syn.pair_batch(8, 1001), syn.PAIR_HEADS
    cfg, fi, ti, f, t, o = _pair_step_tensors(b, hd)
    lens = upload_batch(b)
    meta = M.alloc_meta(cfg)
    st = torch.cuda.Stream()

    def step():
        M.pack(cfg, *lens, meta, st)
        M.attn_full_fwd(cfg, meta, f["q"], f["k"], f["v"], f["u"], f["gamma"], f["beta"],
                        o["Y_f"], o["A_f"], o["S_f"], st)
        M.attn_target_fwd(cfg, meta, t["q"], t["k"], t["v"], t["u"], t["gamma"], t["beta"],
                          o["Y_t"], o["A_t"], o["S_t"], st)

    with torch.cuda.stream(st):
        step()
    torch.cuda.synchronize()
    M.pack_check(meta)
    eager = {k: v.clone() for k, v in o.items()}
    for v in o.values():
        v.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        step()
    with torch.cuda.stream(st):
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    M.pack_check(meta)
    for k in ("A_f", "Y_f", "S_f"):
        assert torch.equal(o[k], eager[k]), k
    for k in ("A_t", "Y_t", "S_t"):
        torch.testing.assert_close(o[k], eager[k], rtol=1e-5, atol=1e-6)
    ref_f = O.full_fwd(b, hd, fi)
    ref_t = O.target_fwd(b, hd, ti)
    assert_close(o["Y_f"].cpu().numpy(), ref_f["Y"], "Y full")
    assert_close(o["Y_t"].cpu().numpy(), ref_t["Y"], "Y target")


def test_stack_graph_replay(cuda_ok):
    b, hd, d = syn.pair_batch(4, 1002), syn.PAIR_HEADS, 128
    cfg = config_for(b, hd)
    meta = M.alloc_meta(cfg)
    M.pack(cfg, *upload_batch(b), meta)
    M.pack_check(meta)
    layers = []
    for lw in syn.stack_weights(hd, d, seed=7, kinds=("F", "T")):
        layers.append(M.LayerWeights(lw.kind, f32_tensor(lw.rms_w), bf16_tensor(lw.w_in),
                                     None if lw.w_kv is None else bf16_tensor(lw.w_kv), bf16_tensor(lw.w_o),
                                     f32_tensor(lw.gamma), f32_tensor(lw.beta)))
    x0 = torch.from_numpy(syn.bf16_bits_to_f32(syn.stack_input(b, d, seed=7))).float().cuda()
    ws = torch.empty(M.stack_workspace_bytes(cfg, d), dtype=torch.uint8, device="cuda")
    st = torch.cuda.Stream()
    x_eager = x0.clone()
    with torch.cuda.stream(st):
        M.stack_fwd(cfg, meta, d, layers, x_eager, ws, st)
    torch.cuda.synchronize()
    x = x0.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        M.stack_fwd(cfg, meta, d, layers, x, ws, st)
    x.copy_(x0)
    with torch.cuda.stream(st):
        g.replay()
    torch.cuda.synchronize()
    M.pack_check(meta)
    torch.testing.assert_close(x, x_eager, rtol=1e-5, atol=1e-5)
