"""The allocation-free Target-layer backward (mtfm_attn_target_bwd_static).

Callers that cannot allocate device memory (inside another allocator's pool,
or with all device memory reserved up front) use this entry point: it takes
no scratch block and runs on the library's own fixed device array.  Its
results must match mtfm_attn_target_bwd, which runs the same kernels on a
caller-provided scratch block, on two calls in a row (the second call sees
the array the first call left behind).

The first call on a device may commit the array (CUDA loads the module that
holds it lazily); the second call is checked to leave free device memory
unchanged.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes
import gc

import numpy as np
import pytest
import torch

import mtfm_synth as syn
from gpu_helpers import assert_close, packed, upload_layer

pytestmark = pytest.mark.gpu


def _outputs(batch, heads, seed):
    inp = syn.layer_inputs(batch, heads, target=True, seed=seed, gln=True, with_dy=True)
    s = packed(batch, heads)
    d = upload_layer(inp)
    y, a, st = s.target_fwd(d["q"], d["k"], d["v"], d["u"], d["gamma"], d["beta"])
    return s, d, a, st


def test_static_scratch_backward_matches_workspace_backward(cuda_ok):
    from hybrid_masked_attention_b200 import attn_target_bwd_static
    b, hd = syn.pair_batch(32, 1001), syn.PAIR_HEADS
    s, d, a, st = _outputs(b, hd, seed=23)
    ref = s.target_bwd(d["q"], d["k"], d["v"], d["u"], d["gamma"], d["beta"], a, st, d["dy"])
    torch.cuda.synchronize()
    f32 = dict(dtype=torch.float32, device="cuda")
    D, Dkv, N, T = hd.dq, hd.dkv, b.total_tokens, b.total_t
    for call in range(2):
        out = {"dq": torch.full((T, D), float("nan"), **f32), "dk": torch.full((N, Dkv), float("nan"), **f32),
               "dv": torch.full((N, Dkv), float("nan"), **f32), "du": torch.full((T, D), float("nan"), **f32),
               "dgamma": torch.full((3, D), float("nan"), **f32), "dbeta": torch.full((3, D), float("nan"), **f32)}
        torch.cuda.synchronize()
        # Python's cycle collector would otherwise free tensors left by earlier tests in the
        # middle of the measured call (torch's allocated-bytes counter then drops)
        gc.collect()
        gc.disable()
        try:
            free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
            attn_target_bwd_static(s.cfg, s.meta, d["q"], d["k"], d["v"], d["u"], d["gamma"], d["beta"], a, st,
                                   d["dy"], out["dq"], out["dk"], out["dv"], out["du"], out["dgamma"],
                                   out["dbeta"])
            torch.cuda.synchronize()
            free1, alloc1 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        finally:
            gc.enable()
        if call == 1:
            # the first call may load the library module that holds the array; the
            # second must not take any device memory
            assert free1 == free0, "the second call changed free device memory"
            assert alloc1 == alloc0, "the second call allocated through torch"
        for name in ("dq", "dk", "dv", "du", "dgamma", "dbeta"):
            assert_close(out[name].cpu().numpy(), ref[name].cpu().numpy(), f"call {call} {name}")


def test_static_scratch_rejects_oversized_problem(cuda_ok):
    import hybrid_masked_attention_b200 as M
    # about 20k T rows at hq*head_dim = 512 needs more than the 24 MiB array
    cfg = M.Config(batch=1, total_tokens=40000, total_r=0, total_t=20000, hq=8, hkv=2, head_dim=64)
    c = cfg.c()
    assert M._lib.mtfm_bwd_workspace_bytes(ctypes.byref(c), 1) > (24 << 20)
    st = M._lib.mtfm_attn_target_bwd_static(ctypes.byref(c), *([None] * 16), None)
    assert st == 4  # MTFM_ERR_WORKSPACE_TOO_SMALL, nothing launched
