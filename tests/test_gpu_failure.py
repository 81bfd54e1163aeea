"""Failure detection on the GPU without a fault: a bounded wait that runs out is
reported through the metadata block, later kernels on that block do nothing, and
the context stays usable (a fresh pack on the same block works again)."""
import time

import numpy as np
import pytest
import torch

import mtfm_synth as syn
from gpu_helpers import assert_close, packed, upload_layer
from oracle import mtfm_oracle as O

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_ok):
    import hybrid_masked_attention_b200 as M
    b, hd = syn.tiny_batch(), syn.TINY_HEADS
    s = packed(b, hd)
    t0 = time.perf_counter()
    M.selftest_wait_timeout(s.meta, 2_000_000)   # ~1 ms of SM clock
    with pytest.raises(M.MtfmError) as e:
        M.pack_check(s.meta)
    assert e.value.status == 6, e.value           # MTFM_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 30.0
    # every later kernel on this block is a no-op: outputs keep their sentinel
    inp = upload_layer(syn.layer_inputs(b, hd, target=False, seed=3))
    y = torch.full((b.total_tokens, hd.dq), 7.0, device="cuda")
    a = torch.full_like(y, 7.0)
    st = torch.empty(b.total_tokens, 2, device="cuda")
    s.full_fwd(inp["q"], inp["k"], inp["v"], inp["u"], inp["gamma"], inp["beta"], out=(y, a, st))
    torch.cuda.synchronize()
    assert bool((a == 7.0).all()) and bool((y == 7.0).all())
    # the context is healthy: re-pack the same block and compute
    from gpu_helpers import upload_batch
    s.pack(*upload_batch(b), check=True)
    y, a, _ = s.full_fwd(inp["q"], inp["k"], inp["v"], inp["u"], inp["gamma"], inp["beta"])
    torch.cuda.synchronize()
    ref = O.full_fwd(b, hd, syn.layer_inputs(b, hd, target=False, seed=3))
    assert_close(a.cpu().numpy(), ref["A"], "A after recovery")
