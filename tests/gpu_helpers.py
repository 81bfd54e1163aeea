"""Shared helpers of the GPU parity tests: upload seeded inputs, call the C ABI, compare."""
from __future__ import annotations

import numpy as np
import torch

import mtfm_synth as syn

# Parity bar for floating-point outputs (bf16 inputs, fp32 accumulation):
# relative L2 <= 1e-2 and max |err| <= 2e-2 * RMS(reference), per output tensor.
REL_L2 = 1e-2
MAX_ABS_RMS = 2e-2


def close_report(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if ref.size == 0:
        return 0.0, 0.0, 0.0
    err = got - ref
    nref = np.linalg.norm(ref)
    rms = float(np.sqrt(np.mean(ref * ref)))
    rel = float(np.linalg.norm(err) / nref) if nref > 0 else float(np.linalg.norm(err))
    mx = float(np.abs(err).max())
    return rel, mx, rms


def assert_close(got, ref, name=""):
    got = np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    rel, mx, rms = close_report(got, ref)
    assert rel <= REL_L2, f"{name}: rel-L2 {rel:.3e} > {REL_L2}"
    bound = MAX_ABS_RMS * rms if rms > 0 else 1e-6
    assert mx <= bound, f"{name}: max-abs {mx:.3e} > {MAX_ABS_RMS} * RMS ({bound:.3e})"


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def f32_tensor(x, device="cuda"):
    if x is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def config_for(batch: syn.JaggedBatch, heads: syn.Heads, **kw):
    from hybrid_masked_attention_b200 import Config
    return Config(batch.B, batch.total_tokens, batch.total_r, batch.total_t, heads.hq, heads.hkv,
                  heads.dh, batch.v2_subtokens, **kw)


def upload_batch(batch: syn.JaggedBatch, device="cuda"):
    it = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dtype=dt)).to(device)
    return (it(batch.L_H, np.int32), it(batch.L_R, np.int32), it(batch.L_T, np.int32),
            it(batch.r_ts, np.int64), it(batch.t_exp, np.int64))


def packed(batch, heads, device="cuda", **kw):
    from hybrid_masked_attention_b200.session import HybridAttention
    cfg = config_for(batch, heads, **kw)
    s = HybridAttention(cfg, device)
    s.pack(*upload_batch(batch, device), check=True)
    return s


def upload_layer(inp: syn.LayerInputs, device="cuda"):
    return dict(q=bf16_tensor(inp.q, device), k=bf16_tensor(inp.k, device),
                v=bf16_tensor(inp.v, device), u=bf16_tensor(inp.u, device),
                gamma=f32_tensor(inp.gamma, device), beta=f32_tensor(inp.beta, device),
                dy=None if inp.dy is None else bf16_tensor(inp.dy, device))


def gpu_mask_rows(meta: dict, batch: syn.JaggedBatch, u: int) -> np.ndarray:
    """Dense visibility of user u rebuilt from the GPU metadata: prefix [0, kv_end) + sibling block."""
    so = int(meta["seq_off"][u])
    LH, LR, LT = int(batch.L_H[u]), int(batch.L_R[u]), int(batch.L_T[u])
    N = LH + LR + LT
    kv = meta["kv_end"][so:so + N]
    cols = np.arange(N)
    M = cols[None, :] < kv[:, None]
    s = batch.v2_subtokens
    for i in range(LH + LR, N):
        lo = LH + LR + ((i - LH - LR) // s) * s
        M[i, lo:lo + s] = True
    return M
