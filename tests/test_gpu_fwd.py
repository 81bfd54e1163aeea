"""Full and Target forward on the GPU (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import mtfm_synth as syn
from gpu_cases import BATCHES, HEADS
from gpu_helpers import assert_close, packed, upload_layer
from oracle import mtfm_oracle as O

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", "tiny", True), ("tiny", "tiny", False),
    ("pair", "pair", True), ("pair", "pair", False),
    ("edge", "pair", True), ("edge", "dh128", True), ("edge", "r8", True),
    ("edge", "dh256", True), ("v2_n512", "dh256", True), ("tiny", "dh256", False),
    ("pair", "dh256", True), ("v1_n2048", "dh256", False),
    ("v2_n512", "pair", True), ("v2_n1024", "pair", True), ("v1_n2048", "pair", True),
    ("pair", "r1", True), ("edge", "r1", True), ("pair", "r2", True), ("edge", "r2", True),
    ("v2_n512", "r2", True), ("v1_n2048", "r1", False),
    # head_dim 32 on the tcgen05 kernels: the tiny heads (r = 2) on larger batches, r = 1 and 4
    ("pair", "tiny", True), ("edge", "tiny", True), ("v1_n2048", "tiny", False),
    ("pair", "dh32_r1", True), ("edge", "dh32_r1", False), ("pair", "dh32_r4", True),
    ("edge", "dh32_r4", True), ("v2_n512", "dh32_r4", True),
    # r = 8: both tcgen05 kernels at head_dim 32 (16 T rows per Target sub-tile), the Target one at 64
    ("pair", "r8", True), ("v2_n512", "r8", True), ("pair", "r8_dh64", True), ("edge", "r8_dh64", False),
]


def _run(batch, heads, target, gln, seed=11):
    inp = syn.layer_inputs(batch, heads, target=target, seed=seed, gln=gln)
    s = packed(batch, heads)
    d = upload_layer(inp)
    f = s.target_fwd if target else s.full_fwd
    y, a, st = f(d["q"], d["k"], d["v"], d["u"], d["gamma"], d["beta"])
    torch.cuda.synchronize()
    ref = (O.target_fwd if target else O.full_fwd)(batch, heads, inp)
    return y.cpu().numpy(), a.cpu().numpy(), (None if st is None else st.cpu().numpy()), ref


@pytest.mark.parametrize("bname,hname,gln", CASES)
@pytest.mark.parametrize("target", [False, True], ids=["full", "target"])
def test_fwd_parity(bname, hname, gln, target, cuda_ok):
    b, hd = BATCHES[bname](), HEADS[hname]
    y, a, st, ref = _run(b, hd, target, gln)
    assert_close(a, ref["A"], "A")
    assert_close(y, ref["Y"], "Y")
    if gln and len(st):
        assert_close(st[:, 0], ref["mean"], "mean")
        assert_close(st[:, 1], ref["rstd"], "rstd")


def test_target_equals_full_t_rows_on_gpu(cuda_ok):
    """Target layer == T rows of a Full layer fed the same Q/U rows (GPU vs GPU)."""
    b, hd = BATCHES["pair"](), HEADS["pair"]
    full = syn.layer_inputs(b, hd, target=False, seed=21)
    so = O.offsets(b.N)
    trows = np.concatenate([np.arange(so[u] + b.L_H[u] + b.L_R[u], so[u + 1]) for u in range(b.B)])
    tgt = syn.LayerInputs(full.q[trows], full.k, full.v, full.u[trows], full.gamma, full.beta)
    s = packed(b, hd)
    df, dt = upload_layer(full), upload_layer(tgt)
    yf, af, _ = s.full_fwd(df["q"], df["k"], df["v"], df["u"], df["gamma"], df["beta"])
    yt, at, _ = s.target_fwd(dt["q"], dt["k"], dt["v"], dt["u"], dt["gamma"], dt["beta"])
    torch.cuda.synchronize()
    assert_close(at.cpu().numpy(), af.cpu().numpy()[trows], "A_T vs A_full[T]")
    assert_close(yt.cpu().numpy(), yf.cpu().numpy()[trows], "Y_T vs Y_full[T]")


def test_fwd_deterministic(cuda_ok):
    b, hd = BATCHES["pair"](), HEADS["pair"]
    inp = upload_layer(syn.layer_inputs(b, hd, target=False, seed=3))
    s = packed(b, hd)
    y1, a1, _ = s.full_fwd(inp["q"], inp["k"], inp["v"], inp["u"], inp["gamma"], inp["beta"])
    y2, a2, _ = s.full_fwd(inp["q"], inp["k"], inp["v"], inp["u"], inp["gamma"], inp["beta"])
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(a1, a2)


def test_work_counters_rewind(cuda_ok):
    """The persistent forward kernels draw work from counters in the metadata
    header and set them back to zero: repeated and interleaved Full / Target
    calls on one block all cover every tile."""
    b, hd = BATCHES["pair"](), HEADS["pair"]
    s = packed(b, hd)
    full = upload_layer(syn.layer_inputs(b, hd, target=False, seed=5))
    tgt = upload_layer(syn.layer_inputs(b, hd, target=True, seed=6))
    outs = []
    for _ in range(3):
        outs.append((s.full_fwd(full["q"], full["k"], full["v"], full["u"], full["gamma"], full["beta"]),
                     s.target_fwd(tgt["q"], tgt["k"], tgt["v"], tgt["u"], tgt["gamma"], tgt["beta"])))
    torch.cuda.synchronize()
    hdr = s.meta[:64].view(torch.int32).cpu().numpy()
    assert hdr[8] == 0, "error flag"
    assert (hdr[12:14] == 0).all(), f"work counters not rewound: {hdr[12:14]}"
    assert hdr[14] == 128 // (hd.hq // hd.hkv), "T rows per Target sub-tile"
    (yf0, af0, _), (yt0, at0, _) = outs[0]
    for (yf, af, _), (yt, at, _) in outs[1:]:
        assert torch.equal(af, af0) and torch.equal(yf, yf0)
        # Target A sums key-range partials with atomics: equal up to summation order
        assert_close(at.cpu().numpy(), at0.cpu().numpy(), "A_T repeat")
    ref_f = O.full_fwd(b, hd, syn.layer_inputs(b, hd, target=False, seed=5))
    ref_t = O.target_fwd(b, hd, syn.layer_inputs(b, hd, target=True, seed=6))
    for (yf, af, _), (yt, at, _) in outs:
        assert_close(af.cpu().numpy(), ref_f["A"], "A full")
        assert_close(at.cpu().numpy(), ref_t["A"], "A target")


@pytest.mark.parametrize("bname,hname", [("pair", "pair"), ("edge", "pair"), ("tiny", "tiny")])
@pytest.mark.parametrize("target", [False, True], ids=["full", "target"])
def test_bf16y_is_rounded_fp32_y(bname, hname, target, cuda_ok):
    """The bf16-Y entry points store exactly the fp32 entry points' Y rounded to nearest bf16,
    with the same A and row statistics; the fp32 Y is checked against the oracle above."""
    import hybrid_masked_attention_b200 as M
    b, hd = BATCHES[bname](), HEADS[hname]
    inp = syn.layer_inputs(b, hd, target=target, seed=13, gln=True)
    s = packed(b, hd)
    d = upload_layer(inp)
    rows = b.total_t if target else b.total_tokens
    f32 = dict(dtype=torch.float32, device="cuda")
    y, a, st = (torch.empty(rows, hd.dq, **f32), torch.empty(rows, hd.dq, **f32), torch.empty(rows, 2, **f32))
    yb = torch.empty(rows, hd.dq, dtype=torch.bfloat16, device="cuda")
    ab, stb = torch.empty_like(a), torch.empty_like(st)
    f, fb = (M.attn_target_fwd, M.attn_target_fwd_bf16y) if target else (M.attn_full_fwd, M.attn_full_fwd_bf16y)
    f(s.cfg, s.meta, d["q"], d["k"], d["v"], d["u"], d["gamma"], d["beta"], y, a, st)
    fb(s.cfg, s.meta, d["q"], d["k"], d["v"], d["u"], d["gamma"], d["beta"], yb, ab, stb)
    M.pack_check(s.meta)
    torch.cuda.synchronize()
    if not target:  # one unit writes each row of A: both calls compute the same bits
        assert torch.equal(ab, a) and torch.equal(stb, st)
        assert torch.equal(yb, y.to(torch.bfloat16)), "bf16 Y differs from the rounded fp32 Y"
    else:  # key chunks may add into A in either order: Y within half a bf16 ulp (+ that noise)
        assert torch.allclose(ab, a, rtol=1e-5, atol=1e-6)
        yf = yb.float()
        bound = y.abs() * 2.0 ** -8 + 1e-5 * y.pow(2).mean().sqrt()
        assert bool(((yf - y).abs() <= bound).all()), "bf16 Y is not the rounded fp32 Y"
    ref = (O.target_fwd if target else O.full_fwd)(b, hd, inp)
    assert_close(y.cpu().numpy(), ref["Y"], "Y (fp32 entry)")
