"""The C-ABI library builds, loads and exports every symbol include/mtfm.h declares;
host-side argument checks reject bad input before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _build():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_mtfm_build", os.path.join(ROOT, "hybrid_masked_attention_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="module")
def lib():
    path = _build()
    return ctypes.CDLL(path)


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "mtfm.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mtfm_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    syms = declared_symbols()
    assert len(syms) >= 10
    for s in syms:
        assert hasattr(lib, s), f"{s} missing from libmtfm.so"


def test_binding_wraps_every_symbol(lib):
    import hybrid_masked_attention_b200 as m
    assert set(declared_symbols()) == set(m.EXPORTED)


def _cfg(**kw):
    import hybrid_masked_attention_b200 as m
    base = dict(batch=2, total_tokens=20, total_r=4, total_t=4, hq=8, hkv=2, head_dim=64)
    base.update(kw)
    return m.Config(**base).c()


@pytest.mark.parametrize("kw,status", [
    (dict(hq=6, hkv=4), 1),           # hq % hkv != 0
    (dict(head_dim=48), 3),           # unsupported head_dim
    (dict(hq=16, hkv=1, head_dim=32), 3),   # r > 8
    (dict(batch=-1), 1),
    (dict(total_r=30), 1),            # R + T exceed the token total
    (dict(v2_subtokens=3), 1),
])
def test_invalid_config_rejected_before_launch(lib, kw, status):
    import hybrid_masked_attention_b200 as m
    c = _cfg(**kw)
    assert m._lib.mtfm_meta_bytes(ctypes.byref(c)) == 0
    st = m._lib.mtfm_pack(ctypes.byref(c), None, None, None, None, None, None, 0, None)
    assert st == status


def test_null_and_misaligned_pointers_rejected(lib):
    import hybrid_masked_attention_b200 as m
    c = _cfg()
    # null metadata block
    assert m._lib.mtfm_pack(ctypes.byref(c), 1024, 1024, 1024, 1024, 1024, None, 1 << 20, None) == 1
    # metadata block not 256-byte aligned
    assert m._lib.mtfm_pack(ctypes.byref(c), 1024, 1024, 1024, 1024, 1024, 4096 + 16, 1 << 20, None) == 1
    # too small
    need = m._lib.mtfm_meta_bytes(ctypes.byref(c))
    assert m._lib.mtfm_pack(ctypes.byref(c), 1024, 1024, 1024, 1024, 1024, 4096, need - 1, None) == 4
    # attention with missing K
    assert m._lib.mtfm_attn_full_fwd(ctypes.byref(c), 4096, 4096, None, 4096, 4096, None, None,
                                     4096, 4096, None, None) == 1
    # misaligned Q
    assert m._lib.mtfm_attn_full_fwd(ctypes.byref(c), 4096, 4096 + 2, 4096, 4096, 4096, None, None,
                                     4096, 4096, None, None) == 1
    # gamma without beta
    assert m._lib.mtfm_attn_target_fwd(ctypes.byref(c), 4096, 4096, 4096, 4096, 4096, 4096, None,
                                       4096, 4096, 4096, None) == 1
    # the bf16-Y forwards check the same arguments: missing K, misaligned Y, gamma without beta
    assert m._lib.mtfm_attn_full_fwd_bf16y(ctypes.byref(c), 4096, 4096, None, 4096, 4096, None, None,
                                           4096, 4096, None, None) == 1
    assert m._lib.mtfm_attn_full_fwd_bf16y(ctypes.byref(c), 4096, 4096, 4096, 4096, 4096, None, None,
                                           4096 + 2, 4096, None, None) == 1
    assert m._lib.mtfm_attn_target_fwd_bf16y(ctypes.byref(c), 4096, 4096, 4096, 4096, 4096, 4096, None,
                                             4096, 4096, 4096, None) == 1
    # cached-prefix Target attention: missing candidate keys, misaligned Q, and a head shape
    # the tensor-core Target kernel does not take
    c64 = _cfg(head_dim=64)
    assert m._lib.mtfm_attn_target_cached(ctypes.byref(c64), 4096, 4096, 4096, 4096, None, 4096, 4096, None) == 1
    assert m._lib.mtfm_attn_target_cached(ctypes.byref(c64), 4096, 4096 + 2, 4096, 4096, 4096, 4096, 4096,
                                          None) == 1
    assert m._lib.mtfm_attn_target_cached_fwd(ctypes.byref(c64), 4096, 4096, 4096, 4096, 4096, 4096, 4096,
                                              4096, None, 4096, 4096, None, None) == 1   # gamma without beta
    c128 = _cfg(head_dim=128)   # head_dim 128: no tensor-core Target kernel
    assert m._lib.mtfm_attn_target_cached(ctypes.byref(c128), 4096, 4096, 4096, 4096, 4096, 4096, 4096,
                                          None) == 3
    c8 = _cfg(hq=8, hkv=1, head_dim=32)   # r = 8 at head_dim 32 is taken: the missing candidate V is the error
    assert m._lib.mtfm_attn_target_cached(ctypes.byref(c8), 4096, 4096, 4096, 4096, 4096, None, 4096,
                                          None) == 1
    c3 = _cfg(hq=6, hkv=2, head_dim=64)   # r = 3: none either
    assert m._lib.mtfm_attn_target_cached(ctypes.byref(c3), 4096, 4096, 4096, 4096, 4096, 4096, 4096,
                                          None) == 3
    # backward workspace too small
    ws = m._lib.mtfm_bwd_workspace_bytes(ctypes.byref(c), 0)
    assert ws > 0
    args = [4096] * 17
    args[5], args[6], args[14], args[15] = None, None, None, None   # no GLN
    assert m._lib.mtfm_attn_full_bwd(ctypes.byref(c), *args, ws - 1, None) == 4


def test_status_strings(lib):
    import hybrid_masked_attention_b200 as m
    for s in range(9):
        assert m._lib.mtfm_status_string(s)
        assert b"unknown" not in m._lib.mtfm_status_string(s)
    assert b"unknown" in m._lib.mtfm_status_string(99)


def test_debug_bounds_queries(lib):
    """The shipped library is the normal build; the site query checks its arguments."""
    import hybrid_masked_attention_b200 as m
    assert m._lib.mtfm_debug_bounds_build() == 0
    assert m._lib.mtfm_debug_site(None, None, None) == 1


def test_meta_capacity_bounds(lib):
    import hybrid_masked_attention_b200 as m
    c = _cfg(batch=3, total_tokens=300, total_r=10, total_t=129)
    assert m._lib.mtfm_max_items(ctypes.byref(c), 0) == (300 + 127) // 128 + 3
    assert m._lib.mtfm_max_items(ctypes.byref(c), 1) == (129 + 127) // 128 + 3


def test_stack_arguments_rejected_before_launch(lib):
    import hybrid_masked_attention_b200 as m
    c = _cfg()
    W = m.CLayerWeights
    assert m._lib.mtfm_stack_workspace_bytes(ctypes.byref(c), 512) > 0
    assert m._lib.mtfm_stack_workspace_bytes(ctypes.byref(c), 96) == 0     # d_model not a multiple of 64
    assert m._lib.mtfm_stack_workspace_bytes(ctypes.byref(c), 2048) == 0   # d_model above 1024
    ws = m._lib.mtfm_stack_workspace_bytes(ctypes.byref(c), 512)
    full = W(4096, 4096, None, 4096, 4096, 4096)
    tgt = W(4096, 4096, 4096, 4096, None, None)
    # Full layer given a w_kv, Target layer without one
    assert m._lib.mtfm_layer_fwd(ctypes.byref(c), 4096, 512, 0, ctypes.byref(tgt), 4096, 4096, ws, None) == 1
    assert m._lib.mtfm_layer_fwd(ctypes.byref(c), 4096, 512, 1, ctypes.byref(full), 4096, 4096, ws, None) == 1
    # gamma without beta
    bad = W(4096, 4096, None, 4096, 4096, None)
    assert m._lib.mtfm_layer_fwd(ctypes.byref(c), 4096, 512, 0, ctypes.byref(bad), 4096, 4096, ws, None) == 1
    # misaligned X, workspace too small or misaligned
    assert m._lib.mtfm_layer_fwd(ctypes.byref(c), 4096, 512, 0, ctypes.byref(full), 4096 + 4, 4096, ws, None) == 1
    assert m._lib.mtfm_layer_fwd(ctypes.byref(c), 4096, 512, 0, ctypes.byref(full), 4096, 4096, ws - 1, None) == 4
    assert m._lib.mtfm_layer_fwd(ctypes.byref(c), 4096, 512, 0, ctypes.byref(full), 4096, 4096 + 16, ws, None) == 1
    # unknown layer kind; one bad layer among good ones stops the whole stack
    arr = (W * 2)(full, tgt)
    assert m._lib.mtfm_stack_fwd(ctypes.byref(c), 4096, 512, 2, b"FX", arr, 4096, 4096, ws, None) == 1
    arr2 = (W * 2)(full, full)
    assert m._lib.mtfm_stack_fwd(ctypes.byref(c), 4096, 512, 2, b"FT", arr2, 4096, 4096, ws, None) == 1
    # no layers: nothing to do
    assert m._lib.mtfm_stack_fwd(ctypes.byref(c), 4096, 512, 0, None, None, 4096, 4096, ws, None) == 0


def test_selftest_arguments(lib):
    import hybrid_masked_attention_b200 as m
    assert m._lib.mtfm_selftest_wait_timeout(None, 1000, None) == 1
    assert m._lib.mtfm_selftest_wait_timeout(4096 + 16, 1000, None) == 1
    assert m._lib.mtfm_selftest_wait_timeout(4096, 0, None) == 1
    assert m._lib.mtfm_selftest_wait_timeout(4096, 5_000_000_000, None) == 1


def test_v2_layer_host_checks(lib):
    import hybrid_masked_attention_b200 as m
    ok = m.Config(batch=2, total_tokens=40, total_r=8, total_t=8, hq=8, hkv=2, head_dim=64, v2_subtokens=4)
    assert lib.mtfm_v2_workspace_bytes(ctypes.byref(ok.c()), 512, 1024) > 0
    v1 = m.Config(batch=2, total_tokens=40, total_r=8, total_t=8, hq=8, hkv=2, head_dim=64)
    assert lib.mtfm_v2_workspace_bytes(ctypes.byref(v1.c()), 512, 1024) == 0     # needs 4 sub-tokens
    assert lib.mtfm_v2_workspace_bytes(ctypes.byref(ok.c()), 512, 1000) == 0     # d_ff multiple of 64
    assert lib.mtfm_v2_workspace_bytes(ctypes.byref(ok.c()), 520, 1024) == 0     # d_model multiple of 64
    odd = m.Config(batch=2, total_tokens=40, total_r=8, total_t=6, hq=8, hkv=2, head_dim=64, v2_subtokens=4)
    assert lib.mtfm_v2_workspace_bytes(ctypes.byref(odd.c()), 512, 1024) == 0    # T rows in targets of 4
    # null weights: rejected before any launch
    st = lib.mtfm_v2_target_layer_fwd(ctypes.byref(ok.c()), ctypes.c_void_p(256), 512, 1024, None, None, None,
                                      ctypes.c_size_t(0), None)
    assert st == 1
