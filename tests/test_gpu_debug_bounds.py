"""The small parity cases once more under the bounds-checked build of the library.

The bounds-checked build (-DMTFM_DEBUG_BOUNDS) tests every TMA coordinate (inner
coordinate 16-byte aligned, box inside its tensor) and the global row indices the
kernels compute before using them, records a failure in the metadata header
(MTFM_ERR_BOUNDS from mtfm_pack_check, the site from mtfm_debug_site) and skips the
access.  It stands in for a device memory checker.  The test builds that variant,
then runs the tiny and edge-batch parity tests of every kernel family (tcgen05 and
mma.sync forward and backward, head_dim 32 / 64 / 128 / 256, GQA r = 1 .. 8, the
cached-prefix layer, the stack's GEMMs) in a child process that loads it; those
tests call mtfm_pack_check after their launches, which raises on a recorded failure.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CASES = ["tests/test_gpu_fwd.py", "tests/test_gpu_bwd.py", "tests/test_gpu_cached.py",
         "tests/test_gpu_stack.py", "tests/test_gpu_debug_bounds.py"]


def test_small_cases_under_bounds_checked_build(cuda_ok):
    if os.environ.get("MTFM_LIBRARY"):
        pytest.skip("already running under another build")
    sys.path.insert(0, os.path.join(ROOT, "hybrid_masked_attention_b200"))
    import build
    lib = build.build(debug_bounds=True)
    env = dict(os.environ, MTFM_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", *CASES, "-q", "-x", "-m", "gpu", "-k",
                        "tiny or edge or bounds_checked_build_loaded", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail


def test_bounds_checked_build_loaded(cuda_ok):
    """Inside the child process: the loaded library is the checked build, no site recorded."""
    if not os.environ.get("MTFM_LIBRARY"):
        pytest.skip("runs in the bounds-checked child process only")
    import hybrid_masked_attention_b200 as M
    import mtfm_synth as syn
    from gpu_helpers import config_for, upload_batch
    assert M.debug_bounds_build()
    b = syn.tiny_batch()
    cfg = config_for(b, syn.TINY_HEADS)
    meta = M.alloc_meta(cfg)
    M.pack(cfg, *upload_batch(b), meta)
    M.pack_check(meta)
    assert M.debug_site(meta) == 0
