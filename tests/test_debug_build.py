"""The debug build (libgdr_debug.so, in-kernel bounds checks; see include/gdr.h).

On the CPU: the debug library exports the same C ABI as the release library and says which
build it is.  On the GPU: the small-shape parity suite (every kernel family: tensor-core
and CUDA-core forward, the split, the cross-GPU split's maps, the mixer, the backward, the
decode step, the wait-expiry path) runs once in a child process with GDR_DEBUG=1, where
tests/conftest.py checks after every test that no bounds check failed."""
import ctypes
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "linear_attention_recurrence_wy_b200")


def test_debug_library_exports_the_release_abi():
    rel, dbg = os.path.join(PKG, "libgdr.so"), os.path.join(PKG, "libgdr_debug.so")
    if not (os.path.exists(rel) and os.path.exists(dbg)):
        pytest.skip("libraries not built")
    from test_boundary import declared_functions
    L_rel, L_dbg = ctypes.CDLL(rel), ctypes.CDLL(dbg)
    for name in declared_functions():
        getattr(L_rel, name)
        getattr(L_dbg, name)
    assert L_rel.gdr_debug_build() == 0 and L_dbg.gdr_debug_build() == 1
    assert L_rel.gdr_debug_bounds_site() == 0 and L_dbg.gdr_debug_bounds_site() == 0


@pytest.mark.gpu
def test_small_shape_suite_passes_under_the_bounds_checks(cuda_ok):
    env = dict(os.environ, GDR_DEBUG="1")
    env.pop("GDR_PARITY_TABLE", None)
    files = ["tests/test_parity_chunk.py", "tests/test_parity_split.py", "tests/test_parity_seqpar.py",
             "tests/test_parity_mixer.py", "tests/test_parity_bwd.py", "tests/test_parity_decode.py",
             "tests/test_wait_expiry.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", *files, "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        "-k", "not full_size and not all_heads and not 1000_steps and not long_context"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-15:])
    assert r.returncode == 0, tail
    assert " passed" in tail
