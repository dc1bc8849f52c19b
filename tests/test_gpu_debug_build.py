"""The debug build (libkvq_debug.so, KVQ_DEBUG=1): its kernels check every
index they compute -- plan entries, window slots, pool chunks, split-K record
slots, and each shared-memory page a warp reads against the pages its unit's
copies filled -- and report a failure in the device error word instead of
making the access.  On valid inputs no check may fire: a child process with
KVQ_DEBUG=1 loads the debug library and runs parity suites whose every call
asserts a clean error word (and matches the oracle), the corrupted-table case
included."""
import os
import subprocess
import sys

import pytest

from quantized_kv_cache_14_b200 import build as kbuild

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_runs_parity_with_a_clean_error_word():
    kbuild.build(debug=True)
    env = dict(os.environ, KVQ_DEBUG="1")
    which = subprocess.run([sys.executable, "-c", "from quantized_kv_cache_14_b200 import kvq; print(kvq.lib()._name)"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert which.returncode == 0, which.stderr[-2000:]
    assert which.stdout.strip().endswith("libkvq_debug.so"), which.stdout
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        "tests/test_gpu_parity.py", "-k",
                        "small_bulk or split_k or merge_rows or shared_prefix or corrupted or bad_lengths",
                        "tests/test_gpu_edges.py"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    summary = r.stdout.strip().splitlines()[-1]
    assert " passed" in summary and "failed" not in summary, summary
