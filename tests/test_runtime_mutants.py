"""The CPU tests of the C ABI must catch plausible mistakes in the library's
host runtime (config validation, the layout geometry, the memory formula and
the append planner: free-list order, admission, block placement, prefix
sharing).  Each case plants one mistake in a copy of csrc/kvq_runtime.cpp,
compiles it with the library's flags, links it with the library's kernel
objects, and runs tests/test_abi.py against that build (host-only handles, no
GPU): at least one test must fail.  The unaltered copy, built the same way,
must pass them all.  The committed sources are never modified, and the case
runs only on a machine without a GPU, so no altered build ever meets one
(host-only handles launch nothing in any case).  (Alignment
changes to the chunk sections are not in the list: with pages of at least 16
tokens every section is already a multiple of 32 bytes, so they change
nothing.)"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

import pytest

from quantized_kv_cache_14_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(kbuild.CSRC, "kvq_runtime.cpp")

# (name, text in the runtime's source, the planted mistake)
MUTANTS = [
    ("splitmix64_shift", "  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;",
     "  z = (z ^ (z >> 28)) * 0x94D049BB133111EBull;"),
    ("fisher_yates_range", "    const uint64_t j = splitmix64(sm) % uint64_t(i + 1);",
     "    const uint64_t j = splitmix64(sm) % uint64_t(i);"),
    ("pages_rounded_down", "  if (c.residual == 0) return (len + c.page - 1) / c.page;",
     "  if (c.residual == 0) return len / c.page;"),
    ("blocks_needed_not_net", "    need += nb - h->nblk[size_t(s)];", "    need += nb;"),
    ("blocks_taken_from_the_back", "  auto take = [&]() { return h->freelist[size_t(allocs++)]; };",
     "  auto take = [&]() { return h->freelist[h->freelist.size() - 1 - size_t(allocs++)]; };"),
    ("freed_blocks_to_front", "    if (--h->refcnt[size_t(e)] == 0) h->freelist.push_back(e);",
     "    if (--h->refcnt[size_t(e)] == 0) h->freelist.push_front(e);"),
    ("prefix_shared_by_page_under_a_window", "  const int32_t unit = c.residual ? c.residual : c.page;",
     "  const int32_t unit = c.page;"),
    ("key_scale_slice", "    g.kslice = D / (c.g_k / c.page);", "    g.kslice = D / c.g_k;"),
    ("formula_without_key_metadata",
     "  const uint64_t kmeta = (elems * meta + uint64_t(cfg->g_k) - 1) / uint64_t(cfg->g_k);",
     "  const uint64_t kmeta = 0;"),
    ("page_of_8_accepted", "  if (c->page < 16 || (c->page & (c->page - 1)) != 0)",
     "  if (c->page < 8 || (c->page & (c->page - 1)) != 0)"),
    ("fail_alloc_after_off_by_one", "  if (c.fail_alloc_after >= 0 && h->alloc_count + need > c.fail_alloc_after)",
     "  if (c.fail_alloc_after >= 0 && h->alloc_count + need >= c.fail_alloc_after)"),
    ("table_width_off_by_one", "    if (nb > MB) return fail(KVQ_ERR_OOM", "    if (nb >= MB) return fail(KVQ_ERR_OOM"),
    ("new_blocks_not_held", "  for (int64_t j = 0; j < allocs; ++j) h->refcnt[size_t(h->freelist[size_t(j)])] = 1;",
     "  for (int64_t j = 0; j < allocs; ++j) h->refcnt[size_t(h->freelist[size_t(j)])] = 2;"),
    ("shared_blocks_not_counted", "    ++h->refcnt[size_t(b)];", "    (void)b;"),
    ("group_flushed_one_token_early", "      if (pos % R == R - 1) {", "      if (pos % R == R - 2) {"),
    ("value_group_of_16_accepted",
     "  if (c->g_v != 32 && c->g_v != 64 && c->g_v != 128) return fail(KVQ_ERR_UNSUPPORTED",
     "  if (c->g_v != 16 && c->g_v != 32 && c->g_v != 64 && c->g_v != 128) return fail(KVQ_ERR_UNSUPPORTED"),
    ("window_length_not_checked", "    if (c->residual != c->g_k) return fail(KVQ_ERR_INVALID_ARG",
     "    if (c->residual < 0) return fail(KVQ_ERR_INVALID_ARG"),
]

_RUN = ("import sys, pytest\n"
        "import quantized_kv_cache_14_b200.kvq as k\n"
        "k.LIB_PATH = sys.argv[1]\n"
        "sys.exit(pytest.main(['tests/test_abi.py', '-x', '-q', '-p', 'no:cacheprovider', '-m', 'not gpu']))\n")


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    """Builds the unaltered copy and every mutant of the runtime, links each
    with the library's kernel objects and runs the ABI tests on it (several
    at once); maps name -> (return code, output tail)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("altered builds of the library run on machines without a GPU only")
    if shutil.which(kbuild.NVCC) is None and not os.path.exists(kbuild.NVCC):
        pytest.skip("nvcc is not available")
    kbuild.build()   # the kernel objects the copies link with
    objs = [os.path.join(kbuild.BUILD, os.path.splitext(s)[0] + ".o") for s in kbuild.SOURCES
            if s != "kvq_runtime.cpp"]
    with open(SRC) as f:
        src = f.read()
    cases = [("unaltered", src)]
    for name, old, new in MUTANTS:
        assert src.count(old) == 1, f"{name}: the text to alter must occur once in the runtime"
        cases.append((name, src.replace(old, new)))
    root = tmp_path_factory.mktemp("runtime_mutants")

    def one(case):
        name, text = case
        d = root / name
        d.mkdir()
        cpp, obj, lib = d / "kvq_runtime.cpp", d / "kvq_runtime.o", d / "libkvq.so"
        cpp.write_text(text)
        subprocess.run([kbuild.NVCC, *kbuild.FLAGS, "-c", str(cpp), "-o", str(obj)], check=True,
                       capture_output=True)
        subprocess.run([kbuild.NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", str(obj), *objs,
                        "-o", str(lib), "-lcudart"], check=True, capture_output=True)
        r = subprocess.run([sys.executable, "-c", _RUN, str(lib)], cwd=ROOT, capture_output=True, text=True,
                           timeout=600)
        for built in (obj, lib):   # 8 MB each: not kept once the run is over
            built.unlink()
        return name, (r.returncode, (r.stdout + r.stderr)[-3000:])

    with cf.ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        return dict(ex.map(one, cases))


def test_unaltered_copy_passes_the_abi_tests(outcomes):
    rc, tail = outcomes["unaltered"]
    assert rc == 0, tail


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_abi_tests_catch_a_planted_mistake(outcomes, name):
    rc, tail = outcomes[name]
    # a failing test (exit 1), or a test run that the mistake crashes (killed by a signal)
    assert rc == 1 or rc < 0, f"no test failed (pytest exit {rc}) with the mistake {name} planted:\n{tail}"
