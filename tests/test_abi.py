"""The C ABI on a machine without a GPU: the library loads, exports every
symbol include/kvq.h declares, validates configs, and its host-side planner
(host_only handles: no device memory, no kernels) places blocks exactly as the
oracle's allocator does."""
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import oracle as O
from quantized_kv_cache_14_b200 import build as kbuild
from quantized_kv_cache_14_b200 import kvq
from tests.conftest import ROOT, read_golden


@pytest.fixture(scope="module", autouse=True)
def built():
    kbuild.build()


def header_functions():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", src)))


def test_exports_match_header():
    declared = header_functions()
    assert declared == sorted(kvq.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", kvq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (kvq_[a-z0-9_]+)$", out, flags=re.M))
    assert set(declared) <= exported
    L = kvq.lib()
    for name in declared:
        assert getattr(L, name) is not None


FMTS = {
    "int8_tok_p16": dict(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=16),
    "int8_tok_p512_fp32": dict(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=1, residual=0, page=512),
    "int4_chan64": dict(bits=4, asym=0, k_axis=1, g_k=64, g_v=64, scale_fp32=0, residual=64, page=16),
    "int2_asym_chan32": dict(bits=2, asym=1, k_axis=1, g_k=32, g_v=32, scale_fp32=0, residual=32, page=16),
    "int4_chan64_p32": dict(bits=4, asym=0, k_axis=1, g_k=64, g_v=32, scale_fp32=0, residual=64, page=32),
    "int4_asym_tok32": dict(bits=4, asym=1, k_axis=0, g_k=32, g_v=32, scale_fp32=0, residual=0, page=32),
    "bf16_control_p16": dict(bits=16, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=16),
    "fp8_p32": dict(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=32, fp8=1),
}


def cfg_of(name, host_only=1, **kw):
    f = dict(FMTS[name])
    base = dict(h_q=8, h_kv=2, d_h=128, max_seqs=4, num_blocks=200, max_blocks_per_seq=128,
                seed=11, fail_alloc_after=-1, host_only=host_only, device=0)
    base.update(kw)
    return kvq.make_config(**f, **base), {**f, **base}


@pytest.mark.parametrize("name", list(FMTS))
def test_layout_matches_oracle_geometry(name):
    cfg, d = cfg_of(name)
    lay = kvq.kvq_layout(cfg)
    oc = O.OracleCache(**{k: v for k, v in d.items() if k not in ("host_only", "device")})
    ol = oc.layout
    assert lay["chunk_bytes"] == ol["chunk_bytes"]
    assert lay["block_bytes"] == ol["block_bytes"]
    assert lay["off_v"] == ol["off_V"] and lay["off_vmeta"] == ol["off_Vm"]
    assert lay["off_kmeta"] == ol["off_Km"] and lay["kslice"] == ol["kslice"]
    assert lay["row_bytes"] == ol["row_bytes"] and lay["sub_bytes"] == ol["sub_bytes"]
    oc.close()


@pytest.mark.parametrize("name", list(FMTS))
def test_planner_block_placement_matches_oracle(name):
    cfg, d = cfg_of(name, max_seqs=5, num_blocks=400)
    h = kvq.kvq_create(cfg)
    oc = O.OracleCache(**{k: v for k, v in d.items() if k not in ("host_only", "device")})
    rng = np.random.default_rng(3)
    D = 128
    for step in range(30):
        n = int(rng.integers(1, 90)) if step % 3 else int(rng.integers(100, 300))
        ids = rng.integers(0, 5, size=n).astype(np.int32)
        kb = np.zeros((n, 2, D), np.uint16)
        assert oc.append(kb, kb, ids) == 0
        kvq.kvq_append(h, 0, 0, ids, n)
        if step == 17:
            oc.free_seq(2)
            kvq.kvq_free_seq(h, 2)
        for s in range(5):
            assert kvq.kvq_seq_len(h, s) == oc.seq_len(s)
            assert kvq.kvq_block_table_host(h, s).tolist() == oc.block_table(s).tolist()
    st = kvq.kvq_stats(h)
    assert st["blocks_free"] == oc.free_count()
    assert st["tokens_stored"] == sum(oc.seq_len(s) for s in range(5))
    kvq.kvq_destroy(h)
    oc.close()


def test_admission_counts_only_the_blocks_a_call_adds():
    """The planner admits an append that needs exactly the free blocks left
    (only the blocks its new tokens open count), refuses one more token with
    KVQ_ERR_OOM and an id equal to max_seqs with KVQ_ERR_BAD_SEQ, both with
    no state change, as the oracle does."""
    cfg, d = cfg_of("int8_tok_p16", num_blocks=3, max_seqs=2)
    h = kvq.kvq_create(cfg)
    oc = O.OracleCache(**{k: v for k, v in d.items() if k not in ("host_only", "device")})
    kb = np.zeros((32, 2, 128), np.uint16)
    for n in (32, 16):
        kvq.kvq_append(h, 0, 0, np.zeros(n, np.int32), n)
        assert oc.append(kb[:n], kb[:n], np.zeros(n, np.int32)) == 0
    assert kvq.kvq_stats(h)["blocks_free"] == oc.free_count() == 0
    assert kvq.kvq_block_table_host(h, 0).tolist() == oc.block_table(0).tolist()
    for ids, status in ((np.zeros(1, np.int32), kvq.KVQ_ERR_OOM), (np.full(1, 2, np.int32), kvq.KVQ_ERR_BAD_SEQ)):
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_append(h, 0, 0, ids, 1)
        assert e.value.status == status
    assert kvq.kvq_seq_len(h, 0) == 48 and kvq.kvq_seq_len(h, 1) == 0
    kvq.kvq_destroy(h)
    oc.close()


def test_errors_leave_state_unchanged():
    cfg, _ = cfg_of("int8_tok_p16", num_blocks=6, max_seqs=2)
    h = kvq.kvq_create(cfg)
    kvq.kvq_append(h, 0, 0, np.zeros(40, np.int32), 40)     # 3 blocks
    table = kvq.kvq_block_table_host(h, 0).tolist()
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_append(h, 0, 0, np.zeros(100, np.int32), 100)
    assert e.value.status == kvq.KVQ_ERR_OOM
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_append(h, 0, 0, np.array([0, 5], np.int32), 2)
    assert e.value.status == kvq.KVQ_ERR_BAD_SEQ
    assert "out of range" in kvq.kvq_last_error()
    assert kvq.kvq_seq_len(h, 0) == 40 and kvq.kvq_block_table_host(h, 0).tolist() == table
    assert kvq.kvq_stats(h)["blocks_free"] == 3
    kvq.kvq_destroy(h)


def test_fail_alloc_after_and_table_width():
    cfg, _ = cfg_of("int8_tok_p16", fail_alloc_after=2)
    h = kvq.kvq_create(cfg)
    kvq.kvq_append(h, 0, 0, np.zeros(32, np.int32), 32)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_append(h, 0, 0, np.zeros(1, np.int32), 1)
    assert e.value.status == kvq.KVQ_ERR_OOM and kvq.kvq_seq_len(h, 0) == 32
    kvq.kvq_destroy(h)
    cfg, _ = cfg_of("int8_tok_p16", max_blocks_per_seq=2)
    h = kvq.kvq_create(cfg)
    kvq.kvq_append(h, 0, 0, np.zeros(32, np.int32), 32)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_append(h, 0, 0, np.zeros(1, np.int32), 1)
    assert e.value.status == kvq.KVQ_ERR_OOM
    kvq.kvq_destroy(h)


@pytest.mark.parametrize("field,value,status", [
    ("bits", 3, kvq.KVQ_ERR_INVALID_ARG),
    ("d_h", 64, kvq.KVQ_ERR_UNSUPPORTED),
    ("h_q", 6, kvq.KVQ_ERR_UNSUPPORTED),
    ("h_q", 3, kvq.KVQ_ERR_INVALID_ARG),
    ("residual", 32, kvq.KVQ_ERR_INVALID_ARG),
    ("page", 24, kvq.KVQ_ERR_INVALID_ARG),
    ("page", 48, kvq.KVQ_ERR_INVALID_ARG),
    ("page", 128, kvq.KVQ_ERR_UNSUPPORTED),
    ("g_v", 48, kvq.KVQ_ERR_UNSUPPORTED),
    ("g_v", 16, kvq.KVQ_ERR_UNSUPPORTED),      # value groups are 32, 64 or 128 channels
    ("page", 8, kvq.KVQ_ERR_INVALID_ARG),      # a page holds at least one 16-token sub-tile
    ("num_blocks", 0, kvq.KVQ_ERR_INVALID_ARG),
    ("k_axis", 2, kvq.KVQ_ERR_INVALID_ARG),
    ("bits", 16, kvq.KVQ_ERR_INVALID_ARG),     # the BF16 control takes token-axis keys, no window
])
def test_config_validation(field, value, status):
    cfg, _ = cfg_of("int4_chan64")
    setattr(cfg, field, value)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_create(cfg)
    assert e.value.status == status


def test_null_and_host_only_guards():
    cfg, _ = cfg_of("int4_chan64")
    h = kvq.kvq_create(cfg)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attn(h, 16, 0, 0, 16, None, 1, 16)
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG       # host-only handle
    with pytest.raises(kvq.KvqError):
        kvq.kvq_append(h, 0, 0, None, 3)                     # null seq ids
    kvq.kvq_append(h, 0, 0, np.zeros(0, np.int32), 0)        # empty append is fine
    for args in [(16, 16, np.zeros(1, np.int32), 16, 1, 16),       # host-only handle
                 (0, 0, np.zeros(1, np.int32), 16, 1, 16),         # rows without k / v
                 (16, 16, np.zeros(1, np.int32), 16, 99, 16),      # batch above max_seqs
                 (16, 16, np.zeros(1, np.int32), 0, 1, 0)]:        # decode rows without q / out
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_step_host(h, *args)
        assert e.value.status == kvq.KVQ_ERR_INVALID_ARG
    assert kvq.kvq_seq_len(h, 0) == 0
    kvq.kvq_destroy(h)


def test_cache_bytes_formula_worked_example():
    g = read_golden("memory_formula.txt")
    cfg, _ = cfg_of("int4_chan64")
    got = kvq.kvq_cache_bytes(g["worked_layers"], g["worked_tokens"], g["worked_h_kv"],
                              g["worked_d_h"], cfg)
    assert got == g["worked_4bit_fp16_per64_mib"] * 2 ** 20
    cfg8, _ = cfg_of("int8_tok_p16")
    # INT8 with fp16 scales per 128: 2 * elems * (1 + 2/128)
    elems = 32 * 8192 * 8 * 128
    assert kvq.kvq_cache_bytes(32, 8192, 8, 128, cfg8) == 2 * elems + 2 * elems * 2 // 128
    cfg2, _ = cfg_of("int2_asym_chan32")
    assert kvq.kvq_cache_bytes(1, 100, 8, 128, cfg2) == 2 * 102400 // 4 + 2 * 102400 * 4 // 32
    cfg16, _ = cfg_of("bf16_control_p16")      # BF16: 2 bytes per element, no metadata
    assert kvq.kvq_cache_bytes(32, 8192, 8, 128, cfg16) == 2 * elems * 2


def test_fp8_config_rules():
    for field, value in (("bits", 4), ("asym", 1), ("scale_fp32", 1), ("g_k", 64), ("fp8", 2)):
        cfg, _ = cfg_of("fp8_p32")
        setattr(cfg, field, value)
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_create(cfg)
        assert e.value.status == kvq.KVQ_ERR_INVALID_ARG
    cfg, _ = cfg_of("fp8_p32")
    h = kvq.kvq_create(cfg)
    kvq.kvq_set_fp8_scales(h, [0.5, 2.0], [1.0, 1.0])
    with pytest.raises(kvq.KvqError):
        kvq.kvq_set_fp8_scales(h, [0.0, 1.0], [1.0, 1.0])       # not positive
    kvq.kvq_append(h, 0, 0, np.zeros(3, np.int32), 3)
    with pytest.raises(kvq.KvqError):
        kvq.kvq_set_fp8_scales(h, [1.0, 1.0], [1.0, 1.0])       # tokens stored already
    kvq.kvq_destroy(h)
    cfg, _ = cfg_of("int8_tok_p16")
    h = kvq.kvq_create(cfg)
    with pytest.raises(kvq.KvqError):
        kvq.kvq_set_fp8_scales(h, [1.0, 1.0], [1.0, 1.0])       # not an FP8 cache
    kvq.kvq_destroy(h)


def test_bf16_control_config_rules():
    for field, value in (("residual", 64), ("asym", 1), ("scale_fp32", 1), ("g_k", 64), ("g_v", 64)):
        cfg, _ = cfg_of("bf16_control_p16")
        setattr(cfg, field, value)
        if field == "residual":
            cfg.k_axis = 1
            cfg.g_k = 64
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_create(cfg)
        assert e.value.status == kvq.KVQ_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["int8_tok_p16", "int4_chan64", "int4_asym_tok32"])
def test_share_prefix_planner_matches_oracle(name):
    cfg, d = cfg_of(name, max_seqs=4, num_blocks=300)
    h = kvq.kvq_create(cfg)
    oc = O.OracleCache(**{k: v for k, v in d.items() if k not in ("host_only", "device")})
    unit = d["residual"] or d["page"]
    z = np.zeros((1, 2, 128), np.uint16)

    def both_append(n, s):
        ids = np.full(n, s, np.int32)
        kb = np.zeros((n, 2, 128), np.uint16)
        assert oc.append(kb, kb, ids) == 0
        kvq.kvq_append(h, 0, 0, ids, n)

    both_append(5 * unit + 7, 0)
    kvq.kvq_share_prefix(h, 0, 1, 3 * unit)
    assert oc.share_prefix(0, 1, 3 * unit) == 0
    both_append(2 * unit + 1, 1)
    both_append(unit, 0)
    kvq.kvq_share_prefix(h, 1, 2, 2 * unit)
    assert oc.share_prefix(1, 2, 2 * unit) == 0
    for s in (0, 1, 2):
        assert kvq.kvq_seq_len(h, s) == oc.seq_len(s)
        assert kvq.kvq_block_table_host(h, s).tolist() == oc.block_table(s).tolist()
    for s in (0, 2, 1):
        kvq.kvq_free_seq(h, s)
        assert oc.free_seq(s) == 0
        assert kvq.kvq_stats(h)["blocks_free"] == oc.free_count()
    both_append(4 * unit, 3)     # blocks come back in the same order on both sides
    assert kvq.kvq_block_table_host(h, 3).tolist() == oc.block_table(3).tolist()
    # format check and other errors, with no state change; with a window only
    # whole key groups share (a page-sized prefix is refused on both sides)
    bad = [((3, 0, unit + 1), kvq.KVQ_ERR_INVALID_ARG), ((3, 3, unit), kvq.KVQ_ERR_INVALID_ARG),
           ((3, 0, 99 * unit), kvq.KVQ_ERR_INVALID_ARG), ((3, 9, unit), kvq.KVQ_ERR_BAD_SEQ)]
    if d["residual"]:
        bad.append(((3, 0, d["page"]), kvq.KVQ_ERR_INVALID_ARG))
        assert oc.share_prefix(0, 3, d["page"]) == 4
    for args, status in bad:
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_share_prefix(h, *args)
        assert e.value.status == status
    assert kvq.kvq_seq_len(h, 0) == 0
    kvq.kvq_destroy(h)
    oc.close()
