"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.  Codes, scales, zero-points, packing and block placement
must match bit for bit (the whole pool, the live residual slots and the block
tables); attention output must be within 2e-3 (max abs) of the oracle's fp64
attention over the same dequantized cache."""
import os

import numpy as np
import pytest
import torch

from quantized_kv_cache_14_b200 import build as kbuild
from quantized_kv_cache_14_b200 import kvq
from quantized_kv_cache_14_b200.workloads import Draws, random_bf16, workload
from tests.gpu_util import ATOL, Pair, bits_to_cuda_bf16

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kbuild.build()


FMTS = {
    "int8_tok_p16": dict(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=16),
    "int8_tok_p512_fp32": dict(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=1, residual=0, page=512),
    "int4_chan64": dict(bits=4, asym=0, k_axis=1, g_k=64, g_v=64, scale_fp32=0, residual=64, page=16),
    "int2_asym_chan32": dict(bits=2, asym=1, k_axis=1, g_k=32, g_v=32, scale_fp32=0, residual=32, page=16),
    "int4_chan64_p32_gv32": dict(bits=4, asym=0, k_axis=1, g_k=64, g_v=32, scale_fp32=0, residual=64, page=32),
    "int4_asym_tok32": dict(bits=4, asym=1, k_axis=0, g_k=32, g_v=32, scale_fp32=0, residual=0, page=32),
    "int8_asym_chan128_p64": dict(bits=8, asym=1, k_axis=1, g_k=128, g_v=128, scale_fp32=0, residual=128, page=64),
    "int2_sym_tok64_fp32": dict(bits=2, asym=0, k_axis=0, g_k=64, g_v=64, scale_fp32=1, residual=0, page=16),
    "int4_chan16": dict(bits=4, asym=0, k_axis=1, g_k=16, g_v=128, scale_fp32=0, residual=16, page=16),
    "int4_chan64_fp32": dict(bits=4, asym=0, k_axis=1, g_k=64, g_v=64, scale_fp32=1, residual=64, page=16),
    # the pages' unquantized BF16 cache on the same paged path (control)
    "bf16_control_p16": dict(bits=16, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=16),
    "bf16_control_p64": dict(bits=16, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=64),
    # FP8 E4M3 with one scale per kv head (1.0 unless a test sets them)
    "fp8_p16": dict(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=16, fp8=1),
    "fp8_p32": dict(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=32, fp8=1),
}


def outlier_keys(rng, n, h_kv, gain=20.0):
    k = rng.standard_normal((n, h_kv, D), dtype=np.float32)
    k[:, :, 3] *= gain
    k[:, :, 77] *= gain
    from quantized_kv_cache_14_b200.workloads import to_bf16_bits
    return to_bf16_bits(k)


@pytest.mark.parametrize("name", list(FMTS))
@pytest.mark.parametrize("lens", [[1], [15, 16, 17], [63, 64, 65], [200, 1, 129], [0, 31, 33]])
def test_small_bulk_append_and_decode(name, lens):
    rng = np.random.default_rng(sum(lens) + len(name))
    h_q, h_kv = 8, 2
    p = Pair(FMTS[name], h_q, h_kv, max_seqs=3, num_blocks=120, mbps=64, seed=5)
    ids = np.repeat(np.arange(len(lens), dtype=np.int32), lens)
    n = int(ids.size)
    if n:
        p.append(outlier_keys(rng, n, h_kv), random_bf16(rng, (n, h_kv, D)), ids)
    p.check_state()
    q = random_bf16(rng, (len(lens), h_q, D))
    p.check_decode(q, lens)
    p.close()


@pytest.mark.parametrize("name", list(FMTS))
def test_incremental_appends_interleaved(name):
    """Appends of random sizes to interleaved sequences equal the oracle's
    one-token-at-a-time definition, with decode checked along the way."""
    rng = np.random.default_rng(7)
    h_q, h_kv = 4, 1
    p = Pair(FMTS[name], h_q, h_kv, max_seqs=3, num_blocks=300, mbps=128, seed=9)
    lens = [0, 0, 0]
    for step in range(14):
        n = int(rng.integers(1, 70))
        ids = rng.integers(0, 3, size=n).astype(np.int32)
        p.append(outlier_keys(rng, n, h_kv), random_bf16(rng, (n, h_kv, D)), ids)
        for s in ids:
            lens[int(s)] += 1
        if step % 4 == 3:
            p.check_state()
            p.check_decode(random_bf16(rng, (3, h_q, D)), lens)
    p.check_state()
    p.close()


@pytest.mark.parametrize("name", ["int4_chan64", "int2_asym_chan32", "int4_chan16", "int8_asym_chan128_p64"])
def test_append_launch_shapes(name):
    """The append's launch shapes give the oracle's bytes: decode steps where
    some sequences complete a key group (flush and window rows in one launch,
    plan in the launch parameters), a multi-token append that completes a
    group and leaves tokens of the same sequence behind (window rows after the
    flush), and a bulk append whose plan is uploaded.  Decode over the
    library's own stored lengths equals decode over explicit lengths."""
    rng = np.random.default_rng(11)
    R = FMTS[name]["residual"]
    h_q, h_kv, S = 8, 2, 4
    p = Pair(FMTS[name], h_q, h_kv, max_seqs=S, num_blocks=400, mbps=128, seed=2)
    # bulk (plan uploaded): lengths R-2, R-1, 2R-1, 3
    lens = [R - 2, R - 1, 2 * R - 1, 3]
    ids = np.repeat(np.arange(S, dtype=np.int32), lens)
    p.append(outlier_keys(rng, ids.size, h_kv), random_bf16(rng, (ids.size, h_kv, D)), ids)
    p.check_state()
    # decode steps: one token per sequence; sequences 1 and 2 flush at once
    for _ in range(3):
        ids = np.arange(S, dtype=np.int32)
        p.append(outlier_keys(rng, S, h_kv), random_bf16(rng, (S, h_kv, D)), ids)
        lens = [L + 1 for L in lens]
        p.check_state()
    # sequence 0 completes its group and keeps 5 tokens in one call; sequence 3 gains 2
    ids = np.array([0] * (R - lens[0] % R + 5) + [3, 3], dtype=np.int32)
    p.append(outlier_keys(rng, ids.size, h_kv), random_bf16(rng, (ids.size, h_kv, D)), ids)
    lens[0] += R - lens[0] % R + 5
    lens[3] += 2
    p.check_state()
    q = random_bf16(rng, (S, h_q, D))
    got, want = p.decode(q, lens)
    assert np.max(np.abs(got - want)) <= ATOL
    out = torch.full((S, h_q, D), float("nan"), dtype=torch.float32, device="cuda")
    p.gpu.decode(bits_to_cuda_bf16(q), None, out)
    torch.cuda.synchronize()
    assert p.gpu.sync_status() == 0
    assert np.array_equal(out.cpu().numpy(), got.astype(np.float32))
    p.close()


@pytest.mark.parametrize("name", ["int4_chan64", "int2_asym_chan32", "int8_asym_chan128_p64", "int4_chan16",
                                  "int4_chan64_p32_gv32", "int4_chan64_fp32"])
def test_bulk_flush_matches_oracle(name):
    """Calls that complete many key groups at once (the bulk prefill shape:
    one CTA per group and head) give the oracle's bytes, with groups whose
    tokens come partly from the window and partly from the call."""
    rng = np.random.default_rng(31)
    R = FMTS[name]["residual"]
    h_q, h_kv, S = 8, 2, 20
    p = Pair(FMTS[name], h_q, h_kv, max_seqs=S, num_blocks=S * (3 * R // 16 + 4), mbps=3 * R // 16 + 4, seed=6)
    lens = [int(x) for x in rng.integers(R // 2, R, size=S)]     # every window partly filled
    ids = np.repeat(np.arange(S, dtype=np.int32), lens)
    p.append(outlier_keys(rng, ids.size, h_kv), random_bf16(rng, (ids.size, h_kv, D)), ids)
    add = [int(x) for x in rng.integers(R, 2 * R, size=S)]       # each call completes 1-2 groups per sequence
    ids = np.repeat(np.arange(S, dtype=np.int32), add)
    rng.shuffle(ids)
    p.append(outlier_keys(rng, ids.size, h_kv), random_bf16(rng, (ids.size, h_kv, D)), ids)
    lens = [a + b for a, b in zip(lens, add)]
    p.check_state()
    p.check_decode(random_bf16(rng, (S, h_q, D)), lens)
    p.close()


@pytest.mark.parametrize("name", ["int4_chan64", "int8_tok_p16", "fp8_p16"])
def test_step_host_equals_device_calls(name):
    """kvq_step_host (host buffers in, host output back, one call) appends the
    same bytes and returns the same output as kvq_append + kvq_decode_attn on
    device buffers, and both match the oracle."""
    rng = np.random.default_rng(21)
    h_q, h_kv, S = 8, 2, 3
    fmt = FMTS[name]
    a = Pair(fmt, h_q, h_kv, max_seqs=S, num_blocks=300, mbps=128, seed=4)
    b = kvq.KVCache(kvq.Format(**fmt), h_q, h_kv, S, 300, 128, seed=4)
    lens = [70, 5, 129]
    ids = np.repeat(np.arange(S, dtype=np.int32), lens)
    k0, v0 = outlier_keys(rng, ids.size, h_kv), random_bf16(rng, (ids.size, h_kv, D))
    a.append(k0, v0, ids)
    b.append(bits_to_cuda_bf16(k0), bits_to_cuda_bf16(v0), ids)

    def host(bits, pinned=True):
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
        return t.pin_memory() if pinned else t.clone()

    def packed(k, v, q, pinned=True):
        # one host buffer holding k | v | q back to back
        buf = host(np.concatenate([k.ravel(), v.ravel(), q.ravel()]), pinned)
        return buf[:k.size].view(k.shape), buf[k.size:2 * k.size].view(v.shape), buf[2 * k.size:].view(q.shape)

    for step in range(72):   # crosses group boundaries of every sequence
        ids = np.arange(S, dtype=np.int32)
        k, v, q = outlier_keys(rng, S, h_kv), random_bf16(rng, (S, h_kv, D)), random_bf16(rng, (S, h_q, D))
        lens = [L + 1 for L in lens]
        a.append(k, v, ids)
        mode = step % 4
        pinned_out = mode in (0, 2)
        out_h = torch.full((S, h_q, D), float("nan"), dtype=torch.float32)
        if pinned_out:   # the output written straight into page-locked memory
            out_h = out_h.pin_memory()
        if mode == 0:    # page-locked k | v | q back to back: one copy
            kh, vh, qh = packed(k, v, q)
        elif mode == 1:  # separate page-locked buffers
            kh, vh, qh = host(k), host(v), host(q)
        elif mode == 2:  # pageable k | v | q back to back: one copy of all three
            kh, vh, qh = packed(k, v, q, pinned=False)
        else:            # separate pageable buffers: three copies
            kh, vh, qh = host(k, False), host(v, False), host(q, False)
        b.step_host(kh, vh, ids, qh, out_h)
        torch.cuda.synchronize()
        if step % 23 == 0 or step >= 68:
            got, want = a.decode(q, lens)
            assert np.array_equal(out_h.numpy(), got.astype(np.float32))
            assert np.max(np.abs(got - want)) <= ATOL
    a.check_state()
    assert np.array_equal(b.pool(), a.gpu.pool())
    assert b.sync_status() == 0
    b.close()
    a.close()


@pytest.mark.parametrize("name", ["int4_chan64", "int8_tok_p16"])
def test_large_batch(name):
    """A thousand sequences of 0 to 140 tokens in one bulk append, then one
    decode of every row and one of 700 shuffled rows with shorter prefixes.
    At this batch the per-row work list no longer fits beside two
    warp-specialised CTAs per SM, so the generic kernel runs, and its prefix
    scan over the rows takes several rows per thread."""
    rng = np.random.default_rng(97)
    h_q, h_kv, S = 8, 2, 1000
    p = Pair(FMTS[name], h_q, h_kv, max_seqs=S, num_blocks=S * 9, mbps=9, seed=11)
    lens = [int(x) for x in rng.integers(0, 141, size=S)]
    ids = rng.permutation(np.repeat(np.arange(S, dtype=np.int32), lens)).astype(np.int32)
    p.append(outlier_keys(rng, ids.size, h_kv), random_bf16(rng, (ids.size, h_kv, D)), ids)
    p.check_state()
    p.check_decode(random_bf16(rng, (S, h_q, D)), lens)
    rows = rng.permutation(S)[:700].astype(np.int32)
    attend = [int(rng.integers(0, lens[r] + 1)) for r in rows]
    p.check_decode(random_bf16(rng, (rows.size, h_q, D)), attend, seq_ids=rows)
    p.close()


@pytest.mark.parametrize("name", ["int4_chan64", "int8_tok_p16", "int2_asym_chan32", "bf16_control_p16", "fp8_p16"])
def test_split_k_merge_is_invariant_to_grid(name):
    rng = np.random.default_rng(3)
    h_q, h_kv = 16, 4
    p = Pair(FMTS[name], h_q, h_kv, max_seqs=4, num_blocks=900, mbps=256, seed=1)
    lens = [1500, 3, 640, 999]
    ids = np.repeat(np.arange(4, dtype=np.int32), lens)
    n = int(ids.size)
    p.append(outlier_keys(rng, n, h_kv), random_bf16(rng, (n, h_kv, D)), ids)
    q = random_bf16(rng, (4, h_q, D))
    outs = []
    for grid in (0, 1, 2, 7, 64, 1000):
        p.gpu.set_decode_grid(grid)
        got, want = p.decode(q, lens)
        assert np.max(np.abs(got - want)) <= ATOL, grid
        outs.append(got)
    for o in outs[1:]:
        assert np.max(np.abs(o - outs[0])) <= 1e-4
    p.close()


@pytest.mark.parametrize("name", ["int4_chan64", "int8_tok_p16", "int2_asym_chan32", "bf16_control_p16"])
def test_shared_prefix_decode(name):
    """Prefix sharing: a sequence holding another's quantized blocks decodes as
    the oracle says, before and after both sequences grow past the share."""
    rng = np.random.default_rng(8)
    fmt = FMTS[name]
    unit = fmt["residual"] or fmt["page"]
    h_q, h_kv = 8, 2
    p = Pair(fmt, h_q, h_kv, max_seqs=3, num_blocks=400, mbps=64, seed=6)
    n0 = 6 * unit + 9
    p.append(outlier_keys(rng, n0, h_kv), random_bf16(rng, (n0, h_kv, D)), np.zeros(n0, np.int32))
    p.share_prefix(0, 1, 4 * unit)
    p.share_prefix(0, 2, 2 * unit)
    p.check_state()
    p.check_decode(random_bf16(rng, (3, h_q, D)), [n0, 4 * unit, 2 * unit])
    for s, n in ((1, 3 * unit + 2), (0, unit + 4), (2, 5)):
        p.append(outlier_keys(rng, n, h_kv), random_bf16(rng, (n, h_kv, D)), np.full(n, s, np.int32))
    p.check_state()
    lens = [p.orc.seq_len(s) for s in range(3)]
    p.check_decode(random_bf16(rng, (3, h_q, D)), lens)
    p.gpu.free_seq(0)
    assert p.orc.free_seq(0) == 0
    p.check_state()
    p.check_decode(random_bf16(rng, (3, h_q, D)), [0] + lens[1:])
    p.close()


@pytest.mark.parametrize("name", ["int4_chan64", "int8_tok_p16", "int2_asym_chan32"])
def test_chunked_prefill_attention(name):
    """Chunked prefill: append a chunk, then each chunk token attends its own
    causal prefix (rows straddle the quantized/window boundary and span more
    rows than max_seqs, so the call takes several launches)."""
    rng = np.random.default_rng(12)
    fmt = FMTS[name]
    h_q, h_kv, S = 8, 2, 3
    p = Pair(fmt, h_q, h_kv, max_seqs=S, num_blocks=300, mbps=64, seed=7)
    pre = [150, 37, 64]
    ids = np.repeat(np.arange(S, dtype=np.int32), pre)
    p.append(outlier_keys(rng, ids.size, h_kv), random_bf16(rng, (ids.size, h_kv, D)), ids)
    chunk = [45, 20, 9]
    cids = np.repeat(np.arange(S, dtype=np.int32), chunk)
    p.append(outlier_keys(rng, cids.size, h_kv), random_bf16(rng, (cids.size, h_kv, D)), cids)
    pos = np.concatenate([np.arange(pre[s], pre[s] + chunk[s]) for s in range(S)]).astype(np.int32)
    q = random_bf16(rng, (cids.size, h_q, D))
    out = torch.full((cids.size, h_q, D), float("nan"), dtype=torch.float32, device="cuda")
    p.gpu.prefill_attn(bits_to_cuda_bf16(q), cids, pos, out)
    torch.cuda.synchronize()
    assert p.gpu.sync_status() == 0
    want = p.orc.decode(q, (pos + 1).tolist(), seq_ids=cids)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    err = float(np.max(np.abs(got - want)))
    assert err <= 2e-3, f"max abs error {err}"
    with pytest.raises(kvq.KvqError):   # a position that is not stored yet
        p.gpu.prefill_attn(bits_to_cuda_bf16(q[:1]), [0], [pre[0] + chunk[0]], out)
    p.close()


@pytest.mark.parametrize("name,h_q,h_kv", [
    ("int4_chan64", 8, 2), ("int4_chan64", 4, 2), ("int4_chan64", 2, 2), ("int2_asym_chan32", 8, 2),
    ("int4_chan64_p32_gv32", 8, 2), ("int8_asym_chan128_p64", 4, 1), ("int4_chan16", 8, 2)])
def test_prefill_kernel_blocks(name, h_q, h_kv):
    """The shared-tile prefill kernel: chunks of several sequences with rows in
    shuffled order, long prefixes (the key range split over CTAs and merged),
    a sequence whose chunk sits only in the window, and a single-split call."""
    rng = np.random.default_rng(31)
    fmt = FMTS[name]
    S = 3
    p = Pair(fmt, h_q, h_kv, max_seqs=S, num_blocks=900, mbps=256, seed=3)
    pre = [1500, 64, 0]
    ids = np.repeat(np.arange(S, dtype=np.int32), pre)
    p.append(outlier_keys(rng, ids.size, h_kv), random_bf16(rng, (ids.size, h_kv, D)), ids)
    chunk = [100, 70, 9]
    cids = np.concatenate([np.full(c, s, np.int32) for s, c in enumerate(chunk)])
    p.append(outlier_keys(rng, cids.size, h_kv), random_bf16(rng, (cids.size, h_kv, D)), cids)
    pos = np.concatenate([np.arange(pre[s], pre[s] + chunk[s]) for s in range(S)]).astype(np.int32)
    perm = rng.permutation(cids.size)
    cids, pos = cids[perm], pos[perm]
    q = random_bf16(rng, (cids.size, h_q, D))
    out = torch.full((cids.size, h_q, D), float("nan"), dtype=torch.float32, device="cuda")
    p.gpu.prefill_attn(bits_to_cuda_bf16(q), cids, pos, out)
    torch.cuda.synchronize()
    assert p.gpu.sync_status() == 0
    want = p.orc.decode(q, (pos + 1).tolist(), seq_ids=cids)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    err = float(np.max(np.abs(got - want)))
    assert err <= ATOL, f"max abs error {err}"
    # one short chunk of one sequence: a single split writes the output directly
    q1 = random_bf16(rng, (5, h_q, D))
    ids1 = np.full(5, 1, np.int32)
    pos1 = np.arange(60, 65, dtype=np.int32)
    out1 = torch.full((5, h_q, D), float("nan"), dtype=torch.float32, device="cuda")
    p.gpu.prefill_attn(bits_to_cuda_bf16(q1), ids1, pos1, out1)
    torch.cuda.synchronize()
    want1 = p.orc.decode(q1, (pos1 + 1).tolist(), seq_ids=ids1)
    assert np.max(np.abs(out1.cpu().numpy().astype(np.float64) - want1)) <= ATOL
    p.close()


def test_prefill_shared_memory_limit_only_rises():
    """Two caches whose prefill runs one kernel instance (4-bit symmetric
    keys per channel, the mma.sync kernel) with different stage sizes: the
    smaller one's first call, which also sizes its residency, must not lower
    the kernel's shared-memory limit under the larger one's next launch."""
    rng = np.random.default_rng(71)
    # 16-token key groups stage 4 pages of 2336 B, 64-token groups 4 of 2176 B
    pairs = [Pair(FMTS["int4_chan16"], 8, 2, max_seqs=1, num_blocks=200, mbps=64, seed=7),
             Pair(FMTS["int4_chan64"], 4, 2, max_seqs=1, num_blocks=200, mbps=64, seed=8)]
    n_pre, n_chunk = 300, 24
    for p in pairs:
        ids = np.zeros(n_pre + n_chunk, np.int32)
        p.append(outlier_keys(rng, ids.size, p.h_kv), random_bf16(rng, (ids.size, p.h_kv, D)), ids)
    pos = np.arange(n_pre, n_pre + n_chunk, dtype=np.int32)
    cids = np.zeros(n_chunk, np.int32)
    for which in (0, 1, 0):
        p = pairs[which]
        q = random_bf16(rng, (n_chunk, p.h_q, D))
        out = torch.full((n_chunk, p.h_q, D), float("nan"), dtype=torch.float32, device="cuda")
        p.gpu.prefill_attn(bits_to_cuda_bf16(q), cids, pos, out)
        torch.cuda.synchronize()
        assert p.gpu.sync_status() == 0
        want = p.orc.decode(q, (pos + 1).tolist(), seq_ids=cids)
        err = float(np.max(np.abs(out.cpu().numpy().astype(np.float64) - want)))
        assert err <= ATOL, f"cache {which}: max abs error {err}"
    for p in pairs:
        p.close()


@pytest.mark.parametrize("name", ["int4_chan64", "int2_asym_chan32"])
def test_prefill_repeated_split_calls(name):
    """Repeated split prefill calls on one cache give bit-identical outputs
    (plan buffers and split records reused across calls, the merge a
    programmatic dependent launch), with a smaller call in between, and match
    the oracle."""
    rng = np.random.default_rng(53)
    fmt = FMTS[name]
    h_q, h_kv = 8, 2
    p = Pair(fmt, h_q, h_kv, max_seqs=2, num_blocks=900, mbps=256, seed=5)
    pre = [2000, 700]
    ids = np.repeat(np.arange(2, dtype=np.int32), pre)
    p.append(outlier_keys(rng, ids.size, h_kv), random_bf16(rng, (ids.size, h_kv, D)), ids)
    chunk = [96, 40]
    cids = np.concatenate([np.full(c, s, np.int32) for s, c in enumerate(chunk)])
    p.append(outlier_keys(rng, cids.size, h_kv), random_bf16(rng, (cids.size, h_kv, D)), cids)
    pos = np.concatenate([np.arange(pre[s], pre[s] + chunk[s]) for s in range(2)]).astype(np.int32)
    q = random_bf16(rng, (cids.size, h_q, D))
    qd = bits_to_cuda_bf16(q)
    outs = []
    for it in range(3):
        if it == 1:
            small = torch.empty((8, h_q, D), dtype=torch.float32, device="cuda")
            p.gpu.prefill_attn(bits_to_cuda_bf16(q[-8:]), cids[-8:], pos[-8:], small)
        out = torch.full((cids.size, h_q, D), float("nan"), dtype=torch.float32, device="cuda")
        p.gpu.prefill_attn(qd, cids, pos, out)
        outs.append(out)
    torch.cuda.synchronize()
    assert p.gpu.sync_status() == 0
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    want = p.orc.decode(q, (pos + 1).tolist(), seq_ids=cids)
    got = outs[0].cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - want)) <= ATOL
    want_small = p.orc.decode(q[-8:], (pos[-8:] + 1).tolist(), seq_ids=cids[-8:])
    assert np.max(np.abs(small.cpu().numpy().astype(np.float64) - want_small)) <= ATOL
    p.close()


@pytest.mark.parametrize("name", ["int4_chan64", "int2_asym_chan32", "int4_chan64_fp32", "int8_tok_p16"])
def test_prefill_over_shared_prefix(name):
    """Chunked prefill of sequences that hold another sequence's blocks: the
    rows read the shared pages through their own block tables (the prefill
    kernel for the channel-axis fp16-scale formats, decode rows for the
    others) and match the oracle."""
    rng = np.random.default_rng(41)
    fmt = FMTS[name]
    unit = fmt["residual"] or fmt["page"]
    h_q, h_kv = 8, 2
    p = Pair(fmt, h_q, h_kv, max_seqs=3, num_blocks=600, mbps=128, seed=8)
    n0 = 12 * unit + 5
    p.append(outlier_keys(rng, n0, h_kv), random_bf16(rng, (n0, h_kv, D)), np.zeros(n0, np.int32))
    p.share_prefix(0, 1, 8 * unit)
    p.share_prefix(0, 2, 3 * unit)
    chunk = [(1, 2 * unit + 7), (2, 40)]
    ids = np.concatenate([np.full(c, s, np.int32) for s, c in chunk])
    p.append(outlier_keys(rng, ids.size, h_kv), random_bf16(rng, (ids.size, h_kv, D)), ids)
    pos = np.concatenate([np.arange(b, b + c) for b, (s, c) in zip((8 * unit, 3 * unit), chunk)]).astype(np.int32)
    q = random_bf16(rng, (ids.size, h_q, D))
    out = torch.full((ids.size, h_q, D), float("nan"), dtype=torch.float32, device="cuda")
    p.gpu.prefill_attn(bits_to_cuda_bf16(q), ids, pos, out)
    torch.cuda.synchronize()
    assert p.gpu.sync_status() == 0
    want = p.orc.decode(q, (pos + 1).tolist(), seq_ids=ids)
    assert np.max(np.abs(out.cpu().numpy().astype(np.float64) - want)) <= ATOL
    p.close()


@pytest.mark.parametrize("page", [16, 32])
def test_fp8_per_head_scales(page):
    """FP8 with per-head scales from amax / 448 of a sample, keys with large
    outliers, and values beyond the scaled range (saturation at +-448)."""
    rng = np.random.default_rng(31)
    fmt = dict(FMTS["fp8_p16"], page=page)
    h_q, h_kv, S = 8, 2, 3
    p = Pair(fmt, h_q, h_kv, max_seqs=S, num_blocks=200, mbps=64, seed=3)
    lens = [300, 45, 129]
    ids = np.repeat(np.arange(S, dtype=np.int32), lens)
    k = outlier_keys(rng, ids.size, h_kv, gain=40.0)
    v = random_bf16(rng, (ids.size, h_kv, D), 2.0)
    from oracle import oracle as O
    kf, vf = O.bf16_bits_to_f32(k), O.bf16_bits_to_f32(v)
    ks = (np.abs(kf[:100]).max(axis=(0, 2)) / 448.0).astype(np.float32)   # amax of a sample per head
    vs = (np.abs(vf[:100]).max(axis=(0, 2)) / 448.0 / 2.0).astype(np.float32)   # half: values saturate
    p.gpu.set_fp8_scales(ks, vs)
    assert p.orc.set_fp8_scales(ks, vs) == 0
    p.append(k, v, ids)
    p.check_state()
    p.check_decode(random_bf16(rng, (S, h_q, D)), lens)
    with pytest.raises(kvq.KvqError):          # scales are fixed once tokens are stored
        p.gpu.set_fp8_scales(ks, vs)
    p.close()


def test_prefix_lengths_empty_rows_and_seq_map():
    rng = np.random.default_rng(4)
    fmt = FMTS["int4_chan64"]
    h_q, h_kv = 8, 2
    p = Pair(fmt, h_q, h_kv, max_seqs=4, num_blocks=200, mbps=64, seed=2)
    lens = [300, 64, 129, 0]
    ids = np.repeat(np.arange(4, dtype=np.int32), lens)
    n = int(ids.size)
    p.append(outlier_keys(rng, n, h_kv), random_bf16(rng, (n, h_kv, D)), ids)
    q = random_bf16(rng, (4, h_q, D))
    # attend to prefixes (inside quantized groups and inside the window)
    p.check_decode(q, [250, 64, 100, 0])
    p.check_decode(q, [1, 0, 129, 0])
    # rows mapped to other sequences, repeated
    seq_ids = np.array([2, 2, 0, 1], np.int32)
    p.check_decode(q, [129, 65, 300, 64], seq_ids=seq_ids)
    p.close()


def test_caller_block_table():
    rng = np.random.default_rng(5)
    fmt = FMTS["int8_tok_p16"]
    h_q, h_kv = 4, 1
    p = Pair(fmt, h_q, h_kv, max_seqs=3, num_blocks=100, mbps=40, seed=2)
    lens = [100, 37, 250]
    ids = np.repeat(np.arange(3, dtype=np.int32), lens)
    n = int(ids.size)
    p.append(outlier_keys(rng, n, h_kv), random_bf16(rng, (n, h_kv, D)), ids)
    # batch rows (2, 0): a caller-built table of those rows, stride 20
    rows = [2, 0]
    bt = np.full((2, 20), -1, np.int32)
    for r, s in enumerate(rows):
        t = p.orc.block_table(s)
        bt[r, :len(t)] = t
    q = random_bf16(rng, (2, h_q, D))
    got, want = p.decode(q, [lens[2], lens[0]], seq_ids=np.array(rows, np.int32),
                         block_table=torch.tensor(bt, device="cuda"), bt_stride=20)
    assert np.max(np.abs(got - want)) <= ATOL
    p.close()


def test_free_and_reuse_blocks():
    rng = np.random.default_rng(6)
    fmt = FMTS["int4_chan64"]
    p = Pair(fmt, 4, 1, max_seqs=3, num_blocks=40, mbps=40, seed=8)
    for s, L in ((0, 130), (1, 70)):
        p.append(outlier_keys(rng, L, 1), random_bf16(rng, (L, 1, D)), np.full(L, s, np.int32))
    p.check_state()
    p.gpu.free_seq(0)
    assert p.orc.free_seq(0) == 0
    p.append(outlier_keys(rng, 200, 1), random_bf16(rng, (200, 1, D)), np.full(200, 2, np.int32))
    p.check_state()
    p.check_decode(random_bf16(rng, (3, 4, D)), [0, 70, 200])
    p.close()


def test_device_check_flags_bad_lengths():
    rng = np.random.default_rng(2)
    fmt = FMTS["int4_chan64"]
    p = Pair(fmt, 4, 1, max_seqs=2, num_blocks=20, mbps=20, seed=1)
    p.append(outlier_keys(rng, 80, 1), random_bf16(rng, (80, 1, D)), np.zeros(80, np.int32))
    q = bits_to_cuda_bf16(random_bf16(rng, (2, 4, D)))
    sl = torch.tensor([500, -3], dtype=torch.int32, device="cuda")   # beyond the stored length
    out = torch.zeros((2, 4, D), dtype=torch.float32, device="cuda")
    p.gpu.decode(q, sl, out)
    from quantized_kv_cache_14_b200 import kvq
    bits = p.gpu.sync_status()
    assert bits & kvq.KVQ_DEVERR_SEQ_LEN
    assert p.gpu.sync_status() == 0        # cleared
    p.close()


# ----------------------------------------------------------- full workloads

def pool_blocks(lengths, growth, page, residual):
    return int(sum((L + growth + page - 1) // page for L in lengths)) + 64


def run_full(idx, steps_checked=(), max_steps=0, check_every_pool=False):
    w = workload(idx)
    dr = Draws(w, steps=max_steps)
    f = w.fmt
    fmt = dict(bits=f.bits, asym=f.asym, k_axis=f.k_axis, g_k=f.g_k, g_v=f.g_v,
               scale_fp32=f.scale_fp32, residual=f.residual, page=f.page)
    nb = pool_blocks(dr.lengths, max_steps, f.page, f.residual)
    mbps = max((L + max_steps) // f.page + 2 for L in dr.lengths)
    p = Pair(fmt, w.h_q, w.h_kv, max_seqs=w.batch, num_blocks=nb, mbps=mbps, seed=w.seed)
    p.append(dr.k, dr.v, dr.seq_ids)
    p.check_state()
    lens = list(dr.lengths)
    errs = [p.check_decode(dr.q, lens, nthreads=os.cpu_count() or 8)]
    for step in range(max_steps):
        k, v, q = dr.step()
        p.append(k, v, np.arange(w.batch, dtype=np.int32))
        lens = [L + 1 for L in lens]
        if step in steps_checked:
            p.check_state(pool=check_every_pool or step in (0, max_steps - 1))
            errs.append(p.check_decode(q, lens, nthreads=os.cpu_count() or 8))
    p.close()
    return errs


def test_workload_1_tiny_int8():
    run_full(1)


def test_workload_2_int8_paged_gqa():
    run_full(2)


def test_workload_3_int4_kivi():
    run_full(3)


def test_workload_4_int2_asym_long_context():
    run_full(4)


def test_workload_4_without_residual_tail():
    w = workload(4)
    dr = Draws(w, length_override=[131072])
    f = w.fmt
    fmt = dict(bits=f.bits, asym=f.asym, k_axis=f.k_axis, g_k=f.g_k, g_v=f.g_v,
               scale_fp32=f.scale_fp32, residual=f.residual, page=f.page)
    p = Pair(fmt, w.h_q, w.h_kv, max_seqs=1, num_blocks=131072 // 16 + 64, mbps=131072 // 16 + 4,
             seed=w.seed)
    p.append(dr.k, dr.v, dr.seq_ids)
    p.check_state(pool=False)
    p.check_decode(dr.q, [131072], nthreads=os.cpu_count() or 8)
    p.close()


def test_workload_5_continuous_batching():
    steps = int(os.environ.get("KVQ_CB_STEPS", "100"))
    checked = set(range(steps)) if os.environ.get("KVQ_CB_FULL") else {0, 1, 2, 49, 98, 99}
    run_full(5, steps_checked={s for s in checked if s < steps}, max_steps=steps)


@pytest.mark.parametrize("name", ["int4_chan64", "int2_asym_chan32"])
def test_merge_rows_and_repeats(name):
    """Split-K merge of the warp-specialised KIVI kernels: rows that attend
    nothing sit between live rows, and calls alternate batch size and grid
    (pairs move between CTAs, a grid may exceed the resident CTAs and the unit
    count); every call must match the oracle, empty rows giving zeros."""
    rng = np.random.default_rng(12)
    fmt = FMTS[name]
    h_q, h_kv = 8, 2
    p = Pair(fmt, h_q, h_kv, max_seqs=5, num_blocks=700, mbps=128, seed=2)
    lens = [700, 1, 0, 333, 97]
    ids = np.repeat(np.arange(5, dtype=np.int32), lens)
    n = int(ids.size)
    p.append(outlier_keys(rng, n, h_kv), random_bf16(rng, (n, h_kv, D)), ids)
    for grid, attend in ((0, [700, 0, 0, 333, 97]), (3, [0, 1, 0, 0, 97]), (0, [700, 1, 0, 333]),
                         (1024, [650, 1, 0, 300, 0]), (0, [700, 1, 0, 333, 97]), (7, [0, 0])):
        p.gpu.set_decode_grid(grid)
        q = random_bf16(rng, (len(attend), h_q, D))
        got, want = p.decode(q, attend)
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - want)) <= ATOL, (grid, attend)
        for r, L in enumerate(attend):
            if L == 0:
                assert not np.any(got[r]), (grid, r)
    assert p.gpu.sync_status() == 0
    p.close()


@pytest.mark.parametrize("name", ["int4_chan64", "int2_asym_chan32", "int8_tok_p16"])
def test_device_check_flags_corrupted_caller_table(name):
    """A caller block table with entries outside [0, num_blocks) sets
    KVQ_DEVERR_BLOCK_ID: the kernels skip those copies instead of faulting,
    and the next call on the same context decodes as the oracle says."""
    rng = np.random.default_rng(9)
    fmt = FMTS[name]
    h_q, h_kv, S, stride = 8, 2, 2, 40
    p = Pair(fmt, h_q, h_kv, max_seqs=S, num_blocks=120, mbps=stride, seed=4)
    lens = [300, 170]
    ids = np.repeat(np.arange(S, dtype=np.int32), lens)
    p.append(outlier_keys(rng, ids.size, h_kv), random_bf16(rng, (ids.size, h_kv, D)), ids)
    bt = np.full((S, stride), -1, np.int32)
    for s in range(S):
        row = p.gpu.block_table_host(s)
        bt[s, :len(row)] = row
    bad = bt.copy()
    bad[0, 1] = -5
    bad[1, 2] = 120 + 3
    q = random_bf16(rng, (S, h_q, D))
    p.gpu.decode(bits_to_cuda_bf16(q), torch.tensor(lens, dtype=torch.int32, device="cuda"),
                 torch.zeros((S, h_q, D), dtype=torch.float32, device="cuda"),
                 block_table=torch.from_numpy(bad).cuda(), bt_stride=stride)
    from quantized_kv_cache_14_b200 import kvq
    bits = p.gpu.sync_status()
    assert bits & kvq.KVQ_DEVERR_BLOCK_ID, bits
    assert p.gpu.sync_status() == 0
    got, want = p.decode(q, lens, block_table=torch.from_numpy(bt).cuda(), bt_stride=stride)
    assert np.max(np.abs(got - want)) <= ATOL
    assert p.gpu.sync_status() == 0
    p.close()
