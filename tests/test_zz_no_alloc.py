"""kvq_decode_attn_noalloc: decode for callers that cannot allocate device
memory while they decode (a runtime that gives the library a fixed arena, a
process that allocates only at start-up, a serving path where allocation is
forbidden).  The caller owns every buffer; the library's scratch is a fixed
device array.  Its output must match kvq_decode_attn's on the same cache and
the CPU oracle's fp64 attention, call after call; sizes past the fixed scratch
are refused with a message; and a small allocation-free plan must not break a
live handle planned for a larger batch.  Collected last, so a failure here
comes after every other test has run."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_kv_cache_14_b200 import build as kbuild
from quantized_kv_cache_14_b200 import kvq
from quantized_kv_cache_14_b200.workloads import random_bf16

pytestmark = pytest.mark.gpu

ATOL = 2e-3
D = 128


def _dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kbuild.build()


def _caller_buffers(cache, fmt, S, stride):
    """Caller-owned device copies of a handle's cache in the library's format."""
    pool = torch.from_numpy(cache.pool()).cuda()
    if fmt["residual"]:
        kw, vw = cache.residual()
        kwin = torch.from_numpy(kw.view(np.int16)).cuda()
        vwin = torch.from_numpy(vw.view(np.int16)).cuda()
    else:
        kwin = vwin = None
    bt = np.full((S, stride), -1, np.int32)
    for s in range(S):
        row = cache.block_table_host(s)
        bt[s, :len(row)] = row
    return pool, kwin, vwin, torch.from_numpy(bt).cuda()


@pytest.mark.parametrize("fmt", [
    dict(bits=4, asym=0, k_axis=1, g_k=64, g_v=64, scale_fp32=0, residual=64, page=16),
    dict(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=16),
    dict(bits=2, asym=1, k_axis=1, g_k=32, g_v=32, scale_fp32=0, residual=32, page=16),
])
def test_noalloc_decode_matches_handle_decode_and_oracle(fmt):
    rng = np.random.default_rng(21)
    h_q, h_kv, S, stride = 8, 2, 3, 24
    cache = kvq.KVCache(kvq.Format(**fmt), h_q, h_kv, max_seqs=S, num_blocks=80,
                        max_blocks_per_seq=stride, seed=4)
    orc = O.OracleCache(**fmt, h_q=h_q, h_kv=h_kv, d_h=D, max_seqs=S, num_blocks=80,
                        max_blocks_per_seq=stride, seed=4, fail_alloc_after=-1)
    lens = [200, 77, 131]
    ids = np.repeat(np.arange(S, dtype=np.int32), lens)
    k, v = random_bf16(rng, (ids.size, h_kv, D), 3.0), random_bf16(rng, (ids.size, h_kv, D))
    cache.append(_dev_bf16(k), _dev_bf16(v), ids)
    assert orc.append(k, v, ids) == 0
    torch.cuda.synchronize()
    pool, kwin, vwin, bt = _caller_buffers(cache, fmt, S, stride)
    kptr = kwin.data_ptr() if kwin is not None else 0
    vptr = vwin.data_ptr() if vwin is not None else 0
    stored = torch.tensor(lens, dtype=torch.int32, device="cuda")
    err = torch.full((1,), 0xFFFF, dtype=torch.int32, device="cuda")

    # two calls in a row on the shared scratch: full lengths, then prefixes
    for call, attend in enumerate((lens, [150, 77, 65])):
        qb = random_bf16(rng, (S, h_q, D))
        q = _dev_bf16(qb)
        sl = torch.tensor(attend, dtype=torch.int32, device="cuda")
        ref = torch.empty((S, h_q, D), dtype=torch.float32, device="cuda")
        got = torch.full((S, h_q, D), float("nan"), dtype=torch.float32, device="cuda")
        cache.decode(q, sl, ref)
        kvq.kvq_decode_attn_noalloc(cache.cfg, pool.data_ptr(), kptr, vptr, bt.data_ptr(), stride,
                                    stored.data_ptr(), sl.data_ptr(), q.data_ptr(), S, got.data_ptr(),
                                    err.data_ptr(), torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"device check bits {err.item():#x} on call {call}"
        assert torch.isfinite(got).all()
        diff = float((got - ref).abs().max())
        assert diff <= ATOL, f"call {call}: max abs difference to kvq_decode_attn {diff}"
        want = orc.decode(qb, attend)
        err_orc = float(np.max(np.abs(got.cpu().numpy().astype(np.float64) - want)))
        assert err_orc <= ATOL, f"call {call}: max abs error to the oracle {err_orc}"
    assert cache.sync_status() == 0

    # a batch beyond max_seqs is refused with a clear message
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attn_noalloc(cache.cfg, pool.data_ptr(), kptr, vptr, bt.data_ptr(), stride,
                                    stored.data_ptr(), stored.data_ptr(), q.data_ptr(), S + 1,
                                    got.data_ptr(), 0, 0)
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG
    cache.close()
    orc.close()


def test_noalloc_refuses_batches_past_the_fixed_scratch():
    """batch within max_seqs whose split-K records outgrow the fixed array:
    refused before any launch, with both sizes in the message."""
    fmt = dict(bits=4, asym=0, k_axis=1, g_k=64, g_v=64, scale_fp32=0, residual=64, page=16)
    cfg = kvq.make_config(**fmt, h_q=32, h_kv=8, d_h=D, max_seqs=512, num_blocks=16, max_blocks_per_seq=4)
    buf = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    p = buf.data_ptr()
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attn_noalloc(cfg, p, p, p, p, 4, p, p, p, 300, p, 0, 0)
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG
    assert "too large for the fixed decode scratch" in str(e.value)


def test_small_noalloc_plan_keeps_a_larger_handle_working():
    """The decode kernel's shared-memory limit is shared by every caller on a
    device: an allocation-free call planned for 3 rows must not lower it
    under a live handle planned for 64."""
    fmt = dict(bits=4, asym=0, k_axis=1, g_k=64, g_v=64, scale_fp32=0, residual=64, page=16)
    rng = np.random.default_rng(5)
    h_q, h_kv, S = 8, 2, 64
    big = kvq.KVCache(kvq.Format(**fmt), h_q, h_kv, max_seqs=S, num_blocks=400, max_blocks_per_seq=16, seed=1)
    lens = [int(x) for x in rng.integers(1, 150, size=S)]
    ids = np.repeat(np.arange(S, dtype=np.int32), lens)
    big.append(_dev_bf16(random_bf16(rng, (ids.size, h_kv, D))), _dev_bf16(random_bf16(rng, (ids.size, h_kv, D))),
               ids)
    q = _dev_bf16(random_bf16(rng, (S, h_q, D)))
    before = torch.empty((S, h_q, D), dtype=torch.float32, device="cuda")
    big.decode(q, None, before)
    torch.cuda.synchronize()

    small = kvq.KVCache(kvq.Format(**fmt), h_q, h_kv, max_seqs=3, num_blocks=40, max_blocks_per_seq=8, seed=2)
    n = 70
    small.append(_dev_bf16(random_bf16(rng, (n, h_kv, D))), _dev_bf16(random_bf16(rng, (n, h_kv, D))),
                 np.zeros(n, np.int32))
    torch.cuda.synchronize()
    pool, kwin, vwin, bt = _caller_buffers(small, fmt, 3, 8)
    stored = torch.tensor([n, 0, 0], dtype=torch.int32, device="cuda")
    qs = _dev_bf16(random_bf16(rng, (3, h_q, D)))
    out = torch.empty((3, h_q, D), dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attn_noalloc(small.cfg, pool.data_ptr(), kwin.data_ptr(), vwin.data_ptr(), bt.data_ptr(), 8,
                                stored.data_ptr(), stored.data_ptr(), qs.data_ptr(), 3, out.data_ptr(), 0,
                                torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()

    after = torch.empty_like(before)
    big.decode(q, None, after)      # the 64-row launch still fits its limit
    torch.cuda.synchronize()
    assert big.sync_status() == 0
    assert torch.equal(before, after)
    big.close()
    small.close()
