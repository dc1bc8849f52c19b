"""kvq_decode_attn_noalloc: decode for callers that cannot allocate device
memory while they decode (a runtime that gives the library a fixed arena, a
process that allocates only at start-up, a serving path where allocation is
forbidden).  The caller owns every buffer; the library's scratch is a fixed
device array.  Its output must match kvq_decode_attn's on the same cache, call
after call.  Collected last, so a failure here comes after every other test
has run."""
import numpy as np
import pytest
import torch

from quantized_kv_cache_14_b200 import build as kbuild
from quantized_kv_cache_14_b200 import kvq
from quantized_kv_cache_14_b200.workloads import random_bf16

pytestmark = pytest.mark.gpu

ATOL = 2e-3
D = 128


def _dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("fmt", [
    dict(bits=4, asym=0, k_axis=1, g_k=64, g_v=64, scale_fp32=0, residual=64, page=16),
    dict(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=16),
])
def test_noalloc_decode_matches_handle_decode(fmt):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kbuild.build()
    rng = np.random.default_rng(21)
    h_q, h_kv, S = 8, 2, 3
    cache = kvq.KVCache(kvq.Format(**fmt), h_q, h_kv, max_seqs=S, num_blocks=80,
                        max_blocks_per_seq=24, seed=4)
    lens = [200, 77, 130]
    ids = np.repeat(np.arange(S, dtype=np.int32), lens)
    cache.append(_dev_bf16(random_bf16(rng, (ids.size, h_kv, D), 3.0)),
                 _dev_bf16(random_bf16(rng, (ids.size, h_kv, D))), ids)
    torch.cuda.synchronize()

    # caller-owned copies of the cache in the library's format
    pool = torch.from_numpy(cache.pool()).cuda()
    if fmt["residual"]:
        kw, vw = cache.residual()
        kwin = torch.from_numpy(kw.view(np.int16)).cuda()
        vwin = torch.from_numpy(vw.view(np.int16)).cuda()
        kptr, vptr = kwin.data_ptr(), vwin.data_ptr()
    else:
        kptr = vptr = 0
    stride = 24
    bt = np.full((S, stride), -1, np.int32)
    for s in range(S):
        row = cache.block_table_host(s)
        bt[s, :len(row)] = row
    bt = torch.from_numpy(bt).cuda()
    stored = torch.tensor(lens, dtype=torch.int32, device="cuda")
    err = torch.full((1,), 0xFFFF, dtype=torch.int32, device="cuda")

    # two calls in a row on the shared scratch: full lengths, then prefixes
    for call, attend in enumerate((lens, [150, 77, 65])):
        q = _dev_bf16(random_bf16(rng, (S, h_q, D)))
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
        assert diff <= ATOL, f"call {call}: max abs difference {diff}"
    assert cache.sync_status() == 0

    # a batch beyond max_seqs is refused with a clear message
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attn_noalloc(cache.cfg, pool.data_ptr(), kptr, vptr, bt.data_ptr(), stride,
                                    stored.data_ptr(), stored.data_ptr(), q.data_ptr(), S + 1,
                                    got.data_ptr(), 0, 0)
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG
    cache.close()
