"""Helpers for the GPU parity tests: drive the CUDA library and the CPU oracle
with the same seeded inputs and compare them."""
import numpy as np
import torch

from oracle import oracle as O
from quantized_kv_cache_14_b200 import kvq

ATOL = 2e-3     # attention output: max-abs error against the fp64 oracle


def bits_to_cuda_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


_CUDART = None


def d2h(ptr: int, nbytes: int) -> np.ndarray:
    """Copies nbytes of device memory at ptr to a new host array (cudart)."""
    global _CUDART
    import ctypes
    if _CUDART is None:
        _CUDART = ctypes.CDLL("libcudart.so.12")
        _CUDART.cudaMemcpy.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int]
    out = np.empty(nbytes, dtype=np.uint8)
    torch.cuda.synchronize()
    assert _CUDART.cudaMemcpy(out.ctypes.data, ptr, nbytes, 2) == 0   # device to host
    return out


class Pair:
    """A GPU cache and its oracle twin, built from one format dict."""

    def __init__(self, fmt: dict, h_q: int, h_kv: int, max_seqs: int, num_blocks: int,
                 mbps: int, seed: int = 0, d_h: int = 128):
        self.fmt = dict(fmt)
        self.h_q, self.h_kv, self.d_h = h_q, h_kv, d_h
        self.gpu = kvq.KVCache(kvq.Format(**fmt), h_q, h_kv, max_seqs, num_blocks, mbps, d_h=d_h,
                               seed=seed)
        self.orc = O.OracleCache(**fmt, h_q=h_q, h_kv=h_kv, d_h=d_h, max_seqs=max_seqs,
                                 num_blocks=num_blocks, max_blocks_per_seq=mbps, seed=seed,
                                 fail_alloc_after=-1)
        self.max_seqs = max_seqs

    def close(self):
        self.gpu.close()
        self.orc.close()

    def append(self, k_bits, v_bits, ids):
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        self.gpu.append(bits_to_cuda_bf16(k_bits), bits_to_cuda_bf16(v_bits), ids)
        assert self.orc.append(k_bits, v_bits, ids) == 0

    def share_prefix(self, src, dst, tokens):
        self.gpu.share_prefix(src, dst, tokens)
        assert self.orc.share_prefix(src, dst, tokens) == 0

    def check_state(self, pool=True):
        torch.cuda.synchronize()
        assert self.gpu.sync_status() == 0
        for s in range(self.max_seqs):
            assert self.gpu.seq_len(s) == self.orc.seq_len(s)
            assert self.gpu.block_table_host(s).tolist() == self.orc.block_table(s).tolist()
        # the device copy of the block table equals the host one
        ptr, stride = kvq.kvq_block_table(self.gpu.h)
        dev = d2h(ptr, self.max_seqs * stride * 4).view(np.int32).reshape(self.max_seqs, stride)
        for s in range(self.max_seqs):
            bt = self.orc.block_table(s)
            assert dev[s, :len(bt)].tolist() == bt.tolist()
            assert np.all(dev[s, len(bt):] == -1)
        if pool:
            g, o = self.gpu.pool(), self.orc.pool()
            if not np.array_equal(g, o):
                bad = np.nonzero(g != o)[0]
                raise AssertionError(f"pool differs at {bad.size} bytes, first {bad[:8]}")
        R = self.fmt["residual"]
        if R:
            kr, vr = self.gpu.residual()
            for s in range(self.max_seqs):
                L = self.orc.seq_len(s)
                occ = L % R
                for h in range(self.h_kv):
                    ok_, ov_ = self.orc.residual(s, h)
                    for j in range(occ):
                        slot = (L - occ + j) % R
                        assert np.array_equal(kr[s, h, slot], ok_[slot])
                        assert np.array_equal(vr[s, h, slot], ov_[slot])

    def decode(self, q_bits, lens, seq_ids=None, block_table=None, bt_stride=0, nthreads=8):
        B = q_bits.shape[0]
        q = bits_to_cuda_bf16(q_bits)
        sl = torch.tensor(np.asarray(lens, dtype=np.int32), device="cuda")
        out = torch.full((B, self.h_q, self.d_h), float("nan"), dtype=torch.float32, device="cuda")
        self.gpu.decode(q, sl, out, block_table=block_table, bt_stride=bt_stride, seq_ids=seq_ids)
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64)
        want = self.orc.decode(q_bits, lens, seq_ids=seq_ids, nthreads=nthreads)
        return got, want

    def check_decode(self, q_bits, lens, **kw):
        got, want = self.decode(q_bits, lens, **kw)
        assert self.gpu.sync_status() == 0
        assert np.all(np.isfinite(got))
        err = float(np.max(np.abs(got - want))) if got.size else 0.0
        assert err <= ATOL, f"max abs error {err}"
        return err
