"""Thin Python binding of libkvq.so (include/kvq.h): argument marshalling only.

Every step of the cache runs in the library's CUDA kernels; there is no Python
or CPU fallback.  If libkvq.so has not been built this module raises on first
use (build it with `python -m quantized_kv_cache_14_b200.build`).

Functions keep the C names (kvq_create, kvq_append, kvq_decode_attn, ...).
Device pointers are passed as ints (e.g. torch.Tensor.data_ptr()), host arrays
as numpy arrays, streams as ints (torch.cuda.Stream.cuda_stream) or 0.
`KVCache` bundles a handle with torch-tensor conveniences.
"""
import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# KVQ_DEBUG=1 in the environment selects the debug build (kernels check every
# index they compute; build.py --debug)
LIB_PATH = os.path.join(_HERE, "libkvq_debug.so" if os.environ.get("KVQ_DEBUG") == "1" else "libkvq.so")

KVQ_OK = 0
KVQ_ERR_INVALID_ARG = 1
KVQ_ERR_OOM = 2
KVQ_ERR_BAD_SEQ = 3
KVQ_ERR_CUDA = 4
KVQ_ERR_DEVICE_CHECK = 5
KVQ_ERR_UNSUPPORTED = 6

KVQ_DEVERR_BLOCK_ID = 0x1
KVQ_DEVERR_SEQ_LEN = 0x2
KVQ_DEVERR_TIMEOUT = 0x4
KVQ_DEVERR_SEQ_ID = 0x8
KVQ_DEVERR_SMEM = 0x10
KVQ_DEVERR_INDEX = 0x20

KVQ_AXIS_TOKEN = 0
KVQ_AXIS_CHANNEL = 1

# Every symbol of include/kvq.h (checked by tests/test_abi.py).
EXPORTS = (
    "kvq_create", "kvq_destroy", "kvq_append", "kvq_decode_attn", "kvq_block_table",
    "kvq_block_table_host", "kvq_seq_len", "kvq_seq_lens_device", "kvq_free_seq", "kvq_share_prefix",
    "kvq_stats", "kvq_cache_bytes", "kvq_layout", "kvq_read_pool", "kvq_read_residual",
    "kvq_sync_status", "kvq_set_decode_grid", "kvq_set_decode_event", "kvq_decode_attn_noalloc",
    "kvq_prefill_attn", "kvq_set_fp8_scales", "kvq_step_host", "kvq_last_error",
    "kvq_pool_device", "kvq_read_floor",
)


class KvqError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"kvq status {status}: {msg}")
        self.status = status


class KvqConfig(ctypes.Structure):
    _fields_ = [
        ("bits", ctypes.c_int32), ("asym", ctypes.c_int32), ("k_axis", ctypes.c_int32),
        ("g_k", ctypes.c_int32), ("g_v", ctypes.c_int32), ("scale_fp32", ctypes.c_int32),
        ("residual", ctypes.c_int32), ("page", ctypes.c_int32),
        ("h_q", ctypes.c_int32), ("h_kv", ctypes.c_int32), ("d_h", ctypes.c_int32),
        ("max_seqs", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32), ("seed", ctypes.c_uint64),
        ("fail_alloc_after", ctypes.c_int32), ("host_only", ctypes.c_int32),
        ("device", ctypes.c_int32), ("fp8", ctypes.c_int32),
    ]


class KvqLayoutInfo(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in (
        "row_bytes", "sub_bytes", "off_v", "off_vmeta", "off_kmeta", "chunk_bytes",
        "block_bytes", "kslice")]


class KvqStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in (
        "blocks_used", "blocks_free", "tokens_stored", "bytes_pool", "bytes_residual",
        "bytes_workspace", "bytes_formula", "kernel_launches")]


_LIB = None


def lib():
    """Loads libkvq.so; raises if it is missing (no fallback path exists)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run python -m quantized_kv_cache_14_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64
        st = ctypes.c_int
        sig = {
            "kvq_create": (st, [ctypes.POINTER(KvqConfig), ctypes.POINTER(P)]),
            "kvq_destroy": (None, [P]),
            "kvq_append": (st, [P, P, P, P, I32, P]),
            "kvq_decode_attn": (st, [P, P, P, I32, P, P, I32, P, P]),
            "kvq_block_table": (st, [P, ctypes.POINTER(P), ctypes.POINTER(I32)]),
            "kvq_block_table_host": (st, [P, I32, P, I32, ctypes.POINTER(I32)]),
            "kvq_seq_len": (st, [P, I32, ctypes.POINTER(I32)]),
            "kvq_seq_lens_device": (st, [P, ctypes.POINTER(P)]),
            "kvq_free_seq": (st, [P, I32, P]),
            "kvq_share_prefix": (st, [P, I32, I32, I32, P]),
            "kvq_prefill_attn": (st, [P, P, P, P, I32, P, P]),
            "kvq_step_host": (st, [P, P, P, P, I32, P, I32, P, P]),
            "kvq_set_fp8_scales": (st, [P, P, P]),
            "kvq_stats": (st, [P, ctypes.POINTER(KvqStats)]),
            "kvq_cache_bytes": (U64, [I32, ctypes.c_int64, I32, I32, ctypes.POINTER(KvqConfig)]),
            "kvq_layout": (st, [ctypes.POINTER(KvqConfig), ctypes.POINTER(KvqLayoutInfo)]),
            "kvq_read_pool": (st, [P, P, U64, P]),
            "kvq_read_residual": (st, [P, P, P, U64, P]),
            "kvq_sync_status": (st, [P, P, ctypes.POINTER(ctypes.c_uint32)]),
            "kvq_set_decode_grid": (st, [P, I32]),
            "kvq_set_decode_event": (st, [P, P]),
            "kvq_decode_attn_noalloc": (st, [ctypes.POINTER(KvqConfig), P, P, P, P, I32, P, P, P, I32,
                                             P, P, P]),
            "kvq_last_error": (ctypes.c_char_p, []),
            "kvq_pool_device": (st, [P, ctypes.POINTER(P), ctypes.POINTER(U64)]),
            "kvq_read_floor": (st, [P, P, ctypes.c_int64, ctypes.c_int64, I32, I32, I32, I32, I32, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _check(status):
    if status != KVQ_OK:
        raise KvqError(status, lib().kvq_last_error().decode())


def _host_i32(a):
    if a is None:
        return None, None
    arr = np.ascontiguousarray(a, dtype=np.int32)
    return arr, ctypes.c_void_p(arr.ctypes.data)


def make_config(bits, asym, k_axis, g_k, g_v, scale_fp32, residual, page, h_q, h_kv, d_h,
                max_seqs, num_blocks, max_blocks_per_seq, seed=0, fail_alloc_after=-1,
                host_only=0, device=0, fp8=0) -> KvqConfig:
    return KvqConfig(bits, asym, k_axis, g_k, g_v, scale_fp32, residual, page, h_q, h_kv, d_h,
                     max_seqs, num_blocks, max_blocks_per_seq, seed, fail_alloc_after,
                     host_only, device, fp8)


# ---- the C calls, same names --------------------------------------------------

def kvq_create(cfg: KvqConfig):
    h = ctypes.c_void_p()
    _check(lib().kvq_create(ctypes.byref(cfg), ctypes.byref(h)))
    return h


def kvq_destroy(h):
    lib().kvq_destroy(h)


def kvq_append(h, k_ptr: int, v_ptr: int, seq_ids, n: int, stream: int = 0):
    arr, p = _host_i32(seq_ids)
    _check(lib().kvq_append(h, ctypes.c_void_p(k_ptr), ctypes.c_void_p(v_ptr), p, int(n),
                            ctypes.c_void_p(stream)))


def kvq_decode_attn(h, q_ptr: int, block_table_ptr: int, bt_stride: int, seq_lens_ptr: int,
                    seq_ids, batch: int, out_ptr: int, stream: int = 0):
    arr, p = _host_i32(seq_ids)
    _check(lib().kvq_decode_attn(h, ctypes.c_void_p(q_ptr), ctypes.c_void_p(block_table_ptr or None),
                                 int(bt_stride), ctypes.c_void_p(seq_lens_ptr), p, int(batch),
                                 ctypes.c_void_p(out_ptr), ctypes.c_void_p(stream)))


def kvq_block_table(h):
    p, s = ctypes.c_void_p(), ctypes.c_int32()
    _check(lib().kvq_block_table(h, ctypes.byref(p), ctypes.byref(s)))
    return p.value, s.value


def kvq_block_table_host(h, seq: int):
    n = ctypes.c_int32()
    _check(lib().kvq_block_table_host(h, int(seq), None, 0, ctypes.byref(n)))
    out = np.zeros(max(n.value, 1), dtype=np.int32)
    _check(lib().kvq_block_table_host(h, int(seq), ctypes.c_void_p(out.ctypes.data), n.value,
                                      ctypes.byref(n)))
    return out[:n.value]


def kvq_seq_len(h, seq: int) -> int:
    n = ctypes.c_int32()
    _check(lib().kvq_seq_len(h, int(seq), ctypes.byref(n)))
    return n.value


def kvq_seq_lens_device(h) -> int:
    p = ctypes.c_void_p()
    _check(lib().kvq_seq_lens_device(h, ctypes.byref(p)))
    return p.value


def kvq_free_seq(h, seq: int, stream: int = 0):
    _check(lib().kvq_free_seq(h, int(seq), ctypes.c_void_p(stream)))


def kvq_prefill_attn(h, q_ptr: int, seq_ids, positions, out_ptr: int, stream: int = 0):
    ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    assert ids.shape == pos.shape
    V = ctypes.c_void_p
    _check(lib().kvq_prefill_attn(h, V(q_ptr), V(ids.ctypes.data), V(pos.ctypes.data), int(ids.size), V(out_ptr),
                                  V(stream)))


def kvq_step_host(h, k_ptr: int, v_ptr: int, seq_ids, q_ptr: int, batch: int, out_ptr: int,
                  stream: int = 0):
    """Host pointers: k, v bf16 [n][h_kv][d_h]; q bf16 [batch][h_q][d_h]; out fp32."""
    arr, p = _host_i32(seq_ids)
    n = 0 if arr is None else int(arr.size)
    V = ctypes.c_void_p
    _check(lib().kvq_step_host(h, V(k_ptr or None), V(v_ptr or None), p, n, V(q_ptr or None), int(batch),
                               V(out_ptr or None), V(stream)))


def kvq_set_fp8_scales(h, k_scales, v_scales):
    k = np.ascontiguousarray(k_scales, dtype=np.float32)
    v = np.ascontiguousarray(v_scales, dtype=np.float32)
    _check(lib().kvq_set_fp8_scales(h, ctypes.c_void_p(k.ctypes.data), ctypes.c_void_p(v.ctypes.data)))


def kvq_share_prefix(h, src_seq: int, dst_seq: int, tokens: int, stream: int = 0):
    _check(lib().kvq_share_prefix(h, int(src_seq), int(dst_seq), int(tokens), ctypes.c_void_p(stream)))


def kvq_stats(h) -> dict:
    s = KvqStats()
    _check(lib().kvq_stats(h, ctypes.byref(s)))
    return {n: getattr(s, n) for n, _ in KvqStats._fields_}


def kvq_cache_bytes(layers: int, tokens: int, h_kv: int, d_h: int, cfg: KvqConfig) -> int:
    return int(lib().kvq_cache_bytes(int(layers), int(tokens), int(h_kv), int(d_h), ctypes.byref(cfg)))


def kvq_layout(cfg: KvqConfig) -> dict:
    li = KvqLayoutInfo()
    _check(lib().kvq_layout(ctypes.byref(cfg), ctypes.byref(li)))
    return {n: getattr(li, n) for n, _ in KvqLayoutInfo._fields_}


def kvq_read_pool(h, nbytes: int, stream: int = 0) -> np.ndarray:
    out = np.empty(int(nbytes), dtype=np.uint8)
    _check(lib().kvq_read_pool(h, ctypes.c_void_p(out.ctypes.data), int(nbytes), ctypes.c_void_p(stream)))
    return out


def kvq_read_residual(h, nbytes: int, stream: int = 0):
    k = np.empty(int(nbytes) // 2, dtype=np.uint16)
    v = np.empty_like(k)
    _check(lib().kvq_read_residual(h, ctypes.c_void_p(k.ctypes.data), ctypes.c_void_p(v.ctypes.data),
                                   int(nbytes), ctypes.c_void_p(stream)))
    return k, v


def kvq_sync_status(h, stream: int = 0) -> int:
    """Returns the device error bits; raises KvqError on a CUDA error."""
    bits = ctypes.c_uint32()
    st = lib().kvq_sync_status(h, ctypes.c_void_p(stream), ctypes.byref(bits))
    if st not in (KVQ_OK, KVQ_ERR_DEVICE_CHECK):
        _check(st)
    return bits.value


def kvq_set_decode_grid(h, ctas: int):
    _check(lib().kvq_set_decode_grid(h, int(ctas)))


def kvq_set_decode_event(h, event: int):
    _check(lib().kvq_set_decode_event(h, ctypes.c_void_p(event or None)))


def kvq_decode_attn_noalloc(cfg: KvqConfig, pool_ptr: int, k_window_ptr: int, v_window_ptr: int,
                            block_table_ptr: int, bt_stride: int, stored_lens_ptr: int,
                            seq_lens_ptr: int, q_ptr: int, batch: int, out_ptr: int,
                            error_bits_ptr: int = 0, stream: int = 0):
    """Decode over caller-owned device buffers; the library allocates nothing
    (its scratch is a fixed device array).  Pointers are device addresses."""
    V = ctypes.c_void_p
    _check(lib().kvq_decode_attn_noalloc(ctypes.byref(cfg), V(pool_ptr), V(k_window_ptr or None),
                                         V(v_window_ptr or None), V(block_table_ptr), int(bt_stride),
                                         V(stored_lens_ptr), V(seq_lens_ptr), V(q_ptr), int(batch),
                                         V(out_ptr), V(error_bits_ptr or None), V(stream)))


def kvq_pool_device(h):
    """(device address, bytes) of the handle's block pool."""
    p, n = ctypes.c_void_p(), ctypes.c_uint64()
    _check(lib().kvq_pool_device(h, ctypes.byref(p), ctypes.byref(n)))
    return p.value, n.value


def kvq_read_floor(base_ptr: int, offsets_ptr: int, n_chunks: int, span_bytes: int, chunk_bytes: int,
                   mode: int, ctas: int, stages: int, per_unit: int, sink_ptr: int, stream: int = 0):
    """The HBM read-floor measurement kernel (device pointers as ints)."""
    V = ctypes.c_void_p
    _check(lib().kvq_read_floor(V(base_ptr), V(offsets_ptr or None), int(n_chunks), int(span_bytes),
                                int(chunk_bytes), int(mode), int(ctas), int(stages), int(per_unit),
                                V(sink_ptr), V(stream)))


def kvq_last_error() -> str:
    return lib().kvq_last_error().decode()


# ---- convenience wrapper --------------------------------------------------------

@dataclass
class Format:
    bits: int
    asym: int
    k_axis: int
    g_k: int
    g_v: int
    scale_fp32: int
    residual: int
    page: int
    fp8: int = 0


class KVCache:
    """One layer's quantized paged cache on a CUDA device (torch tensors in/out)."""

    def __init__(self, fmt, h_q, h_kv, max_seqs, num_blocks, max_blocks_per_seq, d_h=128,
                 seed=0, device=0, fail_alloc_after=-1, host_only=False):
        self.fmt = fmt
        self.cfg = make_config(fmt.bits, fmt.asym, fmt.k_axis, fmt.g_k, fmt.g_v, fmt.scale_fp32,
                               fmt.residual, fmt.page, h_q, h_kv, d_h, max_seqs, num_blocks,
                               max_blocks_per_seq, seed, fail_alloc_after, int(host_only), device,
                               int(getattr(fmt, "fp8", 0)))
        self.h = kvq_create(self.cfg)
        self.h_q, self.h_kv, self.d_h = h_q, h_kv, d_h
        self.layout = kvq_layout(self.cfg)

    def close(self):
        if getattr(self, "h", None):
            kvq_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @staticmethod
    def _stream(stream):
        if stream is None:
            import torch
            return torch.cuda.current_stream().cuda_stream
        return int(stream)

    def append(self, k, v, seq_ids, stream=None):
        """k, v: CUDA bf16 tensors [n, h_kv, d_h]; seq_ids: host int sequence ids."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
        n = int(ids.size)
        if n == 0:
            return
        kp = k.data_ptr() if k is not None else 0
        vp = v.data_ptr() if v is not None else 0
        kvq_append(self.h, kp, vp, ids, n, 0 if self.cfg.host_only else self._stream(stream))

    def decode(self, q, seq_lens, out, block_table=None, bt_stride=0, seq_ids=None, stream=None):
        """q: CUDA bf16 [B, h_q, d_h]; seq_lens: CUDA int32 [B], or None to attend
        over every stored token of sequences 0..B-1 (the library's own device
        lengths, so no length update is needed between appends and decodes);
        out: CUDA fp32 [B, h_q, d_h]."""
        B = int(q.shape[0])
        bt = block_table.data_ptr() if block_table is not None else 0
        if seq_lens is None:
            if seq_ids is not None or block_table is not None:
                raise ValueError("seq_lens=None needs rows 0..B-1 to be sequences 0..B-1")
            sl = kvq_seq_lens_device(self.h)
        else:
            sl = seq_lens.data_ptr()
        kvq_decode_attn(self.h, q.data_ptr(), bt, bt_stride, sl, seq_ids, B,
                        out.data_ptr(), self._stream(stream))

    def step_host(self, k, v, seq_ids, q, out, stream=None):
        """One decode step from host memory (kvq_step_host): CPU tensors k, v
        bf16 [n, h_kv, d_h] (pinned for asynchronous copies), seq_ids int32 [n],
        q bf16 [B, h_q, d_h]; out, CPU fp32 [B, h_q, d_h], is written once the
        stream reaches the end of the step."""
        for t in (k, v, q, out):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("step_host takes contiguous CPU tensors")
        kvq_step_host(self.h, k.data_ptr(), v.data_ptr(), seq_ids, q.data_ptr(), int(q.shape[0]),
                      out.data_ptr(), self._stream(stream))

    def seq_len(self, s):
        return kvq_seq_len(self.h, s)

    def block_table_host(self, s):
        return kvq_block_table_host(self.h, s)

    def free_seq(self, s, stream=None):
        kvq_free_seq(self.h, s, 0 if self.cfg.host_only else self._stream(stream))

    def prefill_attn(self, q, seq_ids, positions, out, stream=None):
        """q: cuda bf16 [n, h_q, d_h]; out: cuda fp32 [n, h_q, d_h]; row i attends
        positions 0..positions[i] of sequence seq_ids[i]."""
        kvq_prefill_attn(self.h, q.data_ptr(), seq_ids, positions, out.data_ptr(), self._stream(stream))

    def set_fp8_scales(self, k_scales, v_scales):
        kvq_set_fp8_scales(self.h, k_scales, v_scales)

    def share_prefix(self, src, dst, tokens, stream=None):
        kvq_share_prefix(self.h, src, dst, tokens, 0 if self.cfg.host_only else self._stream(stream))

    def pool(self, stream=None):
        return kvq_read_pool(self.h, self.cfg.num_blocks * self.layout["block_bytes"], self._stream(stream))

    def residual(self, stream=None):
        c = self.cfg
        nbytes = c.max_seqs * c.h_kv * c.residual * c.d_h * 2
        k, v = kvq_read_residual(self.h, nbytes, self._stream(stream))
        shape = (c.max_seqs, c.h_kv, c.residual, c.d_h)
        return k.reshape(shape), v.reshape(shape)

    def sync_status(self, stream=None):
        return kvq_sync_status(self.h, self._stream(stream))

    def stats(self):
        return kvq_stats(self.h)

    def pool_device(self):
        return kvq_pool_device(self.h)

    def set_decode_grid(self, ctas):
        kvq_set_decode_grid(self.h, ctas)

    def set_decode_event(self, event):
        """event: torch.cuda.Event (recorded between attention and merge) or None."""
        kvq_set_decode_event(self.h, event.cuda_event if event is not None else 0)
