"""Python face of the CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this module.  It wraps oracle/liboracle.so (plain C++, fp64 attention) and
shares nothing with the CUDA library.  The cache model follows the pages on
KV-cache quantization (llmdaily.org day-65 sections "From BF16 to INT8, INT4,
or even fewer bits", "Why scales and groups matter", "Why some systems keep a
full-precision window", "How this connects to paging and prefix caching";
oh-bug.com "KV Cache Quantization in Practice", KIVI paragraph).

Functions with no independent pin: none -- every exported routine is pinned by
tests/test_oracle_*.py against closed forms, the pages' worked numbers, numpy or
brute force, and tests/test_oracle_mutants.py checks that those pins fail when a
plausible mistake is planted in a copy of the oracle's source.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


class OracleConfig(ctypes.Structure):
    _fields_ = [
        ("bits", ctypes.c_int32), ("asym", ctypes.c_int32), ("k_axis", ctypes.c_int32),
        ("g_k", ctypes.c_int32), ("g_v", ctypes.c_int32), ("scale_fp32", ctypes.c_int32),
        ("residual", ctypes.c_int32), ("page", ctypes.c_int32),
        ("h_q", ctypes.c_int32), ("h_kv", ctypes.c_int32), ("d_h", ctypes.c_int32),
        ("max_seqs", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32), ("seed", ctypes.c_uint64),
        ("fail_alloc_after", ctypes.c_int32), ("fp8", ctypes.c_int32),
    ]


def lib():
    """Loads liboracle.so (built on demand).  KVQ_ORACLE_LIB, when set, names
    another build of the oracle's source to load instead: the pin suites run
    against copies with a planted mistake this way (tests/test_oracle_mutants.py)."""
    global _LIB
    if _LIB is None:
        path = os.environ.get("KVQ_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        L.orc_f32_to_f16.restype = ctypes.c_uint16
        L.orc_f32_to_f16.argtypes = [ctypes.c_float]
        L.orc_f16_to_f32.restype = ctypes.c_float
        L.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_stored_value.restype = ctypes.c_float
        L.orc_stored_value.argtypes = [ctypes.c_float, ctypes.c_int32]
        L.orc_quant_sym.argtypes = [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, P]
        L.orc_quant_asym.argtypes = [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, P, P]
        L.orc_cache_bytes_formula.restype = ctypes.c_double
        L.orc_cache_bytes_formula.argtypes = [ctypes.c_int64] * 4 + [ctypes.c_int32] * 4
        L.orc_splitmix64.argtypes = [ctypes.c_uint64, ctypes.c_int32, P]
        L.orc_free_list.argtypes = [ctypes.c_int32, ctypes.c_uint64, P]
        L.orc_create.restype = P
        L.orc_create.argtypes = [ctypes.POINTER(OracleConfig)]
        L.orc_destroy.argtypes = [P]
        L.orc_layout.argtypes = [P, P]
        L.orc_append.restype = ctypes.c_int32
        L.orc_append.argtypes = [P, P, P, P, ctypes.c_int32]
        L.orc_f32_to_e4m3.restype = ctypes.c_uint8
        L.orc_f32_to_e4m3.argtypes = [ctypes.c_float]
        L.orc_e4m3_to_f32.restype = ctypes.c_float
        L.orc_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        L.orc_set_fp8_scales.restype = ctypes.c_int32
        L.orc_set_fp8_scales.argtypes = [P, P, P]
        L.orc_free_seq.restype = ctypes.c_int32
        L.orc_free_seq.argtypes = [P, ctypes.c_int32]
        L.orc_share_prefix.restype = ctypes.c_int32
        L.orc_share_prefix.argtypes = [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
        L.orc_seq_len.restype = ctypes.c_int32
        L.orc_seq_len.argtypes = [P, ctypes.c_int32]
        L.orc_pool_bytes.restype = ctypes.c_int64
        L.orc_pool_bytes.argtypes = [P]
        L.orc_free_count.restype = ctypes.c_int64
        L.orc_free_count.argtypes = [P]
        L.orc_block_table.restype = ctypes.c_int32
        L.orc_block_table.argtypes = [P, ctypes.c_int32, P, ctypes.c_int32]
        L.orc_read_pool.argtypes = [P, P]
        L.orc_read_residual.argtypes = [P, ctypes.c_int32, ctypes.c_int32, P, P]
        L.orc_dequant.argtypes = [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, P, P]
        L.orc_k_loc.argtypes = [P, ctypes.c_int32, ctypes.c_int32, P, P]
        L.orc_v_loc.argtypes = [P, ctypes.c_int32, ctypes.c_int32, P, P]
        L.orc_decode.argtypes = [P, P, P, P, ctypes.c_int32, P, ctypes.c_int32]
        _LIB = L
    return _LIB


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


# ---- scalar routines --------------------------------------------------------

def f32_to_f16_bits(x: float) -> int:
    return lib().orc_f32_to_f16(float(x))


def f32_to_e4m3(x: float) -> int:
    return int(lib().orc_f32_to_e4m3(float(x)))


def e4m3_to_f32(c: int) -> float:
    return float(lib().orc_e4m3_to_f32(int(c)))


def f16_bits_to_f32(h: int) -> float:
    return lib().orc_f16_to_f32(int(h))


def stored_value(s: float, scale_fp32: bool = False) -> float:
    return lib().orc_stored_value(float(s), int(scale_fp32))


def quant_sym(x, bits: int, scale_fp32: bool = False):
    """Symmetric group quantizer on fp32 values -> (stored scale, int codes)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(x.size, dtype=np.int32)
    sc = np.zeros(1, dtype=np.float32)
    lib().orc_quant_sym(_ptr(x), x.size, bits, int(scale_fp32), _ptr(sc), _ptr(codes))
    return float(sc[0]), codes


def quant_asym(x, bits: int, scale_fp32: bool = False):
    """Asymmetric group quantizer -> (stored scale, stored zero, unsigned codes)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(x.size, dtype=np.int32)
    sc = np.zeros(1, dtype=np.float32)
    z = np.zeros(1, dtype=np.float32)
    lib().orc_quant_asym(_ptr(x), x.size, bits, int(scale_fp32), _ptr(sc), _ptr(z), _ptr(codes))
    return float(sc[0]), float(z[0]), codes


def cache_bytes_formula(layers, tokens, h_kv, d_h, bits, g_k, g_v, meta_bytes):
    return lib().orc_cache_bytes_formula(layers, tokens, h_kv, d_h, bits, g_k, g_v, meta_bytes)


def splitmix64(seed: int, n: int):
    out = np.zeros(n, dtype=np.uint64)
    lib().orc_splitmix64(ctypes.c_uint64(seed), n, _ptr(out))
    return [int(v) for v in out]


def free_list(n: int, seed: int):
    out = np.zeros(n, dtype=np.int32)
    lib().orc_free_list(n, ctypes.c_uint64(seed), _ptr(out))
    return out


# ---- the cache model --------------------------------------------------------

LAYOUT_KEYS = ("n", "row_bytes", "sub_bytes", "secK", "secV", "secVm", "secKm",
               "off_V", "off_Vm", "off_Km", "chunk_bytes", "block_bytes", "kslice")


class OracleCache:
    """CPU model of one layer's quantized paged cache (see kvq_oracle.cpp)."""

    def __init__(self, **cfg):
        self.cfg = dict(cfg)
        c = OracleConfig()
        defaults = dict(asym=0, scale_fp32=0, residual=0, seed=0, fail_alloc_after=-1, fp8=0)
        for k, _ in OracleConfig._fields_:
            setattr(c, k, int(cfg.get(k, defaults.get(k, 0))))
        self._c = c
        self.h = lib().orc_create(ctypes.byref(c))
        arr = np.zeros(13, dtype=np.int64)
        lib().orc_layout(self.h, _ptr(arr))
        self.layout = dict(zip(LAYOUT_KEYS, (int(v) for v in arr)))

    def close(self):
        if self.h:
            lib().orc_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def append(self, k_bits, v_bits, seq_ids) -> int:
        k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
        v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
        seq = np.ascontiguousarray(seq_ids, dtype=np.int32)
        return lib().orc_append(self.h, _ptr(k_bits), _ptr(v_bits), _ptr(seq), int(seq.size))

    def free_seq(self, s: int) -> int:
        return lib().orc_free_seq(self.h, int(s))

    def set_fp8_scales(self, k_scales, v_scales) -> int:
        k = np.ascontiguousarray(k_scales, dtype=np.float32)
        v = np.ascontiguousarray(v_scales, dtype=np.float32)
        return lib().orc_set_fp8_scales(self.h, _ptr(k), _ptr(v))

    def share_prefix(self, src: int, dst: int, tokens: int) -> int:
        return lib().orc_share_prefix(self.h, int(src), int(dst), int(tokens))

    def seq_len(self, s: int) -> int:
        return lib().orc_seq_len(self.h, int(s))

    def free_count(self) -> int:
        return lib().orc_free_count(self.h)

    def block_table(self, s: int):
        n = lib().orc_block_table(self.h, int(s), None, 0)
        out = np.zeros(max(n, 1), dtype=np.int32)
        lib().orc_block_table(self.h, int(s), _ptr(out), n)
        return out[:n]

    def pool(self):
        out = np.zeros(lib().orc_pool_bytes(self.h), dtype=np.uint8)
        lib().orc_read_pool(self.h, _ptr(out))
        return out

    def residual(self, s: int, h: int):
        R, D = self.cfg["residual"], self.cfg["d_h"]
        k = np.zeros((R, D), dtype=np.uint16)
        v = np.zeros((R, D), dtype=np.uint16)
        lib().orc_read_residual(self.h, int(s), int(h), _ptr(k), _ptr(v))
        return k, v

    def dequant(self, s: int, h: int, count: int):
        D = self.cfg["d_h"]
        k = np.zeros((max(count, 1), D), dtype=np.float64)
        v = np.zeros_like(k)
        lib().orc_dequant(self.h, int(s), int(h), int(count), _ptr(k), _ptr(v))
        return k[:count], v[:count]

    def code_loc(self, kind: str, tok: int, ch: int):
        """(byte, bit) of a key ('k') or value ('v') code inside its section."""
        b = np.zeros(1, dtype=np.int64)
        sh = np.zeros(1, dtype=np.int32)
        fn = lib().orc_k_loc if kind == "k" else lib().orc_v_loc
        fn(self.h, int(tok), int(ch), _ptr(b), _ptr(sh))
        return int(b[0]), int(sh[0])

    def decode(self, q_bits, seq_lens, seq_ids=None, nthreads: int = 1):
        q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
        B = q_bits.shape[0]
        lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
        ids = None if seq_ids is None else np.ascontiguousarray(seq_ids, dtype=np.int32)
        out = np.zeros((B, self.cfg["h_q"], self.cfg["d_h"]), dtype=np.float64)
        lib().orc_decode(self.h, _ptr(q_bits), _ptr(ids), _ptr(lens), B, _ptr(out), int(nthreads))
        return out


def bf16_bits_to_f32(bits):
    """bf16 bit patterns -> float32 values (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)
