"""GPU parity on the quantizer's edge cases (llmdaily.org day-65, "From BF16
to INT8, INT4, or even fewer bits", with the readings of its silent points):
all-zero groups, constant groups, exact ties x / s = k + 1/2, fp16 scales that
saturate (the clip fires) or underflow to 0, and fp16 subnormal scales, fed
through the CUDA append kernels of every format family -- token-axis keys,
channel-axis keys (the window flush), asymmetric zero-points, fp32 scales and
FP8.  The whole pool must equal the oracle's byte for byte.  Sequence 0 holds
every kind but saturation and is also decoded (attention within 2e-3);
sequence 1 adds the saturating groups, whose huge values make attention
meaningless, so only its bytes are compared."""
import numpy as np
import pytest
import torch

from quantized_kv_cache_14_b200 import build as kbuild
from quantized_kv_cache_14_b200.workloads import random_bf16
from tests.gpu_util import Pair
from tests.quant_edges import KINDS, MILD, edge_rows
from tests.test_gpu_parity import FMTS

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kbuild.build()


FAMILIES = ["int8_tok_p16", "int8_tok_p512_fp32", "int4_chan64", "int4_chan64_fp32", "int2_asym_chan32",
            "int4_asym_tok32", "int8_asym_chan128_p64", "int2_sym_tok64_fp32", "fp8_p16"]


@pytest.mark.parametrize("name", FAMILIES)
def test_quantizer_edges_bit_exact(name):
    fmt = FMTS[name]
    rng = np.random.default_rng(len(name))
    h_q, h_kv = 8, 2
    unit = fmt["residual"] or 64
    p = Pair(fmt, h_q, h_kv, max_seqs=2, num_blocks=200, mbps=64, seed=3)
    # bulk: two whole key groups (or 128 tokens) per sequence plus a tail
    n0 = 2 * unit + 5
    k0, v0 = edge_rows(fmt, n0, h_kv, D, MILD, rng)
    k1, v1 = edge_rows(fmt, n0, h_kv, D, KINDS, rng, phase=3)
    p.append(np.concatenate([k0, k1]), np.concatenate([v0, v1]),
             np.repeat(np.arange(2, dtype=np.int32), n0))
    p.check_state()
    # single-token steps up to the next group boundary (flush inside a step)
    steps = unit - 5 + 2
    ks0, vs0 = edge_rows(fmt, steps, h_kv, D, MILD, rng, phase=1)
    ks1, vs1 = edge_rows(fmt, steps, h_kv, D, KINDS, rng, phase=5)
    for t in range(steps):
        p.append(np.stack([ks0[t], ks1[t]]), np.stack([vs0[t], vs1[t]]), np.arange(2, dtype=np.int32))
    p.check_state()
    L = n0 + steps
    q = random_bf16(rng, (1, h_q, D))
    p.check_decode(q, [L])
    p.close()


@pytest.mark.parametrize("name", ["int4_chan64", "int2_asym_chan32"])
def test_large_key_scales_decode(name):
    """Keys of a few times 2^14 (fp16 scales in the thousands, well short of
    saturation) with q near 2^-14, so the scores are ordinary: the key scale times q must
    not overflow fp16 on any decode path, including the whole-unit paths of the
    KIVI formats that weight parts of q by powers of two."""
    fmt = FMTS[name]
    rng = np.random.default_rng(11)
    h_q, h_kv = 8, 2
    p = Pair(fmt, h_q, h_kv, max_seqs=2, num_blocks=200, mbps=64, seed=5)
    lens = [3 * fmt["g_k"] + 7, 2 * fmt["g_k"] + 40]
    ids = np.repeat(np.arange(2, dtype=np.int32), lens)
    k = random_bf16(rng, (ids.size, h_kv, D), 2.0 ** 14)
    v = random_bf16(rng, (ids.size, h_kv, D))
    p.append(k, v, ids)
    p.check_state()
    q = random_bf16(rng, (2, h_q, D), 2.0 ** -14)
    p.check_decode(q, lens)
    p.check_decode(q, [lens[0] - 20, lens[1] - 45])   # prefixes that end inside key groups
    p.close()
