"""Pins of the CPU oracle's scalar routines against things other than itself:
the pages' printed numbers, closed forms, IEEE conversions done by numpy,
published generator vectors and brute force.  CPU only."""
import math

import numpy as np
import torch
import pytest

from oracle import oracle as O
from tests.conftest import read_golden


# ---------------------------------------------------------------- fp16 / bf16

def test_f32_to_f16_matches_numpy_random():
    rng = np.random.default_rng(123)
    mant = rng.standard_normal(400_000).astype(np.float32)
    expo = rng.integers(-30, 18, size=mant.size)
    x = (mant * np.float32(2.0) ** expo.astype(np.float32)).astype(np.float32)
    want = x.astype(np.float16).view(np.uint16)
    got = np.array([O.f32_to_f16_bits(v) for v in x], dtype=np.uint16)
    assert np.array_equal(got, want)


def test_f32_to_f16_edge_cases():
    cases = np.array([0.0, -0.0, 1.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9,
                      2.0 ** -14, 2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0001, 3 * 2.0 ** -26,
                      1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2.0 ** -26, 6e-8, 5.96e-8,
                      np.inf, -np.inf], dtype=np.float32)
    want = cases.astype(np.float16).view(np.uint16)
    got = np.array([O.f32_to_f16_bits(v) for v in cases], dtype=np.uint16)
    assert np.array_equal(got, want)
    assert O.f32_to_f16_bits(float("nan")) & 0x7C00 == 0x7C00


def test_f16_to_f32_all_patterns():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = pats.view(np.float16).astype(np.float32)
    got = np.array([O.f16_bits_to_f32(int(p)) for p in pats], dtype=np.float32)
    finite = np.isfinite(want)
    assert np.array_equal(got[finite], want[finite])
    assert np.all(np.isnan(got[np.isnan(want)]))


def test_stored_value_saturates_and_rounds():
    assert O.stored_value(70000.0) == 65504.0
    assert O.stored_value(-70000.0) == -65504.0
    assert O.stored_value(1.0) == 1.0
    assert O.stored_value(0.1) == float(np.float16(0.1))
    assert O.stored_value(0.1, scale_fp32=True) == float(np.float32(0.1))


# ---------------------------------------------------------------- quantizers

def _groups(rng, n_groups, size, bits):
    for gi in range(n_groups):
        scale = float(10.0 ** rng.uniform(-3, 3))
        x = (rng.standard_normal(size) * scale).astype(np.float32)
        if gi % 5 == 0:
            x[rng.integers(size)] *= 40.0        # an outlier inside the group
        yield x


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("fp32", [False, True])
def test_quant_sym_nearest_level_and_bounds(bits, fp32):
    """The page's quantizer: s = max|x|/Q, q = clip(round(x/s), -Q, Q) -- checked
    by its defining properties, not by re-evaluating it."""
    rng = np.random.default_rng(bits * 10 + fp32)
    Q = 2 ** (bits - 1) - 1
    for x in _groups(rng, 300, 64, bits):
        s, q = O.quant_sym(x, bits, fp32)
        amax = float(np.max(np.abs(x)))
        # the stored scale is max|x|/Q up to the storage rounding: fp16 rounds with
        # relative error 2^-11 in its normal range and absolute error 2^-25 below it
        if fp32:
            assert abs(s * Q - amax) <= amax * 2.0 ** -22
        else:
            assert abs(s - amax / Q) <= max((amax / Q) * 2.0 ** -11, 2.0 ** -25) + amax / Q * 2.0 ** -23
        assert np.all(np.abs(q) <= Q)
        # the largest-magnitude element maps to +-Q
        i = int(np.argmax(np.abs(x)))
        assert abs(int(q[i])) == Q and np.sign(q[i]) == np.sign(x[i])
        r = x.astype(np.float64) / s
        # nearest level: every code is within 1/2 (+ one fp32 rounding of x/s) of x/s,
        # unless clipped at +-Q
        unclipped = np.abs(r) <= Q + 0.5
        assert np.all(np.abs(q[unclipped] - r[unclipped]) <= 0.5 + 2.0 ** -22 * np.abs(r[unclipped]) + 1e-12)
        assert np.all(np.abs(q[~unclipped]) == Q)
        # reconstruction bound |x - s q| <= s/2 for unclipped elements
        err = np.abs(x.astype(np.float64) - s * q)
        assert np.all(err[unclipped] <= s / 2 * (1 + 2.0 ** -21) + 1e-30)


def test_quant_sym_ties_round_half_even():
    # amax = 7 at 4 bits -> s = 7/7 = 1 exactly, so x/s lands on the ties
    x = np.array([7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5], dtype=np.float32)
    s, q = O.quant_sym(x, 4)
    assert s == 1.0
    assert list(q) == [7, 0, 2, 2, 0, -2, -2, 4]


def test_quant_sym_symmetry_and_power_of_two_scaling():
    rng = np.random.default_rng(7)
    for bits in (2, 4, 8):
        for _ in range(100):
            x = rng.standard_normal(32).astype(np.float32)
            s, q = O.quant_sym(x, bits)
            s2, q2 = O.quant_sym(-x, bits)
            assert s2 == s and np.array_equal(q2, -q)
            s4, q4 = O.quant_sym(x * np.float32(4.0), bits)
            assert s4 == 4 * s and np.array_equal(q4, q)


def test_quant_zero_group():
    s, q = O.quant_sym(np.zeros(16, np.float32), 4)
    assert s == 0.0 and not q.any()
    s, z, q = O.quant_asym(np.full(16, 2.5, np.float32), 2)
    assert s == 0.0 and z == 2.5 and not q.any()


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_quant_asym_properties(bits):
    rng = np.random.default_rng(100 + bits)
    Qa = 2 ** bits - 1
    for x in _groups(rng, 300, 32, bits):
        s, z, q = O.quant_asym(x, bits)
        mn, mx = float(x.min()), float(x.max())
        assert np.all((q >= 0) & (q <= Qa))
        assert q[int(np.argmin(x))] == 0
        assert q[int(np.argmax(x))] == Qa
        assert abs(z - mn) <= max(abs(mn) * 2.0 ** -11, 2.0 ** -25)
        d = (mx - mn) / Qa
        assert abs(s - d) <= max(d * 2.0 ** -11, 2.0 ** -25) + d * 2.0 ** -22
        r = (x.astype(np.float64) - z) / s
        inside = (r >= -0.5) & (r <= Qa + 0.5)
        assert np.all(np.abs(q[inside] - r[inside]) <= 0.5 + 2.0 ** -21 * (np.abs(r[inside]) + 1))
        xhat = s * q + z
        assert np.all(np.abs(x - xhat)[inside] <= s / 2 * (1 + 2.0 ** -20) + 1e-30)


def test_quant_asym_exact_levels():
    x = np.array([0.0, 1.0, 2.0, 3.0, 0.5, 1.5, 2.5], dtype=np.float32)
    s, z, q = O.quant_asym(x, 2)
    assert (s, z) == (1.0, 0.0)
    assert list(q) == [0, 1, 2, 3, 0, 2, 2]


# ------------------------------------------------- the page's outlier example

def test_outlier_vector_one_scale_vs_groups():
    g = read_golden("outlier_vector.txt")
    x = np.array(g["values_bf16"], dtype=np.float32)
    # the bf16 listing is the rounding of the printed decimals
    import torch
    assert np.array_equal(
        torch.tensor(g["values"], dtype=torch.float32).to(torch.bfloat16).float().numpy(), x)
    small, large = g["small"], g["large"]
    # one scale for the whole vector at 4 bits: the small values all round to zero
    s, q = O.quant_sym(x, 4)
    assert not q[small].any() and q[large] == 7
    # one scale per group (A = small values, B = large value): they survive
    sA, qA = O.quant_sym(x[small], 4)
    sB, qB = O.quant_sym(x[[large]], 4)
    assert np.all(qA != 0) and qB[0] == 7 and sA < sB
    errA = np.abs(x[small] - sA * qA).max()
    assert errA < np.abs(x[small] - s * q[small]).max() / 10


def test_outlier_vector_hand_derived_codes():
    """Codes derived by hand.  8 bits: 6.40625/127 = 0.0504429...; on the fp16
    grid of [2^-5, 2^-4) (step 2^-15) that is 1652.91 steps -> 1653 * 2^-15 =
    0.050445556640625; x/s = 0.595, -1.384, 2.381, 1.781, 126.99.
    4 bits: 6.40625/7 = 0.91517...; fp16 step 2^-11 in [0.5, 1) -> 1874.29 ->
    1874 * 2^-11 = 0.9150390625; x/s = 0.033, -0.076, 0.131, 0.098, 7.0009."""
    x = np.array(read_golden("outlier_vector.txt")["values_bf16"], dtype=np.float32)
    s, q = O.quant_sym(x, 8)
    assert s == 1653 * 2.0 ** -15 and list(q) == [1, -1, 2, 2, 127]
    s, q = O.quant_sym(x, 4)
    assert s == 1874 * 2.0 ** -11 and list(q) == [0, 0, 0, 0, 7]
    s, q = O.quant_sym(x, 2)       # Q = 1: s = 6.40625 exactly
    assert s == 6.40625 and list(q) == [0, 0, 0, 0, 1]
    # group A alone (4 bits): 0.1201171875/7 = 0.017159...; step 2^-16 -> 1124.57 ->
    # 1125 * 2^-16 = 0.0171661376953125; x/s = 1.749, -4.067, 6.997, 5.234
    s, q = O.quant_sym(x[:4], 4)
    assert s == 1125 * 2.0 ** -16 and list(q) == [2, -4, 7, 5]


# ---------------------------------------------------------- memory formula

def test_memory_formula_worked_examples():
    g = read_golden("memory_formula.txt")
    L, H, D, T = g["worked_layers"], g["worked_h_kv"], g["worked_d_h"], g["worked_tokens"]
    bf16 = O.cache_bytes_formula(L, T, H, D, 16, 0, 0, 0)
    assert bf16 == g["worked_bf16_bytes"] == 2 ** 30
    ideal4 = O.cache_bytes_formula(L, T, H, D, 4, 0, 0, 0)
    assert ideal4 == g["worked_ideal_4bit_mib"] * 2 ** 20
    q4 = O.cache_bytes_formula(L, T, H, D, 4, 64, 64, 2)
    assert q4 / (2 * L * T * H * D) == g["worked_4bit_fp16_per64_bytes_per_elem"]
    assert q4 == g["worked_4bit_fp16_per64_mib"] * 2 ** 20 == 285_212_672
    assert round(bf16 / q4, 2) == g["worked_reduction"]
    assert round(100 * bf16 / 2 ** 30) == g["worked_100_contexts_bf16_gib"]
    assert round(100 * q4 / 2 ** 30, 1) == g["worked_100_contexts_4bit_gib"]


def test_memory_formula_llama7b():
    g = read_golden("memory_formula.txt")
    # hidden 4096 = all heads x head dim (no GQA in that example): H_kv*d_h = 4096
    per_tok = O.cache_bytes_formula(g["llama7b_layers"], 1, 32, 128, 16, 0, 0, 0)
    assert per_tok == g["llama7b_bytes_per_token"]
    seq = O.cache_bytes_formula(g["llama7b_layers"], g["llama7b_seq_tokens"], 32, 128, 16, 0, 0, 0)
    assert seq == g["llama7b_seq_bytes_gb"] * 2 ** 30
    assert seq * g["llama7b_batch"] == g["llama7b_batch_gb"] * 2 ** 30
    # "Practical Impact": INT8 halves it, INT4 quarters it (metadata ignored)
    for bits, key in ((16, "practical_fp16_gb"), (8, "practical_int8_gb"), (4, "practical_int4_gb")):
        b = O.cache_bytes_formula(32, 2048, 32, 128, bits, 0, 0, 0) * 32
        assert b == g[key] * 2 ** 30


def test_storage_ratios():
    g = read_golden("storage_ratios.txt")
    bf16 = O.cache_bytes_formula(1, 1000, 8, 128, 16, 0, 0, 0)
    for bits, key in ((8, "int8"), (4, "int4"), (2, "int2")):
        assert bf16 / O.cache_bytes_formula(1, 1000, 8, 128, bits, 0, 0, 0) == g[key]


# ---------------------------------------------------- the allocator's generator

def test_splitmix64_published_vector():
    # splitmix64 (Steele, Lea, Flood 2014) from state 0: the reference outputs
    assert O.splitmix64(0, 3) == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_free_list_is_fisher_yates_permutation():
    for n, seed in ((1, 0), (2, 0), (3, 5), (1000, 42), (4096, 7)):
        p = O.free_list(n, seed)
        assert sorted(p.tolist()) == list(range(n))
    # n = 2: one swap step, j = x1 mod 2
    x1 = O.splitmix64(0, 1)[0]
    assert O.free_list(2, 0).tolist() == ([1, 0] if x1 % 2 == 0 else [0, 1])
    # n = 3: i = 2 swaps with x1 mod 3, then i = 1 with x2 mod 2
    x1, x2 = O.splitmix64(9, 2)
    p = [0, 1, 2]
    j = x1 % 3
    p[2], p[j] = p[j], p[2]
    j = x2 % 2
    p[1], p[j] = p[j], p[1]
    assert O.free_list(3, 9).tolist() == p


# ------------------------------------------------------------------ FP8 E4M3

def _e4m3_value(c):
    """The E4M3 code table written from its definition: sign, 4-bit exponent
    with bias 7, 3-bit mantissa, subnormals at exponent 0, S.1111.111 NaN."""
    sign = -1.0 if c & 0x80 else 1.0
    E, m = (c >> 3) & 15, c & 7
    if E == 15 and m == 7:
        return float("nan")
    if E == 0:
        return sign * m / 8.0 * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (E - 7)


def test_e4m3_code_table_and_exact_values():
    for c in range(256):
        want = _e4m3_value(c)
        got = O.e4m3_to_f32(c)
        if np.isnan(want):
            assert np.isnan(got)
            continue
        assert got == want, (c, got, want)
        assert O.f32_to_e4m3(want) == c      # every value encodes to its own code (-0 keeps its sign)
    assert _e4m3_value(0x7E) == 448.0 and _e4m3_value(0x08) == 2.0 ** -6 and _e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_round_to_nearest_even_and_saturation():
    vals = sorted({_e4m3_value(c) for c in range(0x7F)})            # non-negative finite values
    codes = {v: O.f32_to_e4m3(v) for v in vals}
    for lo, hi in zip(vals, vals[1:]):
        mid = np.float32((lo + hi) / 2.0)
        assert float(mid) == (lo + hi) / 2.0                          # midpoints are exact in fp32
        even = lo if (codes[lo] & 1) == 0 else hi
        assert O.f32_to_e4m3(float(mid)) == codes[even]
        assert O.f32_to_e4m3(float(np.nextafter(mid, np.float32(0)))) == codes[lo]
        assert O.f32_to_e4m3(float(np.nextafter(mid, np.float32(np.inf)))) == codes[hi]
    for x in (448.0, 449.0, 463.9, 464.0, 1e6, float("inf")):
        assert O.f32_to_e4m3(x) == 0x7E and O.f32_to_e4m3(-x) == 0xFE
    assert O.f32_to_e4m3(float("nan")) & 0x7F == 0x7F


def test_e4m3_matches_torch_float8_in_range():
    """Independent library check inside the finite range (torch's e4m3fn cast
    rounds to nearest even; beyond 448 it does not saturate, so stay inside)."""
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.normal(0, 1, 20000),
                        rng.normal(0, 2.0 ** -8, 20000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([O.f32_to_e4m3(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(got, ref)
