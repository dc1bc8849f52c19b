"""Hand-built bf16 rows whose quantization groups hit every edge of the
quantizer of llmdaily.org day-65, "From BF16 to INT8, INT4, or even fewer
bits" (s = max|x| / Q, q = clip(round(x / s), -Q, Q), and the zero-point
variant), under the readings of its silent points: round half to even, the
stored (rounded) scale divides, an fp16 scale saturates at 65504 and one that
rounds to 0 makes a zero group.

Each group is one of these kinds:
  zero       every element 0: scale 0, codes 0;
  constant   every element equal: codes +-Q (symmetric), or a zero-scale
             group whose zero-point carries the value (asymmetric);
  ties       a power-of-two scale u (max |x| = Q u, or min 0 and max Qa u) and
             elements at (k + 1/2) u, so x / s is an exact half-integer;
  saturate   max|x| / Q above 65504: the fp16 scale saturates and the largest
             element's code clips;
  underflow  max|x| / Q below 2^-25: the fp16 scale rounds to 0;
  subnormal  s = 2.5 * 2^-24 rounds (half to even) to the fp16 subnormal
             2^-23 < s, so the largest element's code clips (2^-23 exactly for
             8-bit codes);
  normal     standard normal values.
For the FP8 format (no groups, one scale per kv head, 1.0 here) the kinds are
e4m3 ties, saturation at +-448, values below half the smallest subnormal, and
small subnormals.  Every value is exactly representable in bf16."""
import numpy as np

from quantized_kv_cache_14_b200.workloads import to_bf16_bits

KINDS = ("zero", "constant", "ties", "saturate", "underflow", "subnormal", "normal")
MILD = tuple(k for k in KINDS if k != "saturate")


def _unit(bits):
    return 2.0 ** -6 if bits == 8 else 2.0 ** -3


def group_values(kind, n, bits, asym, rng):
    """n float32 values of one quantization group of the given kind."""
    x = np.zeros(n, dtype=np.float64)
    Q = (1 << (bits - 1)) - 1
    Qa = (1 << bits) - 1
    u = _unit(bits)
    if kind == "zero":
        pass
    elif kind == "constant":
        x[:] = -1.25
    elif kind == "ties":
        if asym:
            x[0], x[1] = 0.0, Qa * u
            top = min(Qa - 1, 126)
        else:
            x[0] = Q * u
            top = min(Q - 1, 126)
        for i in range(2 if asym else 1, n):
            k = (i * 7) % (top + 1)
            sign = -1.0 if (not asym and i % 2) else 1.0
            x[i] = sign * (k + 0.5) * u
    elif kind == "saturate":
        if asym:
            big = 2.0 ** (24 if bits == 8 else 20)
            x[:] = rng.uniform(-big, big, n)
            x[0], x[1] = -big, big
        else:
            big = 2.0 ** (24 if bits == 8 else 20)
            x[:] = rng.uniform(-big, big, n)
            x[0] = big
    elif kind == "underflow":
        top = (Qa if asym else Q) * 2.0 ** -27
        x[:] = rng.uniform(0.0 if asym else -top, top, n)
        x[0] = top
        if asym:
            x[1] = 0.0
    elif kind == "subnormal":
        if bits == 8:
            top = (Qa if asym else Q) * 2.0 ** -23
        else:
            top = (Qa if asym else Q) * 2.5 * 2.0 ** -24
        x[:] = rng.uniform(0.0 if asym else -top, top, n)
        x[0] = top
        if asym:
            x[1] = 0.0
    elif kind == "normal":
        x[:] = rng.standard_normal(n)
    else:
        raise ValueError(kind)
    x32 = x.astype(np.float32)
    bits16 = to_bf16_bits(x32)
    back = (bits16.astype(np.uint32) << 16).view(np.float32)
    if kind in ("ties", "constant", "zero"):
        assert np.array_equal(back, x32), f"{kind} values are not exact in bf16"
    # the group's extremes must survive bf16 rounding exactly (they fix s)
    assert back[0] == x32[0] and (not asym or back[1] == x32[1]) or kind in ("normal", "zero", "constant")
    return back


def fp8_values(kind, n, rng):
    """n float32 values (exact in bf16) around the e4m3 grid, scale 1."""
    if kind == "ties":   # halfway between e4m3 neighbours: RNE picks the even one
        pool = [1.0625, -1.0625, 1.1875, -1.1875, 9.5, -9.5, 2.0 ** -10, -(2.0 ** -10), 3 * 2.0 ** -10]
    elif kind == "saturate":
        pool = [448.0, 464.0, 500.0, -1000.0, 2.0 ** 20, -(2.0 ** 20)]
    elif kind == "underflow":
        pool = [2.0 ** -11, -(2.0 ** -12), 2.0 ** -20, 0.0]
    elif kind == "subnormal":
        pool = [2.0 ** -9, 3 * 2.0 ** -9, 7 * 2.0 ** -9, -(5 * 2.0 ** -9)]
    elif kind == "zero":
        pool = [0.0]
    elif kind == "constant":
        pool = [-1.25]
    else:
        return to_bf16_f32(rng.standard_normal(n).astype(np.float32))
    x = np.array([pool[i % len(pool)] for i in range(n)], dtype=np.float32)
    assert np.array_equal(to_bf16_f32(x), x)
    return x


def to_bf16_f32(x32):
    return (to_bf16_bits(x32).astype(np.uint32) << 16).view(np.float32)


def edge_rows(fmt, n_tok, h_kv, d_h, kinds, rng, phase=0):
    """(k, v) bf16 bit patterns [n_tok][h_kv][d_h] whose groups cycle through
    `kinds`: value groups (and token-axis key groups) per (token, head, group);
    channel-axis key groups per (token group, head, channel)."""
    bits, asym = fmt["bits"], fmt["asym"]
    fp8 = fmt.get("fp8", 0)
    k = np.zeros((n_tok, h_kv, d_h), dtype=np.float32)
    v = np.zeros((n_tok, h_kv, d_h), dtype=np.float32)
    nk = len(kinds)
    if fp8:
        for t in range(n_tok):
            for h in range(h_kv):
                k[t, h] = fp8_values(kinds[(t + h + phase) % nk], d_h, rng)
                v[t, h] = fp8_values(kinds[(t + 2 * h + 1 + phase) % nk], d_h, rng)
        return to_bf16_bits(k), to_bf16_bits(v)
    gv = fmt["g_v"]
    for t in range(n_tok):
        for h in range(h_kv):
            for j in range(d_h // gv):
                kind = kinds[(t + j + h + phase) % nk]
                v[t, h, j * gv:(j + 1) * gv] = group_values(kind, gv, bits, asym, rng)
    gk = fmt["g_k"]
    if fmt["k_axis"] == 0:
        for t in range(n_tok):
            for h in range(h_kv):
                for j in range(d_h // gk):
                    kind = kinds[(t + 3 * j + h + 1 + phase) % nk]
                    k[t, h, j * gk:(j + 1) * gk] = group_values(kind, gk, bits, asym, rng)
    else:
        for g0 in range(0, n_tok, gk):
            n = min(gk, n_tok - g0)
            for h in range(h_kv):
                for c in range(d_h):
                    kind = kinds[(g0 // gk + c + h + phase) % nk]
                    k[g0:g0 + n, h, c] = group_values(kind, gk, bits, asym, rng)[:n]
    return to_bf16_bits(k), to_bf16_bits(v)
