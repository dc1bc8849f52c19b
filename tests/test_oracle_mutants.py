"""The pins must catch a plausible mistake anywhere in the oracle.  Each case
plants one mistake in a copy of oracle/kvq_oracle.cpp (a dropped term, a wrong
sign, index, bound or rounding rule, a transposed operand), builds the copy on
the CPU, and runs the CPU pin suites against it through KVQ_ORACLE_LIB: at
least one pin must fail.  The unaltered copy, built and run the same way, must
pass them all, so a caught mistake is the pins' doing and not the harness's.
The committed oracle is never modified."""
import concurrent.futures as cf
import os
import subprocess
import sys

import pytest

from oracle import build as obuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "kvq_oracle.cpp")
PIN_SUITES = ["tests/test_oracle_pins.py", "tests/test_oracle_cache.py", "tests/test_quant_edges.py"]

# (name, text in the oracle's source, the planted mistake)
MUTANTS = [
    # the quantizer (day-65 "From BF16 to INT8, INT4, or even fewer bits")
    ("round_half_away_from_zero",
     "float r = std::nearbyint(x[i * stride] / sh);", "float r = std::round(x[i * stride] / sh);"),
    ("scale_divisor_off_by_one", "float s = amax / float(Q);", "float s = amax / float(Q + 1);"),
    ("clip_one_level_too_low",
     "r = std::min(std::max(r, float(-Q)), float(Q));", "r = std::min(std::max(r, float(-Q - 1)), float(Q));"),
    ("zero_point_from_max", "float zh = stored_value(mn, scale_fp32);", "float zh = stored_value(mx, scale_fp32);"),
    ("asym_levels_off_by_one", "const int Qa = (1 << bits) - 1;", "const int Qa = (1 << bits) - 2;"),
    ("asym_zero_point_not_subtracted",
     "float r = std::nearbyint((x[i * stride] - zh) / sh);", "float r = std::nearbyint(x[i * stride] / sh);"),
    ("scale_not_saturated", "if (std::isinf(r)) r = r > 0 ? 65504.0f : -65504.0f;", "(void)0;"),
    # the number formats
    ("fp16_ties_round_up", "if (rem > half || (rem == half && (r & 1))) ++r;", "if (rem >= half) ++r;"),
    ("fp16_subnormal_shift", "uint64_t r = shift_rne(m24, -(e + 1));", "uint64_t r = shift_rne(m24, -e);"),
    ("e4m3_not_saturated", "if (e > 8 || (e == 8 && r > 14)) return uint8_t(sign | 0x7Eu);",
     "if (e > 8) return uint8_t(sign | 0x7Eu);"),
    # the layout (the format contract)
    ("key_list_order_transposed", "return 16 * j + 2 * t + (e & 1) + 8 * (e >> 1);",
     "return 16 * j + 2 * t + 8 * (e & 1) + (e >> 1);"),
    ("word_fields_in_order", "int word_pos(int l, int n) { return (l >> 1) + (n / 2) * (l & 1); }",
     "int word_pos(int l, int n) { return l + 0 * n; }"),
    ("value_registers_transposed", "int reg = 2 * second + upper;", "int reg = 2 * upper + second;"),
    ("codes_not_sign_extended",
     "if (is_signed && (v & (1u << (bits - 1)))) return int32_t(v) - (1 << bits);", "(void)is_signed;"),
    # grouping and the window (day-65 "Why scales and groups matter", "Why some
    # systems keep a full-precision window")
    ("key_groups_along_channels",
     "else quant_sym(&x[chn], R, D, c.bits, c.scale_fp32, &sc, codes.data());",
     "else quant_sym(&x[chn], R, 1, c.bits, c.scale_fp32, &sc, codes.data());"),
    ("window_flushed_one_token_early", "if (slot == R - 1) flush_group(C, s, pos / R);",
     "if (slot == R - 2) flush_group(C, s, pos / R);"),
    ("window_slot_shifted", "int slot = int(pos % R);\n    const uint16_t* kr",
     "int slot = int((pos + 1) % R);\n    const uint16_t* kr"),
    ("fp8_scale_multiplied", "f32_to_e4m3(x[e] / C.fp8_v[size_t(h)])", "f32_to_e4m3(x[e] * C.fp8_v[size_t(h)])"),
    # attention (day-65 "Why the KV cache grows so quickly")
    ("no_1_over_sqrt_d", "sc[size_t(p)] = acc / std::sqrt(double(D));", "sc[size_t(p)] = acc;"),
    ("gqa_heads_interleaved", "int hq = h * G + a;", "int hq = a * c.h_kv + h;"),
    ("softmax_not_normalised", "double w = sc[size_t(p)] / den;", "double w = sc[size_t(p)];"),
    # the allocator and the memory formula
    ("splitmix64_shift", "z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;",
     "z = (z ^ (z >> 28)) * 0x94D049BB133111EBull;"),
    ("fisher_yates_range", "uint64_t j = splitmix64_next(st) % uint64_t(i + 1);",
     "uint64_t j = splitmix64_next(st) % uint64_t(i);"),
    ("freed_blocks_to_front", "if (--C.holders[size_t(b)] == 0) C.freelist.push_back(b);",
     "if (--C.holders[size_t(b)] == 0) C.freelist.push_front(b);"),
    ("formula_without_metadata",
     "double bk = bits / 8.0 + (g_k > 0 ? double(meta_bytes) / g_k : 0.0);", "double bk = bits / 8.0;"),
    # more of the same kinds
    ("zero_scale_not_special_cased",
     "    if (sh == 0.0f) { codes[i] = 0; continue; }\n    float r = std::nearbyint(x[i * stride] / sh);",
     "    float r = std::nearbyint(x[i * stride] / sh);"),
    ("fp16_overflow_threshold", "if (e > 15) return uint16_t(sign | 0x7C00u);",
     "if (e > 16) return uint16_t(sign | 0x7C00u);"),
    ("fp16_subnormal_unit", "float v = float(man) * 5.9604644775390625e-08f;",
     "float v = float(man) * 1.1920928955078125e-07f;"),
    ("e4m3_subnormal_unit", "else if (E == 0) v = float(m) * 0.001953125f;",
     "else if (E == 0) v = float(m) * 0.00390625f;"),
    ("key_code_bit_offset", "size_t(4 * w) + size_t(c.bits * p / 8);", "size_t(4 * w) + size_t(p / 8);"),
    ("zero_point_subtracted_in_dequant", "    vout[e] = sc * q + z;", "    vout[e] = sc * q - z;"),
    ("key_scales_not_striped", "int j = f / L.kslice, off = f % L.kslice;", "int j = 0, off = f % L.kslice;", 2),
    ("window_boundary_off_by_one", "  if (pos >= Lq) {", "  if (pos > Lq) {"),
    ("blocks_taken_from_the_back", "  int32_t b = C.freelist.front();\n  C.freelist.pop_front();",
     "  int32_t b = C.freelist.back();\n  C.freelist.pop_back();"),
    ("fp8_keys_use_value_scale", "f32_to_e4m3(x[e] / C.fp8_k[size_t(h)])", "f32_to_e4m3(x[e] / C.fp8_v[size_t(h)])"),
    ("query_of_the_kv_head", "qv[e] = bf16_to_f32(q[(size_t(i) * HQ + hq) * D + e]);",
     "qv[e] = bf16_to_f32(q[(size_t(i) * HQ + h) * D + e]);"),
    ("last_position_not_attended",
     "for (int64_t p = 0; p < T; ++p) dequant_token(C, s, h, p, &K[size_t(p) * D], &V[size_t(p) * D]);",
     "for (int64_t p = 0; p + 1 < T; ++p) dequant_token(C, s, h, p, &K[size_t(p) * D], &V[size_t(p) * D]);"),
    ("pages_rounded_down", "  if (c.residual == 0) return (len + c.page - 1) / c.page;",
     "  if (c.residual == 0) return len / c.page;"),
    ("new_block_not_zeroed", "  std::memset(&C.pool[size_t(b) * C.L.block_bytes], 0, C.L.block_bytes);", ""),
    ("value_scales_transposed", "    size_t idx = size_t(tok_in_page) * L.nvg + gi;",
     "    size_t idx = gi * size_t(c.page) + size_t(tok_in_page);"),
    ("value_lanes_transposed", "  int lane = 4 * g + t;", "  int lane = 4 * t + g;"),
    ("prefix_shared_by_page_under_a_window", "  const int32_t unit = c.residual ? c.residual : c.page;",
     "  const int32_t unit = c.page;"),
    # admission and the remaining conversions and metadata
    ("sequence_id_bound_off_by_one", "    if (seq_ids[i] < 0 || seq_ids[i] >= c.max_seqs) return 3;",
     "    if (seq_ids[i] < 0 || seq_ids[i] > c.max_seqs) return 3;"),
    ("e4m3_infinity_to_nan", "  if (exp == 0xFF) return man ? uint8_t(sign | 0x7Fu) : uint8_t(sign | 0x7Eu);",
     "  if (exp == 0xFF) return uint8_t(sign | 0x7Fu);"),
    ("e4m3_exponent_bias", "    return uint8_t(sign | (uint32_t(e + 7) << 3) | (uint32_t(r) & 7u));",
     "    return uint8_t(sign | (uint32_t(e + 8) << 3) | (uint32_t(r) & 7u));"),
    ("fp32_scales_rounded_to_fp16", "  if (scale_fp32) return s;", "  if (scale_fp32) return stored_value(s, 0);"),
    ("value_zero_points_over_scales",
     "    if (c.asym) put_meta(ch + L.off_Vm + (size_t(c.page) * L.nvg + idx) * L.es, z, c.scale_fp32);",
     "    if (c.asym) put_meta(ch + L.off_Vm + idx * L.es, z, c.scale_fp32);"),
    ("key_zero_points_over_scales",
     "      if (c.asym) put_meta(km + (size_t(L.kslice) + off) * L.es, z, c.scale_fp32);",
     "      if (c.asym) put_meta(km + size_t(off) * L.es, z, c.scale_fp32);"),
    ("fail_alloc_after_off_by_one",
     "  if (c.fail_alloc_after >= 0 && C.alloc_count + need > c.fail_alloc_after) return 2;",
     "  if (c.fail_alloc_after >= 0 && C.alloc_count + need >= c.fail_alloc_after) return 2;"),
    ("table_width_off_by_one", "    if (nb > c.max_blocks_per_seq) return 2;", "    if (nb >= c.max_blocks_per_seq) return 2;"),
    ("blocks_needed_not_net", "    need += nb - blocks_for_len(c, C.len[size_t(s)]);", "    need += nb;"),
    # the FP8 and BF16 control layouts, the flush's value rows, the window read-back,
    # the threaded decode, the e4m3 decode, token-axis key metadata
    ("fp8_value_bytes_transposed", "size_t(4 * word) + size_t(2 * (reg & 1) + hi), 0};",
     "size_t(4 * word) + size_t((reg & 1) + 2 * hi), 0};"),
    ("bf16_control_keys_in_list_order",
     "    return {size_t(tok / 16) * L.sub_bytes + size_t(tok % 16) * L.row_bytes + size_t(2 * ch), 0};\n  if (c.fp8)",
     "    return {size_t(tok / 16) * L.sub_bytes + size_t(tok % 16) * L.row_bytes + size_t(2 * inv[ch]), 0};\n"
     "  if (c.fp8)"),
    ("flushed_value_rows_shifted",
     "      write_value_row(C, C.table[s][size_t(pos / P)], int(pos % P), h, row.data());",
     "      write_value_row(C, C.table[s][size_t(pos / P)], int((pos + 1) % P), h, row.data());"),
    ("threaded_decode_skips_items",
     "    th.emplace_back([&, w] { for (int64_t it = w; it < items; it += nt) work(it); });",
     "    th.emplace_back([&, w] { for (int64_t it = w; it < items; it += nt + 1) work(it); });"),
    ("e4m3_decode_exponent", "  else v = std::ldexp(float(8 + m), E - 10);", "  else v = std::ldexp(float(8 + m), E - 11);"),
    ("window_keys_and_values_swapped",
     "    for (int e = 0; e < D; ++e) { kout[e] = bf16_to_f32(kr[e]); vout[e] = bf16_to_f32(vr[e]); }",
     "    for (int e = 0; e < D; ++e) { kout[e] = bf16_to_f32(vr[e]); vout[e] = bf16_to_f32(kr[e]); }"),
    ("token_axis_key_scale_index", "      size_t idx = size_t(tok) * L.nkg + size_t(e / c.g_k);",
     "      size_t idx = size_t(tok) + size_t(e / c.g_k);"),
]


def _run_pins(lib):
    env = dict(os.environ, KVQ_ORACLE_LIB=lib)
    return subprocess.run([sys.executable, "-m", "pytest", *PIN_SUITES, "-x", "-q", "-p", "no:cacheprovider",
                           "-m", "not gpu"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    """Builds the unaltered copy and every mutant and runs the pin suites on
    each (several at once); maps name -> (return code, output tail)."""
    with open(SRC) as f:
        src = f.read()
    cases = [("unaltered", src)]
    for name, old, new, *count in MUTANTS:
        n = count[0] if count else 1
        assert src.count(old) == n, f"{name}: the text to alter must occur {n} time(s) in the oracle"
        cases.append((name, src.replace(old, new)))
    root = tmp_path_factory.mktemp("oracle_mutants")

    def one(case):
        name, text = case
        d = root / name
        d.mkdir()
        (d / "kvq_oracle.cpp").write_text(text)
        lib = obuild.compile_to(str(d / "kvq_oracle.cpp"), str(d / "liboracle.so"))
        r = _run_pins(lib)
        return name, (r.returncode, (r.stdout + r.stderr)[-3000:])

    with cf.ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        return dict(ex.map(one, cases))


def test_unaltered_copy_passes_the_pins(outcomes):
    rc, tail = outcomes["unaltered"]
    assert rc == 0, tail


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_pins_catch_a_planted_mistake(outcomes, name):
    rc, tail = outcomes[name]
    # a failing pin (exit 1), or a pin run that the mistake crashes (killed by a signal)
    assert rc == 1 or rc < 0, f"no pin failed (pytest exit {rc}) with the mistake {name} planted:\n{tail}"
