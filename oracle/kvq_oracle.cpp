// kvq_oracle.cpp -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, obviously-correct CPU model of the quantized paged KV cache:
// the symmetric and asymmetric quantizers, group scales, the BF16 residual
// window, the paged block layout with its block table, and fp64 decode
// attention.  It exists to check the CUDA path; only the tests, the smoke
// check and the benchmark's CPU-baseline leg may load it.  It shares no code,
// header, table or constant generator with the CUDA library: every layout rule
// below is written out here from its definition (the format contract), and the
// CUDA side implements the same contract independently.
//
// Sources (the three web pages on KV-cache quantization):
//  * "KV-cache quantization -- making long-context inference fit in memory"
//    (llmdaily.org day-65):
//      - section "Why the KV cache grows so quickly": attention equation
//        softmax(q_t K^T / sqrt(d_h)) V and the memory formula M = 2 L T H_kv d_h b
//      - section "From BF16 to INT8, INT4, or even fewer bits": symmetric
//        quantizer s = max|x| / (2^(b-1) - 1), q = clip(round(x/s), -Q, Q),
//        x_hat = s q; asymmetric zero-points named as a variant
//      - section "Why scales and groups matter": one scale per group, keys and
//        values grouped along different directions
//      - section "Why some systems keep a full-precision window": BF16
//        residual that is quantized and moved into the cache when it fills
//      - section "How this connects to paging and prefix caching": blocks
//        addressed through block tables
//  * "KV Cache Quantization in Practice" (oh-bug.com): keys per channel and
//    values per token (KIVI), asymmetric 2-bit.
//  * "KV Cache Quantization" (chipfoundryservices.com): per-token
//    scale/zero-point quantization.
//
// Readings where the pages are silent:
//  * round() is round-half-to-even; the division is one IEEE fp32 division.
//  * the codes are computed with the STORED scale (fp16-rounded, saturating at
//    65504), so reconstruction uses the same number that divided.
//  * a group whose stored scale is 0 (all zeros, or a scale that rounds to 0)
//    gets all-zero codes.
//  * asymmetric: z = stored(min x), s = (max x - min x) / (2^b - 1),
//    q = clip(round((x - z)/s), 0, 2^b - 1), x_hat = s q + z.
//  * the residual window holds both K and V; it is flushed when it holds R =
//    G_k tokens; one-token-at-a-time appends are the definition of a bulk append.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fno-fast-math -shared -fPIC
// (see oracle/build.py).  No -ffast-math: every float operation is IEEE.

#include <algorithm>
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <deque>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------------------
// IEEE 754 binary16 / bfloat16 helpers, written from the format definitions.
// ---------------------------------------------------------------------------

uint32_t f32_bits(float x) { uint32_t u; std::memcpy(&u, &x, 4); return u; }
float bits_f32(uint32_t u) { float x; std::memcpy(&x, &u, 4); return x; }

// Shift v right by s bits, rounding to nearest, ties to even.
uint64_t shift_rne(uint64_t v, int s) {
  if (s <= 0) return v << (-s);
  if (s >= 64) return 0;
  uint64_t r = v >> s;
  uint64_t rem = v & ((uint64_t(1) << s) - 1);
  uint64_t half = uint64_t(1) << (s - 1);
  if (rem > half || (rem == half && (r & 1))) ++r;
  return r;
}

// fp32 -> binary16, round to nearest even, gradual underflow, overflow -> inf.
uint16_t f32_to_f16(float x) {
  uint32_t u = f32_bits(x);
  uint16_t sign = uint16_t((u >> 16) & 0x8000u);
  int exp = int((u >> 23) & 0xFF);
  uint32_t man = u & 0x7FFFFFu;
  if (exp == 0xFF) return man ? uint16_t(sign | 0x7E00u) : uint16_t(sign | 0x7C00u);
  if (exp == 0) return sign;  // fp32 zero/subnormal (< 2^-126) rounds to zero
  int e = exp - 127;          // value = (2^23 + man) * 2^(e - 23)
  uint64_t m24 = (uint64_t(1) << 23) | man;
  if (e >= -14) {             // binary16 normal range (before rounding)
    uint64_t r = shift_rne(m24, 13);       // 11-bit significand
    if (r == (uint64_t(1) << 11)) { r >>= 1; ++e; }
    if (e > 15) return uint16_t(sign | 0x7C00u);
    return uint16_t(sign | (uint32_t(e + 15) << 10) | (uint32_t(r) & 0x3FFu));
  }
  // subnormal: count of 2^-24 units = m24 * 2^(e - 23 + 24)
  uint64_t r = shift_rne(m24, -(e + 1));
  return uint16_t(sign | uint32_t(r));    // r == 1024 carries into the exponent
}

// fp32 -> FP8 E4M3 (sign, 4 exponent bits with bias 7, 3 mantissa bits; no
// infinities, S.1111.111 is NaN, largest finite 448), round to nearest even,
// saturating: finite values and infinities beyond 448 become +-448, NaN stays
// NaN.  This is the FP8 KV format the oh-bug.com page calls the engineering
// baseline ("FP8 / INT8: Engineering Baseline").
uint8_t f32_to_e4m3(float x) {
  uint32_t u = f32_bits(x);
  uint8_t sign = uint8_t((u >> 24) & 0x80u);
  int exp = int((u >> 23) & 0xFF);
  uint32_t man = u & 0x7FFFFFu;
  if (exp == 0xFF) return man ? uint8_t(sign | 0x7Fu) : uint8_t(sign | 0x7Eu);
  if (exp == 0) return sign;  // fp32 zero/subnormal: far below half of 2^-9
  int e = exp - 127;          // value = m24 * 2^(e - 23)
  uint64_t m24 = (uint64_t(1) << 23) | man;
  if (e >= -6) {              // E4M3 normal range (before rounding)
    uint64_t r = shift_rne(m24, 20);           // 1.mmm as an integer in [8, 16]
    if (r == 16) { r = 8; ++e; }
    if (e > 8 || (e == 8 && r > 14)) return uint8_t(sign | 0x7Eu);   // beyond 448
    return uint8_t(sign | (uint32_t(e + 7) << 3) | (uint32_t(r) & 7u));
  }
  // subnormal: a count of 2^-9 units; a count of 8 is the smallest normal
  uint64_t r = shift_rne(m24, 14 - e);
  return uint8_t(sign | uint32_t(r));
}

float e4m3_to_f32(uint8_t c) {
  const int E = (c >> 3) & 15, m = c & 7;
  float v;
  if (E == 15 && m == 7) v = std::nanf("");
  else if (E == 0) v = float(m) * 0.001953125f;                    // m * 2^-9
  else v = std::ldexp(float(8 + m), E - 10);                       // (1 + m/8) * 2^(E-7)
  return (c & 0x80u) ? -v : v;
}

float f16_to_f32(uint16_t h) {
  uint32_t sign = uint32_t(h & 0x8000u) << 16;
  int exp = (h >> 10) & 0x1F;
  uint32_t man = h & 0x3FFu;
  if (exp == 0x1F) return bits_f32(sign | 0x7F800000u | (man << 13));
  if (exp == 0) {  // zero or subnormal: man * 2^-24, exact in fp32
    float v = float(man) * 5.9604644775390625e-08f;
    return sign ? -v : v;
  }
  return bits_f32(sign | (uint32_t(exp - 15 + 127) << 23) | (man << 13));
}

float bf16_to_f32(uint16_t b) { return bits_f32(uint32_t(b) << 16); }

// ---------------------------------------------------------------------------
// The quantizers (day-65 page, "From BF16 to INT8, INT4, or even fewer bits").
// ---------------------------------------------------------------------------

// The value a scale (or zero-point) takes once stored: fp16 round-to-nearest-
// even saturating at +-65504, or the fp32 value itself.
float stored_value(float s, int scale_fp32) {
  if (scale_fp32) return s;
  float r = f16_to_f32(f32_to_f16(s));
  if (std::isinf(r)) r = r > 0 ? 65504.0f : -65504.0f;
  return r;
}

// Symmetric: s = max|x| / (2^(b-1)-1); q = clip(round(x/s), -Q, Q).
void quant_sym(const float* x, int n, int stride, int bits, int scale_fp32,
               float* scale_out, int32_t* codes) {
  const int Q = (1 << (bits - 1)) - 1;
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) amax = std::max(amax, std::fabs(x[i * stride]));
  float s = amax / float(Q);                 // one IEEE fp32 division
  float sh = stored_value(s, scale_fp32);
  *scale_out = sh;
  for (int i = 0; i < n; ++i) {
    if (sh == 0.0f) { codes[i] = 0; continue; }
    float r = std::nearbyint(x[i * stride] / sh);   // ties to even (FE_TONEAREST)
    r = std::min(std::max(r, float(-Q)), float(Q));
    codes[i] = int32_t(r);
  }
}

// Asymmetric (zero-point) variant: z = min x, s = (max x - min x)/(2^b - 1),
// q = clip(round((x - z)/s), 0, 2^b - 1), x_hat = s q + z.
void quant_asym(const float* x, int n, int stride, int bits, int scale_fp32,
                float* scale_out, float* zero_out, int32_t* codes) {
  const int Qa = (1 << bits) - 1;
  float mn = x[0], mx = x[0];
  for (int i = 1; i < n; ++i) { mn = std::min(mn, x[i * stride]); mx = std::max(mx, x[i * stride]); }
  float zh = stored_value(mn, scale_fp32);
  float s = (mx - mn) / float(Qa);
  float sh = stored_value(s, scale_fp32);
  *scale_out = sh;
  *zero_out = zh;
  for (int i = 0; i < n; ++i) {
    if (sh == 0.0f) { codes[i] = 0; continue; }
    float r = std::nearbyint((x[i * stride] - zh) / sh);
    r = std::min(std::max(r, 0.0f), float(Qa));
    codes[i] = int32_t(r);
  }
}

// ---------------------------------------------------------------------------
// The cache model.
// ---------------------------------------------------------------------------

struct Cfg {
  int32_t bits, asym, k_axis, g_k, g_v, scale_fp32, residual, page;
  int32_t h_q, h_kv, d_h, max_seqs, num_blocks, max_blocks_per_seq;
  uint64_t seed;
  int32_t fail_alloc_after;
  int32_t fp8;   // 1: FP8 E4M3 elements with one scale per kv head (bits 8, no metadata)
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Layout {
  int n;            // codes per 32-bit word
  size_t row_bytes, sub_bytes, es, nvg, nkg, secK, secV, secVm, secKm;
  size_t off_V, off_Vm, off_Km, chunk_bytes, block_bytes;
  int kslice;       // channel-axis keys: scale entries per block (D / (g_k / P))
};

Layout make_layout(const Cfg& c) {
  Layout L{};
  const size_t D = size_t(c.d_h), P = size_t(c.page), A = size_t(1 + c.asym);
  L.n = 32 / c.bits;
  L.row_bytes = D * c.bits / 8;
  L.sub_bytes = 16 * L.row_bytes;
  L.es = c.scale_fp32 ? 4 : 2;
  L.nvg = D / size_t(c.g_v);
  L.secK = (P / 16) * L.sub_bytes;
  L.secV = L.secK;
  L.secVm = align_up(P * L.nvg * L.es * A, 16);
  if (c.fp8) {
    // FP8 E4M3 (oh-bug.com, "FP8 / INT8: Engineering Baseline"): one scale per
    // kv head for keys and for values, no per-group metadata
    L.nkg = 1;
    L.secVm = 0;
    L.secKm = 0;
    L.kslice = 0;
  } else if (c.bits == 16) {
    // The pages' unquantized BF16 cache ("From BF16 to INT8, INT4, or even
    // fewer bits"), kept as a control: rows only, no scales.
    L.nkg = 1;
    L.secVm = 0;
    L.secKm = 0;
    L.kslice = 0;
  } else if (c.k_axis == 0) {
    L.nkg = D / size_t(c.g_k);
    L.secKm = align_up(P * L.nkg * L.es * A, 16);
    L.kslice = 0;
  } else {
    L.nkg = 0;
    L.kslice = int(D / (size_t(c.g_k) / P));
    L.secKm = align_up(size_t(L.kslice) * L.es * A, 16);
  }
  L.off_V = L.secK;
  L.off_Vm = L.off_V + L.secV;
  L.off_Km = L.off_Vm + L.secVm;
  L.chunk_bytes = align_up(L.off_Km + L.secKm, 32);
  L.block_bytes = size_t(c.h_kv) * L.chunk_bytes;
  return L;
}

// Key rows store channels in the order of the list
//   L[32 t + 4 j + e] = 16 j + 2 t + (e & 1) + 8 (e >> 1),
// t in [0,4), j in [0,8), e in [0,4)  (D = 128).
int key_list_channel(int f) {
  int t = f / 32, j = (f % 32) / 4, e = f % 4;
  return 16 * j + 2 * t + (e & 1) + 8 * (e >> 1);
}

// Element l of an n-element word sits at field (l >> 1) + (n/2)(l & 1).
int word_pos(int l, int n) { return (l >> 1) + (n / 2) * (l & 1); }

struct Loc { size_t byte; int shift; };

// Byte/bit of key code (token-in-page, channel) inside the K section of a chunk.
Loc k_loc(const Cfg& c, const Layout& L, const std::vector<int>& inv, int tok, int ch) {
  if (c.bits == 16)   // BF16 control: natural rows, channel ch at bytes 2ch, 2ch+1
    return {size_t(tok / 16) * L.sub_bytes + size_t(tok % 16) * L.row_bytes + size_t(2 * ch), 0};
  if (c.fp8)          // FP8: key-list order, one byte per element in natural order
    return {size_t(tok / 16) * L.sub_bytes + size_t(tok % 16) * L.row_bytes + size_t(inv[ch]), 0};
  int f = inv[ch];
  int w = f / L.n, l = f % L.n, p = word_pos(l, L.n);
  size_t byte = size_t(tok / 16) * L.sub_bytes + size_t(tok % 16) * L.row_bytes +
                size_t(4 * w) + size_t(c.bits * p / 8);
  return {byte, (c.bits * p) % 8};
}

// Byte/bit of value code (token-in-page, channel) inside the V section.
// Within a 16-token sub-tile, lane record (4 g + t) holds, for channel tile i
// (channels 16 i .. 16 i + 15), the four operand registers
//   a0 = (ch 16i+g,   tok 2t | 2t+1)   a1 = (ch 16i+g+8, tok 2t | 2t+1)
//   a2 = (ch 16i+g,   tok 2t+8 | 2t+9) a3 = (ch 16i+g+8, tok 2t+8 | 2t+9)
// (first token of each pair = low element).  Registers are packed into words:
//   8-bit: word 2i = [a0, a1], word 2i+1 = [a2, a3]
//   4-bit: word i  = [a0, a1, a2, a3]
//   2-bit: word i' = [a0(2i'), a1(2i'), a0(2i'+1), a1(2i'+1),
//                     a2(2i'), a3(2i'), a2(2i'+1), a3(2i'+1)]
// and register x of a word has its low element at field x, its high at x + n/2.
Loc v_loc(const Cfg& c, const Layout& L, int tok, int ch) {
  if (c.bits == 16)   // BF16 control: natural rows, like the keys
    return {size_t(tok / 16) * L.sub_bytes + size_t(tok % 16) * L.row_bytes + size_t(2 * ch), 0};
  int sub = tok / 16, tau = tok % 16;
  int i = ch / 16, rr = ch % 16, g = rr % 8, upper = rr / 8;
  int tt = tau % 8, t = tt / 2, hi = tt % 2, second = tau / 8;
  int reg = 2 * second + upper;
  int lane = 4 * g + t;
  int word, x;
  if (c.fp8) {   // FP8: word 2i = [a0 lo, a0 hi, a1 lo, a1 hi], word 2i+1 = a2, a3 likewise
    word = 2 * i + (reg >> 1);
    return {size_t(sub) * L.sub_bytes + size_t(lane) * 64u + size_t(4 * word) + size_t(2 * (reg & 1) + hi), 0};
  }
  if (c.bits == 8) { word = 2 * i + (reg >> 1); x = reg & 1; }
  else if (c.bits == 4) { word = i; x = reg; }
  else { word = i / 2; x = 4 * (reg >> 1) + 2 * (i & 1) + (reg & 1); }
  int p = hi ? x + L.n / 2 : x;
  size_t byte = size_t(sub) * L.sub_bytes + size_t(lane) * size_t(8 * c.bits) +
                size_t(4 * word) + size_t(c.bits * p / 8);
  return {byte, (c.bits * p) % 8};
}

void put_code(uint8_t* base, Loc loc, int bits, int32_t code) {
  if (bits == 16) {   // a whole little-endian 16-bit field
    base[loc.byte] = uint8_t(uint32_t(code) & 0xFFu);
    base[loc.byte + 1] = uint8_t((uint32_t(code) >> 8) & 0xFFu);
    return;
  }
  uint8_t mask = uint8_t((1u << bits) - 1u);
  uint8_t v = uint8_t(uint32_t(code) & mask);
  base[loc.byte] = uint8_t((base[loc.byte] & ~(mask << loc.shift)) | (v << loc.shift));
}

int32_t get_code(const uint8_t* base, Loc loc, int bits, bool is_signed) {
  if (bits == 16) return int32_t(uint32_t(base[loc.byte]) | (uint32_t(base[loc.byte + 1]) << 8));
  uint32_t mask = (1u << bits) - 1u;
  uint32_t v = (uint32_t(base[loc.byte]) >> loc.shift) & mask;
  if (is_signed && (v & (1u << (bits - 1)))) return int32_t(v) - (1 << bits);
  return int32_t(v);
}

void put_meta(uint8_t* p, float v, int scale_fp32) {
  if (scale_fp32) { std::memcpy(p, &v, 4); }
  else { uint16_t h = f32_to_f16(v); std::memcpy(p, &h, 2); }
}

float get_meta(const uint8_t* p, int scale_fp32) {
  if (scale_fp32) { float v; std::memcpy(&v, p, 4); return v; }
  uint16_t h; std::memcpy(&h, p, 2); return f16_to_f32(h);
}

// splitmix64, as published by Steele, Lea and Flood (2014).
uint64_t splitmix64_next(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ull;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

struct Cache {
  Cfg c;
  Layout L;
  std::vector<int> inv;            // channel -> position in the key list
  std::vector<uint8_t> pool;
  std::vector<uint16_t> kres, vres;  // [max_seqs][h_kv][R][D] bf16 bits
  std::vector<int32_t> len;
  std::vector<std::vector<int32_t>> table;
  std::deque<int32_t> freelist;
  int64_t alloc_count = 0;
  std::vector<int32_t> holders;    // per block: table rows holding it (shared prefixes)
  std::vector<float> fp8_k, fp8_v;  // FP8: per kv head scales (1.0 until set)
};

int64_t blocks_for_len(const Cfg& c, int64_t len) {
  if (c.residual == 0) return (len + c.page - 1) / c.page;
  return (len / c.residual) * (c.residual / c.page);
}

int32_t alloc_block(Cache& C) {
  int32_t b = C.freelist.front();
  C.freelist.pop_front();
  ++C.alloc_count;
  C.holders[size_t(b)] = 1;
  std::memset(&C.pool[size_t(b) * C.L.block_bytes], 0, C.L.block_bytes);
  return b;
}

uint8_t* chunk_ptr(Cache& C, int32_t block, int h) {
  return &C.pool[size_t(block) * C.L.block_bytes + size_t(h) * C.L.chunk_bytes];
}

// Quantize one value row (token, head) per token with groups of g_v channels.
void write_value_row(Cache& C, int32_t block, int tok_in_page, int h, const float* x) {
  const Cfg& c = C.c;
  const Layout& L = C.L;
  uint8_t* ch = chunk_ptr(C, block, h);
  if (c.bits == 16) {   // BF16 control: the row itself (x holds bf16 values exactly)
    for (int e = 0; e < c.d_h; ++e)
      put_code(ch + L.off_V, v_loc(c, L, tok_in_page, e), 16, int32_t(f32_bits(x[e]) >> 16));
    return;
  }
  if (c.fp8) {          // FP8: e4m3(x / s_head), an IEEE fp32 division then RNE + saturation
    for (int e = 0; e < c.d_h; ++e)
      put_code(ch + L.off_V, v_loc(c, L, tok_in_page, e), 8, f32_to_e4m3(x[e] / C.fp8_v[size_t(h)]));
    return;
  }
  int32_t codes[128];
  for (size_t gi = 0; gi < L.nvg; ++gi) {
    float s = 0, z = 0;
    const float* xg = x + gi * size_t(c.g_v);
    if (c.asym) quant_asym(xg, c.g_v, 1, c.bits, c.scale_fp32, &s, &z, codes);
    else quant_sym(xg, c.g_v, 1, c.bits, c.scale_fp32, &s, codes);
    for (int e = 0; e < c.g_v; ++e)
      put_code(ch + L.off_V, v_loc(c, L, tok_in_page, int(gi) * c.g_v + e), c.bits, codes[e]);
    size_t idx = size_t(tok_in_page) * L.nvg + gi;
    put_meta(ch + L.off_Vm + idx * L.es, s, c.scale_fp32);
    if (c.asym) put_meta(ch + L.off_Vm + (size_t(c.page) * L.nvg + idx) * L.es, z, c.scale_fp32);
  }
}

// Keys quantized per token with groups of g_k channels (token axis).
void write_key_row_token_axis(Cache& C, int32_t block, int tok_in_page, int h, const float* x) {
  const Cfg& c = C.c;
  const Layout& L = C.L;
  uint8_t* ch = chunk_ptr(C, block, h);
  if (c.bits == 16) {   // BF16 control: the row itself
    for (int e = 0; e < c.d_h; ++e)
      put_code(ch, k_loc(c, L, C.inv, tok_in_page, e), 16, int32_t(f32_bits(x[e]) >> 16));
    return;
  }
  if (c.fp8) {
    for (int e = 0; e < c.d_h; ++e)
      put_code(ch, k_loc(c, L, C.inv, tok_in_page, e), 8, f32_to_e4m3(x[e] / C.fp8_k[size_t(h)]));
    return;
  }
  int32_t codes[128];
  for (size_t gi = 0; gi < L.nkg; ++gi) {
    float s = 0, z = 0;
    const float* xg = x + gi * size_t(c.g_k);
    if (c.asym) quant_asym(xg, c.g_k, 1, c.bits, c.scale_fp32, &s, &z, codes);
    else quant_sym(xg, c.g_k, 1, c.bits, c.scale_fp32, &s, codes);
    for (int e = 0; e < c.g_k; ++e)
      put_code(ch, k_loc(c, L, C.inv, tok_in_page, int(gi) * c.g_k + e), c.bits, codes[e]);
    size_t idx = size_t(tok_in_page) * L.nkg + gi;
    put_meta(ch + L.off_Km + idx * L.es, s, c.scale_fp32);
    if (c.asym) put_meta(ch + L.off_Km + (size_t(c.page) * L.nkg + idx) * L.es, z, c.scale_fp32);
  }
}

// The residual of sequence s holds a complete key group: quantize keys per
// channel over the G_k tokens and values per token, move them into the pages,
// allocating the group's G_k / P blocks.
void flush_group(Cache& C, int s, int64_t group) {
  const Cfg& c = C.c;
  const Layout& L = C.L;
  const int R = c.residual, D = c.d_h, P = c.page;
  const int npg = R / P;
  for (int j = 0; j < npg; ++j) C.table[s].push_back(alloc_block(C));
  std::vector<float> x(size_t(R) * D);
  std::vector<int32_t> codes(R);
  for (int h = 0; h < c.h_kv; ++h) {
    const uint16_t* kr = &C.kres[(size_t(s) * c.h_kv + h) * R * D];
    const uint16_t* vr = &C.vres[(size_t(s) * c.h_kv + h) * R * D];
    for (size_t i = 0; i < size_t(R) * D; ++i) x[i] = bf16_to_f32(kr[i]);
    for (int chn = 0; chn < D; ++chn) {
      float sc = 0, z = 0;
      if (c.asym) quant_asym(&x[chn], R, D, c.bits, c.scale_fp32, &sc, &z, codes.data());
      else quant_sym(&x[chn], R, D, c.bits, c.scale_fp32, &sc, codes.data());
      for (int t = 0; t < R; ++t) {
        int64_t pos = group * R + t;
        int32_t blk = C.table[s][size_t(pos / P)];
        put_code(chunk_ptr(C, blk, h), k_loc(c, L, C.inv, int(pos % P), chn), c.bits, codes[t]);
      }
      // scales in key-list order, striped: block j of the group holds list
      // positions [j * D/npg, (j+1) * D/npg)
      int f = C.inv[chn];
      int j = f / L.kslice, off = f % L.kslice;
      int32_t blk = C.table[s][size_t(group * npg + j)];
      uint8_t* km = chunk_ptr(C, blk, h) + L.off_Km;
      put_meta(km + size_t(off) * L.es, sc, c.scale_fp32);
      if (c.asym) put_meta(km + (size_t(L.kslice) + off) * L.es, z, c.scale_fp32);
    }
    std::vector<float> row(static_cast<size_t>(D));
    for (int t = 0; t < R; ++t) {
      for (int e = 0; e < D; ++e) row[e] = bf16_to_f32(vr[size_t(t) * D + e]);
      int64_t pos = group * R + t;
      write_value_row(C, C.table[s][size_t(pos / P)], int(pos % P), h, row.data());
    }
  }
}

// Dequantized key and value rows of (seq, head, position); fp64.
void dequant_token(const Cache& C, int s, int h, int64_t pos, double* kout, double* vout) {
  const Cfg& c = C.c;
  const Layout& L = C.L;
  const int D = c.d_h, P = c.page, R = c.residual;
  int64_t stored = C.len[s];
  int64_t Lq = R ? (stored / R) * R : stored;
  if (pos >= Lq) {
    int slot = int(pos % R);
    const uint16_t* kr = &C.kres[((size_t(s) * c.h_kv + h) * R + slot) * D];
    const uint16_t* vr = &C.vres[((size_t(s) * c.h_kv + h) * R + slot) * D];
    for (int e = 0; e < D; ++e) { kout[e] = bf16_to_f32(kr[e]); vout[e] = bf16_to_f32(vr[e]); }
    return;
  }
  int32_t blk = C.table[s][size_t(pos / P)];
  int tok = int(pos % P);
  const uint8_t* ch = &C.pool[size_t(blk) * L.block_bytes + size_t(h) * L.chunk_bytes];
  if (c.fp8) {          // FP8: s_head * e4m3 value
    for (int e = 0; e < D; ++e) {
      kout[e] = double(C.fp8_k[size_t(h)]) *
                e4m3_to_f32(uint8_t(get_code(ch, k_loc(c, L, C.inv, tok, e), 8, false)));
      vout[e] = double(C.fp8_v[size_t(h)]) *
                e4m3_to_f32(uint8_t(get_code(ch + L.off_V, v_loc(c, L, tok, e), 8, false)));
    }
    return;
  }
  if (c.bits == 16) {   // BF16 control: the stored rows are the values
    for (int e = 0; e < D; ++e) {
      kout[e] = bf16_to_f32(uint16_t(get_code(ch, k_loc(c, L, C.inv, tok, e), 16, false)));
      vout[e] = bf16_to_f32(uint16_t(get_code(ch + L.off_V, v_loc(c, L, tok, e), 16, false)));
    }
    return;
  }
  bool sgn = !c.asym;
  for (int e = 0; e < D; ++e) {
    int32_t q = get_code(ch + L.off_V, v_loc(c, L, tok, e), c.bits, sgn);
    size_t idx = size_t(tok) * L.nvg + size_t(e / c.g_v);
    double sc = get_meta(ch + L.off_Vm + idx * L.es, c.scale_fp32);
    double z = c.asym ? get_meta(ch + L.off_Vm + (size_t(P) * L.nvg + idx) * L.es, c.scale_fp32) : 0.0;
    vout[e] = sc * q + z;
  }
  for (int e = 0; e < D; ++e) {
    int32_t q = get_code(ch, k_loc(c, L, C.inv, tok, e), c.bits, sgn);
    double sc, z = 0.0;
    if (c.k_axis == 0) {
      size_t idx = size_t(tok) * L.nkg + size_t(e / c.g_k);
      sc = get_meta(ch + L.off_Km + idx * L.es, c.scale_fp32);
      if (c.asym) z = get_meta(ch + L.off_Km + (size_t(P) * L.nkg + idx) * L.es, c.scale_fp32);
    } else {
      int npg = c.g_k / P;
      int64_t group = pos / c.g_k;
      int f = C.inv[e];
      int j = f / L.kslice, off = f % L.kslice;
      int32_t mblk = C.table[s][size_t(group * npg + j)];
      const uint8_t* km = &C.pool[size_t(mblk) * L.block_bytes + size_t(h) * L.chunk_bytes + L.off_Km];
      sc = get_meta(km + size_t(off) * L.es, c.scale_fp32);
      if (c.asym) z = get_meta(km + (size_t(L.kslice) + off) * L.es, c.scale_fp32);
    }
    kout[e] = sc * q + z;
  }
}

}  // namespace

extern "C" {

// ---- scalar helpers (exported for the pin tests) ---------------------------
uint16_t orc_f32_to_f16(float x) { return f32_to_f16(x); }
uint8_t orc_f32_to_e4m3(float x) { return f32_to_e4m3(x); }

// FP8 format: per kv head scales for keys and values (h_kv each).  Returns 0,
// or 4 when the cache is not FP8, holds tokens already, or a scale is not a
// positive finite number.
int32_t orc_set_fp8_scales(void* hh, const float* k, const float* v);
float orc_e4m3_to_f32(uint8_t c) { return e4m3_to_f32(c); }
float orc_f16_to_f32(uint16_t h) { return f16_to_f32(h); }
float orc_bf16_to_f32(uint16_t b) { return bf16_to_f32(b); }
float orc_stored_value(float s, int32_t scale_fp32) { return stored_value(s, scale_fp32); }

void orc_quant_sym(const float* x, int32_t n, int32_t bits, int32_t scale_fp32,
                   float* scale_out, int32_t* codes) {
  std::fesetround(FE_TONEAREST);
  quant_sym(x, n, 1, bits, scale_fp32, scale_out, codes);
}

void orc_quant_asym(const float* x, int32_t n, int32_t bits, int32_t scale_fp32,
                    float* scale_out, float* zero_out, int32_t* codes) {
  std::fesetround(FE_TONEAREST);
  quant_asym(x, n, 1, bits, scale_fp32, scale_out, zero_out, codes);
}

// Memory formula of the day-65 page: M = 2 L T H_kv d_h b, with b the bytes per
// element including group metadata (bits/8 + meta bytes / group size, for K and
// V separately).  Returned in bytes as a double (exact for the worked sizes).
double orc_cache_bytes_formula(int64_t layers, int64_t tokens, int64_t h_kv, int64_t d_h,
                               int32_t bits, int32_t g_k, int32_t g_v, int32_t meta_bytes) {
  double elems = double(layers) * double(tokens) * double(h_kv) * double(d_h);
  double bk = bits / 8.0 + (g_k > 0 ? double(meta_bytes) / g_k : 0.0);
  double bv = bits / 8.0 + (g_v > 0 ? double(meta_bytes) / g_v : 0.0);
  return elems * (bk + bv);
}

// The first n outputs of splitmix64 started from `seed` (for the pin tests).
void orc_splitmix64(uint64_t seed, int32_t n, uint64_t* out) {
  uint64_t st = seed;
  for (int32_t i = 0; i < n; ++i) out[i] = splitmix64_next(st);
}

// Fisher-Yates permutation of [0, n) driven by splitmix64(seed): for i from n-1
// down to 1, swap element i with element (next() mod (i+1)).
void orc_free_list(int32_t n, uint64_t seed, int32_t* out) {
  uint64_t st = seed;
  for (int32_t i = 0; i < n; ++i) out[i] = i;
  for (int32_t i = n - 1; i >= 1; --i) {
    uint64_t j = splitmix64_next(st) % uint64_t(i + 1);
    std::swap(out[i], out[size_t(j)]);
  }
}

void* orc_create(const Cfg* cfg) {
  std::fesetround(FE_TONEAREST);
  Cache* C = new Cache();
  C->c = *cfg;
  C->L = make_layout(C->c);
  C->inv.assign(size_t(C->c.d_h), 0);
  for (int f = 0; f < C->c.d_h; ++f) C->inv[size_t(key_list_channel(f))] = f;
  C->pool.assign(size_t(C->c.num_blocks) * C->L.block_bytes, 0);
  size_t rs = size_t(C->c.max_seqs) * C->c.h_kv * size_t(C->c.residual) * C->c.d_h;
  C->kres.assign(rs, 0);
  C->vres.assign(rs, 0);
  C->len.assign(size_t(C->c.max_seqs), 0);
  C->table.assign(size_t(C->c.max_seqs), {});
  std::vector<int32_t> perm(size_t(C->c.num_blocks));
  orc_free_list(C->c.num_blocks, C->c.seed, perm.data());
  C->freelist.assign(perm.begin(), perm.end());
  C->holders.assign(size_t(C->c.num_blocks), 0);
  C->fp8_k.assign(size_t(C->c.h_kv), 1.0f);
  C->fp8_v.assign(size_t(C->c.h_kv), 1.0f);
  return C;
}

void orc_destroy(void* h) { delete static_cast<Cache*>(h); }

// Layout numbers: out[0..] = n, row_bytes, sub_bytes, secK, secV, secVm,
// secKm, off_V, off_Vm, off_Km, chunk_bytes, block_bytes, kslice.
void orc_layout(void* h, int64_t* out) {
  const Layout& L = static_cast<Cache*>(h)->L;
  int64_t v[13] = {L.n, int64_t(L.row_bytes), int64_t(L.sub_bytes), int64_t(L.secK),
                   int64_t(L.secV), int64_t(L.secVm), int64_t(L.secKm), int64_t(L.off_V),
                   int64_t(L.off_Vm), int64_t(L.off_Km), int64_t(L.chunk_bytes),
                   int64_t(L.block_bytes), int64_t(L.kslice)};
  std::memcpy(out, v, sizeof(v));
}

// Append n tokens (k, v: bf16 bits [n][h_kv][d_h]) one at a time in array
// order.  Returns 0, or 2 (out of blocks / table width) with no state change,
// or 3 (bad sequence id) with no state change.
int32_t orc_append(void* hh, const uint16_t* k, const uint16_t* v, const int32_t* seq_ids, int32_t n) {
  Cache& C = *static_cast<Cache*>(hh);
  const Cfg& c = C.c;
  const int D = c.d_h, H = c.h_kv, R = c.residual, P = c.page;
  // admission: every id valid, enough free blocks, table width respected
  std::vector<int64_t> newlen(C.len.begin(), C.len.end());
  for (int32_t i = 0; i < n; ++i) {
    if (seq_ids[i] < 0 || seq_ids[i] >= c.max_seqs) return 3;
    ++newlen[size_t(seq_ids[i])];
  }
  int64_t need = 0;
  for (int s = 0; s < c.max_seqs; ++s) {
    int64_t nb = blocks_for_len(c, newlen[size_t(s)]);
    if (nb > c.max_blocks_per_seq) return 2;
    need += nb - blocks_for_len(c, C.len[size_t(s)]);
  }
  if (need > int64_t(C.freelist.size())) return 2;
  if (c.fail_alloc_after >= 0 && C.alloc_count + need > c.fail_alloc_after) return 2;

  std::vector<float> row(static_cast<size_t>(D));
  for (int32_t i = 0; i < n; ++i) {
    int s = seq_ids[i];
    int64_t pos = C.len[size_t(s)];
    if (R == 0) {
      if (pos / P == int64_t(C.table[size_t(s)].size())) C.table[size_t(s)].push_back(alloc_block(C));
      int32_t blk = C.table[size_t(s)][size_t(pos / P)];
      for (int h = 0; h < H; ++h) {
        const uint16_t* kr = k + (size_t(i) * H + h) * D;
        const uint16_t* vr = v + (size_t(i) * H + h) * D;
        for (int e = 0; e < D; ++e) row[size_t(e)] = bf16_to_f32(kr[e]);
        write_key_row_token_axis(C, blk, int(pos % P), h, row.data());
        for (int e = 0; e < D; ++e) row[size_t(e)] = bf16_to_f32(vr[e]);
        write_value_row(C, blk, int(pos % P), h, row.data());
      }
      C.len[size_t(s)] = int32_t(pos + 1);
    } else {
      int slot = int(pos % R);
      for (int h = 0; h < H; ++h) {
        std::memcpy(&C.kres[((size_t(s) * H + h) * R + slot) * D], k + (size_t(i) * H + h) * D, size_t(D) * 2);
        std::memcpy(&C.vres[((size_t(s) * H + h) * R + slot) * D], v + (size_t(i) * H + h) * D, size_t(D) * 2);
      }
      C.len[size_t(s)] = int32_t(pos + 1);
      if (slot == R - 1) flush_group(C, s, pos / R);
    }
  }
  return 0;
}

// Layout probes for the tiling tests: (byte, bit) of a key / value code of
// (token-in-page, channel) inside its section of a chunk.
void orc_k_loc(void* hh, int32_t tok, int32_t ch, int64_t* byte, int32_t* shift) {
  Cache& C = *static_cast<Cache*>(hh);
  Loc l = k_loc(C.c, C.L, C.inv, tok, ch);
  *byte = int64_t(l.byte); *shift = l.shift;
}
void orc_v_loc(void* hh, int32_t tok, int32_t ch, int64_t* byte, int32_t* shift) {
  Cache& C = *static_cast<Cache*>(hh);
  Loc l = v_loc(C.c, C.L, tok, ch);
  *byte = int64_t(l.byte); *shift = l.shift;
}

// Returns a sequence's blocks to the back of the free list (in logical order)
// and resets its length.
int32_t orc_free_seq(void* hh, int32_t s) {
  Cache& C = *static_cast<Cache*>(hh);
  if (s < 0 || s >= C.c.max_seqs) return 3;
  // a block is free again when its last holder lets go; freed in logical order
  for (int32_t b : C.table[size_t(s)])
    if (--C.holders[size_t(b)] == 0) C.freelist.push_back(b);
  C.table[size_t(s)].clear();
  C.len[size_t(s)] = 0;
  return 0;
}

// FP8 scales (oh-bug.com, "FP8 / INT8: Engineering Baseline"): one per kv
// head for keys and one for values, set before the first append.  Returns 0;
// 4 for a cache not in the FP8 format, a non-empty cache or a scale that is
// not positive and finite.
int32_t orc_set_fp8_scales(void* hh, const float* k, const float* v) {
  Cache& C = *static_cast<Cache*>(hh);
  if (!C.c.fp8) return 4;
  for (int32_t L : C.len)
    if (L) return 4;
  for (int h = 0; h < C.c.h_kv; ++h)
    if (!(k[h] > 0.0f) || !(v[h] > 0.0f) || !std::isfinite(k[h]) || !std::isfinite(v[h])) return 4;
  C.fp8_k.assign(k, k + C.c.h_kv);
  C.fp8_v.assign(v, v + C.c.h_kv);
  return 0;
}

// Prefix sharing (day-65 page, "How this connects to paging and prefix
// caching"): the empty sequence dst starts with the first `tokens` tokens of
// src by holding src's blocks too.  Only whole blocks that no append writes
// again are shared: tokens a multiple of the page (no window) or of the window
// length R = g_k (whole key groups).  Returns 0; 3 for bad ids; 4 for dst not
// empty, dst == src, tokens out of [0, len(src)] or not aligned; 2 when dst's
// table row is too short.  No state change on error.
int32_t orc_share_prefix(void* hh, int32_t src, int32_t dst, int32_t tokens) {
  Cache& C = *static_cast<Cache*>(hh);
  const Cfg& c = C.c;
  if (src < 0 || src >= c.max_seqs || dst < 0 || dst >= c.max_seqs) return 3;
  if (src == dst || C.len[size_t(dst)] != 0) return 4;
  if (tokens < 0 || tokens > C.len[size_t(src)]) return 4;
  const int32_t unit = c.residual ? c.residual : c.page;
  if (tokens % unit != 0) return 4;
  const int64_t nb = blocks_for_len(c, tokens);
  if (nb > c.max_blocks_per_seq) return 2;
  for (int64_t j = 0; j < nb; ++j) {
    const int32_t b = C.table[size_t(src)][size_t(j)];
    C.table[size_t(dst)].push_back(b);
    ++C.holders[size_t(b)];
  }
  C.len[size_t(dst)] = tokens;
  return 0;
}

int32_t orc_seq_len(void* hh, int32_t s) { return static_cast<Cache*>(hh)->len[size_t(s)]; }
int64_t orc_pool_bytes(void* hh) { return int64_t(static_cast<Cache*>(hh)->pool.size()); }
int64_t orc_free_count(void* hh) { return int64_t(static_cast<Cache*>(hh)->freelist.size()); }

int32_t orc_block_table(void* hh, int32_t s, int32_t* out, int32_t max_entries) {
  const auto& t = static_cast<Cache*>(hh)->table[size_t(s)];
  int32_t n = int32_t(std::min<size_t>(t.size(), size_t(max_entries)));
  for (int32_t i = 0; i < n; ++i) out[i] = t[size_t(i)];
  return int32_t(t.size());
}

void orc_read_pool(void* hh, uint8_t* dst) {
  const auto& p = static_cast<Cache*>(hh)->pool;
  std::memcpy(dst, p.data(), p.size());
}

// Residual rows of (seq, head) as bf16 bits [R][D] (k then v).
void orc_read_residual(void* hh, int32_t s, int32_t h, uint16_t* kdst, uint16_t* vdst) {
  Cache& C = *static_cast<Cache*>(hh);
  size_t n = size_t(C.c.residual) * C.c.d_h;
  size_t off = (size_t(s) * C.c.h_kv + h) * n;
  std::memcpy(kdst, &C.kres[off], n * 2);
  std::memcpy(vdst, &C.vres[off], n * 2);
}

// Dequantized K and V of (seq, head) for positions [0, count): fp64 [count][D].
void orc_dequant(void* hh, int32_t s, int32_t h, int64_t count, double* kout, double* vout) {
  Cache& C = *static_cast<Cache*>(hh);
  const int D = C.c.d_h;
  for (int64_t p = 0; p < count; ++p)
    dequant_token(C, s, h, p, kout + size_t(p) * D, vout + size_t(p) * D);
}

// Decode attention (day-65 page, "Why the KV cache grows so quickly"):
// out[i][hq] = softmax(q K^T / sqrt(d_h)) V over positions [0, seq_lens[i]) of
// sequence seq_ids[i] (or i when seq_ids is null), with query head hq reading
// kv head hq / (h_q / h_kv).  q: bf16 bits [B][h_q][d_h]; out: fp64.
// Empty sequences give zeros.  nthreads > 1 splits (row, kv head) work.
void orc_decode(void* hh, const uint16_t* q, const int32_t* seq_ids, const int32_t* seq_lens,
                int32_t B, double* out, int32_t nthreads) {
  Cache& C = *static_cast<Cache*>(hh);
  const Cfg& c = C.c;
  const int D = c.d_h, HQ = c.h_q, G = c.h_q / c.h_kv;
  auto work = [&](int64_t item) {
    int i = int(item / c.h_kv), h = int(item % c.h_kv);
    int s = seq_ids ? seq_ids[i] : i;
    int64_t T = seq_lens[i];
    std::vector<double> K(size_t(std::max<int64_t>(T, 1)) * D), V(K.size());
    for (int64_t p = 0; p < T; ++p) dequant_token(C, s, h, p, &K[size_t(p) * D], &V[size_t(p) * D]);
    std::vector<double> sc(size_t(std::max<int64_t>(T, 1)));
    for (int a = 0; a < G; ++a) {
      int hq = h * G + a;
      double* o = out + (size_t(i) * HQ + hq) * D;
      for (int e = 0; e < D; ++e) o[e] = 0.0;
      if (T == 0) continue;
      double qv[512];
      for (int e = 0; e < D; ++e) qv[e] = bf16_to_f32(q[(size_t(i) * HQ + hq) * D + e]);
      double mx = -INFINITY;
      for (int64_t p = 0; p < T; ++p) {
        double acc = 0.0;
        for (int e = 0; e < D; ++e) acc += qv[e] * K[size_t(p) * D + e];
        sc[size_t(p)] = acc / std::sqrt(double(D));
        mx = std::max(mx, sc[size_t(p)]);
      }
      double den = 0.0;
      for (int64_t p = 0; p < T; ++p) { sc[size_t(p)] = std::exp(sc[size_t(p)] - mx); den += sc[size_t(p)]; }
      for (int64_t p = 0; p < T; ++p) {
        double w = sc[size_t(p)] / den;
        for (int e = 0; e < D; ++e) o[e] += w * V[size_t(p) * D + e];
      }
    }
  };
  int64_t items = int64_t(B) * c.h_kv;
  int nt = std::max(1, std::min<int>(nthreads, int(items)));
  if (nt == 1) { for (int64_t it = 0; it < items; ++it) work(it); return; }
  std::vector<std::thread> th;
  for (int w = 0; w < nt; ++w)
    th.emplace_back([&, w] { for (int64_t it = w; it < items; it += nt) work(it); });
  for (auto& t : th) t.join();
}

}  // extern "C"
