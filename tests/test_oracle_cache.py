"""Pins of the oracle's cache model (layout, grouping, residual window,
allocator, attention) against properties, hand-derived locations, an
independent library routine (torch SDPA in fp64) and brute force.  CPU only."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_kv_cache_14_b200.workloads import random_bf16

D = 128

FORMATS = {
    # name: (bits, asym, k_axis, g_k, g_v, scale_fp32, residual, page)
    "int8_tok_p16": (8, 0, 0, 128, 128, 0, 0, 16),
    "int8_tok_fp32_p512": (8, 0, 0, 128, 128, 1, 0, 512),
    "int4_chan64_p16": (4, 0, 1, 64, 64, 0, 64, 16),
    "int2_asym_chan32_p16": (2, 1, 1, 32, 32, 0, 32, 16),
    "int4_asym_tok32": (4, 1, 0, 32, 32, 0, 0, 32),
    "int4_chan64_p32": (4, 0, 1, 64, 32, 0, 64, 32),
    "int8_asym_chan128_p64": (8, 1, 1, 128, 128, 0, 128, 64),
}


def make(name, h_kv=2, h_q=4, max_seqs=4, num_blocks=64, mbps=64, seed=3, **kw):
    bits, asym, k_axis, g_k, g_v, fp32, R, P = FORMATS[name]
    cfg = dict(bits=bits, asym=asym, k_axis=k_axis, g_k=g_k, g_v=g_v, scale_fp32=fp32,
               residual=R, page=P, h_q=h_q, h_kv=h_kv, d_h=D, max_seqs=max_seqs,
               num_blocks=num_blocks, max_blocks_per_seq=mbps, seed=seed, fail_alloc_after=-1)
    cfg.update(kw)
    return O.OracleCache(**cfg)


# ------------------------------------------------------------------ layout

@pytest.mark.parametrize("name", list(FORMATS))
def test_layout_fields_tile_the_sections(name):
    c = make(name)
    bits, P = c.cfg["bits"], c.cfg["page"]
    lay = c.layout
    for kind, sec in (("k", lay["secK"]), ("v", lay["secV"])):
        seen = np.zeros(sec * 8, dtype=np.int32)
        owner_tok = -np.ones(sec, dtype=np.int64)
        for tok in range(P):
            for ch in range(D):
                b, sh = c.code_loc(kind, tok, ch)
                assert 0 <= b < sec and sh % bits == 0 and sh + bits <= 8
                seen[b * 8 + sh: b * 8 + sh + bits] += 1
                # every byte belongs to one token (appends write whole bytes)
                assert owner_tok[b] in (-1, tok)
                owner_tok[b] = tok
        assert np.all(seen == 1), "fields must tile the section exactly once"
        if kind == "k":   # a key row is a contiguous run of D*bits/8 bytes
            for tok in range(P):
                bs = [c.code_loc("k", tok, ch)[0] for ch in range(D)]
                assert max(bs) - min(bs) + 1 == D * bits // 8
    c.close()


def test_layout_hand_derived_locations_int4():
    """From the m16n8k16 operand layout (PTX ISA, mma.sync fragments for
    .bf16 A: row = groupID / groupID+8, columns 2*tig + {0,1} and + 8):
    key rows list channels as 16j + 2t + {0, 1, 8, 9}; a word's even elements
    take the low fields, odd elements the high fields."""
    c = make("int4_chan64_p16")
    row = 64
    # key: token 0; channel 0 -> list pos 0 -> word 0 field 0
    assert c.code_loc("k", 0, 0) == (0, 0)
    # channel 1 -> list pos 1 -> field 4 -> byte 2
    assert c.code_loc("k", 0, 1) == (2, 0)
    # channel 8 -> list pos 2 -> field 1 -> byte 0, bits 4..7
    assert c.code_loc("k", 0, 8) == (0, 4)
    # channel 16 (k-step 1) -> list pos 4 -> field 2 -> byte 1
    assert c.code_loc("k", 0, 16) == (1, 0)
    # channel 2 (lane group t=1) -> list pos 32 -> word 4 -> byte 16
    assert c.code_loc("k", 0, 2) == (16, 0)
    # token 3 -> row 3
    assert c.code_loc("k", 3, 0) == (3 * row, 0)
    # value: token 0, channel 0 -> lane 0, reg a0 low -> field 0
    assert c.code_loc("v", 0, 0) == (0, 0)
    # token 1 (a0 high) -> field 4 -> byte 2
    assert c.code_loc("v", 1, 0) == (2, 0)
    # token 8 (a2 low) -> field 2 -> byte 1
    assert c.code_loc("v", 8, 0) == (1, 0)
    # channel 8 (a1 low) -> field 1 -> byte 0 bits 4..7
    assert c.code_loc("v", 0, 8) == (0, 4)
    # channel 1 -> groupID 1 -> lane 4 -> record of 32 bytes
    assert c.code_loc("v", 0, 1) == (4 * 32, 0)
    # token 2 -> tig 1 -> lane 1
    assert c.code_loc("v", 2, 0) == (32, 0)
    # channel 16 -> channel tile 1 -> word 1
    assert c.code_loc("v", 0, 16) == (4, 0)
    # token 16 -> next 16-token sub-tile (P=16 has one; use a P=32 format)
    c.close()
    c = make("int4_chan64_p32")
    assert c.code_loc("v", 16, 0) == (1024, 0)
    assert c.code_loc("k", 16, 0) == (1024, 0)
    c.close()


def test_layout_hand_derived_locations_int2_int8():
    c = make("int2_asym_chan32_p16")
    # int2: 16 fields per word; key channel 16 -> list pos 4 -> field 2 -> bits 4..5
    assert c.code_loc("k", 0, 16) == (0, 4)
    # value channel 16 (tile 1, a0) -> word 0, reg 2 -> field 2 -> bits 4..5
    assert c.code_loc("v", 0, 16) == (0, 4)
    # value token 8 (a2 of tile 0) -> reg 4 -> field 4 -> byte 1
    assert c.code_loc("v", 8, 0) == (1, 0)
    c.close()
    c = make("int8_tok_p16")
    # int8: key channel 1 -> list pos 1 -> field 2 -> byte 2; channel 8 -> byte 1
    assert c.code_loc("k", 0, 1) == (2, 0) and c.code_loc("k", 0, 8) == (1, 0)
    # value: a1 (channel 8) -> byte 1; a2 (token 8) -> word 1
    assert c.code_loc("v", 0, 8) == (1, 0) and c.code_loc("v", 8, 0) == (4, 0)
    assert c.code_loc("v", 0, 1) == (4 * 64, 0)
    c.close()


def test_layout_hand_derived_locations_fp8():
    """FP8, one byte per element: key rows keep the key-list order with bytes
    in natural order (list position = byte); a value lane record (4 g + t,
    64 bytes) holds operand register x of channel tile i in bytes 2x, 2x + 1
    of word 2 i + x / 2, low token first (a0 = channel g, tokens 2t | 2t+1;
    a1 = channel + 8; a2 = tokens + 8; a3 = both)."""
    c = O.OracleCache(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=16, fp8=1,
                      h_q=4, h_kv=2, d_h=D, max_seqs=1, num_blocks=4, max_blocks_per_seq=4, seed=0,
                      fail_alloc_after=-1)
    # keys: channels 0, 1, 8, 9, 16 are list positions 0, 1, 2, 3, 4; channel 2 is 32; rows of 128 bytes
    for ch, byte in ((0, 0), (1, 1), (8, 2), (9, 3), (16, 4), (2, 32)):
        assert c.code_loc("k", 0, ch) == (byte, 0)
    assert c.code_loc("k", 3, 0) == (3 * 128, 0)
    # values: (token, channel) -> byte of the sub-tile
    for tok, ch, byte in ((0, 0, 0),      # a0 low token, word 0 byte 0
                          (1, 0, 1),      # a0 high token, byte 1
                          (0, 8, 2),      # a1 low, bytes 2-3 of word 0
                          (8, 0, 4),      # a2 low, word 1
                          (9, 8, 7),      # a3 high, word 1 byte 3
                          (0, 16, 8),     # channel tile 1: word 2
                          (2, 0, 64),     # t = 1: lane 1
                          (0, 1, 256)):   # g = 1: lane 4
        assert c.code_loc("v", tok, ch) == (byte, 0), (tok, ch)
    c.close()


# -------------------------------------------- grouping direction / round trip

def _expected_dequant(name, k32, v32, R):
    """Per-(token|channel) groups quantized with the scalar quantizer (pinned
    above), dequantized in fp64 -- keys per channel over G_k tokens for the
    channel axis, per token otherwise; values per token over G_v channels."""
    bits, asym, k_axis, g_k, g_v, fp32, _, _ = FORMATS[name]
    T = k32.shape[0]

    def qd(x, g):
        if asym:
            s, z, q = O.quant_asym(x, bits, fp32)
            return s * q.astype(np.float64) + z
        s, q = O.quant_sym(x, bits, fp32)
        return s * q.astype(np.float64)

    Lq = (T // R) * R if R else T
    K = k32.astype(np.float64).copy()
    V = v32.astype(np.float64).copy()
    for t in range(Lq):
        for a in range(0, D, g_v):
            V[t, a:a + g_v] = qd(v32[t, a:a + g_v], g_v)
    if k_axis == 0:
        for t in range(Lq):
            for a in range(0, D, g_k):
                K[t, a:a + g_k] = qd(k32[t, a:a + g_k], g_k)
    else:
        for g0 in range(0, Lq, g_k):
            for ch in range(D):
                K[g0:g0 + g_k, ch] = qd(k32[g0:g0 + g_k, ch].copy(), g_k)
    return K, V


@pytest.mark.parametrize("name", list(FORMATS))
def test_dequant_matches_group_quantizer(name):
    rng = np.random.default_rng(11)
    c = make(name)
    R = c.cfg["residual"]
    T = 150 if R else 137
    k = random_bf16(rng, (T, 2, D))
    k[:, :, 5] = random_bf16(rng, (T, 2), 20.0)  # an outlier channel
    v = random_bf16(rng, (T, 2, D))
    assert c.append(k, v, np.zeros(T, np.int32)) == 0
    for h in range(2):
        K, V = c.dequant(0, h, T)
        k32 = O.bf16_bits_to_f32(k[:, h, :])
        v32 = O.bf16_bits_to_f32(v[:, h, :])
        Ke, Ve = _expected_dequant(name, k32, v32, R)
        assert np.array_equal(K, Ke)
        assert np.array_equal(V, Ve)
    c.close()


# ---------------------------------------------------------- residual window

@pytest.mark.parametrize("name", ["int4_chan64_p16", "int2_asym_chan32_p16", "int8_asym_chan128_p64"])
def test_residual_window_semantics(name):
    rng = np.random.default_rng(5)
    c = make(name, max_seqs=3, num_blocks=200)
    R, P = c.cfg["residual"], c.cfg["page"]
    hist = {s: [] for s in range(3)}
    for step in range(25):
        n = int(rng.integers(1, 40))
        ids = rng.integers(0, 3, size=n).astype(np.int32)
        k = random_bf16(rng, (n, 2, D))
        v = random_bf16(rng, (n, 2, D))
        assert c.append(k, v, ids) == 0
        for i, s in enumerate(ids):
            hist[int(s)].append((k[i], v[i]))
        for s in range(3):
            L = len(hist[s])
            assert c.seq_len(s) == L
            occ = L % R
            assert len(c.block_table(s)) == (L // R) * (R // P)
            for h in range(2):
                kr, vr = c.residual(s, h)
                for j in range(occ):
                    pos = L - occ + j
                    assert np.array_equal(kr[pos % R], hist[s][pos][0][h])
                    assert np.array_equal(vr[pos % R], hist[s][pos][1][h])
    c.close()


@pytest.mark.parametrize("name", ["int4_chan64_p16", "int8_tok_p16", "int2_asym_chan32_p16"])
def test_bulk_append_equals_chunked_appends(name):
    rng = np.random.default_rng(9)
    n = 300
    ids = rng.integers(0, 3, size=n).astype(np.int32)
    k = random_bf16(rng, (n, 2, D), 3.0)
    v = random_bf16(rng, (n, 2, D))
    a = make(name, max_seqs=3, num_blocks=200)
    b = make(name, max_seqs=3, num_blocks=200)
    assert a.append(k, v, ids) == 0
    cut = [0, 1, 2, 50, 51, 170, 299, 300]
    for lo, hi in zip(cut[:-1], cut[1:]):
        assert b.append(k[lo:hi], v[lo:hi], ids[lo:hi]) == 0
    assert np.array_equal(a.pool(), b.pool())
    for s in range(3):
        assert np.array_equal(a.block_table(s), b.block_table(s))
    a.close(); b.close()


# ----------------------------------------------------------------- allocator

def test_blocks_come_from_the_seeded_free_list_in_order():
    c = make("int8_tok_p16", num_blocks=50, seed=77, max_seqs=2)
    rng = np.random.default_rng(1)
    n = 16 * 7 + 3
    k = random_bf16(rng, (n, 2, D)); v = random_bf16(rng, (n, 2, D))
    assert c.append(k, v, np.zeros(n, np.int32)) == 0
    fl = O.free_list(50, 77)
    assert c.block_table(0).tolist() == fl[:8].tolist()
    # interleaved second sequence continues popping from the front
    assert c.append(k[:20], v[:20], np.ones(20, np.int32)) == 0
    assert c.block_table(1).tolist() == fl[8:10].tolist()
    # freeing pushes blocks to the back in logical order
    assert c.free_seq(0) == 0
    assert c.free_count() == 50 - 10 + 8
    c.close()


def test_freed_blocks_are_reused_after_the_untouched_ones():
    c = make("int8_tok_p16", num_blocks=6, seed=1, max_seqs=2)
    rng = np.random.default_rng(2)
    k = random_bf16(rng, (64, 2, D)); v = random_bf16(rng, (64, 2, D))
    fl = O.free_list(6, 1).tolist()
    assert c.append(k[:64], v[:64], np.zeros(64, np.int32)) == 0     # 4 blocks
    assert c.free_seq(0) == 0
    assert c.append(k[:48], v[:48], np.ones(48, np.int32)) == 0      # 3 blocks
    assert c.block_table(1).tolist() == [fl[4], fl[5], fl[0]]
    c.close()


def test_reused_block_reads_zero_in_its_unused_slots():
    """The layout contract zero-fills the pool, so a token slot that no append
    has written reads as zero codes and zero scales.  A block freed with data
    in all 16 slots and reused by a sequence that writes only 5 of them must
    hold zeros in the other 11 (keys, values and metadata of those slots)."""
    c = make("int8_tok_p16", num_blocks=1, seed=1, max_seqs=2)
    rng = np.random.default_rng(8)
    k = random_bf16(rng, (16, 2, D), 3.0); v = random_bf16(rng, (16, 2, D))
    assert c.append(k, v, np.zeros(16, np.int32)) == 0     # the one block, every slot written
    assert c.free_seq(0) == 0
    assert c.append(k[:5], v[:5], np.ones(5, np.int32)) == 0   # the same block again, 5 slots
    assert c.block_table(1).tolist() == [0]
    pool, lay = c.pool(), c.layout
    for h in range(2):
        chunk = pool[h * lay["chunk_bytes"]:(h + 1) * lay["chunk_bytes"]]
        for tok in range(5, 16):
            for ch in range(D):
                for sec, kind in ((0, "k"), (lay["off_V"], "v")):
                    byte, _ = c.code_loc(kind, tok, ch)
                    assert chunk[sec + byte] == 0, (h, kind, tok, ch)
        # metadata of the unwritten slots: one key and one value scale per token (fp16)
        for tok in range(5, 16):
            assert not chunk[lay["off_Vm"] + 2 * tok:lay["off_Vm"] + 2 * tok + 2].any()
            assert not chunk[lay["off_Km"] + 2 * tok:lay["off_Km"] + 2 * tok + 2].any()
    c.close()


def test_admission_counts_only_the_blocks_a_call_adds():
    """Blocks are allocated on demand (day-65 "How this connects to paging and
    prefix caching"): an append needs only the blocks its new tokens open, so
    a pool with exactly that many free blocks admits it, and one more token
    than fits is refused with nothing changed.  Sequence ids run over
    [0, max_seqs): max_seqs itself is refused."""
    c = make("int8_tok_p16", num_blocks=3, max_seqs=2)
    rng = np.random.default_rng(9)
    k = random_bf16(rng, (49, 2, D)); v = random_bf16(rng, (49, 2, D))
    assert c.append(k[:32], v[:32], np.zeros(32, np.int32)) == 0    # 2 blocks, 1 free
    assert c.append(k[32:48], v[32:48], np.zeros(16, np.int32)) == 0  # fills the 3rd block exactly
    assert c.free_count() == 0 and c.seq_len(0) == 48
    pool = c.pool().copy()
    assert c.append(k[48:], v[48:], np.zeros(1, np.int32)) == 2     # a 4th block: none left
    assert c.append(k[48:], v[48:], np.full(1, 2, np.int32)) == 3   # id == max_seqs
    assert c.seq_len(0) == 48 and c.seq_len(1) == 0 and np.array_equal(c.pool(), pool)
    c.close()


@pytest.mark.parametrize("name", ["int8_tok_p16", "int4_chan64_p16"])
def test_out_of_blocks_leaves_state_unchanged(name):
    c = make(name, num_blocks=5, max_seqs=2)
    rng = np.random.default_rng(3)
    k = random_bf16(rng, (200, 2, D)); v = random_bf16(rng, (200, 2, D))
    assert c.append(k[:40], v[:40], np.zeros(40, np.int32)) == 0
    before = (c.pool().copy(), c.seq_len(0), c.block_table(0).tolist(), c.free_count())
    assert c.append(k, v, np.zeros(200, np.int32)) == 2
    after = (c.pool(), c.seq_len(0), c.block_table(0).tolist(), c.free_count())
    assert np.array_equal(before[0], after[0]) and before[1:] == after[1:]
    assert c.append(k[:5], v[:5], np.full(5, 7, np.int32)) == 3     # bad sequence id
    c.close()


def test_fail_alloc_after_hook():
    c = make("int8_tok_p16", num_blocks=40, fail_alloc_after=2)
    rng = np.random.default_rng(4)
    k = random_bf16(rng, (48, 2, D)); v = random_bf16(rng, (48, 2, D))
    assert c.append(k[:32], v[:32], np.zeros(32, np.int32)) == 0    # blocks 0, 1
    assert c.append(k[:1], v[:1], np.zeros(1, np.int32)) == 2       # 3rd allocation fails
    assert c.seq_len(0) == 32
    c.close()


def test_table_width_is_enforced():
    c = make("int8_tok_p16", num_blocks=40, mbps=2)
    rng = np.random.default_rng(4)
    k = random_bf16(rng, (33, 2, D)); v = random_bf16(rng, (33, 2, D))
    assert c.append(k[:32], v[:32], np.zeros(32, np.int32)) == 0
    assert c.append(k[32:], v[32:], np.zeros(1, np.int32)) == 2
    c.close()


# ---------------------------------------------------------------- attention

def _sdpa(q, K, V):
    # torch's scaled_dot_product_attention in fp64: softmax(q K^T / sqrt(d)) V
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(K)[None, None],
        torch.from_numpy(V)[None, None]).numpy()[0, 0]


@pytest.mark.parametrize("name", ["int4_chan64_p16", "int8_tok_p16", "int2_asym_chan32_p16"])
def test_decode_matches_torch_sdpa_fp64(name):
    rng = np.random.default_rng(21)
    c = make(name, h_kv=2, h_q=8, max_seqs=3, num_blocks=100)
    lens = [1, 77, 200]
    ids = np.repeat(np.arange(3, dtype=np.int32), lens)
    n = int(sum(lens))
    k = random_bf16(rng, (n, 2, D), 2.0); v = random_bf16(rng, (n, 2, D))
    assert c.append(k, v, ids) == 0
    q = random_bf16(rng, (3, 8, D))
    out = c.decode(q, lens)
    q64 = O.bf16_bits_to_f32(q).astype(np.float64)
    for i in range(3):
        for hq in range(8):
            K, V = c.dequant(i, hq // 4, lens[i])
            ref = _sdpa(q64[i, hq][None], K, V)[0]
            assert np.allclose(out[i, hq], ref, rtol=0, atol=1e-12)
    out2 = c.decode(q, lens, nthreads=4)
    assert np.array_equal(out, out2)
    c.close()


def test_decode_special_cases():
    rng = np.random.default_rng(8)
    c = make("int8_tok_p16", h_kv=2, h_q=4, max_seqs=4, num_blocks=50)
    # seq 0: one token -> output is that token's dequantized value, every head
    k = random_bf16(rng, (1, 2, D)); v = random_bf16(rng, (1, 2, D))
    assert c.append(k, v, np.zeros(1, np.int32)) == 0
    # seq 1: identical keys -> uniform weights -> mean of the values
    krow = random_bf16(rng, (1, 2, D))
    k1 = np.repeat(krow, 40, axis=0); v1 = random_bf16(rng, (40, 2, D))
    assert c.append(k1, v1, np.ones(40, np.int32)) == 0
    # seq 2: kv head h has constant values h+1 (head mapping hq -> hq // 2)
    k2 = random_bf16(rng, (30, 2, D))
    v2 = np.zeros((30, 2, D), np.uint16)
    v2[:, 0, :] = 0x3F80   # 1.0
    v2[:, 1, :] = 0x4000   # 2.0
    assert c.append(k2, v2, np.full(30, 2, np.int32)) == 0
    q = random_bf16(rng, (4, 4, D))
    out = c.decode(q, [1, 40, 30, 0])
    for hq in range(4):
        _, V = c.dequant(0, hq // 2, 1)
        assert np.allclose(out[0, hq], V[0], atol=1e-15)
        _, V = c.dequant(1, hq // 2, 40)
        assert np.allclose(out[1, hq], V.mean(axis=0), atol=1e-12)
        _, V = c.dequant(2, hq // 2, 30)
        assert np.all(V == V[0, 0]) and abs(V[0, 0] - (1.0 + hq // 2)) < 1e-3
        assert np.allclose(out[2, hq], V[0, 0], atol=1e-12)
    assert not out[3].any()       # empty sequence -> zeros
    c.close()


def test_decode_dominant_score_picks_its_row():
    rng = np.random.default_rng(12)
    c = make("int8_tok_p16", h_kv=1, h_q=1, max_seqs=1, num_blocks=10)
    T = 50
    k = random_bf16(rng, (T, 1, D), 0.01)
    k[17, 0, :] = 0x4120      # 10.0 everywhere -> score ~ 10 * sum(q) / sqrt(D)
    v = random_bf16(rng, (T, 1, D))
    assert c.append(k, v, np.zeros(T, np.int32)) == 0
    q = np.full((1, 1, D), 0x3F80, np.uint16)    # q = 1.0
    out = c.decode(q, [T])
    _, V = c.dequant(0, 0, T)
    assert np.allclose(out[0, 0], V[17], atol=1e-9)
    c.close()


# ------------------------------------------------------------ BF16 control

def _bf16_control(**kw):
    cfg = dict(bits=16, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=16,
               h_q=4, h_kv=2, d_h=D, max_seqs=3, num_blocks=64, max_blocks_per_seq=64, seed=5,
               fail_alloc_after=-1)
    cfg.update(kw)
    return O.OracleCache(**cfg)


@pytest.mark.parametrize("page", [16, 64])
def test_bf16_control_stores_rows_unchanged(page):
    """The control format is the pages' unquantized BF16 cache: the stored
    bytes are the appended bf16 rows (natural order, 256 B per row, 16-row
    sub-tiles), dequantization returns them exactly, and there is no metadata."""
    rng = np.random.default_rng(2)
    c = _bf16_control(page=page)
    lay = c.layout
    assert lay["row_bytes"] == 2 * D and lay["sub_bytes"] == 16 * 2 * D
    assert lay["off_V"] == lay["secK"] == (page // 16) * 16 * 2 * D
    assert lay["off_Vm"] == lay["off_Km"] == 2 * lay["secK"]          # no scales
    T = 3 * page + 5
    k = random_bf16(rng, (T, 2, D), 4.0)
    v = random_bf16(rng, (T, 2, D))
    assert c.append(k, v, np.zeros(T, np.int32)) == 0
    pool = c.pool()
    table = c.block_table(0)
    for tok in (0, 1, 15, 16, page - 1, page, T - 1):
        for ch in (0, 1, 77, D - 1):
            b, sh = c.code_loc("k", tok % page, ch)
            assert sh == 0 and b == (tok % page // 16) * 16 * 2 * D + (tok % 16) * 2 * D + 2 * ch
            for h in range(2):
                base = int(table[tok // page]) * lay["block_bytes"] + h * lay["chunk_bytes"]
                kb = int(pool[base + b]) | (int(pool[base + b + 1]) << 8)
                vb = int(pool[base + lay["off_V"] + b]) | (int(pool[base + lay["off_V"] + b + 1]) << 8)
                assert kb == int(k[tok, h, ch]) and vb == int(v[tok, h, ch])
    for h in range(2):
        K, V = c.dequant(0, h, T)
        assert np.array_equal(K, O.bf16_bits_to_f32(k[:, h, :]).astype(np.float64))
        assert np.array_equal(V, O.bf16_bits_to_f32(v[:, h, :]).astype(np.float64))
    # 2 bytes per element for K and for V, nothing else
    assert O.cache_bytes_formula(32, 8192, 8, 128, 16, 128, 128, 0) == 2 * 32 * 8192 * 8 * 128 * 2
    c.close()


def test_bf16_control_decode_matches_torch_sdpa():
    rng = np.random.default_rng(9)
    c = _bf16_control()
    lens = [1, 40, 97]
    ids = np.repeat(np.arange(3, dtype=np.int32), lens)
    k = random_bf16(rng, (ids.size, 2, D), 3.0)
    v = random_bf16(rng, (ids.size, 2, D))
    assert c.append(k, v, ids) == 0
    q = random_bf16(rng, (3, 4, D))
    got = c.decode(q, lens)
    for i, L in enumerate(lens):
        sel = ids == i
        K = torch.from_numpy(O.bf16_bits_to_f32(k[sel]).astype(np.float64)).permute(1, 0, 2)
        V = torch.from_numpy(O.bf16_bits_to_f32(v[sel]).astype(np.float64)).permute(1, 0, 2)
        Q = torch.from_numpy(O.bf16_bits_to_f32(q[i]).astype(np.float64)).reshape(4, 1, D)
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q, K.repeat_interleave(2, dim=0), V.repeat_interleave(2, dim=0))
        assert np.allclose(got[i], ref.reshape(4, D).numpy(), rtol=0, atol=1e-12)
    c.close()


# ------------------------------------------------------------ prefix sharing

@pytest.mark.parametrize("name", ["int8_tok_p16", "int4_chan64_p16", "int2_asym_chan32_p16", "int4_asym_tok32"])
def test_shared_prefix_equals_an_unshared_copy(name):
    """A sequence that starts from another's shared prefix holds exactly what a
    sequence built by appending the same rows would hold (quantization works
    per group, and only whole groups/pages are shared); appends after the
    share go to fresh blocks and leave the other sequence unchanged."""
    rng = np.random.default_rng(4)
    bits, asym, k_axis, g_k, g_v, fp32, R, P = FORMATS[name]
    unit = R or P
    c = make(name, max_seqs=3, num_blocks=200)
    ref = make(name, max_seqs=3, num_blocks=200)
    T0 = 4 * unit + 3
    k0, v0 = random_bf16(rng, (T0, 2, D), 3.0), random_bf16(rng, (T0, 2, D))
    assert c.append(k0, v0, np.zeros(T0, np.int32)) == 0
    shared = 3 * unit
    assert c.share_prefix(0, 1, shared) == 0
    assert c.seq_len(1) == shared
    assert c.block_table(1).tolist() == c.block_table(0)[:len(c.block_table(1))].tolist()
    # independent copy: seq 1 of `ref` gets the same prefix rows by appending
    assert ref.append(k0[:shared], v0[:shared], np.ones(shared, np.int32)) == 0
    k1, v1 = random_bf16(rng, (2 * unit + 5, 2, D)), random_bf16(rng, (2 * unit + 5, 2, D))
    k2, v2 = random_bf16(rng, (unit + 1, 2, D)), random_bf16(rng, (unit + 1, 2, D))
    for cache in (c, ref):
        assert cache.append(k1, v1, np.ones(len(k1), np.int32)) == 0
    assert c.append(k2, v2, np.zeros(len(k2), np.int32)) == 0
    for h in range(2):
        K1, V1 = c.dequant(1, h, c.seq_len(1))
        Kr, Vr = ref.dequant(1, h, ref.seq_len(1))
        assert np.array_equal(K1, Kr) and np.array_equal(V1, Vr)
        # seq 0: its whole groups/pages from before are unchanged by everything
        # done to seq 1 (its window tail was quantized later by its own appends)
        T0w = (T0 // unit) * unit
        K0, V0 = c.dequant(0, h, T0w)
        solo = make(name, max_seqs=1, num_blocks=200)
        assert solo.append(k0, v0, np.zeros(T0, np.int32)) == 0
        Ks, Vs = solo.dequant(0, h, T0w)
        assert np.array_equal(K0, Ks) and np.array_equal(V0, Vs)
        solo.close()
    c.close()
    ref.close()


def test_shared_blocks_are_freed_by_their_last_holder():
    c = make("int8_tok_p16", max_seqs=3, num_blocks=40)
    k = random_bf16(np.random.default_rng(1), (80, 2, D))
    assert c.append(k, k, np.zeros(80, np.int32)) == 0          # 5 blocks
    free0 = c.free_count()
    assert c.share_prefix(0, 1, 64) == 0                         # 4 blocks shared
    assert c.free_count() == free0
    t0 = c.block_table(0).tolist()
    assert c.free_seq(0) == 0                                    # only the unshared block frees
    assert c.free_count() == free0 + 1
    assert c.free_seq(1) == 0                                    # now the shared ones, in order
    assert c.free_count() == free0 + 5
    # errors leave the state alone
    assert c.append(k[:20], k[:20], np.zeros(20, np.int32)) == 0
    for args, code in (((0, 1, 17), 4), ((0, 0, 16), 4), ((0, 1, 32), 4), ((0, 5, 16), 3)):
        if args[2] == 32:
            assert c.share_prefix(0, 1, 16) == 0                 # dst no longer empty
        assert c.share_prefix(*args) == code
    assert t0 != []
    c.close()


def test_windowed_cache_shares_whole_key_groups_only():
    """With a BF16 window the pages hold whole key groups only (day-65 "Why
    some systems keep a full-precision window": a group moves into the cache
    when it fills); the newest tokens of a group still filling live in the
    source's window, not in a block.  A prefix that is a whole number of pages
    but not of groups is refused, with no state change; whole groups share."""
    c = make("int4_chan64_p16", max_seqs=3, num_blocks=40)
    k = random_bf16(np.random.default_rng(5), (150, 2, D))
    assert c.append(k, k, np.zeros(150, np.int32)) == 0        # 2 groups in 8 blocks, 22 in the window
    free0, t0 = c.free_count(), c.block_table(0).tolist()
    for tokens in (16, 48, 80, 144):                           # pages, not whole groups
        assert c.share_prefix(0, 1, tokens) == 4
        assert c.seq_len(1) == 0 and c.block_table(1).tolist() == [] and c.free_count() == free0
    assert c.share_prefix(0, 1, 128) == 0                      # two whole groups
    assert c.block_table(1).tolist() == t0 and c.seq_len(1) == 128
    c.close()


# ------------------------------------------------------------ FP8 format

def test_fp8_dequant_is_scale_times_e4m3_of_the_scaled_input():
    """FP8 E4M3 with one scale per kv head: the stored byte of element x is
    e4m3(x / s) (pinned converter), read back as s * e4m3; keys keep the
    key-list order one byte per element, values the lane records."""
    rng = np.random.default_rng(6)
    c = O.OracleCache(bits=8, asym=0, k_axis=0, g_k=128, g_v=128, scale_fp32=0, residual=0, page=16, fp8=1,
                      h_q=4, h_kv=2, d_h=D, max_seqs=2, num_blocks=40, max_blocks_per_seq=40, seed=2,
                      fail_alloc_after=-1)
    ks, vs = np.array([0.25, 3.0], np.float32), np.array([1.5, 0.01], np.float32)
    assert c.set_fp8_scales(ks, vs) == 0
    T = 37
    k = random_bf16(rng, (T, 2, D), 5.0)
    v = random_bf16(rng, (T, 2, D), 5.0)
    assert c.append(k, v, np.zeros(T, np.int32)) == 0
    assert c.set_fp8_scales(ks, vs) == 4                     # fixed once tokens are stored
    lay = c.layout
    assert lay["off_Vm"] == lay["off_Km"] == 2 * lay["secK"]   # no metadata
    kf, vf = O.bf16_bits_to_f32(k), O.bf16_bits_to_f32(v)
    for h in range(2):
        K, V = c.dequant(0, h, T)
        for t in (0, 5, 36):
            for ch in (0, 9, 77, 127):
                ck = O.f32_to_e4m3(float(np.float32(kf[t, h, ch]) / ks[h]))
                cv = O.f32_to_e4m3(float(np.float32(vf[t, h, ch]) / vs[h]))
                assert K[t, ch] == float(ks[h]) * O.e4m3_to_f32(ck)
                assert V[t, ch] == float(vs[h]) * O.e4m3_to_f32(cv)
    # values beyond 448 s saturate
    assert np.max(np.abs(c.dequant(0, 1, T)[1])) <= 448 * float(vs[1]) + 1e-12
    # layout: every byte of a section belongs to one element, key rows in list order
    for kind, sec in (("k", lay["secK"]), ("v", lay["secV"])):
        seen = np.zeros(sec, np.int32)
        for tok in range(16):
            for ch in range(D):
                b, sh = c.code_loc(kind, tok, ch)
                assert sh == 0
                seen[b] += 1
        assert np.all(seen == 1)
    c.close()
