"""The V quantiser's packing shortcuts, emulated exactly on the CPU.

v_quant_kernel packs the INT4 codes of 8 consecutive tokens x 8 channels per
thread into 8 words (one per token, channel e in nibble e), transposes the
8 x 8 nibbles in registers with three block swaps (16-bit halves by byte
permutes 0x5410 / 0x7632, bytes by 0x6240 / 0x7351, single nibbles by masks
and shifts), and sums a channel's signed codes from its packed words as
sum(nibbles of w ^ 0x88888888) - 8 per code.  The emulation below performs
the same 32-bit operations (byte permute semantics: result byte k = byte
sel[k] of the 8-byte pair a | b << 32) and checks them against the plain
definitions: the transposed matrix and the column sums of the codes.
"""
import numpy as np

M32 = 0xFFFFFFFF


def prmt(a, b, sel):
    """PTX prmt.b32 default mode: byte k of the result is byte (sel >> 4k) & 7
    of the 64-bit value b:a."""
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    return sum(src[(sel >> (4 * k)) & 7] << (8 * k) for k in range(4))


def transpose8_nibbles(r):
    r = list(r)
    for i in range(4):
        a, b = r[i], r[i + 4]
        r[i], r[i + 4] = prmt(a, b, 0x5410), prmt(a, b, 0x7632)
    for i in (0, 1, 4, 5):
        a, b = r[i], r[i + 2]
        r[i], r[i + 2] = prmt(a, b, 0x6240), prmt(a, b, 0x7351)
    for i in (0, 2, 4, 6):
        a, b = r[i], r[i + 1]
        r[i] = (a & 0x0F0F0F0F) | ((b << 4) & 0xF0F0F0F0)
        r[i + 1] = ((a >> 4) & 0x0F0F0F0F) | (b & 0xF0F0F0F0)
    return [x & M32 for x in r]


def dp4a_u8(a, acc):
    """dp4a with 0x01010101: acc + the four bytes of a (unsigned)."""
    return acc + sum((a >> (8 * i)) & 0xFF for i in range(4))


def nibble_sum_plus64(w, acc):
    x = w ^ 0x88888888
    acc = dp4a_u8(x & 0x0F0F0F0F, acc)
    return dp4a_u8((x >> 4) & 0x0F0F0F0F, acc)


def pack_row(codes):
    """8 signed codes -> one word, code e in bits 4e .. 4e + 3 (two's complement)."""
    return sum((int(c) & 0xF) << (4 * e) for e, c in enumerate(codes))


def test_transpose_matches_the_definition():
    rng = np.random.default_rng(5)
    for _ in range(2000):
        words = [int(x) for x in rng.integers(0, 1 << 32, 8, dtype=np.uint64)]
        t = transpose8_nibbles(words)
        for e in range(8):
            for i in range(8):
                assert (t[e] >> (4 * i)) & 0xF == (words[i] >> (4 * e)) & 0xF


def test_transpose_is_an_involution():
    rng = np.random.default_rng(6)
    for _ in range(500):
        words = [int(x) for x in rng.integers(0, 1 << 32, 8, dtype=np.uint64)]
        assert transpose8_nibbles(transpose8_nibbles(words)) == words


def test_channel_words_and_column_sums_of_a_block():
    """A 64-token block of V codes in [-7, 7] (the symmetric INT4 range): the
    thread layout (8 channels x 8 consecutive tokens) plus the transpose gives
    per channel the 8 words of its 64 tokens in order, and the nibble sums
    give the column sums."""
    rng = np.random.default_rng(7)
    for _ in range(20):
        codes = rng.integers(-7, 8, (64, 128))          # [token][channel]
        words = np.zeros((8, 128), np.uint64)           # [token group][channel]
        for r0 in range(8):                              # token group: tokens 8 r0 .. 8 r0 + 7
            for g in range(16):                          # channels 8 g .. 8 g + 7
                rows = [pack_row(codes[8 * r0 + i, 8 * g:8 * g + 8]) for i in range(8)]
                t = transpose8_nibbles(rows)
                words[r0, 8 * g:8 * g + 8] = t
        for c in range(128):
            total = -512
            for t in range(8):
                w = int(words[t, c])
                assert w == pack_row(codes[8 * t:8 * t + 8, c])   # tokens of the group in order
                total = nibble_sum_plus64(w, total)
            assert total == int(codes[:, c].sum())


def test_nibble_sum_covers_the_full_code_range():
    for code in range(-8, 8):
        w = pack_row([code] * 8)
        assert nibble_sum_plus64(w, -64) == 8 * code
