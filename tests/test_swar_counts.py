"""The word-at-a-time byte counts the decode kernels use, checked exhaustively
on the host against the byte-at-a-time definitions.

Zero-run encoding (3LC review page, "Proposed method" bullet 3): an escape
byte 243..255 stands for a run of 2..14 zero groups (b - 241 groups), any
other byte for one group; literal bytes other than 121 carry a non-zero
value.  The kernels count 16 payload bytes (four little-endian 32-bit words)
at once with carry-free per-byte arithmetic; these tests restate that
arithmetic in numpy (uint32, wrapping) and compare it with the per-byte
definition for every byte value in every byte position and on random words.
"""
import numpy as np

M = np.uint32(0xFFFFFFFF)


def esc_bits(w):
    w = w.astype(np.uint32)
    return w & ((w & np.uint32(0x7F7F7F7F)) + np.uint32(0x0D0D0D0D)) & np.uint32(0x80808080)


def byte_lane_sum(x):
    return ((x.astype(np.uint64) * 0x01010101) & 0xFFFFFFFF) >> 24


def expansion16(words):
    lo = np.zeros(words.shape[0], np.uint32)
    cnt = np.zeros(words.shape[0], np.uint32)
    for k in range(4):
        e = esc_bits(words[:, k]) >> np.uint32(7)
        lo += words[:, k] & np.uint32(0x0F0F0F0F) & (e * np.uint32(0x0F))
        cnt += e
    return 16 + byte_lane_sum(lo).astype(np.int64) - 2 * byte_lane_sum(cnt).astype(np.int64)


def literals16(words):
    cnt = np.zeros(words.shape[0], np.uint32)
    for k in range(4):
        w = words[:, k]
        x = w ^ np.uint32(0x79797979)
        nz = ((x & np.uint32(0x7F7F7F7F)) + np.uint32(0x7F7F7F7F)) | x
        cnt += ((~nz & np.uint32(0x80808080)) | esc_bits(w)) >> np.uint32(7)
    return 16 - byte_lane_sum(cnt).astype(np.int64)


def by_bytes(b):
    """Per-byte definitions: groups and non-zero literals of rows of 16 bytes."""
    b = b.astype(np.int64)
    groups = np.where(b >= 243, b - 241, 1).sum(axis=1)
    lits = ((b < 243) & (b != 121)).sum(axis=1)
    return groups, lits


def words_of(b):
    return b.astype(np.uint8).reshape(-1, 16).view("<u4").reshape(-1, 4)


def test_every_byte_value_in_every_position():
    rows = []
    for pos in range(16):
        for v in range(256):
            r = np.full(16, 121, np.uint8)
            r[pos] = v
            rows.append(r)
    b = np.stack(rows)
    g, l = by_bytes(b)
    w = words_of(b)
    assert np.array_equal(expansion16(w), g)
    assert np.array_equal(literals16(w), l)


def test_random_and_extreme_rows():
    rng = np.random.default_rng(7)
    b = [rng.integers(0, 256, (20000, 16)),
         rng.integers(240, 256, (20000, 16)),          # escapes and their neighbours
         np.full((1, 16), 255), np.full((1, 16), 243), np.full((1, 16), 242),
         np.full((1, 16), 121), np.zeros((1, 16), int)]
    b = np.concatenate(b).astype(np.uint8)
    g, l = by_bytes(b)
    w = words_of(b)
    assert np.array_equal(expansion16(w), g)
    assert np.array_equal(literals16(w), l)
    assert expansion16(words_of(np.full((1, 16), 255, np.uint8)))[0] == 16 * 14
