"""Host-side model of the tensor-core attention kernel's operand layout
(no GPU): the coordinate permutation, nibble-to-code conversions and
fragment assignment of kvq_attn_tc_kernel, written against the m16n8k16
fragment layout of the PTX ISA (lane = 4 g + c; A rows g, g + 8 and columns
2c, 2c + 1, 2c + 8, 2c + 9; B rows 2c, 2c + 1, 2c + 8, 2c + 9 of column g),
must reproduce the direct products K q and p V of one 16-token chunk."""
import numpy as np
import pytest


def nib_code(n):
    return (n ^ 8) - 8


def lo_pair(x):  # codes of the low nibbles of bytes 0 and 2
    return nib_code(x & 0xF), nib_code((x >> 16) & 0xF)


def hi_pair(x):  # the high nibbles (the kernel shifts x down by 4 first)
    return lo_pair(x >> 4)


def coord(d, c, s, e):
    b = (d // 8) * c + 4 * (s >> 1)
    return 2 * b + 2 * (s & 1) + (e >> 1) + 4 * (e & 1)


def byte_perm(x, y, sel):
    bs = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    return sum(bs[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))


def rows_as_bytes(codes):
    t, d = codes.shape
    b = np.zeros((t, d // 2), dtype=np.int64)
    for i in range(d // 2):
        b[:, i] = (codes[:, 2 * i] & 0xF) | ((codes[:, 2 * i + 1] & 0xF) << 4)
    return b


def word(rows, t, byte0):
    return int(sum(int(rows[t, byte0 + i]) << (8 * i) for i in range(4)))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_coordinate_permutation_is_a_bijection(d):
    seen = sorted(coord(d, c, s, e) for c in range(4) for s in range(d // 16) for e in range(4))
    assert seen == list(range(d))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_score_fragments_match_direct_product(d):
    rng = np.random.default_rng(1)
    codes = rng.integers(-8, 8, size=(16, d))
    rows = rows_as_bytes(codes)
    q = rng.standard_normal((4, d))
    S = np.zeros((16, 8))
    for s in range(d // 16):
        A = np.zeros((16, 16))
        B = np.zeros((16, 8))
        for lane in range(32):
            g, c = lane >> 2, lane & 3
            w0 = word(rows, g, (d // 8) * c + 4 * (s // 2))
            w8 = word(rows, g + 8, (d // 8) * c + 4 * (s // 2))
            if s & 1:
                w0, w8 = w0 >> 8, w8 >> 8
            A[g, 2 * c:2 * c + 2] = lo_pair(w0)
            A[g + 8, 2 * c:2 * c + 2] = lo_pair(w8)
            A[g, 2 * c + 8:2 * c + 10] = hi_pair(w0)
            A[g + 8, 2 * c + 8:2 * c + 10] = hi_pair(w8)
            for e, row in ((0, 2 * c), (1, 2 * c + 1), (2, 2 * c + 8), (3, 2 * c + 9)):
                B[row, g] = q[g >> 1, coord(d, c, s, e)] if g % 2 == 0 else 0.0
        S += A @ B
    got = np.stack([S[:, 2 * k] + S[:, 2 * k + 1] for k in range(4)], 1)
    np.testing.assert_allclose(got, codes @ q.T, rtol=0, atol=1e-9)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_accumulation_fragments_match_direct_product(d):
    rng = np.random.default_rng(2)
    codes = rng.integers(-8, 8, size=(16, d))
    rows = rows_as_bytes(codes)
    p = rng.random((4, 16))
    O = np.zeros((d, 8))
    for mt in range(d // 16):
        A = np.zeros((16, 16))
        B = np.zeros((16, 8))
        sel = (mt & 3) | ((4 + (mt & 3)) << 8)
        for lane in range(32):
            g, c = lane >> 2, lane & 3
            wa, wb, wc, wd = (word(rows, t, (d // 16) * g + 4 * (mt >> 2))
                              for t in (2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9))
            x01, x89 = byte_perm(wa, wb, sel), byte_perm(wc, wd, sel)
            A[g, 2 * c:2 * c + 2] = lo_pair(x01)
            A[g + 8, 2 * c:2 * c + 2] = hi_pair(x01)
            A[g, 2 * c + 8:2 * c + 10] = lo_pair(x89)
            A[g + 8, 2 * c + 8:2 * c + 10] = hi_pair(x89)
            for row in (2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9):
                B[row, g] = p[g >> 1, row] if g % 2 == 0 else 0.0
        Ot = A @ B
        for g in range(8):
            O[2 * ((d // 16) * g + mt)] += Ot[g]
            O[2 * ((d // 16) * g + mt) + 1] += Ot[g + 8]
    got = np.stack([O[:, 2 * k] + O[:, 2 * k + 1] for k in range(4)], 0)
    np.testing.assert_allclose(got, p @ codes, rtol=0, atol=1e-9)


def test_bf16_nibble_codes_exact():
    import struct

    def bf16(bits):
        return struct.unpack("<f", struct.pack("<I", (bits & 0xFFFF) << 16))[0]

    for n in range(16):
        v = bf16((n ^ 0x4308) & 0xFFFF)  # (x & 0xF) ^ 0x4308 for x = n
        assert v == 136 + nib_code(n)
        assert v * 1.0 - 136.0 == nib_code(n)
