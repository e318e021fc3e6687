"""Host-side model of the tensor-core attention kernel's operand layout
(no GPU): the coordinate permutation, nibble-to-code conversions and
fragment assignment of kvq_attn_tc_kernel, written against the fragment
layouts of the PTX ISA (lane = 4 g + c): the scores as m16n8k32 u8 x s8
products of offset codes and fixed-point query slices, the accumulation as
m16n8k16 bf16 products (A rows g, g + 8 and columns 2c, 2c + 1, 2c + 8,
2c + 9; B rows 2c, 2c + 1, 2c + 8, 2c + 9 of column g).  Both must
reproduce the direct products K q and p V of one 16-token chunk."""
import numpy as np
import pytest


def nib_code(n):
    return (n ^ 8) - 8


def lo_pair(x):  # codes of the low nibbles of bytes 0 and 2
    return nib_code(x & 0xF), nib_code((x >> 16) & 0xF)


def hi_pair(x):  # the high nibbles (the kernel shifts x down by 4 first)
    return lo_pair(x >> 4)


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


def u_bytes(x):  # (x & 0x0F0F0F0F) ^ 0x08080808: the offset codes q + 8 of the low nibbles
    return [((x >> (8 * i)) & 0xF) ^ 8 for i in range(4)]


def p2(n):
    return float(np.ldexp(np.float32(1.0), n))


def query_slices(y):
    """The kernel's fixed-point split of one pre-scaled fp32 query: exponent
    k with max |y| < 2^k, then four signed 7-bit slices B_j (|B_j| <= 64)
    with y ~ 2^(k-6) (B_0 + B_1 2^-7 + B_2 2^-14 + B_3 2^-21), every step
    exact in fp32."""
    y = np.asarray(y, dtype=np.float32)
    amax = np.float32(np.abs(y).max())
    e = int((amax.view(np.uint32) >> 23) & 0xFF)
    k = min(max(e - 126, -90), 120)
    t = y * np.float32(p2(6 - k))
    B = []
    for j in range(4):
        b = np.rint(t).astype(np.float32)
        B.append(b.astype(np.int64))
        t = ((t - b) * np.float32(128.0)).astype(np.float32)
    return k, np.stack(B)


@pytest.mark.parametrize("scale", [1.0, 1e-3, 37.0, 1e-30, 0.0])
def test_query_slices_error_bound(scale):
    rng = np.random.default_rng(5)
    y = (rng.standard_normal(256) * scale).astype(np.float32)
    y[3] *= 40
    k, B = query_slices(y)
    assert np.abs(B).max() <= 64
    amax = float(np.abs(y).max())
    assert amax < p2(k) or amax == 0.0
    rec = sum(B[j].astype(np.float64) * p2(k - 6 - 7 * j) for j in range(4))
    # |error| <= 2^(k-28) <= 2^-27 max|y| (amax >= 2^(k-1) unless k was clamped)
    assert np.all(np.abs(rec - y.astype(np.float64)) <= p2(k - 28))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_score_fragments_match_direct_product(d):
    """m16n8k32 u8 x s8 -> s32 (A rows g, g + 8 and columns 4c .. 4c + 3,
    16 + 4c .. 16 + 4c + 3; B rows 4c .., 16 + 4c .. of column g): A holds the
    offset codes of the low and high nibbles of one 32-bit word of tokens g
    and g + 8, B the query slices of the same coordinates, column n = query
    n / 2, slice n % 2 (first product) or 2 + n % 2 (second); the
    accumulator starts at -8 sum_i B_j[i]."""
    rng = np.random.default_rng(1)
    codes = rng.integers(-8, 8, size=(16, d))
    rows = rows_as_bytes(codes)
    q = rng.standard_normal((4, d)).astype(np.float32)
    q[1] *= 1e-3
    ks, Bs = zip(*(query_slices(q[i]) for i in range(4)))
    even = [B[:, 0::2] for B in Bs]  # slices of coordinates 2m
    odd = [B[:, 1::2] for B in Bs]   # ... and 2m + 1
    acc = []
    for half in range(2):  # slices (0, 1) and (2, 3)
        C = np.zeros((16, 8), dtype=np.int64)
        for n in range(8):
            C[:, n] = -8 * Bs[n >> 1][2 * half + (n & 1)].sum()
        for s in range(d // 32):
            A = np.zeros((16, 32), dtype=np.int64)
            B = np.zeros((32, 8), dtype=np.int64)
            for lane in range(32):
                g, c = lane >> 2, lane & 3
                m0 = (d // 8) * c + 4 * s
                w0, w8 = word(rows, g, m0), word(rows, g + 8, m0)
                A[g, 4 * c:4 * c + 4] = u_bytes(w0)
                A[g + 8, 4 * c:4 * c + 4] = u_bytes(w8)
                A[g, 16 + 4 * c:20 + 4 * c] = u_bytes(w0 >> 4)
                A[g + 8, 16 + 4 * c:20 + 4 * c] = u_bytes(w8 >> 4)
                j = 2 * half + (g & 1)
                B[4 * c:4 * c + 4, g] = even[g >> 1][j, m0:m0 + 4]
                B[16 + 4 * c:20 + 4 * c, g] = odd[g >> 1][j, m0:m0 + 4]
            C = C + A @ B
        acc.append(C)
    for qi in range(4):
        for j in range(4):  # exact integer products of the signed codes
            np.testing.assert_array_equal(acc[j >> 1][:, 2 * qi + (j & 1)], codes @ Bs[qi][j])
        # the kernel's combination: two exact integer pairs, then fp32
        hi = (acc[0][:, 2 * qi] * 128 + acc[0][:, 2 * qi + 1]).astype(np.float32)
        lo = (acc[1][:, 2 * qi] * 128 + acc[1][:, 2 * qi + 1]).astype(np.float32)
        got = lo * np.float32(p2(ks[qi] - 27)) + hi * np.float32(p2(ks[qi] - 13))
        ref = codes @ q[qi].astype(np.float64)
        tol = 8 * d * p2(ks[qi] - 28) + 2.0 ** -22 * np.abs(codes) @ np.abs(q[qi].astype(np.float64))
        assert np.all(np.abs(got - ref) <= tol)


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
