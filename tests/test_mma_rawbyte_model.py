"""CPU model of the 2-bit decode's raw-byte tensor-core operands (no GPU).

A 2-bit code word holds four codes per byte (bits 0, 2, 4, 6).  Instead of splitting a byte into its
four codes (a shift and four masks per word), the kernel feeds mma.sync m16n8k32 the word itself and
three masked copies of it, whose bytes are

    V0 = c0 + 4 c1 + 16 c2 + 64 c3,   V1 = 4 c1 + 16 c2 + 64 c3,   V2 = 16 c2 + 64 c3,   V3 = 64 c3,

against the operand values X0 = 64 Q0, X1 = 16 Q1 - 64 Q0, X2 = 4 Q2 - 16 Q1, X3 = Q3 - 4 Q2 of the
byte's four elements (Q = fixed-point q * s on the K side, p * s on the V side).  Then
V0 X0 + V1 X1 + V2 X2 + V3 X3 = 64 (c0 Q0 + c1 Q1 + c2 Q2 + c3 Q3) exactly.  Each X (|X| < 2^30) is
stored as four balanced signed byte digits (the bytes of X + 0x80808080, each minus 128), one B
column per digit, and a 4 x 4 byte transpose puts the digits of four byte positions into one word.

This module restates the kernel's index maps (which token each A row carries, which lane builds which
operand word, the transpose, the digit slots, the zero operand of the other tile, the exchange that
combines the digit columns), runs them through a model of the PTX m16n8k32 fragment layout and checks
every output against the plain integer dot product, for one query per KV head and for several.
"""
import numpy as np
import pytest

RNG = np.random.default_rng(77)
M32 = 0xFFFFFFFF


def variants(w):
    w = int(w) & M32
    return [w, w & 0xFCFCFCFC, w & 0xF0F0F0F0, w & 0xC0C0C0C0]


def x_of(k, q, q_prev):
    """Operand value of variant k of a byte from its element's Q and the previous element's."""
    return (64 >> (2 * k)) * q - ((256 >> (2 * k)) * q_prev if k else 0)


def prmt(a, b, sel):
    """PTX prmt.b32 (default mode): byte i of the result is byte (sel >> 4 i) & 7 of {b, a}."""
    src = (int(a) & M32) | ((int(b) & M32) << 32)
    return sum(((src >> (8 * ((sel >> (4 * i)) & 7))) & 255) << (8 * i) for i in range(4))


def transpose4(u):
    """The kernel's 4 x 4 byte transpose: word d holds byte d of u[0..3] (u[m] at byte m)."""
    t0, t1 = prmt(u[0], u[1], 0x5140), prmt(u[0], u[1], 0x7362)
    t2, t3 = prmt(u[2], u[3], 0x5140), prmt(u[2], u[3], 0x7362)
    return [prmt(t0, t2, 0x5410), prmt(t0, t2, 0x7632), prmt(t1, t3, 0x5410), prmt(t1, t3, 0x7632)]


def digit_words(xs):
    """Balanced signed digits of four operand values: word d holds digit d of xs[m] in byte m."""
    assert all(-(2 ** 30) <= x < 2 ** 30 for x in xs)
    u = [(x + 0x80808080) & M32 for x in xs]
    return [w ^ 0x80808080 for w in transpose4(u)]


def bytes_of(x, signed):
    b = [(int(x) >> (8 * i)) & 255 for i in range(4)]
    return [v - 256 if signed and v >= 128 else v for v in b]


def mma(a_regs, b_regs, acc, b_signed):
    """D += A B for one warp: a_regs[l] = (a0..a3), b_regs[l] = (b0, b1), acc[l] = [d0..d3]."""
    A = np.zeros((16, 32), np.int64)
    B = np.zeros((32, 8), np.int64)
    for l in range(32):
        g, t = l >> 2, l & 3
        a = [bytes_of(r, False) for r in a_regs[l]]
        b = [bytes_of(r, b_signed) for r in b_regs[l]]
        for i in range(4):
            A[g, 4 * t + i], A[g + 8, 4 * t + i] = a[0][i], a[1][i]
            A[g, 16 + 4 * t + i], A[g + 8, 16 + 4 * t + i] = a[2][i], a[3][i]
            B[4 * t + i, g], B[16 + 4 * t + i, g] = b[0][i], b[1][i]
    D = A @ B
    for l in range(32):
        g, t = l >> 2, l & 3
        acc[l][0] += D[g, 2 * t]
        acc[l][1] += D[g, 2 * t + 1]
        acc[l][2] += D[g + 8, 2 * t]
        acc[l][3] += D[g + 8, 2 * t + 1]
        for v in acc[l]:
            assert -(2 ** 31) <= v < 2 ** 31, "int32 accumulator"


def gather4(acc):
    """Digit columns (3, 2) sit in even lanes, (1, 0) in odd lanes; each lane forms c0 * 256 + c1
    for its two rows, scales by 2^16 if even, and one exchange with lane ^ 1 leaves row g in the even
    lane and row g + 8 in the odd lane."""
    part = []
    for l in range(32):
        c = acc[l]
        sc = 1 if l & 1 else 65536
        for v in (c[0] * 256 + c[1], c[2] * 256 + c[3]):
            assert -(2 ** 31) <= v < 2 ** 31
        part.append(((c[0] * 256 + c[1]) * sc, (c[2] * 256 + c[3]) * sc))
    out = []
    for l in range(32):
        odd = l & 1
        keep = part[l][1] if odd else part[l][0]
        recv = part[l ^ 1][0] if (l ^ 1) & 1 else part[l ^ 1][1]
        out.append(keep + recv)
    return out


def word_index(row, slot, var):
    """Operand word (row, digit slot, variant) of the shared-memory layout; slot s holds digit 3 - s."""
    return 16 * row + 4 * (slot ^ ((row >> 1) & 3)) + var


def uint4(words, idx):
    return [int(words[4 * idx + e]) for e in range(4)]


ZERO4 = [0, 0, 0, 0]


def k_words(codes):  # token-major, 16 channels per word
    return [sum(int(codes[T, 16 * w + j]) << (2 * j) for j in range(16)) for T in range(128) for w in range(8)]


def v_words(codes):  # word (row r, channel c) holds tokens 16 r .. 16 r + 15
    return [sum(int(codes[16 * r + j, c]) << (2 * j) for j in range(16)) for r in range(8) for c in range(128)]


def q_operands(Q):
    """build_q: lane (i, k) forms variant k of K word i for bytes m = 0..3 (channels 16 i + 4 m + k);
    the previous channel's Q comes from lane - 1 (k - 1, same word)."""
    words = np.zeros(128, np.int64)
    for lane in range(32):
        i, k = lane >> 2, lane & 3
        xs = [x_of(k, int(Q[16 * i + 4 * m + k]), int(Q[16 * i + 4 * m + k - 1]) if k else 0) for m in range(4)]
        for d, wd in enumerate(digit_words(xs)):
            words[word_index(i, 3 - d, k)] = wd
    return words


def mha_token(g, t, j):
    """Token whose logit lane (g, t) holds for tile pair j (one query per KV head)."""
    return 16 * ((g >> 2) + 2 * (t & 1) + 4 * (t >> 1)) + 4 * j + (g & 3)


def p_operands_mha(P):
    """softmax: lane (g, t) holds tokens 16 r + 4 m + v (m = tile pair) with r = g / 4 + 2 (t % 2) +
    4 (t / 2), v = g % 4; the previous token's P comes from lane - 4."""
    words = np.zeros(128, np.int64)
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        r, v = (g >> 2) + 2 * (t & 1) + 4 * (t >> 1), g & 3
        assert all(mha_token(g, t, m) == 16 * r + 4 * m + v for m in range(4))
        prev_lane = lane - 4
        if v:
            pg, pt = prev_lane >> 2, prev_lane & 3
            assert all(mha_token(pg, pt, m) == 16 * r + 4 * m + v - 1 for m in range(4))
        xs = [x_of(v, int(P[16 * r + 4 * m + v]), int(P[16 * r + 4 * m + v - 1]) if v else 0) for m in range(4)]
        for d, wd in enumerate(digit_words(xs)):
            words[word_index(r, 3 - d, v)] = wd
    return words


def test_transpose_and_digits():
    for _ in range(200):
        xs = [int(x) for x in RNG.integers(-(2 ** 30), 2 ** 30, 4)]
        w = digit_words(xs)
        for m in range(4):
            digits = [bytes_of(w[d], True)[m] for d in range(4)]
            assert sum(dg * 256 ** d for d, dg in enumerate(digits)) == xs[m]


def test_variant_identity():
    for _ in range(500):
        c = RNG.integers(0, 4, 4)
        q = [int(x) for x in RNG.integers(-(2 ** 23), 2 ** 23, 4)]
        w = int(c[0] + 4 * c[1] + 16 * c[2] + 64 * c[3])
        vs = [bytes_of(x, False)[0] for x in variants(w)]
        xs = [x_of(k, q[k], q[k - 1] if k else 0) for k in range(4)]
        assert sum(a * b for a, b in zip(vs, xs)) == 64 * sum(int(ci) * qi for ci, qi in zip(c, q))


def test_one_query_k_tiles():
    codes = RNG.integers(0, 4, (128, 128))
    codes[:5] = 3
    Q = RNG.integers(-(2 ** 23), 2 ** 23 + 1, 128)
    Q[:8] = 2 ** 23   # the largest operand values
    kt, qw = k_words(codes), q_operands(Q)
    got = {}
    for j in range(4):
        acc = [[0] * 4 for _ in range(32)]
        for b in range(2):
            for x in range(2):
                for sp in range(2):
                    a_regs, b_regs = [], []
                    for lane in range(32):
                        g, t = lane >> 2, lane & 3
                        own = (g < 4) if b == 0 else (g >= 4)
                        B = uint4(qw, 8 * t + 4 * x + ((g & 3) ^ t)) if own else ZERO4
                        tg = 16 * ((g >> 2) + 4 * b) + 4 * j + (g & 3)
                        vg, vh = variants(kt[tg * 8 + 2 * t + x]), variants(kt[(tg + 32) * 8 + 2 * t + x])
                        a_regs.append((vg[2 * sp], vh[2 * sp], vg[2 * sp + 1], vh[2 * sp + 1]))
                        b_regs.append((B[2 * sp], B[2 * sp + 1]))
                    mma(a_regs, b_regs, acc, True)
        for lane, val in enumerate(gather4(acc)):
            got[mha_token(lane >> 2, lane & 3, j)] = val
    want = codes @ Q.astype(np.int64) * 64
    assert sorted(got) == list(range(128)) and all(got[T] == want[T] for T in range(128))


def test_one_query_v_tiles():
    codes = RNG.integers(0, 4, (128, 128))
    P = RNG.integers(0, 2 ** 24 - 127, 128)
    P[:16] = 2 ** 24 - 128
    vt, pw = v_words(codes), p_operands_mha(P)
    out = {}
    for v in range(4):
        acc = [[0] * 4 for _ in range(32)]
        for x in range(2):
            for b in range(2):
                for sp in range(2):
                    a_regs, b_regs = [], []
                    for lane in range(32):
                        g, t = lane >> 2, lane & 3
                        own = (g < 4) if b == 0 else (g >= 4)
                        B = uint4(pw, 8 * t + 4 * x + ((g & 3) ^ t)) if own else ZERO4
                        row = 2 * t + x
                        vg = variants(vt[row * 128 + 16 * g + 8 * b + v])        # channel 16 g + 8 b + v: row g
                        vh = variants(vt[row * 128 + 16 * g + 8 * b + 4 + v])    # + 4: row g + 8
                        a_regs.append((vg[2 * sp], vh[2 * sp], vg[2 * sp + 1], vh[2 * sp + 1]))
                        b_regs.append((B[2 * sp], B[2 * sp + 1]))
                    mma(a_regs, b_regs, acc, True)
        for lane, val in enumerate(gather4(acc)):
            out[4 * lane + v] = val
    want = P.astype(np.int64) @ codes * 64
    assert all(out[c] == want[c] for c in range(128))


def gqa_token(g, t, tau):
    """Token whose logit lane (g, t) holds in tile tau (several queries per KV head)."""
    return 16 * ((g >> 2) + 2 * (t & 1) + 4 * (tau >> 2)) + 4 * (tau & 3) + (g & 3)


def p_operands_gqa(P, q):
    """softmax (several queries): lanes with t / 2 == q % 2 hold query q's tokens 16 (r0 + 4 h) + 4 m + v
    (tile tau = 4 h + m), r0 = g / 4 + 2 (t % 2), v = g % 4; the previous token's P is in lane - 4."""
    words = np.zeros(128, np.int64)
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        if (t >> 1) != q % 2:
            continue
        r0, v = (g >> 2) + 2 * (t & 1), g & 3
        for h in range(2):
            r = r0 + 4 * h
            assert all(gqa_token(g, t, 4 * h + m) == 16 * r + 4 * m + v for m in range(4))
            xs = [x_of(v, int(P[16 * r + 4 * m + v]), int(P[16 * r + 4 * m + v - 1]) if v else 0) for m in range(4)]
            for d, wd in enumerate(digit_words(xs)):
                words[word_index(r, 3 - d, v)] = wd
    return words


@pytest.mark.parametrize("G", [2, 4, 8])
def test_several_queries_k_tiles(G):
    nb = G // 2
    codes = RNG.integers(0, 4, (128, 128))
    Q = RNG.integers(-(2 ** 23), 2 ** 23 + 1, (G, 128))
    kt = k_words(codes)
    qw = [q_operands(Q[q]) for q in range(G)]
    want = codes @ Q.T.astype(np.int64) * 64      # [token][query]
    seen = set()
    for tau in range(8):
        acc = [[[0] * 4 for _ in range(32)] for _ in range(nb)]
        for x in range(2):
            for sp in range(2):
                for p in range(nb):
                    a_regs, b_regs = [], []
                    for lane in range(32):
                        g, t = lane >> 2, lane & 3
                        B = uint4(qw[2 * p + (g >> 2)], 8 * t + 4 * x + ((g & 3) ^ t))
                        tg = 16 * ((g >> 2) + 4 * (tau >> 2)) + 4 * (tau & 3) + (g & 3)
                        vg, vh = variants(kt[tg * 8 + 2 * t + x]), variants(kt[(tg + 32) * 8 + 2 * t + x])
                        a_regs.append((vg[2 * sp], vh[2 * sp], vg[2 * sp + 1], vh[2 * sp + 1]))
                        b_regs.append((B[2 * sp], B[2 * sp + 1]))
                    mma(a_regs, b_regs, acc[p], True)
        for p in range(nb):
            for lane, val in enumerate(gather4(acc[p])):
                g, t = lane >> 2, lane & 3
                T, q = gqa_token(g, t, tau), 2 * p + (t >> 1)
                assert val == want[T, q]
                seen.add((T, q))
    assert len(seen) == 128 * G


@pytest.mark.parametrize("G", [2, 4, 8])
def test_several_queries_v_tiles(G):
    nb = G // 2
    codes = RNG.integers(0, 4, (128, 128))
    P = RNG.integers(0, 2 ** 24 - 127, (G, 128))
    vt = v_words(codes)
    pw = [p_operands_gqa(P[q], q) for q in range(G)]
    o = [[[None] * 4 for _ in range(G)] for _ in range(32)]
    for b in range(2):
        acc = [[[[0] * 4 for _ in range(32)] for _ in range(nb)] for _ in range(4)]
        for x in range(2):
            for v in range(4):
                for sp in range(2):
                    for p in range(nb):
                        a_regs, b_regs = [], []
                        for lane in range(32):
                            g, t = lane >> 2, lane & 3
                            B = uint4(pw[2 * p + (g >> 2)], 8 * t + 4 * x + ((g & 3) ^ t))
                            row = 2 * t + x
                            vg = variants(vt[row * 128 + 16 * g + 8 * b + v])
                            vh = variants(vt[row * 128 + 16 * g + 8 * b + 4 + v])
                            a_regs.append((vg[2 * sp], vh[2 * sp], vg[2 * sp + 1], vh[2 * sp + 1]))
                            b_regs.append((B[2 * sp], B[2 * sp + 1]))
                        mma(a_regs, b_regs, acc[v][p], True)
        for v in range(4):
            for p in range(nb):
                for lane, val in enumerate(gather4(acc[v][p])):
                    o[lane][2 * p + b][v] = val
    want = P.astype(np.int64) @ codes * 64
    for lane in range(32):   # tensor-core layout: query 2 p + t / 2, channel 16 g + 8 b + 4 (t % 2) + v
        g, t = lane >> 2, lane & 3
        for p in range(nb):
            for b in range(2):
                for v in range(4):
                    assert o[lane][2 * p + b][v] == want[2 * p + (t >> 1), 16 * g + 8 * b + 4 * (t & 1) + v]
