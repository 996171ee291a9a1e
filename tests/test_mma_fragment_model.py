"""CPU model of the decode kernel's tensor-core fragment maps (no GPU).

The 2-bit decode feeds mma.sync m16n8k32 tiles from registers: code words are unpacked by one shift
and four masks (sets 1 and 3 read 4 * code), B holds byte limbs of the fixed-point q * s or p * s in
a swizzled shared-memory layout, two tiles (or two queries) share one accumulator through B columns
0..2 and 4..6, and one exchange with the partner lane combines the three limbs.  This module restates
those index maps, runs them through a model of the PTX m16n8k32 fragment layout (A rows g, g + 8 and
columns 4 t .. 4 t + 3, 16 + 4 t ..; B column g; D rows g, g + 8 and columns 2 t, 2 t + 1 for lane
(g, t) = (lane / 4, lane % 4)), and checks that every output equals the plain integer dot product:
one query per KV head (K and V), several queries per KV head (K, V and the layout swap), and the
fine-grained V tiles.  The GPU parity tests check the kernel itself against the oracle.
"""
import numpy as np
import pytest

RNG = np.random.default_rng(2024)


def masks2(w):
    w4 = w >> 4
    return [w & 0x03030303, w & 0x0C0C0C0C, w4 & 0x03030303, w4 & 0x0C0C0C0C]


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


def gather(acc):
    """The limb exchange: lane t % 2 == 0 ends with row g, odd lanes with row g + 8."""
    out = []
    for l in range(32):
        odd, p = l & 1, acc[l ^ 1]
        r1 = p[0] if (l ^ 1) & 1 else p[2]
        hi, mid, lo = (r1, p[3], acc[l][2]) if odd else (acc[l][0], acc[l][1], r1)
        out.append(hi * 65536 + mid * 256 + lo)
    return out


def pick(xs, b):
    return sum(((int(x) & 0xFFFFFFFF) >> (8 * b) & 255) << (8 * m) for m, x in enumerate(xs))


def k_limb_rows(Q):
    """Shared-memory Q limb words: (word i, slot, set) at 16 i + 4 (slot ^ (i / 2 % 4)) + set, balanced
    signed digits (bytes of Q + 32896, Q + 128, Q); slot 3 stays zero."""
    qw = np.zeros(128, np.uint64)
    for lane in range(32):
        i, k = lane >> 2, lane & 3
        sw = (i >> 1) & 3
        qs = [int(Q[16 * i + 4 * m + k]) for m in range(4)]
        qw[16 * i + 4 * (0 ^ sw) + k] = pick([q + 32896 for q in qs], 2)
        qw[16 * i + 4 * (1 ^ sw) + k] = pick([q + 128 for q in qs], 1)
        qw[16 * i + 4 * (2 ^ sw) + k] = pick(qs, 0)
    return qw


def p_limb_rows(P, rows_of_lane):
    """Shared-memory P limb bytes: token T goes to byte (T / 4) % 4 of word (T / 16, slot, T % 4)."""
    b = bytearray(512)
    for lane in range(32):
        for T in rows_of_lane(lane):
            r, st, m = T >> 4, T & 3, (T >> 2) & 3
            for slot, sh in ((0, 16), (1, 8), (2, 0)):
                b[64 * r + 16 * (slot ^ ((r >> 1) & 3)) + 4 * st + m] = (int(P[T]) >> sh) & 255
    return np.frombuffer(bytes(b), np.uint32).astype(np.uint64)


def uint4(rows, idx):
    return [int(rows[4 * idx + e]) for e in range(4)]


def k_words(codes):  # token-major, 16 channels per word
    return [sum(int(codes[T, 16 * w + j]) << (2 * j) for j in range(16)) for T in range(128) for w in range(8)]


def v_words(codes):  # word (row r, channel c) holds tokens 16 r .. 16 r + 15
    return [sum(int(codes[16 * r + j, c]) << (2 * j) for j in range(16)) for r in range(8) for c in range(128)]


def weights(x):  # sets 1 and 3 read 4 * code, so their limbs carry 1/4: effective weight 4 x
    return np.array([int(v) * (4 if (i & 3) & 1 else 1) for i, v in enumerate(x)])


def test_one_query_k_tiles():
    codes = RNG.integers(0, 4, (128, 128))
    Q = RNG.integers(-(2 ** 23 - 2 ** 16), 2 ** 23 - 2 ** 16, 128)
    kt, qw = k_words(codes), k_limb_rows(Q)
    got = {}
    for j in range(4):
        acc = [[0] * 4 for _ in range(32)]
        for b in range(2):
            for w in range(2):
                for sp in range(2):
                    a_regs, b_regs = [], []
                    for lane in range(32):
                        g, t = lane >> 2, lane & 3
                        slot = (g - 4 if g >= 4 else 3) if b else (g if g < 4 else 3)
                        B = uint4(qw, 8 * t + 4 * w + (slot ^ t))
                        mg = masks2(kt[(32 * j + 16 * b + g) * 8 + 2 * t + w])
                        mh = masks2(kt[(32 * j + 16 * b + g + 8) * 8 + 2 * t + w])
                        a_regs.append((mg[2 * sp], mh[2 * sp], mg[2 * sp + 1], mh[2 * sp + 1]))
                        b_regs.append((B[2 * sp], B[2 * sp + 1]))
                    mma(a_regs, b_regs, acc, True)
        for lane, val in enumerate(gather(acc)):
            g, t = lane >> 2, lane & 3
            got[32 * j + 16 * (t >> 1) + 8 * (t & 1) + g] = val
    want = codes @ weights(Q)
    assert sorted(got) == list(range(128)) and all(got[T] == want[T] for T in range(128))


def test_one_query_v_tiles():
    codes = RNG.integers(0, 4, (128, 128))
    P = RNG.integers(0, 2 ** 24 - 128, 128)
    vt = v_words(codes)
    pw = p_limb_rows(P, lambda l: [32 * j + 16 * ((l & 3) >> 1) + 8 * (l & 1) + (l >> 2) for j in range(4)])
    out = {}
    for v in range(4):
        acc = [[0] * 4 for _ in range(32)]
        for x in range(2):
            for b in range(2):
                for sp in range(2):
                    a_regs, b_regs = [], []
                    for lane in range(32):
                        g, t = lane >> 2, lane & 3
                        slot = (g - 4 if g >= 4 else 3) if b else (g if g < 4 else 3)
                        B = uint4(pw, 8 * t + 4 * x + (slot ^ t))
                        row = 2 * t + x
                        mg = masks2(vt[row * 128 + 16 * g + 8 * b + v])       # channel 16 g + 8 b + v: row g
                        mh = masks2(vt[row * 128 + 16 * g + 8 * b + 4 + v])   # + 4: row g + 8
                        a_regs.append((mg[2 * sp], mh[2 * sp], mg[2 * sp + 1], mh[2 * sp + 1]))
                        b_regs.append((B[2 * sp], B[2 * sp + 1]))
                    mma(a_regs, b_regs, acc, False)
        for lane, val in enumerate(gather(acc)):
            out[4 * lane + v] = val
    want = weights(P) @ codes
    assert all(out[c] == want[c] for c in range(128))


@pytest.mark.parametrize("G", [2, 4])
def test_several_queries_v_tiles_and_layout_swap(G):
    nb = G // 2
    codes = RNG.integers(0, 4, (128, 128))
    P = RNG.integers(0, 2 ** 24 - 128, (G, 128))
    vt = v_words(codes)
    pw = []
    for q in range(G):   # lane (g, t) writes query 2 p + t / 2, tokens 16 tau + 8 (t % 2) + g
        pw.append(p_limb_rows(P[q], lambda l, q=q: [16 * tau + 8 * (l & 1) + (l >> 2) for tau in range(8)
                                                    if ((l & 3) >> 1) == q % 2]))
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
                            mg = masks2(vt[row * 128 + 16 * g + 8 * b + v])
                            mh = masks2(vt[row * 128 + 16 * g + 8 * b + 4 + v])
                            a_regs.append((mg[2 * sp], mh[2 * sp], mg[2 * sp + 1], mh[2 * sp + 1]))
                            b_regs.append((B[2 * sp], B[2 * sp + 1]))
                        mma(a_regs, b_regs, acc[v][p], False)
        for v in range(4):
            for p in range(nb):
                for lane, val in enumerate(gather(acc[v][p])):
                    o[lane][2 * p + b][v] = val
    want = np.stack([weights(P[q]) @ codes for q in range(G)])
    for lane in range(32):   # tensor-core layout: query 2 p + t / 2, channel 16 g + 8 b + 4 (t % 2) + v
        g, t = lane >> 2, lane & 3
        for p in range(nb):
            for b in range(2):
                for v in range(4):
                    assert o[lane][2 * p + b][v] == want[2 * p + (t >> 1), 16 * g + 8 * b + 4 * (t & 1) + v]
    swapped = [[row[:] for row in o[lane]] for lane in range(32)]
    for lane in range(32):   # exchange o[2 p + 1 - t / 2][v] with lane t ^ 2
        h, ph = (lane >> 1) & 1, ((lane ^ 2) >> 1) & 1
        for p in range(nb):
            for v in range(4):
                swapped[lane][2 * p + (1 - h)][v] = o[lane ^ 2][2 * p + (1 - ph)][v]
    for lane in range(32):   # residual layout: query q, channel 4 lane + e
        for q in range(G):
            for e in range(4):
                assert swapped[lane][q][e] == want[q, 4 * lane + e]


@pytest.mark.parametrize("gv", [32, 64, 128])
def test_fine_grained_v_tiles(gv):
    ngv = 128 // gv
    codes = RNG.integers(0, 4, (128, 128))
    P = RNG.integers(0, 2 ** 24 - 128, (ngv, 128))
    vt = v_words(codes)
    lanes_tokens = lambda l: [32 * j + 16 * ((l & 3) >> 1) + 8 * (l & 1) + (l >> 2) for j in range(4)]
    pw = [p_limb_rows(P[gc], lanes_tokens) for gc in range(ngv)]
    out = {}
    for v in range(4):
        gc = 32 * v // gv
        acc = [[0] * 4 for _ in range(32)]
        for x in range(2):
            for b in range(2):
                for sp in range(2):
                    a_regs, b_regs = [], []
                    for lane in range(32):
                        g, t = lane >> 2, lane & 3
                        slot = (g - 4 if g >= 4 else 3) if b else (g if g < 4 else 3)
                        B = uint4(pw[gc], 8 * t + 4 * x + (slot ^ t))
                        ch = 32 * v + 16 * b + 2 * g   # tile (v, b): row g on ch, row g + 8 on ch + 1
                        row = 2 * t + x
                        mg, mh = masks2(vt[row * 128 + ch]), masks2(vt[row * 128 + ch + 1])
                        a_regs.append((mg[2 * sp], mh[2 * sp], mg[2 * sp + 1], mh[2 * sp + 1]))
                        b_regs.append((B[2 * sp], B[2 * sp + 1]))
                    mma(a_regs, b_regs, acc, False)
        for lane, val in enumerate(gather(acc)):
            g, t = lane >> 2, lane & 3
            out[32 * v + 16 * (t >> 1) + 2 * g + (t & 1)] = val
    want = [int(weights(P[c // gv]) @ codes[:, c]) for c in range(128)]
    assert sorted(out) == list(range(128)) and all(out[c] == want[c] for c in range(128))
