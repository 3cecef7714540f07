"""CPU model of the decode projection kernel's operand layout (gemv_dec.cu):
the code pairs each lane extracts from its packed words (the lop3 / prmt /
HFMA2 bit tricks, emulated bit for bit on fp16 values), the k step and slot
each pair feeds, and the position the staging step writes each activation to.
Summing A x B over every lane, k step and slot of a chunk must give the plain
dot product of the codes with the activations, for INT4 and INT3 rows, for
every lane and chunk position (the INT3 groups may straddle a lane's codes).
The slot and position tables are read from the kernel source, so a change
there is checked here."""
import os
import re

import numpy as np
import pytest

from oracle import tinyloop_oracle as o

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = open(os.path.join(ROOT, "weight_shared_looped_b200", "csrc", "gemv_dec.cu")).read()


def _f16(bits):
    return np.array([bits & 0xFFFF], dtype=np.uint16).view(np.float16)[0]


def _halves(x):
    return float(_f16(x)), float(_f16(x >> 16))


def _hfma2(x, m, a):
    lo, hi = _halves(x)
    r = [np.float16(np.float64(v) * mm + aa) for v, mm, aa in ((lo, m[0], a[0]), (hi, m[1], a[1]))]
    return float(r[0]), float(r[1])


def _lop3_ea(a, b, c):
    return ((a & b) | c) & 0xFFFFFFFF


def _prmt(a, b, sel):
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    return sum(src[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))


def _const(pattern):
    m = re.search(pattern, SRC)
    assert m, pattern
    return m


# ---------------------------------------------------------------- the kernel's extraction steps
def int4_pairs(w):
    w8 = w >> 8
    lo = lambda x: _hfma2(_lop3_ea(x, 0x000F000F, 0x64006400), (1.0, 1.0), (-1032.0, -1032.0))
    hi = lambda x: _hfma2(_lop3_ea(x, 0x00F000F0, 0x64006400), (0.0625, 0.0625), (-72.0, -72.0))
    return [lo(w), hi(w), lo(w8), hi(w8)]


def int3_pair_i6(w, i):
    return _hfma2(_lop3_ea(w >> (3 * i), 0x001C0007, 0x64006400), (1.0, 0.25), (-1028.0, -260.0))


def int3_pair_c4(a, b):
    return _hfma2(_lop3_ea(_prmt(a, b, 0x0501), 0x00700070, 0x64006400), (0.0625, 0.0625),
                  (-68.0, -68.0))


def int3_pair_c5(a, b):
    return _hfma2(_lop3_ea(_prmt(a, b, 0x6521), 0x03800380, 0x64006400), (0.0078125, 0.0078125),
                  (-12.0, -12.0))


def test_extraction_constants_match_the_kernel():
    for c in ("0x001C0007u, 0x64006400u", "h2c(1.f, 0.25f), h2c(-1028.f, -260.f)",
              "prmt(a, b, 0x0501u), 0x00700070u", "h2c(-68.f, -68.f)",
              "prmt(a, b, 0x6521u), 0x03800380u", "h2c(-12.f, -12.f)",
              "lop3_ea(w, 0x000F000Fu, 0x64006400u), one, lo_b",
              "lop3_ea(w, 0x00F000F0u, 0x64006400u), sixteenth, hi_b"):
        assert c in SRC, c


# ---------------------------------------------------------------- slot / position tables
def int3_slot(L, t):
    q, i = divmod(L, 10)
    return {0: (2 * q, 2 * t), 6: (2 * q, 2 * t + 1), 1: (2 * q, 2 * t + 8), 7: (2 * q, 2 * t + 9),
            2: (2 * q + 1, 2 * t), 8: (2 * q + 1, 2 * t + 1), 3: (2 * q + 1, 2 * t + 8),
            9: (2 * q + 1, 2 * t + 9), 4: (8 + (q >> 1), 2 * t + (q & 1)),
            5: (8 + (q >> 1), 2 * t + 8 + (q & 1))}[i]


def test_int3_slot_table_matches_the_kernel():
    for i, (j, s) in {0: ("2 * q", "2 * t"), 6: ("2 * q", "2 * t + 1"), 1: ("2 * q", "2 * t + 8"),
                      7: ("2 * q", "2 * t + 9"), 2: ("2 * q + 1", "2 * t"),
                      8: ("2 * q + 1", "2 * t + 1"), 3: ("2 * q + 1", "2 * t + 8"),
                      9: ("2 * q + 1", "2 * t + 9"), 4: ("8 + (q >> 1)", "2 * t + (q & 1)")}.items():
        assert f"case {i}: j = {j}; return {s};" in SRC, i


def xpos(k, bits):
    if bits == 4:
        c, r = divmod(k, 128)
        t, q, e = r >> 5, (r >> 3) & 3, k & 7
        j = 2 * q + ((e >> 1) & 1)
        s = 2 * t + (8 if e & 1 else 0) + (1 if e >= 4 else 0)
        return c * 128 + 16 * j + s
    c, r = divmod(k, 160)
    t, L = divmod(r, 40)
    j, s = int3_slot(L, t)
    return c * 160 + 16 * j + s


@pytest.mark.parametrize("bits,K", [(4, 256), (3, 480)])
def test_staging_positions_are_a_permutation(bits, K):
    pos = [xpos(k, bits) for k in range(K)]
    assert sorted(pos) == list(range(K))


def test_int4_staging_half2_stores_match_xpos():
    # the staging writes (e0,e4) at base, (e1,e5) at +8, (e2,e6) at +16, (e3,e7) at +24
    for k0 in range(0, 512, 8):
        base = xpos(k0, 4)
        for e, off in ((0, 0), (4, 1), (1, 8), (5, 9), (2, 16), (6, 17), (3, 24), (7, 25)):
            assert xpos(k0 + e, 4) == base + off


# ---------------------------------------------------------------- one chunk, all lanes
def _lane_fragments_int4(words):
    """words: the lane's 4 packed words of one row -> {k step: (pair (2t,2t+1), pair (2t+8,2t+9))}"""
    frags = {}
    for q in range(4):
        p = int4_pairs(int(words[q]))
        frags[2 * q] = (p[0], p[1])
        frags[2 * q + 1] = (p[2], p[3])
    return frags


def _lane_fragments_int3(words, scales_of_L):
    """Like the INT4 case; INT3 pairs are scaled in fp16 by their codes' group scales."""
    def sc(pair, La, Lb):
        return (float(np.float16(pair[0] * scales_of_L(La))), float(np.float16(pair[1] * scales_of_L(Lb))))
    frags = {}
    for q in range(4):
        w, L = int(words[q]), 10 * q
        frags[2 * q] = (sc(int3_pair_i6(w, 0), L, L + 6), sc(int3_pair_i6(w, 1), L + 1, L + 7))
        frags[2 * q + 1] = (sc(int3_pair_i6(w, 2), L + 2, L + 8), sc(int3_pair_i6(w, 3), L + 3, L + 9))
    w = [int(x) for x in words]
    frags[8] = (sc(int3_pair_c4(w[0], w[1]), 4, 14), sc(int3_pair_c5(w[0], w[1]), 5, 15))
    frags[9] = (sc(int3_pair_c4(w[2], w[3]), 24, 34), sc(int3_pair_c5(w[2], w[3]), 25, 35))
    return frags


def _mma_dot(frags_per_lane, xs_chunk, cw):
    """Sum over k steps and slots of A[slot] * B[slot], B read where ldmatrix reads it:
    k step j, slot s at position 16 j + s of the chunk's staged row."""
    total = 0.0
    for t, frags in enumerate(frags_per_lane):
        for j, (pa, pb) in frags.items():
            for slot, v in ((2 * t, pa[0]), (2 * t + 1, pa[1]), (2 * t + 8, pb[0]), (2 * t + 9, pb[1])):
                total += v * xs_chunk[16 * j + slot]
    return total


@pytest.mark.parametrize("seed", range(4))
def test_int4_chunk_dot_product(seed):
    rng = np.random.default_rng(seed)
    K = 256
    codes = rng.integers(-8, 8, size=(1, K)).astype(np.int8)
    codes[0, :8] = [-8, 7, -8, 7, 0, -1, 1, 3]
    words = o.pack_codes(codes, 4)[0]
    x = rng.standard_normal(K).astype(np.float16).astype(np.float64)
    xs = np.zeros(K)
    for k in range(K):
        xs[xpos(k, 4)] = x[k]
    for c in range(K // 128):
        frags = [_lane_fragments_int4(words[16 * c + 4 * t:16 * c + 4 * t + 4]) for t in range(4)]
        got = _mma_dot(frags, xs[128 * c:128 * c + 128], 128)
        want = float(codes[0, 128 * c:128 * c + 128].astype(np.float64) @ x[128 * c:128 * c + 128])
        assert abs(got - want) <= 1e-9 * max(1.0, abs(want)), (c, got, want)


@pytest.mark.parametrize("G", [64, 128])
@pytest.mark.parametrize("seed", range(3))
def test_int3_chunk_dot_product_with_straddling_groups(G, seed):
    rng = np.random.default_rng(100 + seed)
    K = 2048                                              # 205 words padded to 208: 13 chunks
    w = rng.standard_normal((1, K)).astype(np.float32) * 0.02
    codes, scales = o.quantize_groupwise(w, 3, G)
    words = o.pack_codes(codes, 3)[0]
    nvec = len(words) // 4
    nch = (nvec + 3) // 4
    x = np.zeros(nch * 160)
    x[:K] = rng.standard_normal(K).astype(np.float16).astype(np.float64)
    xs = np.zeros(nch * 160)
    for k in range(nch * 160):
        xs[xpos(k, 3)] = x[k]
    s = scales[0].astype(np.float64)
    gpr = K // G
    want_total = got_total = 0.0
    for c in range(nch):
        frags = []
        for t in range(4):
            vi = 4 * c + t
            lw = words[4 * vi:4 * vi + 4] if vi < nvec else np.zeros(4, np.uint32)
            k0 = 160 * c + 40 * t
            ga = min(k0 // G, gpr - 1)
            gb = min(ga + 1, gpr - 1)
            bnd = (k0 // G + 1) * G - k0
            frags.append(_lane_fragments_int3(lw, lambda L: s[ga] if L < bnd else s[gb]))
        got_total += _mma_dot(frags, xs[160 * c:160 * c + 160], 160)
    deq = np.array([float(np.float16(codes[0, k] * s[k // G])) for k in range(K)])
    want_total = float(deq @ x[:K])
    assert abs(got_total - want_total) <= 1e-9 * max(1.0, abs(want_total)), (got_total, want_total)


def test_int3_word_slots_match_the_slot_table():
    """The staging by packed word writes each of a word's ten codes where the
    per-element slot table puts it (read from the kernel source)."""
    src = SRC[SRC.index("void int3_word_slots("):]
    src = src[:src.index("\n}\n")]
    exprs = {}
    for i in range(10):
        m = re.search(r"pos\[%d\] = (.*);\s*// i = %d" % (i, i), src)
        assert m, i
        exprs[i] = m.group(1)
    for c in range(3):
        for t in range(4):
            for q in range(4):
                base = c * 160 + 2 * t
                j0, j1, j8 = 16 * (2 * q), 16 * (2 * q + 1), 16 * (8 + (q >> 1))
                for i in range(10):
                    got = eval(exprs[i].replace("(q & 1)", str(q & 1)),
                               {"base": base, "j0": j0, "j1": j1, "j8": j8})
                    assert got == xpos(c * 160 + 40 * t + 10 * q + i, 3), (c, t, q, i)


# ---------------------------------------------------------------- cross-iteration rounding
# The odd-iteration code is code + 1 where the sign-of-frac bit is set and
# code - 1 where it is clear (oracle.odd_iteration_codes).  The kernels add
# the fp16 pair pm1(x) (bits 15 and 31 of x -> +-1) to each exact code pair;
# the bit manipulations below are the kernels', read from their sources.
TC_SRC = open(os.path.join(ROOT, "weight_shared_looped_b200", "csrc", "gemm_tc.cu")).read()
M32 = 0xFFFFFFFF


def pm1(x):
    return (1.0 if (x >> 15) & 1 else -1.0, 1.0 if (x >> 31) & 1 else -1.0)


def int4_sign_fix(sw, q):
    h = sw if q < 2 else sw >> 16
    P = ((h & 0x0F0F) | ((h & 0xF0F0) << 12)) & M32
    base = 7 if q & 1 else 15
    return [pm1((P << (base - i)) & M32) for i in range(4)]


def int3_sign_S(sg_row, vi):
    wi, o = (5 * vi) >> 2, 8 * (vi & 3)
    a = int(sg_row[wi]) if wi < len(sg_row) else 0
    b = int(sg_row[wi + 1]) if wi + 1 < len(sg_row) else 0
    return ((b << 32) | a) >> o


def int3_sign_i6(S, q, I):
    w = (S >> (10 * q)) & 0x3FF
    return pm1(((w | (w << 10)) << (15 - I)) & M32)


def int3_sign_c(S, o, shift):
    u = (S >> o) & 0xC03
    return pm1(((u | (u << 6)) << shift) & M32)


def sign_spread(h16):
    return (h16 & 0x5555) | ((h16 & 0xAAAA) << 15)


def tc_sign_corr(gs, c):
    return pm1((gs[c >> 3] << (15 - 2 * (c & 7))) & M32)


def test_sign_constants_match_the_kernels():
    for c in ('"r"(0x80008000u), "r"(0xBC00BC00u)', "lop3.b32 %0, %1, %2, %3, 0x6A;",
              "const uint32_t P = (h & 0x0F0Fu) | ((h & 0xF0F0u) << 12);",
              "const int base = (q & 1) ? 7 : 15;", "pm1(P << (base - i))",
              "const uint32_t h = q < 2 ? sw : sw >> 16;",
              "return pm1((w | (w << 10)) << (15 - I));", "(uint32_t)(S >> (10 * q)) & 0x3FFu",
              "(uint32_t)(S >> o) & 0xC03u", "return pm1((u | (u << 6)) << 15);",
              "return pm1((u | (u << 6)) << 14);",
              "const int wi = (5 * vi) >> 2, o = 8 * (vi & 3);",
              "int3_sign_c4(S0, 4)", "int3_sign_c5(S0, 24)"):
        assert c in SRC, c
    for c in ("return (h16 & 0x5555u) | ((h16 & 0xAAAAu) << 15);",
              "pm1(gs[c >> 3] << (15 - 2 * (c & 7)))", "gs[1] = sign_spread(ws.sg.x >> 16);",
              "gs[2] = sign_spread(ws.sg.y & 0xFFFFu);"):
        assert c in TC_SRC, c


def test_tc_sign_pairs():
    """Pair c of a 64-code k block (codes 2c, 2c + 1) gets the bits 2c, 2c + 1."""
    rng = np.random.default_rng(5)
    for _ in range(50):
        x, y = (int(v) for v in rng.integers(0, 2**32, size=2, dtype=np.uint64))
        gs = [sign_spread(x & 0xFFFF), sign_spread(x >> 16), sign_spread(y & 0xFFFF),
              sign_spread(y >> 16)]
        bits = [((x | (y << 32)) >> k) & 1 for k in range(64)]
        for c in range(32):
            assert tc_sign_corr(gs, c) == (2.0 * bits[2 * c] - 1, 2.0 * bits[2 * c + 1] - 1), c


@pytest.mark.parametrize("seed", range(3))
def test_int4_chunk_dot_product_odd_iteration(seed):
    rng = np.random.default_rng(40 + seed)
    K = 256
    codes = rng.integers(-8, 8, size=(1, K)).astype(np.int8)
    bits = rng.integers(0, 2, size=(1, K)).astype(np.uint8)
    words = o.pack_codes(codes, 4)[0]
    sg = o.pack_bits(bits)[0]
    odd = o.odd_iteration_codes(codes, bits)[0].astype(np.float64)
    x = rng.standard_normal(K).astype(np.float16).astype(np.float64)
    xs = np.zeros(K)
    for k in range(K):
        xs[xpos(k, 4)] = x[k]
    for c in range(K // 128):
        frags = []
        for t in range(4):
            vi = 4 * c + t
            f = _lane_fragments_int4(words[4 * vi:4 * vi + 4])
            for q in range(4):
                corr = int4_sign_fix(int(sg[vi]), q)
                a, b = f[2 * q], f[2 * q + 1]
                f[2 * q] = ((a[0][0] + corr[0][0], a[0][1] + corr[0][1]),
                            (a[1][0] + corr[1][0], a[1][1] + corr[1][1]))
                f[2 * q + 1] = ((b[0][0] + corr[2][0], b[0][1] + corr[2][1]),
                                (b[1][0] + corr[3][0], b[1][1] + corr[3][1]))
            frags.append(f)
        got = _mma_dot(frags, xs[128 * c:128 * c + 128], 128)
        want = float(odd[128 * c:128 * c + 128] @ x[128 * c:128 * c + 128])
        assert abs(got - want) <= 1e-9 * max(1.0, abs(want)), (c, got, want)


@pytest.mark.parametrize("seed", range(2))
def test_int3_chunk_dot_product_odd_iteration(seed):
    rng = np.random.default_rng(60 + seed)
    K, G = 2048, 64
    w = rng.standard_normal((1, K)).astype(np.float32) * 0.02
    codes, scales = o.quantize_groupwise(w, 3, G)
    bits = o.sign_of_frac(w, G, 3)
    words = o.pack_codes(codes, 3)[0]
    sg = o.pack_bits(bits)[0]
    odd = o.odd_iteration_codes(codes, bits)[0]
    nvec = len(words) // 4
    nch = (nvec + 3) // 4
    x = np.zeros(nch * 160)
    x[:K] = rng.standard_normal(K).astype(np.float16).astype(np.float64)
    xs = np.zeros(nch * 160)
    for k in range(nch * 160):
        xs[xpos(k, 3)] = x[k]
    s = scales[0].astype(np.float64)
    gpr = K // G
    total = 0.0
    for c in range(nch):
        frags = []
        for t in range(4):
            vi = 4 * c + t
            lw = [int(v) for v in (words[4 * vi:4 * vi + 4] if vi < nvec else np.zeros(4, np.uint32))]
            S = int3_sign_S(sg, vi)
            k0 = 160 * c + 40 * t
            ga = min(k0 // G, gpr - 1)
            gb = min(ga + 1, gpr - 1)
            bnd = (k0 // G + 1) * G - k0
            sc = lambda L: s[ga] if L < bnd else s[gb]

            def fx(pair, corr, La, Lb):
                return (float(np.float16((pair[0] + corr[0]) * sc(La))),
                        float(np.float16((pair[1] + corr[1]) * sc(Lb))))
            f = {}
            for q in range(4):
                L = 10 * q
                f[2 * q] = (fx(int3_pair_i6(lw[q], 0), int3_sign_i6(S, q, 0), L, L + 6),
                            fx(int3_pair_i6(lw[q], 1), int3_sign_i6(S, q, 1), L + 1, L + 7))
                f[2 * q + 1] = (fx(int3_pair_i6(lw[q], 2), int3_sign_i6(S, q, 2), L + 2, L + 8),
                                fx(int3_pair_i6(lw[q], 3), int3_sign_i6(S, q, 3), L + 3, L + 9))
            f[8] = (fx(int3_pair_c4(lw[0], lw[1]), int3_sign_c(S, 4, 15), 4, 14),
                    fx(int3_pair_c5(lw[0], lw[1]), int3_sign_c(S, 4, 14), 5, 15))
            f[9] = (fx(int3_pair_c4(lw[2], lw[3]), int3_sign_c(S, 24, 15), 24, 34),
                    fx(int3_pair_c5(lw[2], lw[3]), int3_sign_c(S, 24, 14), 25, 35))
            frags.append(f)
        total += _mma_dot(frags, xs[160 * c:160 * c + 160], 160)
    deq = np.array([float(np.float16(odd[k] * s[k // G])) for k in range(K)])
    want = float(deq @ x[:K])
    assert abs(total - want) <= 1e-9 * max(1.0, abs(want)), (total, want)


# ---------------------------------------------------------------- staged row layout
def dg_row(r):
    return ((r & 1) << 3) | ((r & 8) >> 1) | ((r & 7) >> 1)


def dg_row_off(r, rb):
    pr = dg_row(r)
    return (pr >> 3) * (8 * rb + 64) + (pr & 7) * rb


def test_row_layout_matches_the_kernel():
    assert "return ((r & 1) << 3) | ((r & 8) >> 1) | ((r & 7) >> 1);" in SRC
    assert "return (size_t)8 * row_bytes + 64;" in SRC
    assert "(size_t)(pr >> 3) * dg_grp_bytes(row_bytes) + (size_t)(pr & 7) * row_bytes" in SRC


@pytest.mark.parametrize("rb", [1024, 4096, 832, 3280])   # INT4 and INT3 rows, K 2048 and 8192
def test_staged_rows_are_bank_conflict_free(rb):
    """Two bulk copies per 16-row tile (rows 0-7, rows 8-15 64 bytes after the
    end of the first group): every 16-byte operand load of a quarter warp
    (lanes 8p .. 8p + 7: MMA rows 2p, 2p + 1, vectors 4c .. 4c + 3) touches 32
    distinct banks, for the rows g and for the rows g + 8."""
    assert sorted(dg_row(r) for r in range(16)) == list(range(16))
    for half in (0, 8):
        for c in range(3):
            for p in range(4):
                banks = []
                for lane in range(8 * p, 8 * p + 8):
                    g, t = lane >> 2, lane & 3
                    off = dg_row_off(g + half, rb) + 16 * (4 * c + t)
                    assert off % 16 == 0
                    banks += [(off // 4 + i) % 32 for i in range(4)]
                assert len(set(banks)) == 32, (rb, half, c, p)
