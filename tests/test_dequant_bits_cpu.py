"""The integer-to-fp16 conversions inside the kernels, emulated bit for bit on
the CPU and checked against the oracle's codes over every input pattern that
matters.

Three kernels turn packed codes into fp16 without a conversion instruction:
  * the tcgen05 GEMM (gemm_tc.cu): one byte of an INT4 word -> the fp16 pair
    (code of k = 2c, code of k = 2c + 1), via prmt, lop3 (a & b) | c and one
    HFMA2, then HMUL2 by the group's scale;
  * the decode GEMV (gemm_mma.cu): nibbles (i, i + 4) of a word -> an fp16
    pair, via lop3 and HSUB2 (low nibbles) or HFMA2 (high nibbles);
  * decode attention over an INT8 cache (attention.cu): four codes of a word,
    or byte e of two words, -> fp16 pairs via prmt / lop3 (a & b) ^ c and
    HSUB2.
Each relies on 0x64 in an fp16's high byte making the value 1024 + the low
bits, exactly.  The emulation follows the PTX definitions of prmt (default
mode: selector nibble i picks byte i of the result from {b, a}, bit 3
replicating that byte's sign) and lop3 (bit (a<<2 | b<<1 | c) of the LUT), and
IEEE fp16 with round-to-nearest-even for the half-precision ops; each test
first checks that the kernel source holds the constants it emulates."""
import os
import re

import numpy as np

from oracle import tinyloop_oracle as o

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "weight_shared_looped_b200", "csrc")
U32 = np.uint32


def _src(name):
    with open(os.path.join(CSRC, name)) as f:
        return re.sub(r"\s+", " ", f.read())


# ---------------------------------------------------------------- PTX emulation

def prmt(a, b, sel):
    """prmt.b32 d, a, b, sel (default mode), elementwise over uint32 arrays."""
    a = np.asarray(a, U32)
    b = np.asarray(b, U32)
    src = [(a >> U32(8 * i)) & U32(0xFF) for i in range(4)] + \
          [(b >> U32(8 * i)) & U32(0xFF) for i in range(4)]
    out = np.zeros(np.broadcast(a, b).shape, U32)
    for i in range(4):
        s = (int(sel) >> (4 * i)) & 0xF
        byte = src[s & 7]
        if s & 8:
            byte = np.where(byte & U32(0x80), U32(0xFF), U32(0))
        out |= (byte & U32(0xFF)) << U32(8 * i)
    return out


def lop3(a, b, c, lut):
    a, b, c = (np.asarray(x, U32) for x in (a, b, c))
    full = U32(0xFFFFFFFF)
    out = np.zeros(np.broadcast(a, b, c).shape, U32)
    for idx in range(8):
        if (lut >> idx) & 1:
            out |= ((a if idx & 4 else a ^ full) & (b if idx & 2 else b ^ full)
                    & (c if idx & 1 else c ^ full))
    return out


def halves(w):
    """uint32 -> (low fp16, high fp16) as float64."""
    w = np.asarray(w, U32)
    lo = (w & U32(0xFFFF)).astype(np.uint16).view(np.float16).astype(np.float64)
    hi = (w >> U32(16)).astype(np.uint16).view(np.float16).astype(np.float64)
    return lo, hi


def f16(x):
    """Round float64 values to fp16 (one IEEE rounding)."""
    return np.asarray(x, np.float64).astype(np.float16).astype(np.float64)


def hsub(x, y):
    return f16(x - y)


def hfma(x, m, c):
    return f16(x * m + c)     # exact in float64 for these operands, then one rounding


# ---------------------------------------------------------------- INT4 words

def _int4_words(rng, n):
    """Random INT4 rows of 8 codes packed by the oracle; returns (words, codes)."""
    codes = rng.integers(-8, 8, size=(n, 8)).astype(np.int8)
    words = o.pack_codes(codes, 4).reshape(n).astype(U32)
    assert np.array_equal(o.unpack_codes(words.reshape(n, 1), 8, 4), codes)
    return words, codes


def _all_byte_words():
    """Words whose byte c & 3 takes every value 0..255 in every position."""
    v = np.arange(256, dtype=U32)
    rng = np.random.default_rng(7)
    noise = rng.integers(0, 2**32, size=256, dtype=np.uint64).astype(U32)
    return np.concatenate([(noise & ~(U32(0xFF) << U32(8 * p))) | (v << U32(8 * p))
                           for p in range(4)])


def test_tcgen05_gemm_byte_to_code_pair():
    src = _src("gemm_tc.cu")
    assert '"r"(bb | 0x40u | (bb << 8) | 0x4000u)' in src
    assert 'lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h) : "r"(x), "r"(0x00F0000Fu), "r"(0x64006400u)' in src
    assert "__float2half_rn(1.0f), __float2half_rn(0.0625f)" in src
    assert "__float2half_rn(-1032.0f), __float2half_rn(-72.0f)" in src
    rng = np.random.default_rng(0)
    words, codes = _int4_words(rng, 1 << 15)
    words = np.concatenate([words, _all_byte_words()])
    codes = np.concatenate([codes, o.unpack_codes(words[-1024:].reshape(-1, 1), 8, 4)])
    for bb in range(4):
        sel = bb | 0x40 | (bb << 8) | 0x4000
        x = prmt(words, U32(0), sel)
        h = lop3(x, U32(0x00F0000F), U32(0x64006400), 0xEA)
        lo, hi = halves(h)
        c_lo = hfma(lo, 1.0, -1032.0)
        c_hi = hfma(hi, 0.0625, -72.0)
        assert np.array_equal(c_lo, codes[:, 2 * bb].astype(np.float64))
        assert np.array_equal(c_hi, codes[:, 2 * bb + 1].astype(np.float64))


def test_decode_projection_nibble_pairs():
    src = _src("gemv_dec.cu")
    assert "lop3_ea(w, 0x000F000Fu, 0x64006400u), one, lo_b" in src
    assert "lop3_ea(w, 0x00F000F0u, 0x64006400u), sixteenth, hi_b" in src
    assert "lop3_ea(w8, 0x000F000Fu, 0x64006400u), one, lo_b" in src
    assert "const uint32_t w8 = w >> 8;" in src
    assert "h2c(-1032.f, -1032.f), hi_b = h2c(-72.f, -72.f)" in src
    rng = np.random.default_rng(1)
    words, codes = _int4_words(rng, 1 << 16)
    # pairs (0, 4), (1, 5) from w; (2, 6), (3, 7) from w >> 8
    for sh, (k0, k1) in [(0, (0, 1)), (8, (2, 3))]:
        w = words >> U32(sh)
        lo_a, hi_a = halves(lop3(w, U32(0x000F000F), U32(0x64006400), 0xEA))
        lo_b, hi_b = halves(lop3(w, U32(0x00F000F0), U32(0x64006400), 0xEA))
        assert np.array_equal(hfma(lo_a, 1.0, -1032.0), codes[:, k0])
        assert np.array_equal(hfma(hi_a, 1.0, -1032.0), codes[:, k0 + 4])
        assert np.array_equal(hfma(lo_b, 0.0625, -72.0), codes[:, k1])
        assert np.array_equal(hfma(hi_b, 0.0625, -72.0), codes[:, k1 + 4])


def _int3_words(rng, n):
    codes = rng.integers(-4, 4, size=(n, 10)).astype(np.int8)
    codes[: 8 ** 2] = np.stack(np.meshgrid(np.arange(-4, 4), np.arange(-4, 4)), -1).reshape(-1, 2).repeat(5, 1)
    return o.pack_codes(codes, 3)[:, 0], codes


def test_decode_projection_int3_pairs():
    """The decode kernel's INT3 pairs: codes (i, i + 6) of a word, and codes 4
    and 5 of two words, over every code value in every position."""
    src = _src("gemv_dec.cu")
    for c in ["lop3_ea(w >> (3 * I), 0x001C0007u, 0x64006400u)", "h2c(1.f, 0.25f), h2c(-1028.f, -260.f)",
              "lop3_ea(prmt(a, b, 0x0501u), 0x00700070u, 0x64006400u)", "h2c(0.0625f, 0.0625f), h2c(-68.f, -68.f)",
              "lop3_ea(prmt(a, b, 0x6521u), 0x03800380u, 0x64006400u)",
              "h2c(0.0078125f, 0.0078125f), h2c(-12.f, -12.f)"]:
        assert c in src, c
    rng = np.random.default_rng(5)
    words, codes = _int3_words(rng, 1 << 14)
    for i in range(4):
        lo, hi = halves(lop3(words >> U32(3 * i), U32(0x001C0007), U32(0x64006400), 0xEA))
        assert np.array_equal(hfma(lo, 1.0, -1028.0), codes[:, i])
        assert np.array_equal(hfma(hi, 0.25, -260.0), codes[:, i + 6])
    wa, wb = words, np.roll(words, 1)
    ca, cb = codes, np.roll(codes, 1, axis=0)
    lo, hi = halves(lop3(prmt(wa, wb, 0x0501), U32(0x00700070), U32(0x64006400), 0xEA))
    assert np.array_equal(hfma(lo, 0.0625, -68.0), ca[:, 4])
    assert np.array_equal(hfma(hi, 0.0625, -68.0), cb[:, 4])
    lo, hi = halves(lop3(prmt(wa, wb, 0x6521), U32(0x03800380), U32(0x64006400), 0xEA))
    assert np.array_equal(hfma(lo, 0.0078125, -12.0), ca[:, 5])
    assert np.array_equal(hfma(hi, 0.0078125, -12.0), cb[:, 5])


def test_tcgen05_gemm_int3_consecutive_pairs():
    """The tensor-core GEMM's INT3 pairs (codes 2c, 2c + 1 of a word at an even
    position i): shift, 6-bit mask, multiply by 1 + 2^13, lop3, less 1028."""
    src = _src("gemm_tc.cu")
    for c in ["const uint32_t y = ((v[q] >> (3 * i)) & 0x3Fu) * 8193u;",
              '"r"(y), "r"(0x00070007u), "r"(0x64006400u)', "__float2half_rn(1028.0f)"]:
        assert c in src, c
    rng = np.random.default_rng(6)
    words, codes = _int3_words(rng, 1 << 14)
    for i in (0, 2, 4, 6, 8):
        y = (((words >> U32(3 * i)) & U32(0x3F)) * U32(8193)).astype(U32)
        lo, hi = halves(lop3(y, U32(0x00070007), U32(0x64006400), 0xEA))
        assert np.array_equal(hsub(lo, 1028.0), codes[:, i])
        assert np.array_equal(hsub(hi, 1028.0), codes[:, i + 1])


def _int8_words(rng, n):
    codes = rng.integers(-127, 128, size=(n, 4)).astype(np.int8)
    return codes.view(np.uint8).view("<u4").reshape(n).astype(U32), codes


def test_decode_int8_four_codes_of_a_word():
    src = _src("attention.cu")
    for s in ['const uint32_t u = w ^ 0x80808080u;', '"r"(u), "r"(0x64646464u), "r"(0x4140u)',
              '"r"(u), "r"(0x64646464u), "r"(0x4342u)', "__float2half2_rn(1152.0f)"]:
        assert s in src, s
    # every code value in every byte position, plus random words
    v = np.arange(-128, 128, dtype=np.int8)
    rng = np.random.default_rng(2)
    words, codes = _int8_words(rng, 1 << 16)
    for p in range(4):
        c = rng.integers(-127, 128, size=(256, 4)).astype(np.int8)
        c[:, p] = v
        words = np.concatenate([words, c.view(np.uint8).view("<u4").reshape(256).astype(U32)])
        codes = np.concatenate([codes, c])
    u = words ^ U32(0x80808080)
    lo0, lo1 = halves(prmt(u, U32(0x64646464), 0x4140))
    hi0, hi1 = halves(prmt(u, U32(0x64646464), 0x4342))
    got = np.stack([hsub(lo0, 1152.0), hsub(lo1, 1152.0), hsub(hi0, 1152.0), hsub(hi1, 1152.0)], 1)
    assert np.array_equal(got, codes.astype(np.float64))


def test_decode_int8_byte_pairs_of_two_words():
    src = _src("attention.cu")
    for s in ['"r"((uint32_t)(E | ((E + 4) << 8)))',
              'lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(y) : "r"(x), "r"(0x00FF00FFu), "r"(0x64806480u)']:
        assert s in src, s
    # all 65536 (byte of wa, byte of wb) combinations in each position, other bytes random
    rng = np.random.default_rng(3)
    ca = np.repeat(np.arange(-128, 128), 256).astype(np.int8)
    cb = np.tile(np.arange(-128, 128), 256).astype(np.int8)
    for e in range(4):
        A = rng.integers(-128, 128, size=(65536, 4)).astype(np.int8)
        B = rng.integers(-128, 128, size=(65536, 4)).astype(np.int8)
        A[:, e] = ca
        B[:, e] = cb
        wa = A.view(np.uint8).view("<u4").reshape(-1).astype(U32)
        wb = B.view(np.uint8).view("<u4").reshape(-1).astype(U32)
        x = prmt(wa, wb, e | ((e + 4) << 8))
        lo, hi = halves(lop3(x, U32(0x00FF00FF), U32(0x64806480), 0x6A))
        assert np.array_equal(hsub(lo, 1152.0), ca.astype(np.float64))
        assert np.array_equal(hsub(hi, 1152.0), cb.astype(np.float64))


def test_emulation_matches_ptx_definitions_on_hand_cases():
    """The emulated instructions on hand-worked values (PTX ISA definitions)."""
    a, b = U32(0x33221100), U32(0x77665544)
    assert int(prmt(a, b, 0x3210)) == 0x33221100          # identity
    assert int(prmt(a, b, 0x7654)) == 0x77665544          # all from b
    assert int(prmt(a, b, 0x0404)) == 0x00440044
    assert int(prmt(U32(0x80), U32(0), 0x8888)) == 0xFFFFFFFF   # sign replicate of byte 0
    x, y, z = U32(0xF0F0F0F0), U32(0xCCCCCCCC), U32(0xAAAAAAAA)
    assert int(lop3(x, y, z, 0xEA)) == 0xEAEAEAEA          # LUT = F(0xF0, 0xCC, 0xAA)
    assert int(lop3(x, y, z, 0x6A)) == 0x6A6A6A6A
    assert [float(h) for h in halves(U32(0x64006400))] == [1024.0, 1024.0]
    assert [float(h) for h in halves(U32(0x640F6401))] == [1025.0, 1039.0]
