"""The integer tricks inside the decode kernels, modelled on the host and checked against
the oracle's plain definitions, exhaustively where the domain is small.

The constants (logic-op truth tables, masks, byte-permute selectors, multipliers) are
read from the kernel sources, so a change there that breaks the arithmetic fails here
without a GPU.  The models follow the PTX definitions of the instructions:
  lop3.b32 d, a, b, c, LUT: bit i of d = bit (4 a_i + 2 b_i + c_i) of LUT;
  prmt (__byte_perm(x, y, s)): byte n of the result = byte (s >> 4n) & 7 of y:x;
  mul.hi.u32 / mul.lo.u32 / mad.lo.u32: the high / low 32 bits of the product;
  dp4a.u32.s32: c + sum of unsigned bytes of a times signed bytes of b (mod 2^32)."""
import os
import re

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.cpu

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "ternary_weight_bit_absmean_b200", "csrc")
M32 = 0xFFFFFFFF


def _src(name):
    with open(os.path.join(CSRC, name)) as f:
        return f.read()


def lop3(a, b, c, lut):
    out = np.zeros_like(a)
    for bit in range(32):
        ai, bi, ci = (a >> bit) & 1, (b >> bit) & 1, (c >> bit) & 1
        out |= ((lut >> (4 * ai + 2 * bi + ci)) & 1) << bit
    return out


def prmt(x, y, sel):
    b = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    out = 0
    for n in range(4):
        s = (sel >> (4 * n)) & 0xF
        assert s < 8, "sign-replicate selectors are not modelled"
        out = out | (b[s] << (8 * n))
    return out


# ------------------------------------------------------ the stride-4 2-bit unpack --

def test_stride4_unpack_matches_the_2bit_decode():
    """BL_S4_UNPACK turns one word of 16 codes into four words of int8 64 * code, word i
    holding codes {i, 4 + i, 8 + i, 12 + i} (byte j = code 4j + i); codes 11 read as 0."""
    src = _src("bl_device.cuh")
    mac = src[src.index("#define BL_S4_UNPACK"):]
    mac = mac[:mac.index("\n\n")]
    lx, ly = [int(v, 16) for v in re.findall(r"lop3\.b32 t[xy], [^;]*?0x55555555, (0x[0-9A-Fa-f]+)", mac)]
    mask = int(re.search(r'and\.b32 " O3 ", tv, (0x[0-9A-Fa-f]+)', mac).group(1), 16)
    hi1, two, m4, m16, m64 = [int(eval(v.replace("u", ""))) for v in
                              re.search(r"return S4Mul\{([^}]*)\}", src).group(1).split(",")]
    rng = np.random.default_rng(5)
    words = np.concatenate([rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64),
                            np.array([0, M32, 0x55555555, 0xAAAAAAAA, 0x99999999, 0x66666666], np.uint64)])
    # every 8-bit pattern (four codes) in every byte position
    for pos in range(4):
        words = np.concatenate([words, (np.arange(256, dtype=np.uint64) << np.uint64(8 * pos))])
    w = words.astype(np.uint64)
    ta = (w * np.uint64(hi1)) >> np.uint64(32)
    tx = lop3(w, ta, np.full_like(w, 0x55555555), lx)
    ty = lop3(ta, w, np.full_like(w, 0x55555555), ly)
    tv = (ty * np.uint64(two) + tx) & np.uint64(M32)
    outs = [(tv * np.uint64(m)) & np.uint64(M32) & np.uint64(mask) for m in (m64, m16, m4, 1)]  # o0..o3
    packed = w.astype(np.uint32).view(np.uint8).reshape(-1, 4)
    codes = oracle.unpack(packed, 16).astype(np.int64)  # the oracle's decode of the same word
    for i in range(4):
        for j in range(4):
            byte = ((outs[i] >> np.uint64(8 * j)) & np.uint64(0xFF)).astype(np.int64)
            sbyte = np.where(byte >= 128, byte - 256, byte)
            assert np.array_equal(sbyte, 64 * codes[:, 4 * j + i]), (i, j)


# ------------------------------------------------- the five-per-byte digit decode --

def _tl5_constants():
    src = _src("k_tl5.cu")
    sel_e = int(re.search(r"__byte_perm\(ww\[q\], 0u, (0x[0-9A-Fa-f]+)\);\s*// bytes 0, 2", src).group(1), 16)
    sel_o = int(re.search(r"__byte_perm\(ww\[q\], 0u, (0x[0-9A-Fa-f]+)\);\s*// bytes 1, 3", src).group(1), 16)
    sel_h = int(re.search(r"__byte_perm\(even \* kMul, odd \* kMul, (0x[0-9A-Fa-f]+)\)", src).group(1), 16)
    muls = [int(v) for v in re.findall(r"P == \d \? (\d+)u", src)] + \
        [int(re.search(r"P == 3 \? \d+u : (\d+)u;", src).group(1))]
    return sel_e, sel_o, sel_h, muls


def _tl5_plane_digits(word, sel_e, sel_o, sel_h, muls):
    """Digits (one per byte) of the five planes of a 4-byte word, as the kernel forms them."""
    ev, od = prmt(word, 0, sel_e), prmt(word, 0, sel_o)
    h, out = 0, []
    for mul in muls:
        ye, yo = (ev * mul) & M32, (od * mul) & M32
        hn = prmt(ye, yo, sel_h)
        out.append((hn - 3 * h) & M32)
        h = hn
    return out


def test_tl5_digits_match_the_oracle_for_every_byte():
    sel_e, sel_o, sel_h, muls = _tl5_constants()
    assert muls == [3, 9, 27, 81, 243]
    for pos in range(4):
        for B in range(256):
            word = (B << (8 * pos)) | sum(((37 * i + 11) & 0xFF) << (8 * i) for i in range(4) if i != pos)
            digits = _tl5_plane_digits(word, sel_e, sel_o, sel_h, muls)
            blk = np.full((1, 16), 128, np.uint8)
            for i in range(4):
                blk[0, i] = (word >> (8 * i)) & 0xFF
            ref = oracle.unpack_tl5(blk, 80)[0].astype(np.int64) + 1  # digits t = c + 1
            for p in range(5):
                for i in range(4):
                    assert (digits[p] >> (8 * i)) & 0xFF == ref[16 * p + i], (pos, B, p, i)


def _dp4a_us(a, b, c):
    r = c
    for i in range(4):
        sb = (b >> (8 * i)) & 0xFF
        r += ((a >> (8 * i)) & 0xFF) * (sb - 256 if sb & 0x80 else sb)
    return r & M32


def test_tl5_row_sum_with_token_sum_correction():
    """A whole row as the decode kernel sums it: unsigned digits against x_q, minus the
    token's sum of x_q, planes past K skipped; equal to the oracle's int32 product, for
    arbitrary bytes, ragged K and x_q = -128 everywhere."""
    sel_e, sel_o, sel_h, muls = _tl5_constants()
    rng = np.random.default_rng(8)
    for K in (16, 80, 96, 400, 1296):
        N, RB = 5, oracle.tl5_row_bytes(K)
        w5 = rng.integers(0, 256, size=(N, RB)).astype(np.uint8)
        xq = rng.integers(-128, 128, size=(2, K)).astype(np.int8)
        xq[1] = -128
        ref = oracle.forward_tl5(xq, np.ones(2, np.float32), w5, 1.0, K, oracle.OUT_I32)
        for m in range(2):
            xs = 0
            for k in range(0, K, 4):
                xs = _dp4a_us(0x01010101, int.from_bytes(xq[m, k:k + 4].tobytes(), "little"), xs)
            for n in range(N):
                acc = 0
                for blk in range(RB // 16):
                    for q in range(4):
                        word = int.from_bytes(w5[n, 16 * blk + 4 * q:16 * blk + 4 * q + 4].tobytes(), "little")
                        digits = _tl5_plane_digits(word, sel_e, sel_o, sel_h, muls)
                        for p in range(5):
                            k0 = 80 * blk + 16 * p
                            if k0 >= K:
                                break
                            xw = int.from_bytes(xq[m, k0 + 4 * q:k0 + 4 * q + 4].tobytes(), "little")
                            acc = _dp4a_us(digits[p], xw, acc)
                r = (acc - xs) & M32
                assert (r - (1 << 32) if r & 0x80000000 else r) == ref[m, n], (K, m, n)


# ----------------------------------------- the table unpacks of the other layouts --

def _code_table():
    return int(re.search(r"constexpr uint32_t kCodeTable = (0x[0-9A-Fa-f]+)u;", _src("bl_device.cuh")).group(1), 16)


def _words_under_test():
    rng = np.random.default_rng(9)
    words = [int(v) for v in rng.integers(0, 2 ** 32, size=3000, dtype=np.uint64)]
    words += [0, M32, 0x55555555, 0xAAAAAAAA]
    for pos in range(4):
        words += [b << (8 * pos) for b in range(256)]
    return words


def _as_int8(word):
    return [((word >> (8 * i)) & 0xFF) - (256 if (word >> (8 * i)) & 0x80 else 0) for i in range(4)]


def test_natural_and_evenodd_unpacks_match_the_2bit_decode():
    """unpack16_natural (nibble spread, then a table byte per code) and unpack16_evenodd
    (two masks, then table bytes) give the oracle's codes in their stated orders."""
    tab = _code_table()
    words = _words_under_test()
    packed = np.array(words, dtype=np.uint32).view(np.uint8).reshape(-1, 4)
    codes = oracle.unpack(packed, 16)
    for w, c in zip(words, codes):
        lo, hi = prmt(w, 0, 0x4140), prmt(w, 0, 0x4342)
        lo = (lo | (lo << 4)) & 0x0F0F0F0F
        hi = (hi | (hi << 4)) & 0x0F0F0F0F
        lo = (lo | (lo << 2)) & 0x33333333
        hi = (hi | (hi << 2)) & 0x33333333
        nat = _as_int8(prmt(tab, 0, lo & 0xFFFF)) + _as_int8(prmt(tab, 0, lo >> 16)) + \
            _as_int8(prmt(tab, 0, hi & 0xFFFF)) + _as_int8(prmt(tab, 0, hi >> 16))
        assert nat == list(c), hex(w)
        sa, sb = w & 0x33333333, (w >> 2) & 0x33333333
        e0, e1 = _as_int8(prmt(tab, 0, sa & 0xFFFF)), _as_int8(prmt(tab, 0, sa >> 16))
        o0, o1 = _as_int8(prmt(tab, 0, sb & 0xFFFF)), _as_int8(prmt(tab, 0, sb >> 16))
        assert e0 + e1 == list(c[0::2]) and o0 + o1 == list(c[1::2]), hex(w)


# ---------------------------------------------------- the activation quantiser --

def test_act_quant_rounding_by_magic_add_is_rint():
    """q8_bits rounds x s by adding 1.5 * 2^23 in fp32: the low byte of the sum's bits is
    rint(x s) (half to even) as int8, for every bf16 x and scales of the form
    127 / max(a, eps) with |x| <= a, as the quantiser forms them."""
    src = _src("k_quant.cu")
    magic = np.float32(float(re.search(r"__fmul_rn\(x, s\), ([0-9.]+)f\)", src).group(1)))
    assert magic == np.float32(1.5 * 2 ** 23)
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    x = (bits << 16).view(np.float32)
    x = x[np.isfinite(x)]
    rng = np.random.default_rng(12)
    amax = np.concatenate([np.abs(x[rng.integers(0, x.size, 48)]), np.float32([1.0, 3.0e38, 1.0e-38])])
    for a in amax:
        s = np.float32(127.0) / np.maximum(np.float32(a), np.float32(1e-5))  # s = 127 / max(a, eps)
        xs = x[np.abs(x) <= a]
        prod = xs * s
        got = ((prod + magic).view(np.uint32) & 0xFF).astype(np.int64)
        got = np.where(got >= 128, got - 256, got)
        want = np.clip(np.rint(prod.astype(np.float64)), -128, 127).astype(np.int64)
        assert np.array_equal(got, want), a


def test_bf16_magnitude_order_is_bit_order():
    """The quantiser takes max |x| as an unsigned max of the bf16 bit patterns with the
    sign cleared: for finite values that order is the order of the magnitudes."""
    bits = np.arange(0, 0x7F80, dtype=np.uint32)  # +0 .. the largest finite bf16
    mags = (bits << 16).view(np.float32)
    assert np.all(np.diff(mags.astype(np.float64)) > 0)
    src = _src("k_quant.cu")
    assert src.count("__vmaxu2(m, v.x & 0x7FFF7FFFu)") == 1
