"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with:
  * the hand-worked cases in ``tests/golden/hand_cases.txt`` (values computed by hand
    from the pages' definitions),
  * closed forms (E[gamma] for Gaussian weights, the share of zero codes),
  * invariants (code alphabet, sign symmetry, absmax -> +-127, all-zero inputs,
    K-permutation invariance, linearity),
  * independent library routines (numpy integer matmul, torch round/clamp in fp32,
    torch's bf16 conversion, a float64 matmul of the dequantised operands).
They are plain functions so that ``test_oracle_mutants`` can run the same pins
against deliberately broken builds of the oracle and show that each break is caught.
"""
import math

import numpy as np
import torch

from conftest import parse_golden
from oracle import OUT_BF16, OUT_F32, OUT_I32

EPS = 1e-5


def _floats(v):
    return np.array([float(x) for x in v.split(",")], dtype=np.float32)


def _ints(v, dt=np.int64):
    return np.array([int(x, 0) for x in v.split(",")], dtype=dt)


def _bf16_bits(x_f32):
    t = torch.from_numpy(np.asarray(x_f32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------- hand cases --

def pin_hand_ternarise(O):
    n = 0
    for kind, r in parse_golden("hand_cases.txt"):
        if kind != "ternarise":
            continue
        W = _floats(r["W"])[None, :]
        got = O.ternarise(W, np.float32(float(r["gamma"])))
        assert np.array_equal(got[0].astype(np.int64), _ints(r["codes"])), (r, got)
        n += 1
    assert n >= 2


def pin_hand_absmean(O):
    n = 0
    for kind, r in parse_golden("hand_cases.txt"):
        if kind != "absmean":
            continue
        N, K = int(r["N"]), int(r["K"])
        W = _floats(r["W"]).reshape(N, K)
        g = O.absmean_gamma(W, float(r["eps"]))
        assert g == np.float32(float(r["gamma"])), (r, g)
        codes = O.ternarise(W, g)
        assert np.array_equal(codes.reshape(-1).astype(np.int64), _ints(r["codes"])), (r, codes)
        n += 1
    assert n >= 2


def pin_hand_act(O):
    n = 0
    for kind, r in parse_golden("hand_cases.txt"):
        if kind != "act":
            continue
        x = _floats(r["x"])[None, :]
        bits = _bf16_bits(x)
        # every hand value is exactly representable in bf16
        assert np.array_equal(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
                              .float().numpy(), x)
        xq, s = O.quantize_act(bits, EPS)
        assert s[0] == np.float32(float(r["s"])), (r, s)
        assert np.array_equal(xq[0].astype(np.int64), _ints(r["xq"])), (r, xq)
        n += 1
    assert n >= 3


def pin_hand_pack(O):
    n = 0
    for kind, r in parse_golden("hand_cases.txt"):
        if kind != "pack":
            continue
        codes = _ints(r["codes"], np.int8)[None, :]
        packed, bad = O.pack(codes)
        assert bad == 0
        assert int(packed[0, 0]) == int(r["byte"], 16), (r, hex(packed[0, 0]))
        assert np.array_equal(O.unpack(packed, 4), codes)
        n += 1
    assert n >= 8


def pin_hand_matmul(O):
    n = 0
    for kind, r in parse_golden("hand_cases.txt"):
        if kind != "matmul":
            continue
        K = int(r["K"])
        xq = _ints(r["xq"], np.int8)[None, :]
        codes = np.array([[int(v) for v in row.split(",")] for row in r["codes"].split(";")],
                         dtype=np.int8)
        acc = O.int_matmul(xq, codes)
        assert np.array_equal(acc[0].astype(np.int64), _ints(r["acc"])), (r, acc)
        s = np.array([float(r["s"])], np.float32)
        y = O.dequant(acc, s, np.float32(float(r["gamma"])))
        want = np.array([int(a) / int(r["y_den"]) for a in r["y_num"].split(",")])
        assert np.allclose(y[0].astype(np.float64), want, rtol=1e-7, atol=0), (y, want)
        packed, _ = O.pack(codes)
        y2 = O.forward(xq, s, packed, np.float32(float(r["gamma"])), K)
        assert np.array_equal(y2, y)
        n += 1
    assert n >= 1


# --------------------------------------------------------------- closed forms --

def pin_gaussian_statistics(O):
    """W ~ N(0, sigma): E|w| = sigma sqrt(2/pi); a weight codes to 0 iff |w| <= gamma/2,
    so the zero share is erf(gamma / (2 sigma sqrt 2)) for the sample's own gamma."""
    sigma = 0.02
    for seed in (0, 1, 2):
        g = torch.Generator().manual_seed(seed)
        W = (torch.randn(256, 512, generator=g) * sigma).numpy()
        gamma = float(O.absmean_gamma(W, EPS))
        n = W.size
        mean_abs = sigma * math.sqrt(2 / math.pi)
        sd_mean = sigma * math.sqrt(1 - 2 / math.pi) / math.sqrt(n)
        assert abs((gamma - EPS) - mean_abs) < 5 * sd_mean, (gamma, mean_abs)
        codes = O.ternarise(W, np.float32(gamma))
        zero = float(np.mean(codes == 0))
        p0 = math.erf(gamma / (2 * sigma * math.sqrt(2)))
        assert abs(zero - p0) < 5 * math.sqrt(p0 * (1 - p0) / n), (zero, p0)
        assert abs(zero - 0.3101) < 0.01
        # the two signs are equally likely
        plus, minus = float(np.mean(codes == 1)), float(np.mean(codes == -1))
        assert abs(plus - minus) < 5 * math.sqrt(0.7 / n)


def pin_constant_magnitude(O):
    """|W| constant -> gamma = that constant + eps, codes = sign(W)."""
    rng = np.random.default_rng(5)
    for c in (0.25, 0.015625, 3.0):
        W = np.where(rng.random((64, 128)) < 0.5, -c, c).astype(np.float32)
        g = O.absmean_gamma(W, 2.0 ** -20)
        assert g == np.float32(np.float32(c) + np.float32(2.0 ** -20))
        assert np.array_equal(O.ternarise(W, g), np.sign(W).astype(np.int8))


# ----------------------------------------------------------------- invariants --

def pin_zero_weights(O):
    W = np.zeros((16, 32), np.float32)
    g = O.absmean_gamma(W, EPS)
    assert g == np.float32(EPS)
    codes = O.ternarise(W, g)
    assert not codes.any()
    packed, bad = O.pack(codes)
    assert bad == 0 and not packed.any()
    xq, s = O.quantize_act(_bf16_bits(np.random.default_rng(1).normal(size=(3, 32))), EPS)
    assert not O.forward(xq, s, packed, g, 32).any()


def pin_zero_token(O):
    X = np.random.default_rng(2).normal(size=(4, 64)).astype(np.float32)
    X[2] = 0.0
    xq, s = O.quantize_act(_bf16_bits(X), EPS)
    assert not xq[2].any()
    codes = np.random.default_rng(3).integers(-1, 2, size=(8, 64)).astype(np.int8)
    packed, _ = O.pack(codes)
    y = O.forward(xq, s, packed, np.float32(0.03), 64)
    assert not y[2].any() and y[[0, 1, 3]].any()


def pin_code_alphabet_and_sign_symmetry(O):
    g = torch.Generator().manual_seed(11)
    W = (torch.randn(64, 256, generator=g) * 0.02).numpy()
    gamma = O.absmean_gamma(W, EPS)
    c = O.ternarise(W, gamma)
    assert set(np.unique(c).tolist()) <= {-1, 0, 1}
    assert O.absmean_gamma(-W, EPS) == gamma
    assert np.array_equal(O.ternarise(-W, gamma), -c)


def pin_act_range_and_symmetry(O):
    g = torch.Generator().manual_seed(12)
    X = torch.randn(32, 300, generator=g)
    X[:, 7] *= 20
    bits = _bf16_bits(X.numpy())
    xq, s = O.quantize_act(bits, EPS)
    xf = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.abs(xq.astype(np.int64)).max() <= 127
    am = np.argmax(np.abs(xf), axis=1)
    rows = np.arange(xf.shape[0])
    assert np.array_equal(xq[rows, am].astype(np.int64), (127 * np.sign(xf[rows, am])).astype(np.int64))
    xqn, sn = O.quantize_act(bits ^ np.uint16(0x8000), EPS)
    assert np.array_equal(sn, s) and np.array_equal(xqn, -xq)


def pin_permutation_and_linearity(O):
    rng = np.random.default_rng(4)
    M, N, K = 5, 7, 96
    xa = rng.integers(-63, 64, size=(M, K)).astype(np.int8)
    xb = rng.integers(-63, 64, size=(M, K)).astype(np.int8)
    c = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    acc = O.int_matmul(xa, c)
    perm = rng.permutation(K)
    assert np.array_equal(O.int_matmul(xa[:, perm], c[:, perm]), acc)
    assert np.array_equal(O.int_matmul((xa + xb).astype(np.int8), c), acc + O.int_matmul(xb, c))
    # swapping the roles of two token rows swaps the output rows
    assert np.array_equal(O.int_matmul(xa[[1, 0, 2, 3, 4]], c), acc[[1, 0, 2, 3, 4]])


# -------------------------------------------------- independent implementations --

def pin_matmul_vs_numpy(O):
    rng = np.random.default_rng(6)
    for (M, N, K) in [(1, 1, 4), (3, 17, 64), (16, 40, 260), (33, 9, 1000)]:
        xq = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
        c = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
        want = xq.astype(np.int64) @ c.astype(np.int64).T
        assert np.array_equal(O.int_matmul(xq, c).astype(np.int64), want)
        packed, _ = O.pack(c)
        assert np.array_equal(O.forward(xq, np.ones(M, np.float32), packed, 1.0, K, 2), want)


def pin_ternarise_vs_torch(O):
    g = torch.Generator().manual_seed(7)
    W = torch.randn(128, 192, generator=g) * 0.02
    for gamma in (0.015, 0.0173, 0.02, 1e-3):
        want = torch.round(W / torch.tensor(gamma, dtype=torch.float32)).clamp(-1, 1)
        got = O.ternarise(W.numpy(), np.float32(gamma))
        assert np.array_equal(got, want.to(torch.int8).numpy())
    # values sitting exactly on the +-0.5 boundary
    gamma = np.float32(0.0625)
    Wt = np.array([[0.03125, -0.03125, 0.09375, -0.09375, 0.0312500037]], np.float32)
    want = torch.round(torch.from_numpy(Wt) / torch.tensor(gamma)).clamp(-1, 1).to(torch.int8)
    assert np.array_equal(O.ternarise(Wt, gamma), want.numpy())
    # weights a few ulps either side of gamma/2 for many gammas: here an IEEE division
    # and a multiply by a rounded reciprocal disagree on some codes
    rng = np.random.default_rng(13)
    for gamma in rng.uniform(0.005, 0.05, size=64).astype(np.float32):
        half = np.float32(gamma * np.float32(0.5))
        w = half + np.arange(-8, 9, dtype=np.float32) * np.spacing(half)
        Wb = np.concatenate([w, -w]).astype(np.float32)[None, :]
        want = torch.round(torch.from_numpy(Wb) / torch.tensor(gamma)).clamp(-1, 1).to(torch.int8)
        assert np.array_equal(O.ternarise(Wb, gamma), want.numpy()), gamma


def pin_act_vs_torch(O):
    g = torch.Generator().manual_seed(8)
    X = (torch.randn(64, 512, generator=g) * 3).to(torch.bfloat16)
    X[5] = 0
    X[6, :] = torch.tensor(1e-7).to(torch.bfloat16)
    bits = X.view(torch.int16).numpy().view(np.uint16)
    xf = X.float()
    a = xf.abs().amax(dim=1)
    s = torch.tensor(127.0) / torch.clamp(a, min=EPS)
    xq = torch.round(xf * s[:, None]).clamp(-128, 127).to(torch.int8)
    got_q, got_s = O.quantize_act(bits, EPS)
    assert np.array_equal(got_s, s.numpy())
    assert np.array_equal(got_q, xq.numpy())


def pin_pack_vs_numpy(O):
    rng = np.random.default_rng(9)
    c = rng.integers(-1, 2, size=(13, 88)).astype(np.int8)
    enc = np.where(c == 1, 1, np.where(c == -1, 2, 0)).astype(np.uint8)
    want = (enc[:, 0::4] | (enc[:, 1::4] << 2) | (enc[:, 2::4] << 4) | (enc[:, 3::4] << 6))
    packed, bad = O.pack(c)
    assert bad == 0 and np.array_equal(packed, want.astype(np.uint8))
    assert np.array_equal(O.unpack(packed, 88), c)
    # invalid codes are counted and written as 00
    cb = c.copy()
    cb[0, 0], cb[3, 5] = 2, -7
    packed_b, bad_b = O.pack(cb)
    assert bad_b == 2
    # byte 11 decodes to 0 everywhere
    assert not O.unpack(np.full((2, 3), 0xFF, np.uint8), 12).any()


def pin_dequant_vs_float64(O):
    """y equals the float64 product of the dequantised operands (x_q / s)(gamma c)^T."""
    rng = np.random.default_rng(10)
    M, N, K = 9, 21, 320
    xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    s = (rng.random(M) * 50 + 1).astype(np.float32)
    c = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    gamma = np.float32(0.0173)
    packed, _ = O.pack(c)
    y = O.forward(xq, s, packed, gamma, K)
    want = (xq.astype(np.float64) / s.astype(np.float64)[:, None]) @ (float(gamma) * c.astype(np.float64)).T
    assert np.allclose(y.astype(np.float64), want, rtol=2e-7, atol=1e-12)
    # bf16 output is torch's round-to-nearest-even of the fp32 output
    yb = O.forward(xq, s, packed, gamma, K, 1)
    assert np.array_equal(yb, torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


# ----------------------------------------------- normalisation + quantiser --

def pin_hand_norm(O):
    n = 0
    for kind, r in parse_golden("hand_cases.txt"):
        if kind != "normact":
            continue
        x = _floats(r["x"])[None, :]
        w = _floats(r["w"]) if "w" in r else None
        xq, s, _ = O.norm_quantize_act(_bf16_bits(x), w, int(r["kind"]), float(r["norm_eps"]), EPS)
        assert np.array_equal(xq[0].astype(np.int64), _ints(r["xq"])), (r, xq)
        if "s" in r:
            assert s[0] == np.float32(float(r["s"])), (r, s)
        else:
            assert abs(float(s[0]) / float(r["s_approx"]) - 1.0) < 1e-6, (r, s)
        n += 1
    assert n >= 3


def _torch_norm_quant(xb, w, kind, norm_eps):
    """The same two steps through torch's own norm routines (float64) and fp32 ops."""
    import torch.nn.functional as F
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    K = x.shape[1]
    wt = None if w is None else torch.from_numpy(w).to(torch.float64)
    if kind == 0:
        xn = F.rms_norm(x, (K,), weight=wt, eps=norm_eps)
    else:
        xn = F.layer_norm(x, (K,), weight=wt, bias=None, eps=norm_eps)
    xn = xn.to(torch.float32)
    a = xn.abs().amax(dim=1)
    s = torch.tensor(127.0, dtype=torch.float32) / torch.clamp(a, min=EPS)
    q = torch.round(xn * s[:, None]).clamp(-128, 127)
    return q.numpy().astype(np.int64), s.numpy(), (xn * s[:, None]).numpy()


def pin_norm_vs_torch(O):
    """torch's rms_norm / layer_norm in float64 then the quantiser in fp32: the scale
    within 2^-21 (the oracle normalises each element in fp32, torch in float64), the
    codes equal except where x_n s sits within 1e-3 of a rounding midpoint, and those
    are rare."""
    rng = np.random.default_rng(7)
    for kind in (0, 1):
        for with_w in (False, True):
            x = rng.standard_normal((64, 384)).astype(np.float32) * 3.0 + (0.7 if kind == 1 else 0.0)
            x[:, :4] *= 20.0
            xb = _bf16_bits(x)
            w = (rng.uniform(0.5, 1.5, size=384).astype(np.float32) if with_w else None)
            xq, s, _ = O.norm_quantize_act(xb, w, kind, 1e-5, EPS)
            tq, ts, tv = _torch_norm_quant(xb, w, kind, 1e-5)
            assert np.all(np.abs(s / ts - 1.0) < 2.0 ** -21), (kind, with_w)
            frac = np.abs(tv - np.floor(tv) - 0.5)
            differ = xq.astype(np.int64) != tq
            assert np.all(frac[differ] < 1e-3), (kind, with_w)
            assert differ.mean() < 1e-3


def pin_norm_invariants(O):
    """RMSNorm is exactly invariant to scaling a token by a power of two (no norm_eps);
    a zero token normalises to zero and quantises to zero with s = 127 / eps."""
    rng = np.random.default_rng(8)
    x = rng.standard_normal((8, 64)).astype(np.float32)
    xb1, xb2 = _bf16_bits(x), _bf16_bits(np.float32(4.0) * _bf16_to_f32(_bf16_bits(x)))
    a = O.norm_quantize_act(xb1, None, 0, 0.0, EPS)
    b = O.norm_quantize_act(xb2, None, 0, 0.0, EPS)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    z = np.zeros((2, 32), dtype=np.uint16)
    for kind in (0, 1):
        xq, s, xn = O.norm_quantize_act(z, None, kind, 1e-5, EPS)
        assert not xq.any() and not xn.any()
        assert np.all(s == np.float32(127.0) / np.float32(EPS))


def pin_dequant_rows(O):
    """One gamma per output row: the hand case acc = [10, -4], s = 2, gamma = (0.5, 0.25)
    gives y = 10 * 0.5 / 2 = 2.5 and -4 * 0.25 / 2 = -0.5; with every row's gamma equal
    it is the single-gamma rescale, bit for bit."""
    y = O.dequant_rows(np.array([[10, -4]], dtype=np.int32), np.array([2.0], dtype=np.float32),
                       np.array([0.5, 0.25], dtype=np.float32))
    assert np.array_equal(y, np.array([[2.5, -0.5]], dtype=np.float32)), y
    rng = np.random.default_rng(11)
    acc = rng.integers(-50000, 50000, size=(7, 33)).astype(np.int32)
    s = rng.uniform(0.5, 200.0, size=7).astype(np.float32)
    g = np.float32(0.0173)
    assert np.array_equal(O.dequant_rows(acc, s, np.full(33, g, dtype=np.float32)), O.dequant(acc, s, g))


# ------------------------------------------------------- 1.6-bit packing (TL5) --

def _row_from_nonzero(K, spec):
    row = np.zeros(K, dtype=np.int8)
    for item in spec.split(","):
        k, c = item.split(":")
        row[int(k)] = int(c)
    return row


def pin_hand_tl5(O):
    """Hand-worked bytes of the five-per-byte format (golden file), both directions, and
    hand-decoded bytes that packing never writes."""
    n = 0
    for kind, r in parse_golden("hand_cases.txt"):
        if kind == "tl5":
            K = int(r["K"])
            row = _row_from_nonzero(K, r["nonzero"])[None, :]
            want = _ints(r["bytes"], np.uint8)[None, :]
            packed, bad = O.pack_tl5(row)
            assert bad == 0
            assert np.array_equal(packed, want), (K, packed, want)
            assert np.array_equal(O.unpack_tl5(want, K), row)
            n += 1
        elif kind == "tl5dec":
            blk = np.full((1, 16), 128, dtype=np.uint8)  # 128 = five zero codes
            blk[0, 0] = int(r["byte"])
            codes = O.unpack_tl5(blk, 80)
            assert np.array_equal(codes[0, 0::16], _ints(r["codes"], np.int8)), (r, codes[0, 0::16])
            assert not codes[0].reshape(5, 16)[:, 1:].any()
            n += 1
    assert n >= 7


def pin_tl5_every_value(O):
    """All 3^5 digit patterns of one byte: packing is one to one and order preserving
    (the stored byte grows with v = sum t_p 3^(4-p), p = 0 most significant), and
    reading gives each pattern back.  Every byte value 0..255 reads as codes in
    {-1, 0, +1}, and the value it encodes never decreases with the byte."""
    import itertools
    pats = np.array(list(itertools.product((-1, 0, 1), repeat=5)), dtype=np.int8)  # lexicographic = v order
    rows = np.zeros((pats.shape[0], 80), dtype=np.int8)
    for p in range(5):
        rows[:, 16 * p] = pats[:, p]
    packed, bad = O.pack_tl5(rows)
    assert bad == 0
    b0 = packed[:, 0].astype(np.int64)
    assert np.all(np.diff(b0) > 0) and b0[0] == 0 and b0[-1] == 255
    assert np.array_equal(O.unpack_tl5(packed, 80), rows)
    allb = np.full((256, 16), 128, dtype=np.uint8)
    allb[:, 0] = np.arange(256)
    dec = O.unpack_tl5(allb, 80)[:, 0::16].astype(np.int64) + 1
    assert dec.min() >= 0 and dec.max() <= 2
    v = dec @ np.array([81, 27, 9, 3, 1])
    assert np.all(np.diff(v) >= 0) and v[0] == 0 and v[-1] == 242
    # 256 byte values for 243 patterns: each pattern is read from one or two bytes
    assert len(np.unique(v)) == 243


def pin_tl5_size_and_equivalence(O):
    """Rows take 16 * ceil(K / 80) bytes, 1.6 bits per code when 80 divides K (the
    pages' ~1.6 bits per weight).  For ragged K and several rows, the codes read back
    from the five-per-byte format equal the codes read back from the 2-bit format, and
    the forward from either format is the same, for every output kind."""
    for K, want in ((16, 16), (80, 16), (96, 32), (160, 32), (8192, 1648), (28672, 5744)):
        assert O.tl5_row_bytes(K) == want, (K, O.tl5_row_bytes(K))
    assert O.tl5_row_bytes(8000) * 8 / 8000 == 1.6
    rng = np.random.default_rng(23)
    for N, K in ((7, 16), (5, 96), (3, 400), (9, 1040)):
        c = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
        p5, bad = O.pack_tl5(c)
        assert bad == 0 and p5.shape == (N, O.tl5_row_bytes(K))
        p2, _ = O.pack(c)
        assert np.array_equal(O.unpack_tl5(p5, K), O.unpack(p2, K))
        M = 3
        xq = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
        s = rng.uniform(0.5, 100.0, size=M).astype(np.float32)
        for kind in (OUT_I32, OUT_F32, OUT_BF16):
            assert np.array_equal(O.forward_tl5(xq, s, p5, 0.0271, K, kind), O.forward(xq, s, p2, 0.0271, K, kind))
    # invalid codes are counted and written as 0
    cb = rng.integers(-1, 2, size=(2, 32)).astype(np.int8)
    cb[0, 3], cb[1, 30] = 2, -5
    pb, badb = O.pack_tl5(cb)
    assert badb == 2
    ub = O.unpack_tl5(pb, 32)
    assert ub[0, 3] == 0 and ub[1, 30] == 0


def pin_tl5_padding_not_read(O):
    """Positions past K in the last block carry no code: whatever digits a byte holds
    there, reading gives the same codes for k < K."""
    rng = np.random.default_rng(29)
    c = rng.integers(-1, 2, size=(4, 48)).astype(np.int8)  # block of 80, planes 3 and 4 are padding
    p5, _ = O.pack_tl5(c)
    t = (c.astype(np.int64) + 1).reshape(4, 3, 16)
    for pad3, pad4 in ((0, 0), (2, 2), (0, 2), (1, 0)):
        v = t[:, 0] * 81 + t[:, 1] * 27 + t[:, 2] * 9 + pad3 * 3 + pad4
        other = ((v * 256 + 242) // 243).astype(np.uint8)
        assert np.array_equal(O.unpack_tl5(other, 48), c)
    assert np.array_equal(p5, (((t[:, 0] * 81 + t[:, 1] * 27 + t[:, 2] * 9 + 4) * 256 + 242) // 243).astype(np.uint8))


# ------------------------------------------------ straight-through backward (STE) --

def pin_hand_ste(O):
    """Hand-worked gradients of the straight-through backward (golden file)."""
    n = 0
    for kind, r in parse_golden("hand_cases.txt"):
        if kind != "ste":
            continue
        M, N, K = int(r["M"]), int(r["N"]), int(r["K"])
        g = float(r["gamma"])
        dY = _floats(r["dY"]).reshape(M, N)
        codes = _ints(r["codes"], np.int8).reshape(N, K)
        xq = _ints(r["xq"], np.int8).reshape(M, K)
        s = _floats(r["s"]).reshape(M)
        packed, _ = O.pack(codes)
        assert np.array_equal(O.ste_grad_input(dY, packed, g, K), _floats(r["dX"]).reshape(M, K))
        assert np.array_equal(O.ste_grad_weight(dY, xq, s, g), _floats(r["dW"]).reshape(N, K))
        n += 1
    assert n >= 2


def pin_ste_vs_autograd(O):
    """The pages' quantisation-aware-training forward, written in torch float64 with the
    straight-through estimator (W_eff = W_fp + (W_tern - W_fp).detach(), and the same
    for the activation quantiser), differentiated by autograd: its gradients for the
    shadow weights and for the quantiser's input equal the oracle's, given the same
    codes, x_q, s and gamma."""
    rng = np.random.default_rng(37)
    for M, N, K in ((1, 3, 8), (5, 7, 12), (9, 16, 40)):
        W = torch.from_numpy(rng.normal(0.0, 0.02, size=(N, K)))
        x = torch.from_numpy(rng.normal(0.0, 1.0, size=(M, K)))
        gamma = torch.tensor(float(np.float32(W.abs().mean().item() + 1e-5)), dtype=torch.float64)
        W_tern = torch.clamp(torch.round(W / gamma), -1, 1)
        s = torch.from_numpy((127.0 / x.abs().amax(dim=1).numpy()).astype(np.float32).astype(np.float64))
        x_q = torch.clamp(torch.round(x * s[:, None]), -128, 127)
        dY = torch.from_numpy(rng.normal(0.0, 1.0, size=(M, N)).astype(np.float32).astype(np.float64))

        W_fp = W.clone().requires_grad_(True)
        x_in = x.clone().requires_grad_(True)
        W_eff = W_fp + (W_tern - W_fp).detach()
        xs = x_in * s[:, None]
        x_q_ste = xs + (x_q - xs).detach()
        y = (x_q_ste @ W_eff.T) * (gamma / s)[:, None]
        y.backward(dY)

        packed, _ = O.pack(W_tern.numpy().astype(np.int8))
        dX = O.ste_grad_input(dY.numpy().astype(np.float32), packed, gamma.item(), K)
        dW = O.ste_grad_weight(dY.numpy().astype(np.float32), x_q.numpy().astype(np.int8),
                               s.numpy().astype(np.float32), gamma.item())
        for got, want in ((dX, x_in.grad.numpy()), (dW, W_fp.grad.numpy())):
            assert np.allclose(got, want, rtol=2.0 ** -22, atol=1e-30), (M, N, K, np.abs(got - want).max())


def _bf16_to_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


ALL_PINS = [
    pin_hand_ste, pin_ste_vs_autograd,
    pin_hand_tl5, pin_tl5_every_value, pin_tl5_size_and_equivalence, pin_tl5_padding_not_read,
    pin_hand_norm, pin_norm_vs_torch, pin_norm_invariants, pin_dequant_rows,
    pin_hand_ternarise, pin_hand_absmean, pin_hand_act, pin_hand_pack, pin_hand_matmul,
    pin_gaussian_statistics, pin_constant_magnitude, pin_zero_weights, pin_zero_token,
    pin_code_alphabet_and_sign_symmetry, pin_act_range_and_symmetry,
    pin_permutation_and_linearity, pin_matmul_vs_numpy, pin_ternarise_vs_torch,
    pin_act_vs_torch, pin_pack_vs_numpy, pin_dequant_vs_float64,
]
