"""Parity of the whole path with the oracle on the sweep workload: square and rectangular
ternary GEMMs with K, N in {1024 ... 16384} and M in {1 ... 8192}; weights whose share of
zero codes is 30%, 50% or 70% (the mixtures of the input generator); activations with
0.1-2% outlier channels scaled by 50.

Each case runs the path as the benchmark runs it: absmean ternarisation of the fp32
weights (gamma within 1e-6; the codes bit-exact through the given-scale entry with the
oracle's gamma), per-token quantisation into the stride-4 k16 x_q layout (x_q and s
bit-exact), and the forward with automatic dispatch (the decode GEMV for M <= 16, the
tcgen05 kernels above) in all three output kinds.  Where the oracle would take too long
on every token row, it computes sampled rows (int32 bit-exact, fp32 within 1e-5 relative
/ 1e-6 absolute, bf16 equal up to rounding-midpoint cases), and every row is checked
through the linearity of the integer product: acc . v == x_q . (C^T v) for a random
integer vector v, evaluated in float64 on the device, where every partial sum is an
integer below 2^53 and so exact.

Weights ("1-bit & Ternary LLMs (BitNet b1.58)", "How it works (real mechanics)", block
"BitNet b1.58 (Feb 2024)"): gamma = mean|W| + eps, W~ = RoundClip(W / gamma, -1, 1).
Because absmean is scale invariant, the zero share is set by the shape of the weight
distribution (a fraction of entries drawn with a tiny scale), not by sigma.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import EPS, assert_bf16_match, assert_float_close, bits
from ternary_weight_bit_absmean_b200 import binding as B
from ternary_weight_bit_absmean_b200 import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from ternary_weight_bit_absmean_b200 import build_lib
    build_lib.build()
    B.lib()


def stride4_positions(K):
    """Byte position of element k in the stride-4 k16 layout, from its definition: in
    each group of 16 the bytes hold elements 0,4,8,12, 1,5,9,13, 2,6,10,14, 3,7,11,15."""
    order = [0, 4, 8, 12, 1, 5, 9, 13, 2, 6, 10, 14, 3, 7, 11, 15]
    inv = np.empty(16, dtype=np.int64)
    inv[order] = np.arange(16)
    k = np.arange(K)
    return 16 * (k // 16) + inv[k % 16]


def sample_rows(M, N, K, seed):
    """Every token row when the oracle finishes them quickly, else the first, the last
    and a few random rows."""
    if M * N * K <= 2_000_000_000:
        return np.arange(M)
    n_rand = 1 if N * K >= 16384 * 8192 else 4
    return np.unique(np.r_[0, M - 1, np.random.default_rng(seed).integers(0, M, n_rand)])


def run_case(N, K, zeros, outlier_frac, Ms, layouts=(B.BL_XQ_K16_STRIDE4,)):
    seed = N + 7 * K + zeros
    W = synth.weight(N, K, seed=seed, small_frac=synth.SWEEP_SMALL_FRAC[zeros])
    g_ref, codes_ref, packed_ref = oracle.quantize_weights(W.numpy(), EPS)
    # the mixture gives the zero share it is named for (the oracle's codes)
    assert abs(float(np.mean(codes_ref == 0)) - zeros / 100.0) < 0.015  # a plain Gaussian gives ~31%

    # a1 + a2 on the device
    Wd = W.to(DEV)
    del W
    gamma, packed = B.quantize_weights(Wd, EPS)
    g_dev = torch.tensor([g_ref], dtype=torch.float32, device=DEV)
    packed_given = torch.empty_like(packed)
    B.bitlinear_quantize_weights_with_scale(Wd, g_dev, packed_given)
    torch.cuda.synchronize()
    del Wd
    assert abs(gamma.item() - float(g_ref)) <= 1e-6 * float(g_ref), (gamma.item(), g_ref)
    pk = torch.from_numpy(packed_ref).to(DEV)
    assert torch.equal(packed_given, pk), "codes differ from the oracle's (given gamma)"
    if gamma.item() == float(g_ref):
        assert torch.equal(packed, pk), "codes differ from the oracle's"
    del packed, packed_given

    # C^T v for the linearity check of every row (float64 on the device, exact)
    v = torch.from_numpy(np.random.default_rng(seed).integers(-3, 4, size=N).astype(np.float64)).to(DEV)
    cv = torch.from_numpy(codes_ref).to(DEV).to(torch.float64).T @ v
    del codes_ref
    pos = stride4_positions(K)

    for M in Ms:
        X = synth.activations(M, K, seed=M + K + int(outlier_frac * 10000), outlier_frac=outlier_frac,
                              outlier_scale=synth.SWEEP_OUTLIER_SCALE)
        xq_ref, s_ref = oracle.quantize_act(bits(X), EPS)
        rows = sample_rows(M, N, K, seed + M)
        acc_ref = oracle.forward(xq_ref[rows], s_ref[rows], packed_ref, g_ref, K, oracle.OUT_I32)
        y_ref = oracle.dequant(acc_ref, s_ref[rows], g_ref)
        yb_ref = oracle.f32_to_bf16(y_ref)
        xq_lin = torch.from_numpy(xq_ref).to(DEV).to(torch.float64) @ cv
        rows_dev = torch.from_numpy(rows).to(DEV)
        for lay in layouts:
            what = "N=%d K=%d zeros=%d%% outliers=%g M=%d layout=%d" % (N, K, zeros, outlier_frac, M, lay)
            xq, s = B.quantize_act(X.to(DEV), EPS, layout=lay)
            torch.cuda.synchronize()
            xq_host = xq.cpu().numpy()
            if lay == B.BL_XQ_K16_STRIDE4:
                xq_host = xq_host[:, pos]
            assert np.array_equal(xq_host, xq_ref), "x_q differs: " + what
            assert np.array_equal(s.cpu().numpy(), s_ref), "s differs: " + what
            del xq_host
            acc = B.forward(xq, s, pk, g_dev, torch.int32, layout=lay)
            torch.cuda.synchronize()
            assert np.array_equal(acc[rows_dev].cpu().numpy(), acc_ref), "int32 accumulators differ: " + what
            assert torch.equal(acc.to(torch.float64) @ v, xq_lin), "linearity fails on some row: " + what
            del acc
            y = B.forward(xq, s, pk, g_dev, torch.float32, layout=lay)
            torch.cuda.synchronize()
            assert_float_close(y[rows_dev].cpu().numpy(), y_ref, "fp32 y " + what)
            del y
            yb = B.forward(xq, s, pk, g_dev, torch.bfloat16, layout=lay)
            torch.cuda.synchronize()
            yb_host = yb[rows_dev].view(torch.int16).cpu().numpy().view(np.uint16)
            assert_bf16_match(yb_host, y_ref, yb_ref, "bf16 y " + what)
            del yb, xq, s


# (N, K, zero share %, outlier fraction, token counts): the grid at its default point
# (50% zeros, 1% outliers): the largest square from one token to the largest prefill,
# both rectangular extremes, two mid-size rectangles, and (below) one small square at
# every token count of the grid
GRID = [
    (16384, 16384, 50, 0.01, [1, 16, 64, 1024, 8192]),
    (1024, 16384, 50, 0.01, [4, 256, 8192]),
    (16384, 1024, 50, 0.01, [4, 256, 8192]),
    (4096, 8192, 50, 0.01, [16, 1024]),
    (8192, 4096, 50, 0.01, [1, 64]),
]


@pytest.mark.parametrize("N,K,zeros,ofrac,Ms", GRID, ids=["%dx%d" % (c[0], c[1]) for c in GRID])
def test_sweep_grid(N, K, zeros, ofrac, Ms):
    run_case(N, K, zeros, ofrac, Ms)


def test_sweep_small_square_every_token_count_both_layouts():
    run_case(2048, 2048, 50, 0.01, synth.SWEEP_M, layouts=(B.BL_XQ_ROWMAJOR, B.BL_XQ_K16_STRIDE4))


@pytest.mark.parametrize("zeros", [30, 70])
def test_sweep_zero_mixtures(zeros):
    """K = N = 8192 with 30% and 70% zero codes (50% runs in the outlier cases)."""
    run_case(8192, 8192, zeros, 0.01, [16, 1024])


@pytest.mark.parametrize("ofrac", synth.SWEEP_OUTLIER_FRACS)
def test_sweep_outlier_fractions(ofrac):
    """K = N = 8192, 50% zero codes, outlier channels x50 at 0.1, 0.5, 1 and 2%."""
    run_case(8192, 8192, 50, ofrac, [1, 256])
