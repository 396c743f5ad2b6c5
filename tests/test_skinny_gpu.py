"""Parity of the small-batch tcgen05 forward (BL_PATH_SKINNY: weights expanded to int8 in
shared memory, K split over a thread-block cluster when rows are few) with the oracle: ragged
shapes in every x_q layout and output kind, the LLaMA-70B decode shapes at 17 to 64
tokens (the automatic dispatch's range for this kernel), the largest accumulators,
per-row weight scales, undefined code 11, and repeated launches.

Integers bit-exact, fp32 within 1e-5 relative / 1e-6 absolute, bf16 equal up to
rounding-midpoint cases, and no write outside the output."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import EPS, assert_bf16_match, assert_float_close, bits, check_guard, guarded_empty
from ternary_weight_bit_absmean_b200 import binding as B
from ternary_weight_bit_absmean_b200 import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

DEV = "cuda"
SK = B.BL_PATH_SKINNY


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from ternary_weight_bit_absmean_b200 import build_lib
    build_lib.build()
    B.lib()


def positions(layout, K):
    """Byte position of every element k in the x_q layout, from the layout's definition."""
    k = np.arange(K)
    if layout == B.BL_XQ_ROWMAJOR:
        return k
    e = k % 16
    if layout == B.BL_XQ_K16_EVENODD:
        return 16 * (k // 16) + 8 * (e % 2) + 4 * (e // 8) + (e % 8) // 2
    return 16 * (k // 16) + 4 * (e % 4) + e // 4


def problem(M, N, K, seed, small_frac=0.0):
    W = synth.weight(N, K, seed=seed, small_frac=small_frac)
    X = synth.activations(M, K, seed=seed, outlier_frac=0.01, outlier_scale=20.0)
    g_ref, _, packed_ref = oracle.quantize_weights(W.numpy(), EPS)
    xq_ref, s_ref = oracle.quantize_act(bits(X), EPS)
    return g_ref, packed_ref, xq_ref, s_ref


def run(xq_ref, s_ref, packed_ref, gamma, layout, dtypes, rows=None, path=SK, gamma_rows=None):
    """The forward on the device in the given layout; checks the sampled rows (all rows
    by default) against the oracle, every row of the int32 result through linearity, and
    the canaries around each output."""
    M, K = xq_ref.shape
    N = packed_ref.shape[0]
    sel = np.arange(M) if rows is None else np.asarray(rows)
    acc_ref = oracle.forward(xq_ref[sel], s_ref[sel], packed_ref, gamma, K, oracle.OUT_I32)
    if gamma_rows is None:
        y_ref = oracle.dequant(acc_ref, s_ref[sel], gamma)
    else:
        y_ref = oracle.dequant_rows(acc_ref, s_ref[sel], gamma_rows)
    xl = np.empty_like(xq_ref)
    xl[:, positions(layout, K)] = xq_ref
    xq = torch.from_numpy(xl).to(DEV)
    s = torch.from_numpy(s_ref).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    g = torch.tensor([gamma], dtype=torch.float32, device=DEV)
    gr = None if gamma_rows is None else torch.from_numpy(gamma_rows).to(DEV)
    for dt in dtypes:
        out = guarded_empty((M, N), dt)
        err = torch.zeros(1, dtype=torch.int32, device=DEV)
        if gr is None:
            B.bitlinear_forward(xq, s, packed, g, out, err, path=path, layout=layout)
        else:
            B.bitlinear_forward_rowscale(xq, s, packed, gr, out, err, path=path, layout=layout)
        torch.cuda.synchronize()
        check_guard(out)
        assert err.item() == 0
        what = "M=%d N=%d K=%d layout=%d %s" % (M, N, K, layout, dt)
        if dt == torch.int32:
            got = out.cpu().numpy()
            assert np.array_equal(got[sel], acc_ref), "int32 accumulators differ: " + what
            if rows is not None:
                # every row: acc . v == x_q . (C^T v), in float64 on the device (integers
                # below 2^53, so exact)
                codes = torch.from_numpy(oracle.unpack(packed_ref, K)).to(DEV).to(torch.float64)
                v = torch.from_numpy(np.random.default_rng(M + N).integers(-3, 4, size=N).astype(np.float64)).to(DEV)
                lhs = out.to(torch.float64) @ v
                rhs = torch.from_numpy(xq_ref).to(DEV).to(torch.float64) @ (codes.T @ v)
                assert torch.equal(lhs, rhs), "linearity fails on some row: " + what
                del codes
        elif dt == torch.float32:
            assert_float_close(out.cpu().numpy()[sel], y_ref, "fp32 y " + what)
        else:
            yb = out.view(torch.int16).cpu().numpy().view(np.uint16)[sel]
            assert_bf16_match(yb, y_ref, oracle.f32_to_bf16(y_ref), "bf16 y " + what)


LAYOUTS = [B.BL_XQ_ROWMAJOR, B.BL_XQ_K16_EVENODD, B.BL_XQ_K16_STRIDE4]
ALL = (torch.int32, torch.float32, torch.bfloat16)

# (M, N, K): token tiles of 16, 32, 64 and 128 (and two of 128), ragged rows and tokens,
# K from one stage to 64 stages; few row tiles make the launcher split K over clusters
# of up to 8 blocks (N = 100 .. 2048), many row tiles (N >= 16384) split less or not
RAGGED = [(1, 1, 64), (5, 100, 192), (16, 128, 128), (17, 300, 640), (32, 1000, 1024), (33, 129, 4096),
          (48, 2048, 8192), (64, 4096, 1536), (65, 640, 320), (100, 256, 256), (128, 8192, 512),
          (129, 512, 1024), (3, 16384, 256), (64, 40000, 256)]


@pytest.mark.parametrize("layout", LAYOUTS, ids=["rowmajor", "evenodd", "stride4"])
@pytest.mark.parametrize("M,N,K", RAGGED)
def test_skinny_ragged(M, N, K, layout):
    g, packed, xq, s = problem(M, N, K, seed=M + 3 * N + K)
    run(xq, s, packed, g, layout, ALL)


@pytest.mark.parametrize("name,N,K", [("q", 8192, 8192), ("k", 1024, 8192), ("up", 28672, 8192),
                                      ("down", 8192, 28672)])
def test_skinny_llama70b_decode_batches(name, N, K):
    """The LLaMA-70B layer's projections at 17-64 tokens through the automatic dispatch
    with x_q in the stride-4 layout, as the benchmark runs them (the asynchronous-copy
    GEMV up to 32 tokens, this kernel above): sampled token rows against the oracle,
    every row through linearity; and the forced small-batch kernel at 32 tokens."""
    W = synth.weight(N, K, seed=N + K)
    g, _, packed = oracle.quantize_weights(W.numpy(), EPS)
    del W
    for M in (17, 32, 48, 64):
        X = synth.activations(M, K, seed=N + K + M, outlier_frac=0.01, outlier_scale=20.0)
        xq, s = oracle.quantize_act(bits(X), EPS)
        rows = np.unique(np.r_[0, M - 1, np.random.default_rng(M).integers(0, M, 1)])
        run(xq, s, packed, g, B.BL_XQ_K16_STRIDE4, ALL, rows=rows, path=B.BL_PATH_AUTO)
        if M == 32:
            run(xq, s, packed, g, B.BL_XQ_K16_STRIDE4, (torch.int32,), rows=rows, path=SK)


def test_skinny_extreme_accumulators():
    """|acc| = 128 K at K = 2^17 (the stride-4 kernels sum 64 * code, reaching 2^30), with
    and without a K split."""
    for M, N in ((20, 256), (64, 20000)):
        K = 1 << 17
        xq = torch.full((M, K), -128, dtype=torch.int8, device=DEV)
        xq[1::2] = 127
        packed = torch.full((N, K // 4), 0xAA, dtype=torch.uint8, device=DEV)  # all -1
        packed[::5] = 0x55                                                     # all +1
        want = (xq.long().sum(1)[:, None] * torch.where(torch.arange(N, device=DEV) % 5 == 0, 1, -1)[None, :])
        for layout in LAYOUTS:
            acc = B.forward(xq, torch.ones(M, device=DEV), packed, torch.ones(1, device=DEV), torch.int32,
                            path=SK, layout=layout)
            torch.cuda.synchronize()
            assert torch.equal(acc.long(), want), (M, N, layout)


def test_skinny_per_row_scales():
    """q/k/v-shaped stacked matrices, each with its own gamma, in one launch."""
    M, K = 40, 1536
    parts = [(1536, 1), (512, 2), (512, 3)]
    Ws = [synth.weight(n, K, seed=sd) for n, sd in parts]
    qs = [oracle.quantize_weights(W.numpy(), EPS) for W in Ws]
    packed = np.concatenate([q[2] for q in qs])
    gamma_rows = np.concatenate([np.full(n, q[0], dtype=np.float32) for (n, _), q in zip(parts, qs)])
    X = synth.activations(M, K, seed=9, outlier_frac=0.01)
    xq, s = oracle.quantize_act(bits(X), EPS)
    for layout in LAYOUTS:
        run(xq, s, packed, 1.0, layout, (torch.float32, torch.bfloat16), gamma_rows=gamma_rows)


@pytest.mark.parametrize("layout", LAYOUTS, ids=["rowmajor", "evenodd", "stride4"])
def test_skinny_reads_code_11_as_zero(layout):
    M, N, K = 33, 700, 2048
    rng = np.random.default_rng(layout + 7)
    packed = rng.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    xq = rng.integers(-128, 128, size=(M, K), dtype=np.int8)
    s = rng.uniform(0.5, 2.0, size=M).astype(np.float32)
    run(xq, s, packed, np.float32(0.03), layout, (torch.int32,))


def test_skinny_repeated_launches_after_act_quant():
    """Back-to-back launches, each right after an activation-quantisation launch on the
    same stream, give the same result every time."""
    M, N, K = 64, 8192, 28672
    g, packed_ref, xq_ref, s_ref = problem(M, N, K, seed=77)
    X = synth.activations(M, K, seed=77, outlier_frac=0.01, outlier_scale=20.0).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g], device=DEV)
    first = None
    for _ in range(6):
        xq, s = B.quantize_act(X, EPS, layout=B.BL_XQ_K16_STRIDE4)
        acc = B.forward(xq, s, packed, gamma, torch.int32, path=SK, layout=B.BL_XQ_K16_STRIDE4)
        torch.cuda.synchronize()
        if first is None:
            first = acc.clone()
            acc_ref = oracle.forward(xq_ref[:2], s_ref[:2], packed_ref, g, K, oracle.OUT_I32)
            assert np.array_equal(acc[:2].cpu().numpy(), acc_ref)
        assert torch.equal(acc, first)


def test_skinny_matches_other_paths():
    M, N, K = 24, 4800, 2048
    g, packed_ref, xq_ref, s_ref = problem(M, N, K, seed=21)
    s = torch.from_numpy(s_ref).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g], device=DEV)
    outs = []
    for layout in LAYOUTS:
        xl = np.empty_like(xq_ref)
        xl[:, positions(layout, K)] = xq_ref
        xd = torch.from_numpy(xl).to(DEV)
        for path in (B.BL_PATH_GEMV, B.BL_PATH_TC_1SM, SK):
            outs.append(B.forward(xd, s, packed, gamma, torch.int32, path=path, layout=layout))
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(outs[0], o)
