"""Parity of the decode GEMV fed by per-thread asynchronous copies (BL_PATH_GEMV_STREAM) with
the oracle, and agreement with the TMA-fed GEMV (BL_PATH_GEMV_TMA) and the small-batch
tcgen05 kernel where they apply.

Shapes span one, two and four token tiles (M = 1..16, then groups of 32 tokens up to
M = 64, with a ragged last group), ragged rows (N not a multiple of 16, blocks with
unequal tile counts, and layers with fewer tiles than SMs, whose K is split over a
cluster of blocks that add their partial sums through distributed shared memory), K with a partial last 256-code quarter (K % 256 = 64,
128, 192), the most tiles a block takes, the largest accumulators, per-row weight
scales and the undefined code 11.  Integers bit-exact, fp32 within 1e-5 relative /
1e-6 absolute, bf16 equal up to rounding-midpoint cases, and no write outside the
output."""
import functools

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
ST = B.BL_PATH_GEMV_STREAM
S4 = B.BL_XQ_K16_STRIDE4
ALL = (torch.int32, torch.float32, torch.bfloat16)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from ternary_weight_bit_absmean_b200 import build_lib
    build_lib.build()
    B.lib()


def stride4(xq):
    """x_q rows in the stride-4 k16 layout: inside each group of 16 the bytes hold the
    elements e = 0,4,8,12, 1,5,9,13, 2,6,10,14, 3,7,11,15."""
    M, K = xq.shape
    e = np.arange(16)
    order = (4 * (e % 4) + e // 4)  # element at byte position e
    return np.ascontiguousarray(xq.reshape(M, K // 16, 16)[:, :, order].reshape(M, K))


def problem(M, N, K, seed):
    W = synth.weight(N, K, seed=seed)
    X = synth.activations(M, K, seed=seed + 1, outlier_frac=0.01, outlier_scale=20.0)
    g, _, packed = oracle.quantize_weights(W.numpy(), EPS)
    xq, s = oracle.quantize_act(bits(X), EPS)
    return np.float32(g), packed, xq, s


def run(xq_ref, s_ref, packed_ref, gamma, dtypes=ALL, rows=None, path=ST, gamma_rows=None):
    M, K = xq_ref.shape
    N = packed_ref.shape[0]
    sel = np.arange(M) if rows is None else np.asarray(rows)
    acc_ref = oracle.forward(xq_ref[sel], s_ref[sel], packed_ref, gamma, K, oracle.OUT_I32)
    y_ref = (oracle.dequant(acc_ref, s_ref[sel], gamma) if gamma_rows is None
             else oracle.dequant_rows(acc_ref, s_ref[sel], gamma_rows))
    xq = torch.from_numpy(stride4(xq_ref)).to(DEV)
    s = torch.from_numpy(s_ref).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    g = torch.tensor([gamma], dtype=torch.float32, device=DEV)
    gr = None if gamma_rows is None else torch.from_numpy(gamma_rows).to(DEV)
    outs = {}
    for dt in dtypes:
        out = guarded_empty((M, N), dt)
        err = torch.zeros(1, dtype=torch.int32, device=DEV)
        if gr is None:
            B.bitlinear_forward(xq, s, packed, g, out, err, path=path, layout=S4)
        else:
            B.bitlinear_forward_rowscale(xq, s, packed, gr, out, err, path=path, layout=S4)
        torch.cuda.synchronize()
        check_guard(out)
        assert err.item() == 0
        what = "M=%d N=%d K=%d %s" % (M, N, K, dt)
        if dt == torch.int32:
            assert np.array_equal(out.cpu().numpy()[sel], acc_ref), "int32 accumulators differ: " + what
        elif dt == torch.float32:
            assert_float_close(out.cpu().numpy()[sel], y_ref, "fp32 y " + what)
        else:
            yb = out.view(torch.int16).cpu().numpy().view(np.uint16)[sel]
            assert_bf16_match(yb, y_ref, oracle.f32_to_bf16(y_ref), "bf16 y " + what)
        outs[dt] = out
    return outs


# (M, N, K): one token tile (M <= 8), two (9..16) and groups of 32; N from one row (one
# tile, K split over a cluster) through fewer tiles than SMs to several tiles per SM
# (ragged last tiles); K from one quarter to 40, with partial quarters; activations
# staged in shared memory or read from global memory
SHAPES = [(1, 2368, 64), (3, 2353, 192), (8, 2400, 320), (9, 3000, 1024), (16, 4737, 640), (2, 5000, 2112),
          (7, 9000, 4160), (12, 2400, 10048), (17, 2400, 1024), (32, 2368, 640), (33, 3000, 2112),
          (50, 2353, 320), (64, 4737, 1024),
          # fewer tiles than SMs: one tile per run, K split over a cluster of 2 to 8 blocks
          (1, 1024, 8192), (4, 16, 2048), (9, 300, 640), (1, 1536, 1536), (32, 1024, 8192), (17, 40, 256),
          (2, 1, 4096)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_stream_ragged(M, N, K):
    g, packed, xq, s = problem(M, N, K, seed=M * 7 + N + K)
    run(xq, s, packed, g)


@functools.lru_cache(maxsize=3)
def _layer_weights(N, K):
    W = synth.weight(N, K, seed=N + K)
    g, _, packed = oracle.quantize_weights(W.numpy(), EPS)
    return g, packed


@pytest.mark.parametrize("N,K", [(28672, 8192), (8192, 28672), (8192, 8192)])
@pytest.mark.parametrize("M", [1, 4, 8, 16, 32, 64])
def test_stream_llama70b_decode(M, N, K):
    """The LLaMA-70B layer's wide projections at decode token counts: every row in int32
    against the oracle for M = 1, sampled rows otherwise, and equality on every element
    with the TMA-fed GEMV (M <= 16) or the small-batch tcgen05 kernel (M > 16)."""
    g, packed = _layer_weights(N, K)
    X = synth.activations(M, K, seed=N + K + M, outlier_frac=0.01, outlier_scale=20.0)
    xq, s = oracle.quantize_act(bits(X), EPS)
    rows = None if M == 1 else np.unique(np.r_[0, M - 1, np.random.default_rng(M).integers(0, M, 1)])
    outs = run(xq, s, packed, np.float32(g), dtypes=(torch.int32, torch.bfloat16), rows=rows)
    xd = torch.from_numpy(stride4(xq)).to(DEV)
    other = B.forward(xd, torch.from_numpy(s).to(DEV), torch.from_numpy(packed).to(DEV),
                      torch.tensor([g], device=DEV), torch.int32,
                      path=B.BL_PATH_GEMV_TMA if M <= 16 else B.BL_PATH_SKINNY, layout=S4)
    torch.cuda.synchronize()
    assert torch.equal(outs[torch.int32], other)


def test_stream_most_tiles_per_block():
    """64 tiles per block on every SM (N = SMs * 64 * 16 rows), the kernel's limit, and
    one tile more is refused."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    N, K, M = sms * 64 * 16, 128, 5
    g, packed, xq, s = problem(M, N, K, seed=3)
    run(xq, s, packed, g, dtypes=(torch.int32, torch.float32))
    xd = torch.zeros(M, K, dtype=torch.int8, device=DEV)
    big = torch.zeros(N + 16, K // 4, dtype=torch.uint8, device=DEV)
    with pytest.raises(B.BitLinearError, match="UNSUPPORTED_SHAPE"):
        B.forward(xd, torch.ones(M, device=DEV), big, torch.ones(1, device=DEV), torch.int32, path=ST, layout=S4)


def test_stream_extreme_accumulators():
    """|acc| = 128 K at K = 2^17: the unpack sums 64 * code, reaching 2^30."""
    K, N = 1 << 17, 2400
    for M in (3, 16):
        xq = torch.full((M, K), -128, dtype=torch.int8, device=DEV)
        xq[1::2] = 127
        packed = torch.full((N, K // 4), 0xAA, dtype=torch.uint8, device=DEV)  # all -1
        packed[::5] = 0x55                                                     # all +1
        want = (xq.long().sum(1)[:, None] * torch.where(torch.arange(N, device=DEV) % 5 == 0, 1, -1)[None, :])
        acc = B.forward(xq, torch.ones(M, device=DEV), packed, torch.ones(1, device=DEV), torch.int32, path=ST,
                        layout=S4)  # constant rows: the same in every layout
        torch.cuda.synchronize()
        assert torch.equal(acc.long(), want), M


def test_stream_per_row_scales():
    """Stacked matrices (q/k/v-like), each with its own gamma, in one launch."""
    M, K = 6, 1536
    parts = [(1536, 1), (512, 2), (512, 3)]
    qs = [oracle.quantize_weights(synth.weight(n, K, seed=sd).numpy(), EPS) for n, sd in parts]
    packed = np.concatenate([q[2] for q in qs])
    gamma_rows = np.concatenate([np.full(n, q[0], dtype=np.float32) for (n, _), q in zip(parts, qs)])
    X = synth.activations(M, K, seed=9, outlier_frac=0.01)
    xq, s = oracle.quantize_act(bits(X), EPS)
    run(xq, s, packed, np.float32(1.0), dtypes=(torch.float32, torch.bfloat16), gamma_rows=gamma_rows)


def test_stream_reads_code_11_as_zero():
    M, N, K = 11, 2500, 1024
    rng = np.random.default_rng(11)
    packed = rng.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    xq = rng.integers(-128, 128, size=(M, K), dtype=np.int8)
    s = rng.uniform(0.5, 2.0, size=M).astype(np.float32)
    run(xq, s, packed, np.float32(0.03), dtypes=(torch.int32,))


def test_stream_repeated_launches_after_act_quant():
    """Back-to-back launches, each right after an activation-quantisation launch on the
    same stream, give the same result every time."""
    M, N, K = 8, 28672, 8192
    g, packed_ref, xq_ref, s_ref = problem(M, N, K, seed=77)
    X = synth.activations(M, K, seed=78, outlier_frac=0.01, outlier_scale=20.0).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g], device=DEV)
    first = None
    for _ in range(6):
        xq, s = B.quantize_act(X, EPS, layout=S4)
        acc = B.forward(xq, s, packed, gamma, torch.int32, path=ST, layout=S4)
        torch.cuda.synchronize()
        if first is None:
            first = acc.clone()
            acc_ref = oracle.forward(xq_ref[:2], s_ref[:2], packed_ref, g, K, oracle.OUT_I32)
            assert np.array_equal(acc[:2].cpu().numpy(), acc_ref)
        assert torch.equal(acc, first)


def test_stream_refuses_other_layouts_and_shapes():
    xq = torch.zeros(4, 256, dtype=torch.int8, device=DEV)
    s = torch.ones(4, device=DEV)
    gamma = torch.ones(1, device=DEV)
    wide = torch.zeros(4096, 64, dtype=torch.uint8, device=DEV)
    for packed, layout, M in ((wide, B.BL_XQ_ROWMAJOR, 4), (wide, B.BL_XQ_K16_EVENODD, 4)):
        with pytest.raises(B.BitLinearError, match="UNSUPPORTED_SHAPE"):
            B.forward(xq[:M], s[:M], packed, gamma, torch.int32, path=ST, layout=layout)
    x65 = torch.zeros(65, 256, dtype=torch.int8, device=DEV)
    with pytest.raises(B.BitLinearError, match="UNSUPPORTED_SHAPE"):
        B.forward(x65, torch.ones(65, device=DEV), wide, gamma, torch.int32, path=ST, layout=S4)
