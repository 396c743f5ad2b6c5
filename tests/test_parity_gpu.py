"""Parity of the CUDA path (through the C ABI) with the CPU oracle on the same seeded
inputs.  Integer and byte results (packed codes, x_q, int32 accumulators) must be
bit-exact; gamma within 1e-6 relative; float outputs within 1e-5 relative / 1e-6
absolute; bf16 outputs equal the oracle's except next to a rounding midpoint."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (EPS, assert_bf16_match, assert_float_close, bits, check_guard,
                      guarded_empty)
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


def sync():
    torch.cuda.synchronize()


# ----------------------------------------------------------- activations (a4) --

ACT_SHAPES = [(1, 1), (3, 7), (5, 100), (2, 4), (17, 8), (8192, 256), (4096, 1536), (512, 4096),
              (64, 3200), (16, 8640), (8, 8192), (3, 28672), (33, 1032), (7, 36000)]


@pytest.mark.parametrize("M,K", ACT_SHAPES)
def test_quantize_act_bit_exact(M, K):
    X = synth.activations(M, K, seed=M * 7 + K, outlier_frac=0.01, outlier_scale=20.0)
    if M > 2:
        X[1] = 0  # an all-zero token
    xq_ref, s_ref = oracle.quantize_act(bits(X), EPS)
    Xd = X.to(DEV)
    xq = guarded_empty((M, K), torch.int8)
    s = guarded_empty((M,), torch.float32)
    B.bitlinear_quantize_act(Xd, EPS, xq, s)
    sync()
    check_guard(xq)
    check_guard(s)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(xq.cpu().numpy(), xq_ref)


def test_quantize_act_tiny_rows_use_eps():
    X = torch.full((4, 64), 1e-7, dtype=torch.float32).to(torch.bfloat16)
    xq_ref, s_ref = oracle.quantize_act(bits(X), EPS)
    xq, s = B.quantize_act(X.to(DEV), EPS)
    sync()
    assert np.array_equal(s.cpu().numpy(), s_ref) and np.array_equal(xq.cpu().numpy(), xq_ref)


# ------------------------------------------------------- weights (a1, a2, a3) --

W_SHAPES = [(1, 4), (3, 12), (7, 20), (512, 256), (1536, 1536), (4096, 1536), (1536, 4096),
            (3200, 3200), (8640, 3200), (1024, 8192), (33, 1000)]


@pytest.mark.parametrize("N,K", W_SHAPES)
def test_quantize_weights(N, K):
    W = synth.weight(N, K, seed=N + 3 * K)
    g_ref, codes_ref, packed_ref = oracle.quantize_weights(W.numpy(), EPS)
    Wd = W.to(DEV)
    gamma = torch.empty(1, dtype=torch.float32, device=DEV)
    packed = guarded_empty((N, K // 4), torch.uint8)
    ws = torch.empty(B.bitlinear_workspace_size(N, K), dtype=torch.uint8, device=DEV)
    B.bitlinear_quantize_weights(Wd, EPS, gamma, packed, ws)
    sync()
    check_guard(packed)
    g = np.float32(gamma.item())
    assert abs(float(g) - float(g_ref)) <= 1e-6 * float(g_ref)
    # codes are compared with the oracle's gamma through the given-scale entry
    g_dev = torch.tensor([g_ref], dtype=torch.float32, device=DEV)
    packed2 = guarded_empty((N, K // 4), torch.uint8)
    B.bitlinear_quantize_weights_with_scale(Wd, g_dev, packed2)
    sync()
    check_guard(packed2)
    assert np.array_equal(packed2.cpu().numpy(), packed_ref)
    if g == g_ref:
        assert np.array_equal(packed.cpu().numpy(), packed_ref)
    # gamma is reproducible from run to run
    gamma2 = torch.empty(1, dtype=torch.float32, device=DEV)
    B.bitlinear_quantize_weights(Wd, EPS, gamma2, packed, ws)
    sync()
    assert gamma2.item() == gamma.item()


def test_quantize_weights_given_scale_ties_and_zero_share():
    # weights on the +-gamma/2 rounding boundary and beyond the clip
    gamma = np.float32(0.0625)
    row = np.array([0.03125, -0.03125, 0.09375, -0.09375, 0.5, -0.5, 0.0, 0.0312500037] * 2, np.float32)
    W = torch.from_numpy(np.tile(row, (3, 1)))
    want, _ = oracle.pack(oracle.ternarise(W.numpy(), gamma))
    packed = torch.empty(3, 4, dtype=torch.uint8, device=DEV)
    B.bitlinear_quantize_weights_with_scale(W.to(DEV), torch.tensor([gamma], device=DEV), packed)
    sync()
    assert np.array_equal(packed.cpu().numpy(), want)
    # zero-code share of the 50% / 70% mixtures (reported by the oracle) is reproduced
    for frac in (0.378, 0.664):
        Wm = synth.weight(256, 1024, seed=5, small_frac=frac)
        g_ref, codes, packed_ref = oracle.quantize_weights(Wm.numpy(), EPS)
        g_dev, p_dev = B.quantize_weights(Wm.to(DEV), EPS)
        sync()
        pk = oracle.unpack(p_dev.cpu().numpy(), 1024)
        assert abs(float(np.mean(pk == 0)) - float(np.mean(codes == 0))) < 1e-3


def test_zero_weights():
    W = torch.zeros(64, 256, device=DEV)
    gamma, packed = B.quantize_weights(W, EPS)
    sync()
    assert gamma.item() == np.float32(EPS) and not packed.any().item()


@pytest.mark.parametrize("N,K", [(1, 4), (5, 12), (64, 256), (1536, 4096), (7, 100)])
def test_pack_codes(N, K):
    c = synth.codes(N, K, seed=N * K)
    want, bad = oracle.pack(c.numpy())
    assert bad == 0
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    packed = guarded_empty((N, K // 4), torch.uint8)
    B.bitlinear_pack(c.to(DEV), packed, err)
    sync()
    check_guard(packed)
    assert err.item() == 0
    assert np.array_equal(packed.cpu().numpy(), want)


def test_pack_reports_bad_codes():
    c = synth.codes(16, 64, seed=3)
    c[3, 5] = 2
    c[9, 63] = -100
    want, bad = oracle.pack(c.numpy())
    assert bad == 2
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    packed = torch.empty(16, 16, dtype=torch.uint8, device=DEV)
    B.bitlinear_pack(c.to(DEV), packed, err)
    sync()
    assert err.item() & B.BL_ERRBIT_BAD_CODE
    assert np.array_equal(packed.cpu().numpy(), want)


# ------------------------------------------------------------ forward (a5-a7) --

def make_problem(M, N, K, seed, zero_row=False):
    W = synth.weight(N, K, seed=seed)
    X = synth.activations(M, K, seed=seed, outlier_frac=0.01, outlier_scale=20.0)
    if zero_row and M > 1:
        X[M // 2] = 0
    g_ref, _, packed_ref = oracle.quantize_weights(W.numpy(), EPS)
    xq_ref, s_ref = oracle.quantize_act(bits(X), EPS)
    return g_ref, packed_ref, xq_ref, s_ref


def run_forward(xq_ref, s_ref, packed_ref, g_ref, out_dtype, path):
    M, K = xq_ref.shape
    N = packed_ref.shape[0]
    xq = torch.from_numpy(xq_ref).to(DEV)
    s = torch.from_numpy(s_ref).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g_ref], dtype=torch.float32, device=DEV)
    out = guarded_empty((M, N), out_dtype)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    B.bitlinear_forward(xq, s, packed, gamma, out, err, path=path)
    sync()
    check_guard(out)
    assert err.item() == 0
    return out


def check_forward(M, N, K, path, seed=0, rows=None, zero_row=True):
    g_ref, packed_ref, xq_ref, s_ref = make_problem(M, N, K, seed, zero_row)
    sel = np.arange(M) if rows is None else np.asarray(rows)
    acc_ref = oracle.forward(xq_ref[sel], s_ref[sel], packed_ref, g_ref, K, oracle.OUT_I32)
    y_ref = oracle.dequant(acc_ref, s_ref[sel], g_ref)
    yb_ref = oracle.f32_to_bf16(y_ref)
    acc = run_forward(xq_ref, s_ref, packed_ref, g_ref, torch.int32, path).cpu().numpy()
    assert np.array_equal(acc[sel], acc_ref), "int32 accumulators differ"
    y = run_forward(xq_ref, s_ref, packed_ref, g_ref, torch.float32, path).cpu().numpy()
    assert_float_close(y[sel], y_ref, "fp32 y")
    yb = run_forward(xq_ref, s_ref, packed_ref, g_ref, torch.bfloat16, path)
    yb = yb.view(torch.int16).cpu().numpy().view(np.uint16)
    assert_bf16_match(yb[sel], y_ref, yb_ref, "bf16 y")
    if rows is not None:
        # every row: the integer accumulators are linear in x_q, so the product of the
        # accumulator matrix with a random vector equals x_q times (codes^T times it)
        codes = oracle.unpack(packed_ref, K).astype(np.int64)
        v = np.random.default_rng(seed).integers(-3, 4, size=N).astype(np.int64)
        assert np.array_equal(acc.astype(np.int64) @ v, xq_ref.astype(np.int64) @ (codes.T @ v))


GEMV_CASES = [(1, 1, 64), (1, 256, 64), (2, 300, 192), (3, 512, 256), (8, 1536, 1536),
              (9, 100, 320), (16, 4096, 1536), (16, 3200, 8640), (5, 1024, 8192), (1, 8192, 8192),
              (13, 8640, 3200), (16, 1000, 4160), (40, 200, 256)]


@pytest.mark.parametrize("M,N,K", GEMV_CASES)
def test_forward_gemv(M, N, K):
    check_forward(M, N, K, B.BL_PATH_GEMV, seed=M + N + K)


TC_CASES = [(17, 128, 128), (32, 256, 256), (64, 512, 256), (100, 300, 192), (256, 128, 1536),
            (300, 200, 320), (512, 1536, 1536), (513, 4096, 1536), (1000, 1536, 4096),
            (8192, 512, 256), (130, 640, 8192), (1792, 2304, 320), (1536, 2304, 192)]


@pytest.mark.parametrize("path", [B.BL_PATH_TC_1SM, B.BL_PATH_TC_2SM], ids=["tc1sm", "tc2sm"])
@pytest.mark.parametrize("M,N,K", TC_CASES)
def test_forward_tc(M, N, K, path):
    check_forward(M, N, K, path, seed=M * 3 + N + K)


@pytest.mark.parametrize("M,N,K", [(1, 64, 100), (3, 33, 4), (20, 17, 36), (5, 7, 1000)])
def test_forward_generic_k(M, N, K):
    """K % 64 != 0 runs the plain kernel through the automatic dispatch."""
    check_forward(M, N, K, B.BL_PATH_AUTO, seed=M + 2 * N + K)


def test_forward_paths_agree_and_are_deterministic():
    g_ref, packed_ref, xq_ref, s_ref = make_problem(300, 768, 2048, 11)
    outs = [run_forward(xq_ref, s_ref, packed_ref, g_ref, torch.int32, p)
            for p in (B.BL_PATH_GEMV, B.BL_PATH_TC_1SM, B.BL_PATH_TC_2SM, B.BL_PATH_TC, B.BL_PATH_TC_2SM)]
    for o in outs[1:]:
        assert torch.equal(outs[0], o)


def test_forward_zero_weights_give_zero():
    M, N, K = 300, 256, 512
    xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=DEV)
    s = torch.ones(M, device=DEV)
    packed = torch.zeros(N, K // 4, dtype=torch.uint8, device=DEV)
    gamma = torch.tensor([EPS], device=DEV)
    for path in (B.BL_PATH_GEMV, B.BL_PATH_TC_1SM, B.BL_PATH_TC_2SM):
        y = B.forward(xq, s, packed, gamma, torch.float32, path=path)
        sync()
        assert not y.any().item()


def test_forward_extreme_accumulators():
    """All codes +1 against x_q = -128 or +127 everywhere: |acc| reaches 128 K."""
    M, N, K = 64, 256, 8192
    xq = torch.full((M, K), 127, dtype=torch.int8, device=DEV)
    xq[::2] = -128
    packed = torch.full((N, K // 4), 0x55, dtype=torch.uint8, device=DEV)  # all +1
    packed[::3] = 0xAA                                                     # all -1
    s = torch.ones(M, device=DEV)
    gamma = torch.tensor([1.0], device=DEV)
    want = (xq.long().sum(1)[:, None] * torch.where(torch.arange(N, device=DEV) % 3 == 0, -1, 1)[None, :])
    for path in (B.BL_PATH_GEMV, B.BL_PATH_TC_1SM, B.BL_PATH_TC_2SM):
        acc = B.forward(xq, s, packed, gamma, torch.int32, path=path)
        sync()
        assert torch.equal(acc.long(), want)


# -------------------------------------------------- the workloads' own sizes --

@pytest.mark.parametrize("name", ["toy", "llama700m", "llama3b", "llama70b"])
def test_workload_sizes(name):
    """Every projection of each workload at its decode and prefill token counts, in the
    configuration the benchmark times (automatic dispatch, x_q in the stride-4 k16
    layout) and with row-major x_q; large problems are checked on sampled token rows."""
    spec = synth.WORKLOADS[name]
    projs = spec["proj"]
    if name == "llama70b":
        projs = [p for p in projs if p[0] in ("k", "up", "down")]
    for pi, (pname, N, K) in enumerate(projs):
        W = synth.weight(N, K, seed=pi)
        g_ref, _, packed_ref = oracle.quantize_weights(W.numpy(), EPS)
        g_dev, p_dev = B.quantize_weights(W.to(DEV), EPS)
        sync()
        assert abs(g_dev.item() - float(g_ref)) <= 1e-6 * float(g_ref)
        if g_dev.item() == float(g_ref):
            assert np.array_equal(p_dev.cpu().numpy(), packed_ref)
        Ms = spec["M"] if name != "llama70b" else [1, 16, 64]
        for M in Ms:
            X = synth.activations(M, K, seed=pi + 100 * M, outlier_frac=spec["outlier_frac"])
            xq_ref, s_ref = oracle.quantize_act(bits(X), EPS)
            xq, s = B.quantize_act(X.to(DEV), EPS)
            xq4, s4 = B.quantize_act(X.to(DEV), EPS, layout=B.BL_XQ_K16_STRIDE4)
            sync()
            assert np.array_equal(xq.cpu().numpy(), xq_ref) and np.array_equal(s.cpu().numpy(), s_ref)
            assert np.array_equal(xq4.cpu().numpy()[:, stride4_positions(K)], xq_ref)
            assert np.array_equal(s4.cpu().numpy(), s_ref)
            rows = np.arange(M) if M * N * K <= 4e9 else np.unique(
                np.r_[0, M - 1, np.random.default_rng(M).integers(0, M, 6)])
            acc_ref = oracle.forward(xq_ref[rows], s_ref[rows], packed_ref, g_ref, K, oracle.OUT_I32)
            y_ref = oracle.dequant(acc_ref, s_ref[rows], g_ref)
            gamma = torch.tensor([g_ref], device=DEV)
            pk = torch.from_numpy(packed_ref).to(DEV)
            for lay, xl, sl in ((B.BL_XQ_ROWMAJOR, xq, s), (B.BL_XQ_K16_STRIDE4, xq4, s4)):
                acc = B.forward(xl, sl, pk, gamma, torch.int32, layout=lay).cpu().numpy()
                y = B.forward(xl, sl, pk, gamma, torch.float32, layout=lay).cpu().numpy()
                assert np.array_equal(acc[rows], acc_ref), (name, pname, M, lay)
                assert_float_close(y[rows], y_ref, "%s %s M=%d layout %d" % (name, pname, M, lay))


# ------------------------------------------------ x_q in the k16 layouts --

def stride4_positions(K):
    """Byte position of every element k in the stride-4 k16 layout, built from the
    layout's definition: inside each group of 16 the element order is
    0,4,8,12, 1,5,9,13, 2,6,10,14, 3,7,11,15."""
    order = [0, 4, 8, 12, 1, 5, 9, 13, 2, 6, 10, 14, 3, 7, 11, 15]
    pos = np.empty(K, dtype=np.int64)
    for q in range(K // 16):
        for p, e in enumerate(order):
            pos[16 * q + e] = 16 * q + p
    return pos


def evenodd_positions(K):
    """Byte position of every element k in the even/odd k16 layout, built from the
    layout's definition: inside each group of 16 the element order is
    0,2,4,6, 8,10,12,14, 1,3,5,7, 9,11,13,15."""
    order = [0, 2, 4, 6, 8, 10, 12, 14, 1, 3, 5, 7, 9, 11, 13, 15]
    pos = np.empty(K, dtype=np.int64)
    for q in range(K // 16):
        for p, e in enumerate(order):
            pos[16 * q + e] = 16 * q + p
    return pos


@pytest.mark.parametrize("M,K", [(1, 16), (5, 1536), (33, 4096), (4096, 1536), (3, 28672), (64, 208)])
def test_quantize_act_evenodd_layout(M, K):
    X = synth.activations(M, K, seed=M + 11 * K)
    xq_ref, s_ref = oracle.quantize_act(bits(X), EPS)
    xq = guarded_empty((M, K), torch.int8)
    s = guarded_empty((M,), torch.float32)
    B.bitlinear_quantize_act(X.to(DEV), EPS, xq, s, layout=B.BL_XQ_K16_EVENODD)
    sync()
    check_guard(xq)
    check_guard(s)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    got = xq.cpu().numpy()
    assert np.array_equal(got[:, evenodd_positions(K)], xq_ref)


EO_CASES = [(1, 300, 256, B.BL_PATH_GEMV), (16, 4096, 1536, B.BL_PATH_GEMV), (9, 640, 4160, B.BL_PATH_GEMV),
            (40, 200, 256, B.BL_PATH_GEMV), (5, 64, 208, B.BL_PATH_AUTO), (100, 300, 192, B.BL_PATH_TC_1SM),
            (513, 4096, 1536, B.BL_PATH_TC_1SM), (300, 200, 320, B.BL_PATH_TC_2SM),
            (1000, 1536, 4096, B.BL_PATH_TC_2SM), (4096, 1536, 1536, B.BL_PATH_TC)]


@pytest.mark.parametrize("M,N,K,path", EO_CASES)
def test_forward_evenodd_layout(M, N, K, path):
    g_ref, packed_ref, xq_ref, s_ref = make_problem(M, N, K, seed=M + N + 7 * K, zero_row=True)
    acc_ref = oracle.forward(xq_ref, s_ref, packed_ref, g_ref, K, oracle.OUT_I32)
    y_ref = oracle.dequant(acc_ref, s_ref, g_ref)
    xq_eo = np.empty_like(xq_ref)
    xq_eo[:, evenodd_positions(K)] = xq_ref
    xq = torch.from_numpy(xq_eo).to(DEV)
    s = torch.from_numpy(s_ref).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g_ref], device=DEV)
    for dt in (torch.int32, torch.float32):
        out = guarded_empty((M, N), dt)
        B.bitlinear_forward(xq, s, packed, gamma, out, path=path, layout=B.BL_XQ_K16_EVENODD)
        sync()
        check_guard(out)
        if dt == torch.int32:
            assert np.array_equal(out.cpu().numpy(), acc_ref)
        else:
            assert_float_close(out.cpu().numpy(), y_ref, "evenodd fp32")


@pytest.mark.parametrize("M,K", [(1, 16), (5, 1536), (33, 4096), (4096, 1536), (3, 28672), (64, 208)])
def test_quantize_act_stride4_layout(M, K):
    X = synth.activations(M, K, seed=M + 13 * K)
    xq_ref, s_ref = oracle.quantize_act(bits(X), EPS)
    xq = guarded_empty((M, K), torch.int8)
    s = guarded_empty((M,), torch.float32)
    B.bitlinear_quantize_act(X.to(DEV), EPS, xq, s, layout=B.BL_XQ_K16_STRIDE4)
    sync()
    check_guard(xq)
    check_guard(s)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(xq.cpu().numpy()[:, stride4_positions(K)], xq_ref)


def run_layout_forward(xq_ref, s_ref, packed_ref, g_ref, layout, positions, path, dtypes, rows=None):
    M, K = xq_ref.shape
    N = packed_ref.shape[0]
    sel = np.arange(M) if rows is None else np.asarray(rows)
    acc_ref = oracle.forward(xq_ref[sel], s_ref[sel], packed_ref, g_ref, K, oracle.OUT_I32)
    y_ref = oracle.dequant(acc_ref, s_ref[sel], g_ref)
    xl = np.empty_like(xq_ref)
    xl[:, positions] = xq_ref
    xq = torch.from_numpy(xl).to(DEV)
    s = torch.from_numpy(s_ref).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g_ref], device=DEV)
    for dt in dtypes:
        out = guarded_empty((M, N), dt)
        err = torch.zeros(1, dtype=torch.int32, device=DEV)
        B.bitlinear_forward(xq, s, packed, gamma, out, err, path=path, layout=layout)
        sync()
        check_guard(out)
        assert err.item() == 0
        if dt == torch.int32:
            assert np.array_equal(out.cpu().numpy()[sel], acc_ref), "int32 accumulators differ"
        elif dt == torch.float32:
            assert_float_close(out.cpu().numpy()[sel], y_ref, "fp32 y")
        else:
            yb = out.view(torch.int16).cpu().numpy().view(np.uint16)[sel]
            assert_bf16_match(yb, y_ref, oracle.f32_to_bf16(y_ref), "bf16 y")


# (M, N, K, path): the persistent TMA decode kernel takes M <= 16 with at least one
# 16-row tile per SM; N picks how many tiles each SM owns (1, 2, 4, 13, 18, 32) and so
# how warps share tile pairs; K covers partial 512-code units and ragged 128-code tails
S4_CASES = [(1, 2368, 128, B.BL_PATH_GEMV), (1, 4096, 1536, B.BL_PATH_GEMV), (16, 8192, 640, B.BL_PATH_GEMV),
            (8, 28672, 1536, B.BL_PATH_GEMV), (9, 3001, 3200, B.BL_PATH_GEMV), (2, 40000, 1024, B.BL_PATH_GEMV),
            (16, 75000, 256, B.BL_PATH_GEMV), (3, 9000, 8192, B.BL_PATH_AUTO), (1, 300, 256, B.BL_PATH_GEMV),
            (40, 200, 256, B.BL_PATH_GEMV), (5, 64, 208, B.BL_PATH_AUTO), (100, 300, 192, B.BL_PATH_TC_1SM),
            (513, 4096, 1536, B.BL_PATH_TC_1SM), (300, 200, 320, B.BL_PATH_TC_2SM),
            (1000, 1536, 4096, B.BL_PATH_TC_2SM), (4096, 1536, 1536, B.BL_PATH_TC), (17, 128, 128, B.BL_PATH_TC_1SM)]


@pytest.mark.parametrize("M,N,K,path", S4_CASES)
def test_forward_stride4_layout(M, N, K, path):
    g_ref, packed_ref, xq_ref, s_ref = make_problem(M, N, K, seed=M + N + 5 * K, zero_row=True)
    run_layout_forward(xq_ref, s_ref, packed_ref, g_ref, B.BL_XQ_K16_STRIDE4, stride4_positions(K), path,
                       (torch.int32, torch.float32, torch.bfloat16))


@pytest.mark.parametrize("layout", [B.BL_XQ_ROWMAJOR, B.BL_XQ_K16_EVENODD, B.BL_XQ_K16_STRIDE4],
                         ids=["rowmajor", "evenodd", "stride4"])
@pytest.mark.parametrize("M,N,K,path", [(1, 2400, 1024, B.BL_PATH_GEMV), (16, 512, 512, B.BL_PATH_GEMV),
                                        (200, 384, 512, B.BL_PATH_TC_1SM), (300, 512, 512, B.BL_PATH_TC_2SM)])
def test_forward_reads_code_11_as_zero(M, N, K, path, layout):
    """Packed bytes drawn uniformly from 0..255 hold the unused code 11 in a quarter of
    the fields; every kernel must read it as 0, as the oracle does."""
    rng = np.random.default_rng(M + N + K + layout)
    packed_ref = rng.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    xq_ref = rng.integers(-128, 128, size=(M, K), dtype=np.int8)
    s_ref = rng.uniform(0.5, 2.0, size=M).astype(np.float32)
    pos = {B.BL_XQ_ROWMAJOR: np.arange(K), B.BL_XQ_K16_EVENODD: evenodd_positions(K),
           B.BL_XQ_K16_STRIDE4: stride4_positions(K)}[layout]
    run_layout_forward(xq_ref, s_ref, packed_ref, np.float32(0.03), layout, pos, path, (torch.int32,))


def test_forward_stride4_extreme_accumulators_and_k_limit():
    """The stride-4 kernels sum 64 * code: at K = 2^17 with |x_q| = 128 and every code -1
    the scaled sums reach 2^30 and must still be exact; above 2^17 the tensor-core paths
    refuse the shape and the automatic dispatch runs the unscaled GEMV."""
    N = 2400
    for M, K, path in ((1, 1 << 17, B.BL_PATH_GEMV), (16, 1 << 15, B.BL_PATH_GEMV), (200, 1 << 17, B.BL_PATH_TC_1SM),
                       (300, 1 << 17, B.BL_PATH_TC_2SM), (16, (1 << 17) + 128, B.BL_PATH_AUTO)):
        xq = torch.full((M, K), -128, dtype=torch.int8, device=DEV)
        xq[1::2] = 127
        packed = torch.full((N, K // 4), 0xAA, dtype=torch.uint8, device=DEV)  # all -1
        packed[::5] = 0x55                                                     # all +1
        s = torch.ones(M, device=DEV)
        gamma = torch.tensor([1.0], device=DEV)
        # the layout only permutes x_q inside each 16-group; a row of equal bytes is unchanged
        want = (xq.long().sum(1)[:, None] * torch.where(torch.arange(N, device=DEV) % 5 == 0, 1, -1)[None, :])
        acc = B.forward(xq, s, packed, gamma, torch.int32, path=path, layout=B.BL_XQ_K16_STRIDE4)
        sync()
        assert torch.equal(acc.long(), want), (M, K, path)
    xq = torch.zeros((200, (1 << 17) + 128), dtype=torch.int8, device=DEV)
    packed = torch.zeros((256, xq.shape[1] // 4), dtype=torch.uint8, device=DEV)
    with pytest.raises(B.BitLinearError, match="UNSUPPORTED_SHAPE"):
        B.forward(xq, torch.ones(200, device=DEV), packed, torch.ones(1, device=DEV), torch.int32,
                  path=B.BL_PATH_TC, layout=B.BL_XQ_K16_STRIDE4)


def test_forward_all_paths_and_layouts_agree():
    M, N, K = 16, 4800, 2048
    g_ref, packed_ref, xq_ref, s_ref = make_problem(M, N, K, 21)
    xq = torch.from_numpy(xq_ref).to(DEV)
    s = torch.from_numpy(s_ref).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g_ref], device=DEV)
    outs = []
    for layout, pos in ((B.BL_XQ_ROWMAJOR, np.arange(K)), (B.BL_XQ_K16_EVENODD, evenodd_positions(K)),
                        (B.BL_XQ_K16_STRIDE4, stride4_positions(K))):
        xl = np.empty_like(xq_ref)
        xl[:, pos] = xq_ref
        xd = torch.from_numpy(xl).to(DEV)
        for path in (B.BL_PATH_GEMV, B.BL_PATH_TC_1SM, B.BL_PATH_TC_2SM):
            outs.append(B.forward(xd, s, packed, gamma, torch.int32, path=path, layout=layout))
    sync()
    for o in outs[1:]:
        assert torch.equal(outs[0], o)


@pytest.mark.parametrize("M", [16, 8])
def test_forward_stride4_wide_layer_repeated(M):
    """The LLaMA-70B up projection (28672 x 8192) on the persistent decode kernel, where
    blocks own 12 or 13 tiles and some warps own no tile pair: repeated launches, each
    right after an activation-quantisation launch, must all match the oracle (a warp
    that released stages it did not read once let a stage be refilled under a slower
    pair)."""
    N, K = 28672, 8192
    g_ref, packed_ref, xq_ref, s_ref = make_problem(M, N, K, seed=M + 3)
    acc_ref = oracle.forward(xq_ref, s_ref, packed_ref, g_ref, K, oracle.OUT_I32)
    X = synth.activations(M, K, seed=M + 3, outlier_frac=0.01, outlier_scale=20.0).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g_ref], device=DEV)
    for _ in range(6):
        xq, s = B.quantize_act(X, EPS, layout=B.BL_XQ_K16_STRIDE4)
        acc = B.forward(xq, s, packed, gamma, torch.int32, path=B.BL_PATH_GEMV, layout=B.BL_XQ_K16_STRIDE4)
        sync()
        assert np.array_equal(acc.cpu().numpy(), acc_ref)


# ------------------------------------- normalisation fused into the quantiser --

NORM_SHAPES = [(1, 16), (3, 40), (5, 1536), (33, 4096), (4096, 1536), (7, 8192), (2, 8208), (2, 12288), (3, 28672),
               (2, 36000)]


@pytest.mark.parametrize("M,K", NORM_SHAPES)
@pytest.mark.parametrize("kind", [B.BL_NORM_RMS, B.BL_NORM_LAYER], ids=["rms", "layer"])
def test_norm_quantize_act(M, K, kind):
    X = synth.activations(M, K, seed=M + 3 * K + kind, outlier_frac=0.01, outlier_scale=20.0)
    if kind == B.BL_NORM_LAYER:
        X = (X.float() + 0.75).to(torch.bfloat16)  # a nonzero mean for LayerNorm to remove
    w = torch.from_numpy(np.random.default_rng(M + K).uniform(0.5, 1.5, size=K).astype(np.float32))
    layouts = [B.BL_XQ_ROWMAJOR] + ([B.BL_XQ_K16_EVENODD, B.BL_XQ_K16_STRIDE4] if K % 16 == 0 else [])
    for weight in (None, w):
        xq_ref, s_ref, _ = oracle.norm_quantize_act(bits(X), None if weight is None else weight.numpy(), kind,
                                                    1e-5, EPS)
        for lay in layouts:
            xq = guarded_empty((M, K), torch.int8)
            s = guarded_empty((M,), torch.float32)
            B.bitlinear_norm_quantize_act(X.to(DEV), None if weight is None else weight.to(DEV), kind, 1e-5, EPS,
                                          xq, s, layout=lay)
            sync()
            check_guard(xq)
            check_guard(s)
            assert np.array_equal(s.cpu().numpy(), s_ref), (kind, lay, weight is None)
            pos = {B.BL_XQ_ROWMAJOR: np.arange(K), B.BL_XQ_K16_EVENODD: None, B.BL_XQ_K16_STRIDE4: None}[lay]
            if lay == B.BL_XQ_K16_EVENODD:
                pos = evenodd_positions(K)
            elif lay == B.BL_XQ_K16_STRIDE4:
                pos = stride4_positions(K)
            assert np.array_equal(xq.cpu().numpy()[:, pos], xq_ref), (kind, lay, weight is None)


def test_norm_quantize_act_edge_rows():
    """Zero tokens, a constant token and tiny tokens (norm_eps dominates)."""
    M, K = 6, 256
    X = synth.activations(M, K, seed=5).float()
    X[0] = 0.0
    X[1] = 3.0
    X[2] *= 1e-6
    X = X.to(torch.bfloat16)
    for kind in (B.BL_NORM_RMS, B.BL_NORM_LAYER):
        xq_ref, s_ref, _ = oracle.norm_quantize_act(bits(X), None, kind, 1e-5, EPS)
        xq, s = B.norm_quantize_act(X.to(DEV), None, kind, 1e-5, EPS)
        sync()
        assert np.array_equal(s.cpu().numpy(), s_ref) and np.array_equal(xq.cpu().numpy(), xq_ref), kind


def test_norm_quantize_then_forward():
    """The fused quantiser feeding the forward, against the same two oracle steps."""
    M, N, K = 8, 2400, 1024
    X = synth.activations(M, K, seed=9, outlier_frac=0.01, outlier_scale=20.0)
    W = synth.weight(N, K, seed=9)
    w = torch.from_numpy(np.random.default_rng(9).uniform(0.5, 1.5, size=K).astype(np.float32))
    g_ref, _, packed_ref = oracle.quantize_weights(W.numpy(), EPS)
    xq_ref, s_ref, _ = oracle.norm_quantize_act(bits(X), w.numpy(), B.BL_NORM_RMS, 1e-5, EPS)
    acc_ref = oracle.forward(xq_ref, s_ref, packed_ref, g_ref, K, oracle.OUT_I32)
    y_ref = oracle.dequant(acc_ref, s_ref, g_ref)
    xq, s = B.norm_quantize_act(X.to(DEV), w.to(DEV), B.BL_NORM_RMS, 1e-5, EPS, layout=B.BL_XQ_K16_STRIDE4)
    pk = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g_ref], device=DEV)
    acc = B.forward(xq, s, pk, gamma, torch.int32, layout=B.BL_XQ_K16_STRIDE4)
    y = B.forward(xq, s, pk, gamma, torch.float32, layout=B.BL_XQ_K16_STRIDE4)
    sync()
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_float_close(y.cpu().numpy(), y_ref, "norm + forward fp32")


# ------------------------------------- stacked matrices, one scale per output row --

@pytest.mark.parametrize("M,path,layout", [
    (1, B.BL_PATH_GEMV, B.BL_XQ_K16_STRIDE4), (8, B.BL_PATH_GEMV, B.BL_XQ_ROWMAJOR),
    (16, B.BL_PATH_GEMV, B.BL_XQ_K16_STRIDE4), (40, B.BL_PATH_GEMV, B.BL_XQ_ROWMAJOR),
    (300, B.BL_PATH_TC_1SM, B.BL_XQ_K16_STRIDE4), (300, B.BL_PATH_TC_2SM, B.BL_XQ_K16_STRIDE4),
    (700, B.BL_PATH_TC, B.BL_XQ_ROWMAJOR), (5, B.BL_PATH_AUTO, B.BL_XQ_K16_EVENODD)])
def test_forward_rowscale_stacked_matrices(M, path, layout):
    """q, k and v stacked along N (1536 + 512 + 512 rows; the 2560-row stack puts the
    decode case on the persistent kernel), each with its own absmean gamma: one launch
    against the oracle's per-row rescale."""
    K = 1024
    parts = [synth.weight(n, K, seed=40 + i) for i, n in enumerate((1536, 512, 512))]
    packs, grows = [], []
    for W in parts:
        g, _, p = oracle.quantize_weights(W.numpy(), EPS)
        packs.append(p)
        grows.append(np.full(W.shape[0], g, dtype=np.float32))
    packed_ref = np.concatenate(packs, axis=0)
    gamma_rows = np.concatenate(grows)
    N = packed_ref.shape[0]
    X = synth.activations(M, K, seed=M + 41, outlier_frac=0.01, outlier_scale=20.0)
    xq_ref, s_ref = oracle.quantize_act(bits(X), EPS)
    acc_ref = oracle.forward(xq_ref, s_ref, packed_ref, 1.0, K, oracle.OUT_I32)
    y_ref = oracle.dequant_rows(acc_ref, s_ref, gamma_rows)
    pos = {B.BL_XQ_ROWMAJOR: np.arange(K), B.BL_XQ_K16_EVENODD: evenodd_positions(K),
           B.BL_XQ_K16_STRIDE4: stride4_positions(K)}[layout]
    xl = np.empty_like(xq_ref)
    xl[:, pos] = xq_ref
    xq = torch.from_numpy(xl).to(DEV)
    s = torch.from_numpy(s_ref).to(DEV)
    pk = torch.from_numpy(packed_ref).to(DEV)
    gr = torch.from_numpy(gamma_rows).to(DEV)
    for dt in (torch.int32, torch.float32, torch.bfloat16):
        out = guarded_empty((M, N), dt)
        err = torch.zeros(1, dtype=torch.int32, device=DEV)
        B.bitlinear_forward_rowscale(xq, s, pk, gr, out, err, path=path, layout=layout)
        sync()
        check_guard(out)
        assert err.item() == 0
        if dt == torch.int32:
            assert np.array_equal(out.cpu().numpy(), acc_ref)
        elif dt == torch.float32:
            assert_float_close(out.cpu().numpy(), y_ref, "rowscale fp32")
        else:
            yb = out.view(torch.int16).cpu().numpy().view(np.uint16)
            assert_bf16_match(yb, y_ref, oracle.f32_to_bf16(y_ref), "rowscale bf16")


def test_forward_rowscale_equal_scales_match_single_scale():
    """With every row's scale equal to gamma, the per-row forward is the single-gamma
    forward bit for bit, on every path."""
    M, N, K = 300, 768, 512
    g_ref, packed_ref, xq_ref, s_ref = make_problem(M, N, K, seed=12)
    xq = torch.from_numpy(xq_ref).to(DEV)
    s = torch.from_numpy(s_ref).to(DEV)
    pk = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g_ref], device=DEV)
    gr = torch.full((N,), float(g_ref), device=DEV)
    for path in (B.BL_PATH_GEMV, B.BL_PATH_TC_1SM, B.BL_PATH_TC_2SM):
        a = guarded_empty((M, N), torch.float32)
        b = guarded_empty((M, N), torch.float32)
        B.bitlinear_forward(xq, s, pk, gamma, a, path=path)
        B.bitlinear_forward_rowscale(xq, s, pk, gr, b, path=path)
        sync()
        assert torch.equal(a, b), path


# ------------------------------------------ 1.6-bit weights, five codes per byte --

TL5_PACK_SHAPES = [(1, 16), (3, 80), (5, 96), (7, 1040), (64, 4096), (33, 8192), (2, 28672), (300, 1536)]


@pytest.mark.parametrize("N,K", TL5_PACK_SHAPES)
def test_pack_tl5_and_repack(N, K):
    """Packing int8 codes and converting the 2-bit format give the oracle's bytes."""
    c = synth.codes(N, K, seed=N + K).numpy()
    want, bad = oracle.pack_tl5(c)
    assert bad == 0
    out = guarded_empty(want.shape, torch.uint8)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    B.bitlinear_pack_tl5(torch.from_numpy(c).to(DEV), out, err)
    sync()
    check_guard(out)
    assert err.item() == 0
    assert np.array_equal(out.cpu().numpy(), want)
    packed2, _ = oracle.pack(c)
    out2 = guarded_empty(want.shape, torch.uint8)
    B.bitlinear_repack_tl5(torch.from_numpy(packed2).to(DEV), out2)
    sync()
    check_guard(out2)
    assert np.array_equal(out2.cpu().numpy(), want)


def test_pack_tl5_flags_bad_codes_and_repack_reads_code_11_as_zero():
    c = synth.codes(4, 160, seed=5).numpy().copy()
    c[1, 17], c[3, 159] = 3, -2
    want, bad = oracle.pack_tl5(c)
    assert bad == 2
    out = torch.empty(want.shape, dtype=torch.uint8, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    B.bitlinear_pack_tl5(torch.from_numpy(c).to(DEV), out, err)
    sync()
    assert err.item() & B.BL_ERRBIT_BAD_CODE
    assert np.array_equal(out.cpu().numpy(), want)
    # a 2-bit byte of 0xFF holds four codes 11, read as 0
    packed2, _ = oracle.pack(np.zeros((2, 64), np.int8))
    packed2[0, 3] = 0xFF
    packed2[1, 15] = 0xBF  # 10 11 11 11: -1 then three codes 11
    ref_codes = oracle.unpack(packed2, 64)
    want2, _ = oracle.pack_tl5(ref_codes)
    out2 = torch.empty(want2.shape, dtype=torch.uint8, device=DEV)
    B.bitlinear_repack_tl5(torch.from_numpy(packed2).to(DEV), out2)
    sync()
    assert np.array_equal(out2.cpu().numpy(), want2)


def _tl5_forward(xq_ref, s_ref, tl5_ref, g_ref, out_dtype):
    M, K = xq_ref.shape
    N = tl5_ref.shape[0]
    out = guarded_empty((M, N), out_dtype)
    B.bitlinear_forward_tl5(torch.from_numpy(xq_ref).to(DEV), torch.from_numpy(s_ref).to(DEV),
                            torch.from_numpy(tl5_ref).to(DEV),
                            torch.tensor([g_ref], dtype=torch.float32, device=DEV), out)
    sync()
    check_guard(out)
    return out


def check_forward_tl5(xq_ref, s_ref, tl5_ref, g_ref, rows=None):
    K = xq_ref.shape[1]
    sel = np.arange(xq_ref.shape[0]) if rows is None else np.asarray(rows)
    acc_ref = oracle.forward_tl5(xq_ref[sel], s_ref[sel], tl5_ref, g_ref, K, oracle.OUT_I32)
    y_ref = oracle.dequant(acc_ref, s_ref[sel], g_ref)
    acc = _tl5_forward(xq_ref, s_ref, tl5_ref, g_ref, torch.int32).cpu().numpy()
    assert np.array_equal(acc[sel], acc_ref), "int32 accumulators differ"
    y = _tl5_forward(xq_ref, s_ref, tl5_ref, g_ref, torch.float32).cpu().numpy()
    assert_float_close(y[sel], y_ref, "fp32 y")
    yb = _tl5_forward(xq_ref, s_ref, tl5_ref, g_ref, torch.bfloat16).view(torch.int16).cpu().numpy().view(np.uint16)
    assert_bf16_match(yb[sel], y_ref, oracle.f32_to_bf16(y_ref), "bf16 y")
    return acc


TL5_FWD_CASES = [(1, 1, 16), (1, 37, 80), (2, 100, 96), (3, 300, 1040), (4, 1536, 1536), (5, 1000, 4096),
                 (8, 4096, 1536), (13, 3200, 8640), (16, 8192, 512), (17, 200, 1536), (40, 64, 8192),
                 (1, 3, 28672)]


@pytest.mark.parametrize("M,N,K", TL5_FWD_CASES)
def test_forward_tl5(M, N, K):
    g_ref, packed_ref, xq_ref, s_ref = make_problem(M, N, K, seed=7 * M + N + K)
    tl5_ref, _ = oracle.pack_tl5(oracle.unpack(packed_ref, K))
    check_forward_tl5(xq_ref, s_ref, tl5_ref, g_ref)


def test_forward_tl5_reads_every_byte_value():
    """Arbitrary bytes, including the 13 values packing never writes: the forward reads
    each as the oracle does (and ignores the missing planes of a partial last block)."""
    rng = np.random.default_rng(31)
    for M, N, K in ((1, 64, 400), (3, 50, 1040), (16, 33, 96)):
        tl5 = rng.integers(0, 256, size=(N, oracle.tl5_row_bytes(K))).astype(np.uint8)
        tl5[:, :16] = np.arange(256, dtype=np.uint16).reshape(16, 16)[np.arange(N) % 16].astype(np.uint8)
        xq = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
        s = rng.uniform(0.5, 50.0, size=M).astype(np.float32)
        check_forward_tl5(xq, s, tl5, 0.0213)


def test_forward_tl5_extreme_accumulators():
    """x_q = -128 against all +1 and all -1 rows: |acc| = 128 K at the int32 limit's side."""
    K = 16 * 8192
    xq = np.full((2, K), -128, dtype=np.int8)
    c = np.zeros((3, K), dtype=np.int8)
    c[0] = 1
    c[1] = -1
    c[2, ::2] = 1
    tl5, _ = oracle.pack_tl5(c)
    s = np.array([1.0, 3.0], dtype=np.float32)
    acc = check_forward_tl5(xq, s, tl5, 0.5)
    assert acc[0, 0] == -128 * K and acc[0, 1] == 128 * K and acc[0, 2] == -64 * K


@pytest.mark.parametrize("M,N,K", [(1, 28672, 8192), (4, 8192, 28672), (16, 8640, 3200)])
def test_forward_tl5_full_size_matches_2bit_path(M, N, K):
    """At full layer sizes: the five-per-byte forward equals the 2-bit decode forward bit
    for bit (same exact accumulators, same rescale), and sampled rows equal the oracle."""
    W = synth.weight(N, K, seed=N + K)
    X = synth.activations(M, K, seed=M + K, outlier_frac=0.01, outlier_scale=20.0)
    gamma, packed = B.quantize_weights(W.to(DEV), EPS)
    xq, s = B.quantize_act(X.to(DEV), EPS)
    tl5 = B.repack_tl5(packed)
    for dt in (torch.int32, torch.float32, torch.bfloat16):
        y5 = B.forward_tl5(xq, s, tl5, gamma, dt)
        y2 = B.forward(xq, s, packed, gamma, dt, path=B.BL_PATH_GEMV)
        sync()
        assert torch.equal(y5, y2), dt
    sel = np.array([0, M - 1])
    acc = B.forward_tl5(xq, s, tl5, gamma, torch.int32).cpu().numpy()
    codes = oracle.unpack_tl5(tl5.cpu().numpy(), K)
    cols = np.random.default_rng(3).choice(N, size=64, replace=False)
    acc_ref = oracle.int_matmul(xq.cpu().numpy()[sel], codes[cols])
    assert np.array_equal(acc[np.ix_(sel, cols)], acc_ref)


# ------------------------------------------------ straight-through backward (STE) --

def _ste_inputs(M, N, K, seed):
    W = synth.weight(N, K, seed=seed)
    X = synth.activations(M, K, seed=seed + 1, outlier_frac=0.01, outlier_scale=20.0)
    g_ref, _, packed_ref = oracle.quantize_weights(W.numpy(), EPS)
    xq_ref, s_ref = oracle.quantize_act(bits(X), EPS)
    dY = (torch.randn(M, N, generator=torch.Generator().manual_seed(seed + 2)) * 1e-3).numpy()
    return g_ref, packed_ref, xq_ref, s_ref, dY


def _assert_within_sum_bound(got, want, abs_terms, n_terms, gamma, what, split_err=2.0 ** -16, precise=False):
    """|got - want| <= gamma (e + (2n + 2) 2^-22) sum|terms| + 2^-24 |want|.  The kernels
    carry each fp32 factor as two bf16 parts (hi + lo) within e = 2^-16 relative (plus
    2^-23 for dW's rounded reciprocal), multiply both parts by exact bf16 operands and
    sum the 2n exact products in fp32 on the tensor cores, whose order and rounding are
    not specified: 2^-22 per addition covers rounding or truncation.  The final product
    by gamma rounds once.  With `precise`, the largest error relative to gamma sum|terms|
    must also stay below 2^-17: a typical split-bf16 result is far inside that, while one
    bf16 rounding of the fp32 factor (2^-9 per term) lands far outside it at these sizes."""
    scale = float(gamma) * abs_terms
    bound = (split_err + (2 * n_terms + 2) * 2.0 ** -22) * scale + 2.0 ** -24 * np.abs(want) + 1e-30
    err = np.abs(got.astype(np.float64) - want.astype(np.float64))
    assert (err <= bound).all(), (what, float((err / bound).max()))
    if precise:
        rel = float((err / (scale + 1e-30)).max())
        assert rel < 2.0 ** -17, (what, "largest relative error %g" % rel)


STE_CASES = [(1, 1, 4), (3, 17, 36), (64, 64, 64), (65, 100, 132), (7, 1536, 1536), (130, 300, 1000),
             (200, 130, 516), (257, 64, 1028)]


@pytest.mark.parametrize("M,N,K", STE_CASES)
def test_ste_backward(M, N, K):
    g, packed, xq, s, dY = _ste_inputs(M, N, K, seed=M + 2 * N + 3 * K)
    gd = torch.tensor([g], dtype=torch.float32, device=DEV)
    dX = guarded_empty((M, K), torch.float32)
    dW = guarded_empty((N, K), torch.float32)
    B.bitlinear_ste_backward_input(torch.from_numpy(dY).to(DEV), torch.from_numpy(packed).to(DEV), gd, dX)
    B.bitlinear_ste_backward_weight(torch.from_numpy(dY).to(DEV), torch.from_numpy(xq).to(DEV),
                                    torch.from_numpy(s).to(DEV), gd, dW)
    sync()
    check_guard(dX)
    check_guard(dW)
    codes = oracle.unpack(packed, K).astype(np.float64)
    big = min(M, N) >= 64
    _assert_within_sum_bound(dX.cpu().numpy(), oracle.ste_grad_input(dY, packed, g, K),
                             np.abs(dY.astype(np.float64)) @ np.abs(codes), N, g, "dX", precise=big and N >= 64)
    xs = np.abs(xq.astype(np.float64) / s.astype(np.float64)[:, None])
    _assert_within_sum_bound(dW.cpu().numpy(), oracle.ste_grad_weight(dY, xq, s, g),
                             np.abs(dY.astype(np.float64)).T @ xs, M, g, "dW", split_err=2.0 ** -16 + 2.0 ** -23,
                             precise=big and M >= 64)


@pytest.mark.parametrize("M,N,K", [(4096, 1536, 1536), (4096, 4096, 1536), (2048, 1536, 4096)])
def test_ste_backward_full_size_sampled(M, N, K):
    """LLaMA-700M-shaped projections at 2048-4096 tokens: sampled rows of dX and dW
    against the oracle (which sees only those rows / output features)."""
    g, packed, xq, s, dY = _ste_inputs(M, N, K, seed=11 + N)
    gd = torch.tensor([g], dtype=torch.float32, device=DEV)
    dX, dW = B.ste_backward(torch.from_numpy(dY).to(DEV), torch.from_numpy(packed).to(DEV),
                            torch.from_numpy(xq).to(DEV), torch.from_numpy(s).to(DEV), gd)
    sync()
    rm = np.array([0, 1, M // 2 - 1, M - 1])
    codes = oracle.unpack(packed, K).astype(np.float64)
    _assert_within_sum_bound(dX.cpu().numpy()[rm], oracle.ste_grad_input(dY[rm], packed, g, K),
                             np.abs(dY[rm].astype(np.float64)) @ np.abs(codes), N, g, "dX rows", precise=True)
    rn = np.array([0, 777, N - 1])
    xs = np.abs(xq.astype(np.float64) / s.astype(np.float64)[:, None])
    want = oracle.ste_grad_weight(np.ascontiguousarray(dY[:, rn]), xq, s, g)
    _assert_within_sum_bound(dW.cpu().numpy()[rn], want, np.abs(dY[:, rn].astype(np.float64)).T @ xs, M, g,
                             "dW rows", split_err=2.0 ** -16 + 2.0 ** -23, precise=True)


# ------------------------------------------------------------ bounded device waits --

@pytest.mark.parametrize("path,M,N,K,layout", [
    (B.BL_PATH_TC_1SM, 256, 1024, 4096, B.BL_XQ_K16_STRIDE4),
    (B.BL_PATH_TC_1SM, 300, 640, 2048, B.BL_XQ_ROWMAJOR),
    (B.BL_PATH_SKINNY, 32, 1024, 4096, B.BL_XQ_K16_STRIDE4),
    (B.BL_PATH_SKINNY, 64, 40000, 1024, B.BL_XQ_ROWMAJOR),
    (B.BL_PATH_GEMV, 4, 4736, 32768, B.BL_XQ_K16_STRIDE4),
], ids=["tc1-stride4", "tc1-rowmajor", "skinny-split", "skinny-nosplit", "gemv-tma"])
def test_bounded_wait_runs_out_then_next_call_is_exact(path, M, N, K, layout):
    """Each block's load producer stops after 3 loads and every wait is limited to 1 ms:
    the waits for the fourth load run out, the kernel drains what is in flight, frees its
    tensor memory and reports BL_ERRBIT_TIMEOUT.  The context stays usable: the next
    normal call on the same stream matches the oracle bit for bit."""
    g_ref, packed_ref, xq_ref, s_ref = make_problem(M, N, K, seed=M + N + K)
    pos = {B.BL_XQ_ROWMAJOR: np.arange(K), B.BL_XQ_K16_STRIDE4: stride4_positions(K)}[layout]
    xl = np.empty_like(xq_ref)
    xl[:, pos] = xq_ref
    xq = torch.from_numpy(xl).to(DEV)
    s = torch.from_numpy(s_ref).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g_ref], device=DEV)
    out = guarded_empty((M, N), torch.int32)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    B.bitlinear_forward_stall_test(xq, s, packed, gamma, out, err, 1_000_000, 3, path=path, layout=layout)
    sync()
    check_guard(out)
    assert err.item() & B.BL_ERRBIT_TIMEOUT
    rows = np.unique(np.r_[0, M - 1, np.random.default_rng(M).integers(0, M, 4)])
    acc_ref = oracle.forward(xq_ref[rows], s_ref[rows], packed_ref, g_ref, K, oracle.OUT_I32)
    for _ in range(2):
        err.zero_()
        acc = B.forward(xq, s, packed, gamma, torch.int32, path=path, layout=layout, err_word=err)
        sync()
        assert err.item() == 0
        assert np.array_equal(acc.cpu().numpy()[rows], acc_ref)


def test_bounded_wait_test_rejects_other_paths_and_limits():
    xq = torch.zeros(32, 256, dtype=torch.int8, device=DEV)
    s = torch.ones(32, device=DEV)
    packed = torch.zeros(256, 64, dtype=torch.uint8, device=DEV)
    gamma = torch.ones(1, device=DEV)
    out = torch.empty(32, 256, dtype=torch.int32, device=DEV)
    for path, limit, stall in ((B.BL_PATH_TC_2SM, 1000, 1), (B.BL_PATH_TC_1SM, 0, 1), (B.BL_PATH_TC_1SM, 1000, -1),
                               (B.BL_PATH_TC_1SM, 3_000_000_000, 1)):
        with pytest.raises(B.BitLinearError, match="INVALID_ARG"):
            B.bitlinear_forward_stall_test(xq, s, packed, gamma, out, None, limit, stall, path=path)
    with pytest.raises(B.BitLinearError, match="UNSUPPORTED_SHAPE"):  # no TMA-fed GEMV at this size
        B.bitlinear_forward_stall_test(xq[:4], s[:4], packed, gamma, out[:4], None, 1000, 1, path=B.BL_PATH_GEMV,
                                       layout=B.BL_XQ_K16_STRIDE4)


# ------------------------------------------------- reused buffers, other shapes --

def test_tensor_core_paths_reuse_buffers_with_other_shapes():
    """The same device buffers viewed with different shapes in turn (the launchers keep
    recently encoded tensor maps, keyed by address and shape): every call matches the
    oracle, including a shape repeated after another one used the same addresses."""
    xbuf = torch.empty(1 << 20, dtype=torch.int8, device=DEV)
    pbuf = torch.empty(1 << 20, dtype=torch.uint8, device=DEV)
    shapes = [(300, 256, 1024), (200, 512, 512), (300, 256, 1024), (129, 384, 640)]
    for i, (M, N, K) in enumerate(shapes):
        g_ref, packed_ref, xq_ref, s_ref = make_problem(M, N, K, seed=40 + i)
        xq = xbuf[:M * K].view(M, K)
        xq.copy_(torch.from_numpy(xq_ref))
        packed = pbuf[:N * K // 4].view(N, K // 4)
        packed.copy_(torch.from_numpy(packed_ref))
        s = torch.from_numpy(s_ref).to(DEV)
        gamma = torch.tensor([g_ref], device=DEV)
        acc_ref = oracle.forward(xq_ref, s_ref, packed_ref, g_ref, K, oracle.OUT_I32)
        for path in (B.BL_PATH_TC_1SM, B.BL_PATH_TC_2SM, B.BL_PATH_SKINNY):
            acc = B.forward(xq, s, packed, gamma, torch.int32, path=path)
            sync()
            assert np.array_equal(acc.cpu().numpy(), acc_ref), (M, N, K, path)
