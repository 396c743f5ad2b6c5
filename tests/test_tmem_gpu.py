"""Parity of the tiled tcgen05 forward with the expanded weights in tensor memory
(BL_PATH_TC_TMEM) with the oracle: ragged shapes in every x_q layout and output kind, every
token tile it picks, the LLaMA-3B prefill shapes on sampled rows (every row through
linearity), the largest accumulators, per-row weight scales, undefined code 11, repeated
launches, agreement with the shared-memory kernels, and the bounded waits.

Integers bit-exact, fp32 within 1e-5 relative / 1e-6 absolute, bf16 equal up to
rounding-midpoint cases, and no write outside the output."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import EPS, bits, check_guard, guarded_empty
from test_skinny_gpu import ALL, LAYOUTS, positions, problem, run
from ternary_weight_bit_absmean_b200 import binding as B
from ternary_weight_bit_absmean_b200 import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

DEV = "cuda"
TM = B.BL_PATH_TC_TMEM


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from ternary_weight_bit_absmean_b200 import build_lib
    build_lib.build()
    B.lib()


# (M, N, K): ragged tokens and features, K from one stage to 32 stages with a ragged
# 64-code tail; M and N chosen so that the launcher's token tiles (64 ... 192) and the
# persistent blocks' tile counts (below, at and above one per SM) all occur
RAGGED = [(17, 1, 64), (65, 100, 192), (100, 300, 320), (129, 128, 4096), (300, 1000, 1024), (513, 640, 1536),
          (1000, 2048, 4160), (2048, 1536, 256), (4096, 384, 512), (777, 3200, 3200)]


@pytest.mark.parametrize("layout", LAYOUTS, ids=["rowmajor", "evenodd", "stride4"])
@pytest.mark.parametrize("M,N,K", RAGGED)
def test_tmem_ragged(M, N, K, layout):
    g, packed, xq, s = problem(M, N, K, seed=M + 5 * N + K)
    run(xq, s, packed, g, layout, ALL, path=TM)


@pytest.mark.parametrize("M", [2048, 8192])
@pytest.mark.parametrize("name,N,K", [("q", 3200, 3200), ("up", 8640, 3200), ("down", 3200, 8640)])
def test_tmem_llama3b_prefill(name, N, K, M):
    """The LLaMA-3B projections at 2048 and 8192 tokens, stride-4 x_q (as the benchmark
    runs them): sampled token rows against the oracle, every row through linearity."""
    g, packed, xq, s = problem(M, N, K, seed=N + K + M)
    rows = np.unique(np.r_[0, M - 1, np.random.default_rng(M).integers(0, M, 3)])
    run(xq, s, packed, g, B.BL_XQ_K16_STRIDE4, ALL, rows=rows, path=TM)


def test_tmem_extreme_accumulators():
    """|acc| = 128 K at K = 2^17: the stride-4 sums of 64 * code reach 2^30."""
    M, N, K = 200, 640, 1 << 17
    xq = torch.full((M, K), -128, dtype=torch.int8, device=DEV)
    xq[1::2] = 127
    packed = torch.full((N, K // 4), 0xAA, dtype=torch.uint8, device=DEV)  # all -1
    packed[::5] = 0x55                                                     # all +1
    want = (xq.long().sum(1)[:, None] * torch.where(torch.arange(N, device=DEV) % 5 == 0, 1, -1)[None, :])
    for layout in LAYOUTS:
        acc = B.forward(xq, torch.ones(M, device=DEV), packed, torch.ones(1, device=DEV), torch.int32,
                        path=TM, layout=layout)
        torch.cuda.synchronize()
        assert torch.equal(acc.long(), want), layout


def test_tmem_per_row_scales():
    M, K = 300, 1536
    parts = [(1536, 1), (512, 2), (512, 3)]
    Ws = [synth.weight(n, K, seed=sd) for n, sd in parts]
    qs = [oracle.quantize_weights(W.numpy(), EPS) for W in Ws]
    packed = np.concatenate([q[2] for q in qs])
    gamma_rows = np.concatenate([np.full(n, q[0], dtype=np.float32) for (n, _), q in zip(parts, qs)])
    X = synth.activations(M, K, seed=19, outlier_frac=0.01)
    xq, s = oracle.quantize_act(bits(X), EPS)
    for layout in LAYOUTS:
        run(xq, s, packed, 1.0, layout, (torch.float32, torch.bfloat16), path=TM, gamma_rows=gamma_rows)


@pytest.mark.parametrize("layout", LAYOUTS, ids=["rowmajor", "evenodd", "stride4"])
def test_tmem_reads_code_11_as_zero(layout):
    M, N, K = 300, 700, 2048
    rng = np.random.default_rng(layout + 11)
    packed = rng.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    xq = rng.integers(-128, 128, size=(M, K), dtype=np.int8)
    s = rng.uniform(0.5, 2.0, size=M).astype(np.float32)
    run(xq, s, packed, np.float32(0.03), layout, (torch.int32,), path=TM)


def test_tmem_matches_shared_memory_kernels_repeatedly():
    M, N, K = 4096, 1536, 4096
    g, packed_ref, xq_ref, s_ref = problem(M, N, K, seed=5)
    xl = np.empty_like(xq_ref)
    xl[:, positions(B.BL_XQ_K16_STRIDE4, K)] = xq_ref
    xq = torch.from_numpy(xl).to(DEV)
    s = torch.from_numpy(s_ref).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g], device=DEV)
    want = B.forward(xq, s, packed, gamma, torch.int32, path=B.BL_PATH_TC_2SM, layout=B.BL_XQ_K16_STRIDE4)
    for _ in range(5):
        acc = B.forward(xq, s, packed, gamma, torch.int32, path=TM, layout=B.BL_XQ_K16_STRIDE4)
        torch.cuda.synchronize()
        assert torch.equal(acc, want)


def test_tmem_bounded_wait_runs_out_then_next_call_is_exact():
    M, N, K = 512, 1024, 4096
    g, packed_ref, xq_ref, s_ref = problem(M, N, K, seed=8)
    xq = torch.from_numpy(xq_ref).to(DEV)
    s = torch.from_numpy(s_ref).to(DEV)
    packed = torch.from_numpy(packed_ref).to(DEV)
    gamma = torch.tensor([g], device=DEV)
    out = guarded_empty((M, N), torch.int32)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    B.bitlinear_forward_stall_test(xq, s, packed, gamma, out, err, 1_000_000, 3, path=TM)
    torch.cuda.synchronize()
    check_guard(out)
    assert err.item() & B.BL_ERRBIT_TIMEOUT
    acc_ref = oracle.forward(xq_ref[:4], s_ref[:4], packed_ref, g, K, oracle.OUT_I32)
    err.zero_()
    acc = B.forward(xq, s, packed, gamma, torch.int32, path=TM, err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert np.array_equal(acc[:4].cpu().numpy(), acc_ref)
