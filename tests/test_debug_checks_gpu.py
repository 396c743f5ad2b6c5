"""The debugging build (`build_lib.build(debug=True)`, `libbitlinear_debug.so`): the same
library with the device index checks on (BL_DEBUG_CHECKS=1), which record an index
outside its buffer as BL_ERRBIT_INDEX in the error word and skip the access instead of
trapping.  On correct kernels no check fails: the small-batch tcgen05 kernel, the one
that carries the checks, runs ragged shapes with and without its K split and must match
the oracle bit for bit with an error word of zero."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import EPS, bits
from ternary_weight_bit_absmean_b200 import binding as B
from ternary_weight_bit_absmean_b200 import build_lib, synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

DEV = "cuda"


@pytest.fixture(scope="module")
def debug_lib():
    """Loads the debugging build in place of the normal one for this module's tests."""
    path = build_lib.build(debug=True)
    saved = (B.LIB_PATH, B._lib)
    B.LIB_PATH, B._lib = path, None
    B.lib()
    yield path
    B.LIB_PATH, B._lib = saved


@pytest.mark.parametrize("M,N,K", [(17, 300, 640), (33, 129, 4096), (64, 4096, 1536), (48, 2048, 8192),
                                   (100, 256, 256), (3, 16384, 256)])
def test_debug_build_small_batch_kernel(debug_lib, M, N, K):
    W = synth.weight(N, K, seed=M + N + K)
    X = synth.activations(M, K, seed=M + N + K, outlier_frac=0.01, outlier_scale=20.0)
    g, _, packed_ref = oracle.quantize_weights(W.numpy(), EPS)
    xq_ref, s_ref = oracle.quantize_act(bits(X), EPS)
    acc_ref = oracle.forward(xq_ref, s_ref, packed_ref, g, K, oracle.OUT_I32)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    acc = B.forward(torch.from_numpy(xq_ref).to(DEV), torch.from_numpy(s_ref).to(DEV),
                    torch.from_numpy(packed_ref).to(DEV), torch.tensor([g], device=DEV), torch.int32,
                    path=B.BL_PATH_SKINNY, err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0, "index check failed: err_word = %#x" % err.item()
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
