"""GPU test of bitlinear_quantize_weights_noalloc, the weight-quantisation entry point
for callers that cannot allocate device memory (a serving loop that must not call
cudaMalloc, a plug-in whose host framework owns every device allocation, a deployment
with a fixed memory budget).  It keeps its fp64 partial sums in a fixed array inside the
library instead of a caller workspace.

The test calls the new entry point through the C ABI and compares gamma and the packed
codes with those of bitlinear_quantize_weights (the workspace entry point) on the same
weights, for two calls in a row: a large matrix and then a small one, so the second
call runs with the first call's partial sums still in the shared array.  Both entry
points run the same two kernels with the same number of partial sums, summed in the
same fixed order, so gamma must be bit-identical.  Around the second call, device memory
in use (the driver's free-memory count and PyTorch's allocator) must not change.  It
lives in a file of its own, collected last, and passes alone in a fresh process too.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

EPS = 1e-5


def noalloc_entry():
    from ternary_weight_bit_absmean_b200 import binding, build_lib
    build_lib.build()
    f = binding.lib().bitlinear_quantize_weights_noalloc
    P = ctypes.c_void_p
    f.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_float, P, P, P]
    f.restype = ctypes.c_int
    return f


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row():
    from ternary_weight_bit_absmean_b200 import binding as B
    from ternary_weight_bit_absmean_b200 import synth

    f = noalloc_entry()
    dev = torch.device("cuda")
    stream = torch.cuda.current_stream().cuda_stream
    # first a matrix that uses every partial slot, then one that uses very few
    for i, (N, K) in enumerate([(8640, 3200), (33, 100)]):
        W = synth.weight(N, K, seed=40 + i).to(dev)
        g_ref, p_ref = B.quantize_weights(W, EPS)
        gamma = torch.full((1,), -1.0, dtype=torch.float32, device=dev)
        packed = torch.full((N, K // 4), 0xFF, dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()
        free_before, _ = torch.cuda.mem_get_info()
        torch_before = torch.cuda.memory_allocated()
        status = f(W.data_ptr(), N, K, EPS, gamma.data_ptr(), packed.data_ptr(), stream)
        assert status == 0, B.lib().bitlinear_status_string(status)
        torch.cuda.synchronize()
        if i == 1:
            # the module (and its array) is loaded by now: this call must allocate nothing
            free_after, _ = torch.cuda.mem_get_info()
            assert free_after == free_before, (free_before, free_after)
            assert torch.cuda.memory_allocated() == torch_before
        assert torch.equal(gamma, g_ref), (gamma.item(), g_ref.item())
        assert torch.equal(packed, p_ref)


def test_noalloc_rejects_bad_arguments_before_launch():
    f = noalloc_entry()
    fake = 1 << 20
    assert f(None, 8, 64, EPS, fake, fake, None) == 1          # BL_ERR_INVALID_ARG
    assert f(fake, 8, 66, EPS, fake, fake, None) == 2          # BL_ERR_UNSUPPORTED_SHAPE
    assert f(fake, 8, 64, 0.0, fake, fake, None) == 1
    assert f(fake + 4, 8, 64, EPS, fake, fake, None) == 3      # BL_ERR_MISALIGNED
