"""B200-native BitNet b1.58 BitLinear forward: absmean ternarisation with 2-bit packing,
per-token absmax int8 activations, and a ternary x int8 GEMM with int32 accumulation
(register-unpack GEMV for decode, tcgen05 kind::i8 for prefill), all in CUDA kernels
for sm_100a behind the C ABI in ``include/bitlinear.h``.

Importing the package does not load the CUDA library; the first call through
``binding`` does, and raises if it is missing.
"""
from .binding import (  # noqa: F401
    BL_OUT_BF16, BL_OUT_F32, BL_OUT_I32, BL_PATH_AUTO, BL_PATH_GEMV, BL_PATH_TC,
    BitLinearError, bitlinear_forward, bitlinear_pack, bitlinear_quantize_act,
    bitlinear_quantize_weights, bitlinear_quantize_weights_with_scale, bitlinear_workspace_size,
    forward, quantize_act, quantize_weights,
)
