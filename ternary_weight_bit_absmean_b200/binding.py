"""Thin Python binding of ``libbitlinear.so`` (argument marshalling only).

Each ``bitlinear_*`` function here has the name, arguments and meaning of the C entry
point declared in ``include/bitlinear.h``; it checks that the torch tensors it is given
are CUDA, contiguous and of the expected dtype and shape, passes their device pointers
and the current CUDA stream, and raises ``BitLinearError`` on a non-zero status.  All
arithmetic happens in the library's CUDA kernels.  There is no fallback: if the library
cannot be loaded, every call raises.

The helpers at the end (``quantize_weights``, ``quantize_act``, ``forward``) only
allocate the output tensors with torch and call the entry points above.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitlinear.so")

BL_OK = 0
BL_OUT_F32, BL_OUT_BF16, BL_OUT_I32 = 0, 1, 2
(BL_PATH_AUTO, BL_PATH_GEMV, BL_PATH_TC, BL_PATH_TC_1SM, BL_PATH_TC_2SM, BL_PATH_SKINNY, BL_PATH_GEMV_STREAM,
 BL_PATH_GEMV_TMA) = range(8)
BL_ERRBIT_BAD_CODE, BL_ERRBIT_TIMEOUT, BL_ERRBIT_INDEX = 0x1, 0x2, 0x4
BL_XQ_ROWMAJOR, BL_XQ_K16_EVENODD, BL_XQ_K16_STRIDE4 = 0, 1, 2
BL_NORM_RMS, BL_NORM_LAYER = 0, 1

EXPORTED = [
    "bitlinear_workspace_size", "bitlinear_quantize_weights",
    "bitlinear_quantize_weights_with_scale", "bitlinear_pack", "bitlinear_quantize_act",
    "bitlinear_forward", "bitlinear_forward_path", "bitlinear_quantize_act_layout",
    "bitlinear_forward_layout", "bitlinear_norm_quantize_act", "bitlinear_forward_rowscale",
    "bitlinear_tl5_row_bytes", "bitlinear_pack_tl5", "bitlinear_repack_tl5", "bitlinear_forward_tl5",
    "bitlinear_ste_backward_input", "bitlinear_ste_backward_weight", "bitlinear_forward_stall_test",
    "bitlinear_last_cuda_error",
    "bitlinear_status_string",
]


class BitLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = lib().bitlinear_status_string(status).decode()
        extra = ""
        if name == "BL_ERR_CUDA":
            extra = " (cudaError %d)" % lib().bitlinear_last_cuda_error()
        super().__init__("%s: %s%s" % (where, name, extra))


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libbitlinear.so is not built (run "
                               "`python -m ternary_weight_bit_absmean_b200.build_lib`): %s" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P, I64, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
        S = ctypes.c_int
        L.bitlinear_workspace_size.argtypes = [I64, I64]
        L.bitlinear_workspace_size.restype = ctypes.c_size_t
        L.bitlinear_quantize_weights.argtypes = [P, I64, I64, F, P, P, P, ctypes.c_size_t, P]
        L.bitlinear_quantize_weights.restype = S
        L.bitlinear_quantize_weights_with_scale.argtypes = [P, I64, I64, P, P, P]
        L.bitlinear_quantize_weights_with_scale.restype = S
        L.bitlinear_pack.argtypes = [P, I64, I64, P, P, P]
        L.bitlinear_pack.restype = S
        L.bitlinear_quantize_act.argtypes = [P, I64, I64, F, P, P, P]
        L.bitlinear_quantize_act.restype = S
        L.bitlinear_forward.argtypes = [P, P, P, P, I64, I64, I64, P, S, P, P]
        L.bitlinear_forward.restype = S
        L.bitlinear_forward_path.argtypes = [P, P, P, P, I64, I64, I64, P, S, P, S, P]
        L.bitlinear_forward_path.restype = S
        L.bitlinear_quantize_act_layout.argtypes = [P, I64, I64, F, P, P, S, P]
        L.bitlinear_quantize_act_layout.restype = S
        L.bitlinear_forward_layout.argtypes = [P, P, P, P, I64, I64, I64, P, S, P, S, S, P]
        L.bitlinear_forward_layout.restype = S
        L.bitlinear_forward_rowscale.argtypes = [P, P, P, P, I64, I64, I64, P, S, P, S, S, P]
        L.bitlinear_forward_rowscale.restype = S
        L.bitlinear_norm_quantize_act.argtypes = [P, P, I64, I64, S, F, F, P, P, S, P]
        L.bitlinear_norm_quantize_act.restype = S
        L.bitlinear_tl5_row_bytes.argtypes = [I64]
        L.bitlinear_tl5_row_bytes.restype = I64
        L.bitlinear_pack_tl5.argtypes = [P, I64, I64, P, P, P]
        L.bitlinear_pack_tl5.restype = S
        L.bitlinear_repack_tl5.argtypes = [P, I64, I64, P, P]
        L.bitlinear_repack_tl5.restype = S
        L.bitlinear_forward_tl5.argtypes = [P, P, P, P, I64, I64, I64, P, S, P]
        L.bitlinear_forward_tl5.restype = S
        L.bitlinear_ste_backward_input.argtypes = [P, P, P, I64, I64, I64, P, P]
        L.bitlinear_ste_backward_input.restype = S
        L.bitlinear_ste_backward_weight.argtypes = [P, P, P, P, I64, I64, I64, P, P]
        L.bitlinear_ste_backward_weight.restype = S
        L.bitlinear_forward_stall_test.argtypes = [P, P, P, P, I64, I64, I64, P, S, P, S, S, ctypes.c_uint64,
                                                   ctypes.c_int32, P]
        L.bitlinear_forward_stall_test.restype = S
        L.bitlinear_last_cuda_error.argtypes = []
        L.bitlinear_last_cuda_error.restype = ctypes.c_int
        L.bitlinear_status_string.argtypes = [ctypes.c_int]
        L.bitlinear_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, dtype, name: str, shape=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    return t.data_ptr()


def _opt(t, name):
    return None if t is None else _dev(t, torch.int32, name, (1,))


def _check(status: int, where: str):
    if status != BL_OK:
        raise BitLinearError(status, where)


def bitlinear_workspace_size(N: int, K: int) -> int:
    return int(lib().bitlinear_workspace_size(N, K))


def bitlinear_quantize_weights(W, eps, gamma_out, packed_out, ws, stream=None):
    N, K = W.shape
    _check(lib().bitlinear_quantize_weights(
        _dev(W, torch.float32, "W"), N, K, float(eps), _dev(gamma_out, torch.float32, "gamma_out", (1,)),
        _dev(packed_out, torch.uint8, "packed_out", (N, K // 4)), _dev(ws, torch.uint8, "ws"),
        ws.numel(), _stream(stream)), "bitlinear_quantize_weights")


def bitlinear_quantize_weights_with_scale(W, gamma, packed_out, stream=None):
    N, K = W.shape
    _check(lib().bitlinear_quantize_weights_with_scale(
        _dev(W, torch.float32, "W"), N, K, _dev(gamma, torch.float32, "gamma", (1,)),
        _dev(packed_out, torch.uint8, "packed_out", (N, K // 4)), _stream(stream)),
        "bitlinear_quantize_weights_with_scale")


def bitlinear_pack(codes, packed_out, err_word=None, stream=None):
    N, K = codes.shape
    _check(lib().bitlinear_pack(
        _dev(codes, torch.int8, "codes"), N, K, _dev(packed_out, torch.uint8, "packed_out", (N, K // 4)),
        _opt(err_word, "err_word"), _stream(stream)), "bitlinear_pack")


def bitlinear_quantize_act(X, eps, xq_out, s_out, stream=None, layout=BL_XQ_ROWMAJOR):
    M, K = X.shape
    args = (_dev(X, torch.bfloat16, "X"), M, K, float(eps), _dev(xq_out, torch.int8, "xq_out", (M, K)),
            _dev(s_out, torch.float32, "s_out", (M,)))
    if layout == BL_XQ_ROWMAJOR:
        _check(lib().bitlinear_quantize_act(*args, _stream(stream)), "bitlinear_quantize_act")
    else:
        _check(lib().bitlinear_quantize_act_layout(*args, int(layout), _stream(stream)),
               "bitlinear_quantize_act_layout")


def bitlinear_norm_quantize_act(X, norm_weight, kind, norm_eps, eps, xq_out, s_out, stream=None,
                                layout=BL_XQ_ROWMAJOR):
    M, K = X.shape
    w = None if norm_weight is None else _dev(norm_weight, torch.float32, "norm_weight", (K,))
    _check(lib().bitlinear_norm_quantize_act(
        _dev(X, torch.bfloat16, "X"), w, M, K, int(kind), float(norm_eps), float(eps),
        _dev(xq_out, torch.int8, "xq_out", (M, K)), _dev(s_out, torch.float32, "s_out", (M,)), int(layout),
        _stream(stream)), "bitlinear_norm_quantize_act")


_OUT_DT = {BL_OUT_F32: torch.float32, BL_OUT_BF16: torch.bfloat16, BL_OUT_I32: torch.int32}


def bitlinear_forward(xq, s, packed, gamma, out, err_word=None, stream=None, path=BL_PATH_AUTO,
                      layout=BL_XQ_ROWMAJOR):
    M, K = xq.shape
    N = packed.shape[0]
    kind = {v: k for k, v in _OUT_DT.items()}.get(out.dtype)
    if kind is None:
        raise TypeError("out must be float32, bfloat16 or int32")
    args = (_dev(xq, torch.int8, "xq"), _dev(s, torch.float32, "s", (M,)),
            _dev(packed, torch.uint8, "packed", (N, K // 4)), _dev(gamma, torch.float32, "gamma", (1,)),
            M, N, K, _dev(out, out.dtype, "out", (M, N)), kind, _opt(err_word, "err_word"))
    if layout != BL_XQ_ROWMAJOR:
        _check(lib().bitlinear_forward_layout(*args, int(layout), int(path), _stream(stream)),
               "bitlinear_forward_layout")
    elif path == BL_PATH_AUTO:
        _check(lib().bitlinear_forward(*args, _stream(stream)), "bitlinear_forward")
    else:
        _check(lib().bitlinear_forward_path(*args, int(path), _stream(stream)), "bitlinear_forward_path")


def bitlinear_forward_stall_test(xq, s, packed, gamma, out, err_word, wait_limit_ns, stall_after_loads,
                                 stream=None, path=BL_PATH_TC_1SM, layout=BL_XQ_ROWMAJOR):
    """The forward with every device wait limited to wait_limit_ns and each block's load
    producer stopped after stall_after_loads loads (a test of the bounded waits)."""
    M, K = xq.shape
    N = packed.shape[0]
    kind = {v: k for k, v in _OUT_DT.items()}.get(out.dtype)
    if kind is None:
        raise TypeError("out must be float32, bfloat16 or int32")
    _check(lib().bitlinear_forward_stall_test(
        _dev(xq, torch.int8, "xq"), _dev(s, torch.float32, "s", (M,)),
        _dev(packed, torch.uint8, "packed", (N, K // 4)), _dev(gamma, torch.float32, "gamma", (1,)),
        M, N, K, _dev(out, out.dtype, "out", (M, N)), kind, _opt(err_word, "err_word"), int(layout), int(path),
        int(wait_limit_ns), int(stall_after_loads), _stream(stream)), "bitlinear_forward_stall_test")


def bitlinear_forward_rowscale(xq, s, packed, gamma_rows, out, err_word=None, stream=None, path=BL_PATH_AUTO,
                               layout=BL_XQ_ROWMAJOR):
    M, K = xq.shape
    N = packed.shape[0]
    kind = {v: k for k, v in _OUT_DT.items()}.get(out.dtype)
    if kind is None:
        raise TypeError("out must be float32, bfloat16 or int32")
    _check(lib().bitlinear_forward_rowscale(
        _dev(xq, torch.int8, "xq"), _dev(s, torch.float32, "s", (M,)),
        _dev(packed, torch.uint8, "packed", (N, K // 4)), _dev(gamma_rows, torch.float32, "gamma_rows", (N,)),
        M, N, K, _dev(out, out.dtype, "out", (M, N)), kind, _opt(err_word, "err_word"), int(layout), int(path),
        _stream(stream)), "bitlinear_forward_rowscale")


def bitlinear_tl5_row_bytes(K):
    return int(lib().bitlinear_tl5_row_bytes(int(K)))


def bitlinear_pack_tl5(codes, tl5_out, err_word=None, stream=None):
    N, K = codes.shape
    _check(lib().bitlinear_pack_tl5(
        _dev(codes, torch.int8, "codes"), N, K, _dev(tl5_out, torch.uint8, "tl5_out", (N, bitlinear_tl5_row_bytes(K))),
        _opt(err_word, "err_word"), _stream(stream)), "bitlinear_pack_tl5")


def bitlinear_repack_tl5(packed, tl5_out, stream=None):
    N, KB = packed.shape
    K = 4 * KB
    _check(lib().bitlinear_repack_tl5(
        _dev(packed, torch.uint8, "packed"), N, K,
        _dev(tl5_out, torch.uint8, "tl5_out", (N, bitlinear_tl5_row_bytes(K))), _stream(stream)),
        "bitlinear_repack_tl5")


def bitlinear_forward_tl5(xq, s, tl5, gamma, out, stream=None):
    M, K = xq.shape
    N = tl5.shape[0]
    kind = {v: k for k, v in _OUT_DT.items()}.get(out.dtype)
    if kind is None:
        raise TypeError("out must be float32, bfloat16 or int32")
    _check(lib().bitlinear_forward_tl5(
        _dev(xq, torch.int8, "xq"), _dev(s, torch.float32, "s", (M,)),
        _dev(tl5, torch.uint8, "tl5", (N, bitlinear_tl5_row_bytes(K))), _dev(gamma, torch.float32, "gamma"),
        M, N, K, _dev(out, out.dtype, "out", (M, N)), kind, _stream(stream)), "bitlinear_forward_tl5")


def bitlinear_ste_backward_input(dY, packed, gamma, dX, stream=None):
    M, N = dY.shape
    K = 4 * packed.shape[1]
    _check(lib().bitlinear_ste_backward_input(
        _dev(dY, torch.float32, "dY"), _dev(packed, torch.uint8, "packed", (N, K // 4)),
        _dev(gamma, torch.float32, "gamma"), M, N, K, _dev(dX, torch.float32, "dX", (M, K)), _stream(stream)),
        "bitlinear_ste_backward_input")


def bitlinear_ste_backward_weight(dY, xq, s, gamma, dW, stream=None):
    M, N = dY.shape
    K = xq.shape[1]
    _check(lib().bitlinear_ste_backward_weight(
        _dev(dY, torch.float32, "dY"), _dev(xq, torch.int8, "xq", (M, K)), _dev(s, torch.float32, "s", (M,)),
        _dev(gamma, torch.float32, "gamma"), M, N, K, _dev(dW, torch.float32, "dW", (N, K)), _stream(stream)),
        "bitlinear_ste_backward_weight")


# ----------------------------------------------------------- allocating helpers --

def quantize_weights(W: torch.Tensor, eps: float = 1e-5, stream=None):
    """(gamma [1] fp32, packed [N, K/4] uint8) of an fp32 CUDA weight matrix."""
    N, K = W.shape
    gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    packed = torch.empty(N, K // 4, dtype=torch.uint8, device=W.device)
    ws = torch.empty(max(1, bitlinear_workspace_size(N, K)), dtype=torch.uint8, device=W.device)
    bitlinear_quantize_weights(W, eps, gamma, packed, ws, stream)
    return gamma, packed


def quantize_act(X: torch.Tensor, eps: float = 1e-5, stream=None, layout=BL_XQ_ROWMAJOR):
    """(x_q [M, K] int8, s [M] fp32) of a bf16 CUDA activation matrix."""
    M, K = X.shape
    xq = torch.empty(M, K, dtype=torch.int8, device=X.device)
    s = torch.empty(M, dtype=torch.float32, device=X.device)
    bitlinear_quantize_act(X, eps, xq, s, stream, layout)
    return xq, s


def norm_quantize_act(X: torch.Tensor, norm_weight=None, kind=BL_NORM_RMS, norm_eps: float = 1e-5,
                      eps: float = 1e-5, stream=None, layout=BL_XQ_ROWMAJOR):
    """(x_q [M, K] int8, s [M] fp32) of RMSNorm / LayerNorm(X) for a bf16 CUDA matrix."""
    M, K = X.shape
    xq = torch.empty(M, K, dtype=torch.int8, device=X.device)
    s = torch.empty(M, dtype=torch.float32, device=X.device)
    bitlinear_norm_quantize_act(X, norm_weight, kind, norm_eps, eps, xq, s, stream, layout)
    return xq, s


def forward(xq, s, packed, gamma, out_dtype=torch.float32, stream=None, path=BL_PATH_AUTO, err_word=None,
            layout=BL_XQ_ROWMAJOR):
    """y [M, N] of the BitLinear forward from quantised operands."""
    out = torch.empty(xq.shape[0], packed.shape[0], dtype=out_dtype, device=xq.device)
    bitlinear_forward(xq, s, packed, gamma, out, err_word, stream, path, layout)
    return out


def pack_tl5(codes: torch.Tensor, stream=None):
    """[N, tl5_row_bytes(K)] uint8: int8 codes in the five-per-byte format."""
    N, K = codes.shape
    out = torch.empty(N, bitlinear_tl5_row_bytes(K), dtype=torch.uint8, device=codes.device)
    bitlinear_pack_tl5(codes, out, None, stream)
    return out


def repack_tl5(packed: torch.Tensor, stream=None):
    """[N, tl5_row_bytes(K)] uint8 from the 2-bit format [N, K/4]."""
    N, KB = packed.shape
    out = torch.empty(N, bitlinear_tl5_row_bytes(4 * KB), dtype=torch.uint8, device=packed.device)
    bitlinear_repack_tl5(packed, out, stream)
    return out


def forward_tl5(xq, s, tl5, gamma, out_dtype=torch.float32, stream=None):
    """y [M, N] from row-major x_q and weights in the five-per-byte format."""
    out = torch.empty(xq.shape[0], tl5.shape[0], dtype=out_dtype, device=xq.device)
    bitlinear_forward_tl5(xq, s, tl5, gamma, out, stream)
    return out


def ste_backward(dY, packed, xq, s, gamma, stream=None):
    """(dX [M, K], dW [N, K]) fp32: the straight-through gradients of the forward."""
    M, N = dY.shape
    K = 4 * packed.shape[1]
    dX = torch.empty(M, K, dtype=torch.float32, device=dY.device)
    dW = torch.empty(N, K, dtype=torch.float32, device=dY.device)
    bitlinear_ste_backward_input(dY, packed, gamma, dX, stream)
    bitlinear_ste_backward_weight(dY, xq, s, gamma, dW, stream)
    return dX, dW
