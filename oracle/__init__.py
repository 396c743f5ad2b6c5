"""ctypes front end of the CPU oracle (``bitlinear_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  The CUDA library and its Python
binding never import it, and it imports nothing from them.

Every function takes and returns numpy arrays (C-contiguous); bf16 tensors travel as
their raw ``uint16`` bit patterns.  Each method names the oracle routine it calls; the
C source cites the passage each routine follows.  ``Oracle(path)`` wraps any build of
the oracle source (the tests also load deliberately broken builds to show that the
pins catch them); the module-level functions use the default build.
"""
import ctypes
import numpy as np

from . import build as _build

OUT_F32, OUT_BF16, OUT_I32 = 0, 1, 2


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _vp(a):
    return a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    def __init__(self, path):
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int64
        F = ctypes.c_float
        L.oracle_absmean_gamma.argtypes = [P, I, I, F]
        L.oracle_absmean_gamma.restype = F
        L.oracle_ternarise.argtypes = [P, I, I, F, P]
        L.oracle_ternarise.restype = None
        L.oracle_pack.argtypes = [P, I, I, P]
        L.oracle_pack.restype = I
        L.oracle_unpack.argtypes = [P, I, I, P]
        L.oracle_unpack.restype = None
        L.oracle_quantize_act.argtypes = [P, I, I, F, P, P]
        L.oracle_norm_quantize_act.argtypes = [P, P, I, I, ctypes.c_int, F, F, P, P, P]
        L.oracle_norm_quantize_act.restype = None
        L.oracle_quantize_act.restype = None
        L.oracle_int_matmul.argtypes = [P, P, I, I, I, P]
        L.oracle_int_matmul.restype = I
        L.oracle_dequant.argtypes = [P, P, F, I, I, P]
        L.oracle_dequant.restype = None
        L.oracle_f32_to_bf16.argtypes = [P, I, P]
        L.oracle_dequant_rows.argtypes = [P, P, P, I, I, P]
        L.oracle_dequant_rows.restype = None
        L.oracle_f32_to_bf16.restype = None
        L.oracle_forward.argtypes = [P, P, P, F, I, I, I, ctypes.c_int, P, P, P, P]
        L.oracle_forward.restype = I
        L.oracle_tl5_row_bytes.argtypes = [I]
        L.oracle_tl5_row_bytes.restype = I
        L.oracle_pack_tl5.argtypes = [P, I, I, P]
        L.oracle_pack_tl5.restype = I
        L.oracle_unpack_tl5.argtypes = [P, I, I, P]
        L.oracle_unpack_tl5.restype = None
        L.oracle_forward_tl5.argtypes = [P, P, P, F, I, I, I, ctypes.c_int, P, P, P, P]
        L.oracle_forward_tl5.restype = I
        L.oracle_ste_grad_input.argtypes = [P, P, F, I, I, I, P, P]
        L.oracle_ste_grad_input.restype = None
        L.oracle_ste_grad_weight.argtypes = [P, P, P, F, I, I, I, P]
        L.oracle_ste_grad_weight.restype = None
        self.L = L
        self.path = path

    def absmean_gamma(self, W, eps):
        """gamma = mean|W| + eps (oracle_absmean_gamma)."""
        W, p = _c(W, np.float32)
        N, K = W.shape
        return np.float32(self.L.oracle_absmean_gamma(p, N, K, eps))

    def ternarise(self, W, gamma):
        """codes = clip(round_half_even(W / gamma), -1, 1) (oracle_ternarise)."""
        W, p = _c(W, np.float32)
        N, K = W.shape
        codes = np.empty((N, K), dtype=np.int8)
        self.L.oracle_ternarise(p, N, K, float(gamma), _vp(codes))
        return codes

    def pack(self, codes):
        """2-bit packing, four codes per byte along K (oracle_pack).  Returns (packed, n_bad)."""
        codes, p = _c(codes, np.int8)
        N, K = codes.shape
        assert K % 4 == 0
        packed = np.empty((N, K // 4), dtype=np.uint8)
        bad = self.L.oracle_pack(p, N, K, _vp(packed))
        return packed, int(bad)

    def unpack(self, packed, K):
        """Inverse of pack (oracle_unpack)."""
        packed, p = _c(packed, np.uint8)
        N = packed.shape[0]
        assert packed.shape[1] * 4 == K
        codes = np.empty((N, K), dtype=np.int8)
        self.L.oracle_unpack(p, N, K, _vp(codes))
        return codes

    def quantize_weights(self, W, eps):
        """gamma, codes and packed bytes of one weight matrix."""
        g = self.absmean_gamma(W, eps)
        codes = self.ternarise(W, g)
        packed, bad = self.pack(codes)
        assert bad == 0
        return g, codes, packed

    def quantize_act(self, X_bits, eps):
        """Per-token absmax int8 quantiser (oracle_quantize_act).  X_bits: uint16 bf16 bits."""
        X_bits, p = _c(X_bits, np.uint16)
        M, K = X_bits.shape
        xq = np.empty((M, K), dtype=np.int8)
        s = np.empty((M,), dtype=np.float32)
        self.L.oracle_quantize_act(p, M, K, eps, _vp(xq), _vp(s))
        return xq, s

    def norm_quantize_act(self, X_bits, w, kind, norm_eps, eps):
        """RMSNorm (kind 0) or LayerNorm (kind 1) then the int8 quantiser
        (oracle_norm_quantize_act).  X_bits: uint16 bf16 bits [M, K]; w: fp32 [K] or None.
        Returns (x_q, s, x_n)."""
        X_bits, p = _c(X_bits, np.uint16)
        M, K = X_bits.shape
        wp = None
        if w is not None:
            w, wp = _c(np.asarray(w, dtype=np.float32).reshape(K), np.float32)
        xq = np.empty((M, K), dtype=np.int8)
        s = np.empty((M,), dtype=np.float32)
        xn = np.empty((M, K), dtype=np.float32)
        self.L.oracle_norm_quantize_act(p, wp, M, K, int(kind), float(norm_eps), float(eps), _vp(xq), _vp(s),
                                        _vp(xn))
        return xq, s, xn

    def int_matmul(self, xq, codes):
        """Exact int32 accumulators x_q . codes^T (oracle_int_matmul)."""
        xq, px = _c(xq, np.int8)
        codes, pc = _c(codes, np.int8)
        M, K = xq.shape
        N = codes.shape[0]
        acc = np.empty((M, N), dtype=np.int32)
        over = self.L.oracle_int_matmul(px, pc, M, N, K, _vp(acc))
        assert over == 0, "int32 overflow in the oracle accumulator"
        return acc

    def dequant(self, acc, s, gamma):
        """y = acc * gamma / s (oracle_dequant), fp32."""
        acc, pa = _c(acc, np.int32)
        s, ps = _c(s, np.float32)
        M, N = acc.shape
        y = np.empty((M, N), dtype=np.float32)
        self.L.oracle_dequant(pa, ps, float(gamma), M, N, _vp(y))
        return y

    def dequant_rows(self, acc, s, gamma_rows):
        """y = acc * gamma_n / s_m with one gamma per output row (oracle_dequant_rows)."""
        acc, pa = _c(acc, np.int32)
        M, N = acc.shape
        s, ps = _c(np.asarray(s, dtype=np.float32).reshape(M), np.float32)
        g, pg = _c(np.asarray(gamma_rows, dtype=np.float32).reshape(N), np.float32)
        y = np.empty((M, N), dtype=np.float32)
        self.L.oracle_dequant_rows(pa, ps, pg, M, N, _vp(y))
        return y

    def f32_to_bf16(self, y):
        """Round fp32 to bf16 bits, nearest-even (oracle_f32_to_bf16)."""
        y, p = _c(y, np.float32)
        out = np.empty(y.shape, dtype=np.uint16)
        self.L.oracle_f32_to_bf16(p, y.size, _vp(out))
        return out

    def forward(self, xq, s, packed, gamma, K, out_kind=OUT_F32):
        """Whole forward from packed weights (oracle_forward)."""
        xq, px = _c(xq, np.int8)
        s, ps = _c(s, np.float32)
        packed, pp = _c(packed, np.uint8)
        M = xq.shape[0]
        N = packed.shape[0]
        assert xq.shape[1] == K and packed.shape[1] * 4 == K
        dt = {OUT_F32: np.float32, OUT_BF16: np.uint16, OUT_I32: np.int32}[out_kind]
        out = np.empty((M, N), dtype=dt)
        codes_tmp = np.empty((N, K), dtype=np.int8)
        acc_tmp = np.empty((M, N), dtype=np.int32)
        y_tmp = np.empty((M, N), dtype=np.float32)
        over = self.L.oracle_forward(px, ps, pp, float(gamma), M, N, K, out_kind, _vp(out),
                                     _vp(codes_tmp), _vp(acc_tmp), _vp(y_tmp))
        assert over == 0, "int32 overflow in the oracle accumulator"
        return out


    def tl5_row_bytes(self, K):
        """Bytes per row of the 1.6-bit format (oracle_tl5_row_bytes)."""
        return int(self.L.oracle_tl5_row_bytes(int(K)))

    def pack_tl5(self, codes):
        """Five codes per byte (oracle_pack_tl5): (packed uint8 [N, row_bytes], bad count)."""
        codes, pc = _c(codes, np.int8)
        N, K = codes.shape
        packed = np.empty((N, self.tl5_row_bytes(K)), dtype=np.uint8)
        bad = self.L.oracle_pack_tl5(pc, N, K, _vp(packed))
        return packed, int(bad)

    def unpack_tl5(self, packed, K):
        """Codes from the 1.6-bit format (oracle_unpack_tl5)."""
        packed, pp = _c(packed, np.uint8)
        N = packed.shape[0]
        assert packed.shape[1] == self.tl5_row_bytes(K)
        codes = np.empty((N, K), dtype=np.int8)
        self.L.oracle_unpack_tl5(pp, N, K, _vp(codes))
        return codes

    def forward_tl5(self, xq, s, packed, gamma, K, out_kind=OUT_F32):
        """Whole forward from 1.6-bit weights (oracle_forward_tl5)."""
        xq, px = _c(xq, np.int8)
        s, ps = _c(s, np.float32)
        packed, pp = _c(packed, np.uint8)
        M = xq.shape[0]
        N = packed.shape[0]
        assert xq.shape[1] == K and packed.shape[1] == self.tl5_row_bytes(K)
        dt = {OUT_F32: np.float32, OUT_BF16: np.uint16, OUT_I32: np.int32}[out_kind]
        out = np.empty((M, N), dtype=dt)
        codes_tmp = np.empty((N, K), dtype=np.int8)
        acc_tmp = np.empty((M, N), dtype=np.int32)
        y_tmp = np.empty((M, N), dtype=np.float32)
        over = self.L.oracle_forward_tl5(px, ps, pp, float(gamma), M, N, K, out_kind, _vp(out),
                                         _vp(codes_tmp), _vp(acc_tmp), _vp(y_tmp))
        assert over == 0, "int32 overflow in the oracle accumulator"
        return out

    def ste_grad_input(self, dY, packed, gamma, K):
        """dX = gamma dY C under the straight-through estimator (oracle_ste_grad_input)."""
        dY, pd = _c(dY, np.float32)
        packed, pp = _c(packed, np.uint8)
        M, N = dY.shape
        assert packed.shape == (N, K // 4)
        dX = np.empty((M, K), dtype=np.float32)
        codes_tmp = np.empty((N, K), dtype=np.int8)
        self.L.oracle_ste_grad_input(pd, pp, float(gamma), M, N, K, _vp(dX), _vp(codes_tmp))
        return dX

    def ste_grad_weight(self, dY, xq, s, gamma):
        """dW = gamma sum_m dY[m,n] x_q[m,k] / s[m] (oracle_ste_grad_weight)."""
        dY, pd = _c(dY, np.float32)
        xq, px = _c(xq, np.int8)
        M, N = dY.shape
        K = xq.shape[1]
        s, ps = _c(np.asarray(s, dtype=np.float32).reshape(M), np.float32)
        dW = np.empty((N, K), dtype=np.float32)
        self.L.oracle_ste_grad_weight(pd, px, ps, float(gamma), M, N, K, _vp(dW))
        return dW

_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def absmean_gamma(W, eps): return default().absmean_gamma(W, eps)
def ternarise(W, gamma): return default().ternarise(W, gamma)
def pack(codes): return default().pack(codes)
def unpack(packed, K): return default().unpack(packed, K)
def quantize_weights(W, eps): return default().quantize_weights(W, eps)
def quantize_act(X_bits, eps): return default().quantize_act(X_bits, eps)
def norm_quantize_act(X_bits, w, kind, norm_eps, eps): return default().norm_quantize_act(X_bits, w, kind, norm_eps, eps)
def int_matmul(xq, codes): return default().int_matmul(xq, codes)
def dequant(acc, s, gamma): return default().dequant(acc, s, gamma)
def dequant_rows(acc, s, gamma_rows): return default().dequant_rows(acc, s, gamma_rows)
def f32_to_bf16(y): return default().f32_to_bf16(y)
def forward(xq, s, packed, gamma, K, out_kind=OUT_F32):
    return default().forward(xq, s, packed, gamma, K, out_kind)
def pack_tl5(codes): return default().pack_tl5(codes)
def unpack_tl5(packed, K): return default().unpack_tl5(packed, K)
def tl5_row_bytes(K): return default().tl5_row_bytes(K)
def forward_tl5(xq, s, packed, gamma, K, out_kind=OUT_F32):
    return default().forward_tl5(xq, s, packed, gamma, K, out_kind)
def ste_grad_input(dY, packed, gamma, K): return default().ste_grad_input(dY, packed, gamma, K)
def ste_grad_weight(dY, xq, s, gamma): return default().ste_grad_weight(dY, xq, s, gamma)
