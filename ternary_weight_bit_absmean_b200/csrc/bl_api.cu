// bl_api.cu -- the C ABI of libbitlinear.so (declared in include/bitlinear.h): argument
// validation on the host, workspace checks, and dispatch to the kernels.  No call here
// allocates, frees, copies or synchronises; every kernel is enqueued on the caller's
// stream.
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "bitlinear.h"
#include "bl_internal.h"

namespace {

thread_local int g_last_cuda_error = 0;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool eps_ok(float eps) { return std::isfinite(eps) && eps > 0.0f; }

bl_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return BL_OK;
    g_last_cuda_error = static_cast<int>(e);
    return BL_ERR_CUDA;
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Shapes shared by the weight entry points.
bl_status check_weight_shape(int64_t N, int64_t K) {
    if (N <= 0 || K <= 0) return BL_ERR_INVALID_ARG;
    if (K % 4 != 0) return BL_ERR_UNSUPPORTED_SHAPE;
    if (N > (int64_t(1) << 40) / K) return BL_ERR_UNSUPPORTED_SHAPE;
    return BL_OK;
}

}  // namespace

namespace bl {
void record_cuda_error(int code) { g_last_cuda_error = code; }

namespace {
thread_local WaitTest g_wait_test = {kDefaultWaitNs, -1};
}  // namespace

WaitTest wait_test() { return g_wait_test; }

unsigned long long current_context_id() {
    // the driver functions come through the runtime's entry-point query, so the library
    // does not link the driver library; looked up once (thread-safe static init)
    struct CtxFns {
        CUresult (*get_current)(CUcontext*) = nullptr;
        CUresult (*get_id)(CUcontext, unsigned long long*) = nullptr;
        CtxFns() {
            void* p = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
                    cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                get_current = reinterpret_cast<CUresult (*)(CUcontext*)>(p);
            if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                get_id = reinterpret_cast<CUresult (*)(CUcontext, unsigned long long*)>(p);
        }
    };
    static const CtxFns fns;
    if (fns.get_current == nullptr || fns.get_id == nullptr) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (fns.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (fns.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}
}  // namespace bl

extern "C" {

size_t bitlinear_workspace_size(int64_t N, int64_t K) {
    if (N <= 0 || K <= 0) return 0;
    return static_cast<size_t>(bl::absmean_num_partials(N * K)) * sizeof(double);
}

bl_status bitlinear_quantize_weights(const float* W, int64_t N, int64_t K, float eps, float* gamma_out,
                                     uint8_t* packed_out, void* ws, size_t ws_bytes, void* stream) {
    BL_RANGE("bitlinear_quantize_weights");
    if (W == nullptr || gamma_out == nullptr || packed_out == nullptr || !eps_ok(eps))
        return BL_ERR_INVALID_ARG;
    bl_status st = check_weight_shape(N, K);
    if (st != BL_OK) return st;
    if (!aligned16(W) || !aligned16(packed_out) || !aligned16(gamma_out)) return BL_ERR_MISALIGNED;
    const size_t need = bitlinear_workspace_size(N, K);
    if (ws == nullptr || ws_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(ws)) return BL_ERR_MISALIGNED;
    const int64_t numel = N * K;
    const int nparts = bl::absmean_num_partials(numel);
    double* partials = static_cast<double*>(ws);
    cudaError_t e = bl::launch_absmean_partials(W, numel, partials, nparts, as_stream(stream));
    if (e != cudaSuccess) return cuda_status(e);
    e = bl::launch_ternarise_pack(W, numel, nullptr, partials, nparts, eps, gamma_out, packed_out,
                                  as_stream(stream));
    return cuda_status(e);
}

bl_status bitlinear_quantize_weights_with_scale(const float* W, int64_t N, int64_t K, const float* gamma,
                                                uint8_t* packed_out, void* stream) {
    BL_RANGE("bitlinear_quantize_weights_with_scale");
    if (W == nullptr || gamma == nullptr || packed_out == nullptr) return BL_ERR_INVALID_ARG;
    bl_status st = check_weight_shape(N, K);
    if (st != BL_OK) return st;
    if (!aligned16(W) || !aligned16(packed_out)) return BL_ERR_MISALIGNED;
    cudaError_t e = bl::launch_ternarise_pack(W, N * K, gamma, nullptr, 0, 0.0f, nullptr, packed_out,
                                              as_stream(stream));
    return cuda_status(e);
}

bl_status bitlinear_pack(const int8_t* codes, int64_t N, int64_t K, uint8_t* packed_out, int32_t* err_word,
                         void* stream) {
    BL_RANGE("bitlinear_pack");
    if (codes == nullptr || packed_out == nullptr) return BL_ERR_INVALID_ARG;
    bl_status st = check_weight_shape(N, K);
    if (st != BL_OK) return st;
    if (!aligned16(codes) || !aligned16(packed_out)) return BL_ERR_MISALIGNED;
    cudaError_t e = bl::launch_pack_codes(codes, N * K, packed_out, err_word, as_stream(stream));
    return cuda_status(e);
}

bl_status bitlinear_quantize_act_layout(const uint16_t* X, int64_t M, int64_t K, float eps, int8_t* xq_out,
                                        float* s_out, bl_xq_layout layout, void* stream) {
    BL_RANGE("bitlinear_quantize_act_layout");
    if (X == nullptr || xq_out == nullptr || s_out == nullptr || !eps_ok(eps)) return BL_ERR_INVALID_ARG;
    if (M <= 0 || K <= 0) return BL_ERR_INVALID_ARG;
    if (layout != BL_XQ_ROWMAJOR && layout != BL_XQ_K16_EVENODD && layout != BL_XQ_K16_STRIDE4)
        return BL_ERR_INVALID_ARG;
    if (layout != BL_XQ_ROWMAJOR && (K % 16 != 0 || K > (int64_t(1) << 30))) return BL_ERR_UNSUPPORTED_SHAPE;
    if (M > (int64_t(1) << 40) / K) return BL_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(X) || !aligned16(xq_out) || !aligned16(s_out)) return BL_ERR_MISALIGNED;
    cudaError_t e = bl::launch_quantize_act(X, M, K, eps, xq_out, s_out, static_cast<int>(layout), as_stream(stream));
    return cuda_status(e);
}

bl_status bitlinear_norm_quantize_act(const uint16_t* X, const float* norm_weight, int64_t M, int64_t K,
                                      bl_norm_kind norm_kind, float norm_eps, float eps, int8_t* xq_out, float* s_out,
                                      bl_xq_layout layout, void* stream) {
    BL_RANGE("bitlinear_norm_quantize_act");
    if (X == nullptr || xq_out == nullptr || s_out == nullptr || !eps_ok(eps)) return BL_ERR_INVALID_ARG;
    if (!std::isfinite(norm_eps) || norm_eps < 0.0f) return BL_ERR_INVALID_ARG;
    if (norm_kind != BL_NORM_RMS && norm_kind != BL_NORM_LAYER) return BL_ERR_INVALID_ARG;
    if (M <= 0 || K <= 0) return BL_ERR_INVALID_ARG;
    if (layout != BL_XQ_ROWMAJOR && layout != BL_XQ_K16_EVENODD && layout != BL_XQ_K16_STRIDE4)
        return BL_ERR_INVALID_ARG;
    if (K % (layout == BL_XQ_ROWMAJOR ? 8 : 16) != 0 || K > (int64_t(1) << 30)) return BL_ERR_UNSUPPORTED_SHAPE;
    if (M > (int64_t(1) << 40) / K || M >= (int64_t(1) << 31)) return BL_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(X) || !aligned16(xq_out) || !aligned16(s_out)) return BL_ERR_MISALIGNED;
    if (norm_weight != nullptr && !aligned16(norm_weight)) return BL_ERR_MISALIGNED;
    cudaError_t e = bl::launch_norm_quantize_act(X, norm_weight, M, K, static_cast<int>(norm_kind), norm_eps, eps,
                                                 xq_out, s_out, static_cast<int>(layout), as_stream(stream));
    return cuda_status(e);
}

bl_status bitlinear_quantize_act(const uint16_t* X, int64_t M, int64_t K, float eps, int8_t* xq_out,
                                 float* s_out, void* stream) {
    return bitlinear_quantize_act_layout(X, M, K, eps, xq_out, s_out, BL_XQ_ROWMAJOR, stream);
}

static bl_status forward_impl(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma, int64_t M,
                              int64_t N, int64_t K, void* out, bl_dtype out_dtype, int32_t* err_word,
                              bl_xq_layout xq_layout, bl_path path, bool gamma_per_row, void* stream) {
    if (xq == nullptr || s == nullptr || packed == nullptr || gamma == nullptr || out == nullptr)
        return BL_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0) return BL_ERR_INVALID_ARG;
    if (out_dtype != BL_OUT_F32 && out_dtype != BL_OUT_BF16 && out_dtype != BL_OUT_I32)
        return BL_ERR_INVALID_ARG;
    if (path != BL_PATH_AUTO && path != BL_PATH_GEMV && path != BL_PATH_TC && path != BL_PATH_TC_1SM &&
        path != BL_PATH_TC_2SM && path != BL_PATH_SKINNY && path != BL_PATH_GEMV_STREAM && path != BL_PATH_GEMV_TMA)
        return BL_ERR_INVALID_ARG;
    if (xq_layout != BL_XQ_ROWMAJOR && xq_layout != BL_XQ_K16_EVENODD && xq_layout != BL_XQ_K16_STRIDE4)
        return BL_ERR_INVALID_ARG;
    if (K % 4 != 0) return BL_ERR_UNSUPPORTED_SHAPE;
    if (xq_layout != BL_XQ_ROWMAJOR && K % 16 != 0) return BL_ERR_UNSUPPORTED_SHAPE;
    // |acc| <= 128 K must fit in int32; sizes must fit the kernels' 32-bit indexing.
    if (K > (int64_t(1) << 31) / 128 - 1) return BL_ERR_UNSUPPORTED_SHAPE;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return BL_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(xq) || !aligned16(s) || !aligned16(packed) || !aligned16(out)) return BL_ERR_MISALIGNED;
    const bool k64 = (K % 64) == 0;
    const bool tc = path == BL_PATH_TC || path == BL_PATH_TC_1SM || path == BL_PATH_TC_2SM || path == BL_PATH_SKINNY;
    if (tc && !k64) return BL_ERR_UNSUPPORTED_SHAPE;
    // the tensor-core kernels expand stride-4 codes as 64 * code: 64 * 128 * K must fit
    const bool s4_big = xq_layout == BL_XQ_K16_STRIDE4 && K > (int64_t(1) << 17);
    if (tc && s4_big) return BL_ERR_UNSUPPORTED_SHAPE;
    if (path == BL_PATH_GEMV_STREAM &&
        (xq_layout != BL_XQ_K16_STRIDE4 || !bl::gemv_stream_applicable(M, N, K)))
        return BL_ERR_UNSUPPORTED_SHAPE;
    if (path == BL_PATH_GEMV_TMA && (xq_layout != BL_XQ_K16_STRIDE4 || !bl::gemv_tma_applicable(M, N, K)))
        return BL_ERR_UNSUPPORTED_SHAPE;
    if (path == BL_PATH_AUTO) {
        if (M <= 16 || !k64 || s4_big)
            path = BL_PATH_GEMV;
        else if (M <= 32 && xq_layout == BL_XQ_K16_STRIDE4 && bl::gemv_stream_applicable(M, N, K))
            path = BL_PATH_GEMV_STREAM;  // measured faster than the small-batch kernel up to 32 tokens
        else
            path = M <= 64 ? BL_PATH_SKINNY : BL_PATH_TC;
    }
    if (gamma_per_row && !aligned16(gamma)) return BL_ERR_MISALIGNED;
    const int kind = static_cast<int>(out_dtype) | (gamma_per_row ? bl::kGammaPerRow : 0);
    const int lay = static_cast<int>(xq_layout);
    cudaStream_t st = as_stream(stream);
    cudaError_t e;
    if (path == BL_PATH_TC) {
        e = bl::launch_gemm_tc(xq, s, packed, gamma, M, N, K, out, kind, err_word, lay, st);
    } else if (path == BL_PATH_TC_1SM) {
        e = bl::launch_gemm_tc1(xq, s, packed, gamma, M, N, K, out, kind, err_word, lay, st);
    } else if (path == BL_PATH_TC_2SM) {
        e = bl::launch_gemm_tc2(xq, s, packed, gamma, M, N, K, out, kind, err_word, lay, st);
    } else if (path == BL_PATH_SKINNY) {
        e = bl::launch_gemv_tc(xq, s, packed, gamma, M, N, K, out, kind, err_word, lay, st);
    } else if (path == BL_PATH_GEMV_STREAM) {
        e = bl::launch_gemv_stream(xq, s, packed, gamma, M, N, K, out, kind, st);
    } else if (path == BL_PATH_GEMV_TMA) {
        e = bl::launch_gemv_tma(xq, s, packed, gamma, M, N, K, out, kind, err_word, st);
    } else if (k64 && M <= int64_t(65535) * 16) {
        e = bl::launch_gemv(xq, s, packed, gamma, M, N, K, out, kind, err_word, lay, st);
    } else {
        e = bl::launch_gemv_generic(xq, s, packed, gamma, M, N, K, out, kind, lay, st);
    }
    return cuda_status(e);
}

int64_t bitlinear_tl5_row_bytes(int64_t K) {
    if (K <= 0 || K % 16 != 0) return 0;
    return bl::tl5_row_bytes(K);
}

// Shapes of the TL5 weight entry points: the 2-bit rules plus K % 16 == 0, K < 2^31.
static bl_status check_tl5_shape(int64_t N, int64_t K) {
    bl_status st = check_weight_shape(N, K);
    if (st != BL_OK) return st;
    if (K % 16 != 0 || K >= (int64_t(1) << 31)) return BL_ERR_UNSUPPORTED_SHAPE;
    return BL_OK;
}

bl_status bitlinear_pack_tl5(const int8_t* codes, int64_t N, int64_t K, uint8_t* tl5_out, int32_t* err_word,
                             void* stream) {
    BL_RANGE("bitlinear_pack_tl5");
    if (codes == nullptr || tl5_out == nullptr) return BL_ERR_INVALID_ARG;
    bl_status st = check_tl5_shape(N, K);
    if (st != BL_OK) return st;
    if (!aligned16(codes) || !aligned16(tl5_out)) return BL_ERR_MISALIGNED;
    return cuda_status(bl::launch_tl5_pack(codes, N, K, tl5_out, err_word, as_stream(stream)));
}

bl_status bitlinear_repack_tl5(const uint8_t* packed, int64_t N, int64_t K, uint8_t* tl5_out, void* stream) {
    BL_RANGE("bitlinear_repack_tl5");
    if (packed == nullptr || tl5_out == nullptr) return BL_ERR_INVALID_ARG;
    bl_status st = check_tl5_shape(N, K);
    if (st != BL_OK) return st;
    if (!aligned16(packed) || !aligned16(tl5_out)) return BL_ERR_MISALIGNED;
    return cuda_status(bl::launch_tl5_repack(packed, N, K, tl5_out, as_stream(stream)));
}

bl_status bitlinear_forward_tl5(const int8_t* xq, const float* s, const uint8_t* tl5, const float* gamma, int64_t M,
                                int64_t N, int64_t K, void* out, bl_dtype out_dtype, void* stream) {
    BL_RANGE("bitlinear_forward_tl5");
    if (xq == nullptr || s == nullptr || tl5 == nullptr || gamma == nullptr || out == nullptr)
        return BL_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0) return BL_ERR_INVALID_ARG;
    if (out_dtype != BL_OUT_F32 && out_dtype != BL_OUT_BF16 && out_dtype != BL_OUT_I32) return BL_ERR_INVALID_ARG;
    if (K % 16 != 0) return BL_ERR_UNSUPPORTED_SHAPE;
    // |acc| <= 128 K must fit in int32; token groups of 16 go to grid.y (at most 65535)
    if (K > (int64_t(1) << 31) / 128 - 1) return BL_ERR_UNSUPPORTED_SHAPE;
    if (M > int64_t(65535) * 16 || N >= (int64_t(1) << 31)) return BL_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(xq) || !aligned16(s) || !aligned16(tl5) || !aligned16(out)) return BL_ERR_MISALIGNED;
    return cuda_status(bl::launch_gemv_tl5(xq, s, tl5, gamma, M, N, K, out, static_cast<int>(out_dtype),
                                           as_stream(stream)));
}

bl_status bitlinear_ste_backward_input(const float* dY, const uint8_t* packed, const float* gamma, int64_t M,
                                       int64_t N, int64_t K, float* dX, void* stream) {
    BL_RANGE("bitlinear_ste_backward_input");
    if (dY == nullptr || packed == nullptr || gamma == nullptr || dX == nullptr) return BL_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0) return BL_ERR_INVALID_ARG;
    if (K % 4 != 0) return BL_ERR_UNSUPPORTED_SHAPE;
    const int64_t lim = int64_t(1) << 31;
    if (M >= lim || N >= lim || K >= lim) return BL_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(dY) || !aligned16(packed) || !aligned16(dX)) return BL_ERR_MISALIGNED;
    return cuda_status(bl::launch_ste_grad_input(dY, packed, gamma, M, N, K, dX, as_stream(stream)));
}

bl_status bitlinear_ste_backward_weight(const float* dY, const int8_t* xq, const float* s, const float* gamma,
                                        int64_t M, int64_t N, int64_t K, float* dW, void* stream) {
    BL_RANGE("bitlinear_ste_backward_weight");
    if (dY == nullptr || xq == nullptr || s == nullptr || gamma == nullptr || dW == nullptr) return BL_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0) return BL_ERR_INVALID_ARG;
    if (K % 4 != 0) return BL_ERR_UNSUPPORTED_SHAPE;
    const int64_t lim = int64_t(1) << 31;
    if (M >= lim || N >= lim || K >= lim) return BL_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(dY) || !aligned16(xq) || !aligned16(s) || !aligned16(dW)) return BL_ERR_MISALIGNED;
    return cuda_status(bl::launch_ste_grad_weight(dY, xq, s, gamma, M, N, K, dW, as_stream(stream)));
}

bl_status bitlinear_forward_layout(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                                   int64_t M, int64_t N, int64_t K, void* out, bl_dtype out_dtype,
                                   int32_t* err_word, bl_xq_layout xq_layout, bl_path path, void* stream) {
    BL_RANGE("bitlinear_forward_layout");
    return forward_impl(xq, s, packed, gamma, M, N, K, out, out_dtype, err_word, xq_layout, path, false, stream);
}

bl_status bitlinear_forward_rowscale(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma_rows,
                                     int64_t M, int64_t N, int64_t K, void* out, bl_dtype out_dtype,
                                     int32_t* err_word, bl_xq_layout xq_layout, bl_path path, void* stream) {
    BL_RANGE("bitlinear_forward_rowscale");
    return forward_impl(xq, s, packed, gamma_rows, M, N, K, out, out_dtype, err_word, xq_layout, path, true, stream);
}

bl_status bitlinear_forward_stall_test(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                                      int64_t M, int64_t N, int64_t K, void* out, bl_dtype out_dtype,
                                      int32_t* err_word, bl_xq_layout xq_layout, bl_path path, uint64_t wait_limit_ns,
                                      int32_t stall_after_loads, void* stream) {
    BL_RANGE("bitlinear_forward_stall_test");
    if (wait_limit_ns == 0 || wait_limit_ns > bl::kDefaultWaitNs || stall_after_loads < 0) return BL_ERR_INVALID_ARG;
    // only the kernels that wait on TMA loads: the single-SM tcgen05 kernel, the small-
    // batch tcgen05 kernel, and the TMA-fed decode GEMV (BL_PATH_GEMV names it here)
    if (path != BL_PATH_TC_1SM && path != BL_PATH_SKINNY && path != BL_PATH_GEMV && path != BL_PATH_GEMV_TMA)
        return BL_ERR_INVALID_ARG;
    if (path == BL_PATH_GEMV) path = BL_PATH_GEMV_TMA;
    if (path == BL_PATH_GEMV_TMA && (xq_layout != BL_XQ_K16_STRIDE4 || !bl::gemv_tma_applicable(M, N, K)))
        return BL_ERR_UNSUPPORTED_SHAPE;
    const bl::WaitTest saved = bl::g_wait_test;
    bl::g_wait_test = bl::WaitTest{wait_limit_ns, stall_after_loads};
    const bl_status st =
        forward_impl(xq, s, packed, gamma, M, N, K, out, out_dtype, err_word, xq_layout, path, false, stream);
    bl::g_wait_test = saved;
    return st;
}

bl_status bitlinear_forward_path(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                                 int64_t M, int64_t N, int64_t K, void* out, bl_dtype out_dtype,
                                 int32_t* err_word, bl_path path, void* stream) {
    return bitlinear_forward_layout(xq, s, packed, gamma, M, N, K, out, out_dtype, err_word, BL_XQ_ROWMAJOR, path,
                                    stream);
}

bl_status bitlinear_forward(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                            int64_t M, int64_t N, int64_t K, void* out, bl_dtype out_dtype,
                            int32_t* err_word, void* stream) {
    return bitlinear_forward_path(xq, s, packed, gamma, M, N, K, out, out_dtype, err_word, BL_PATH_AUTO,
                                  stream);
}

int bitlinear_last_cuda_error(void) { return g_last_cuda_error; }

const char* bitlinear_status_string(int status) {
    switch (status) {
        case BL_OK: return "BL_OK";
        case BL_ERR_INVALID_ARG: return "BL_ERR_INVALID_ARG";
        case BL_ERR_UNSUPPORTED_SHAPE: return "BL_ERR_UNSUPPORTED_SHAPE";
        case BL_ERR_MISALIGNED: return "BL_ERR_MISALIGNED";
        case BL_ERR_WORKSPACE: return "BL_ERR_WORKSPACE";
        case BL_ERR_CUDA: return "BL_ERR_CUDA";
        case BL_ERR_TIMEOUT: return "BL_ERR_TIMEOUT";
        case BL_ERR_BAD_CODE: return "BL_ERR_BAD_CODE";
        default: return "BL_ERR_UNKNOWN";
    }
}

}  // extern "C"
