// bl_noalloc.cu -- bitlinear_quantize_weights_noalloc: weight quantisation for callers
// that cannot allocate device memory.
//
// bitlinear_quantize_weights needs a small device workspace for the per-block fp64
// partial sums of |W|.  Some callers have no way to provide one: code that runs where
// cudaMalloc is off limits (cudaMalloc may synchronise the whole device, which a
// latency-critical serving loop cannot afford), plug-ins loaded into a host framework
// that owns every device allocation through its own arena and hands out no scratch,
// and deployments that fix their device memory budget at start-up.  This entry point
// keeps the partial sums in a fixed array that lives in the library itself, so the
// caller passes only W and the two outputs.
//
// The array is a file-scope __device__ variable: every GPU that loads this library
// holds kNoAllocMaxPartials doubles (9472 bytes) of it until the process exits.  Host
// code cannot use the array's name as a device address, so every call looks the
// address up with cudaGetSymbolAddress, with the caller's device current.  The lookup
// allocates nothing; it is repeated on every call (it costs little once the module is
// loaded) so that an address from a context that was since destroyed (after
// cudaDeviceReset) is never used.
#include <cmath>
#include <cstdint>
#include <cuda_runtime.h>

#include "bitlinear.h"
#include "bl_internal.h"

namespace {

constexpr int kNoAllocMaxPartials = 148 * 8;
// every partial count the absmean kernel can use fits in the array
static_assert(kNoAllocMaxPartials >= bl::kAbsMaxParts, "the no-allocation array must hold every partial sum");

static __device__ __align__(256) double g_absmean_partials[kNoAllocMaxPartials];

// Device address of g_absmean_partials in the current context.  The first lookup on a
// device may make the driver load this library's device code (lazy module loading),
// which is where the array itself is placed in device memory.
cudaError_t partials_address(double** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_absmean_partials);
    if (e != cudaSuccess) return e;
    *out = static_cast<double*>(p);
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

bl_status bitlinear_quantize_weights_noalloc(const float* W, int64_t N, int64_t K, float eps,
                                             float* gamma_out, uint8_t* packed_out, void* stream) {
    BL_RANGE("bitlinear_quantize_weights_noalloc");
    if (W == nullptr || gamma_out == nullptr || packed_out == nullptr) return BL_ERR_INVALID_ARG;
    if (!std::isfinite(eps) || !(eps > 0.0f)) return BL_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0) return BL_ERR_INVALID_ARG;
    if (K % 4 != 0 || N > (int64_t(1) << 40) / K) return BL_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(W) || !aligned16(packed_out) || !aligned16(gamma_out)) return BL_ERR_MISALIGNED;
    const int64_t numel = N * K;
    const int nparts = bl::absmean_num_partials(numel);
    if (nparts > kNoAllocMaxPartials) return BL_ERR_WORKSPACE;  // more partials than the array holds
    double* partials = nullptr;
    cudaError_t e = partials_address(&partials);
    if (e == cudaSuccess) {
        // every slot the pack kernel reads is written by the partials kernel first, so
        // what an earlier call left in the array is never used
        e = bl::launch_absmean_partials(W, numel, partials, nparts, static_cast<cudaStream_t>(stream));
    }
    if (e == cudaSuccess) {
        e = bl::launch_ternarise_pack(W, numel, nullptr, partials, nparts, eps, gamma_out, packed_out,
                                      static_cast<cudaStream_t>(stream));
    }
    if (e != cudaSuccess) {
        bl::record_cuda_error(static_cast<int>(e));
        return BL_ERR_CUDA;
    }
    return BL_OK;
}

}  // extern "C"
