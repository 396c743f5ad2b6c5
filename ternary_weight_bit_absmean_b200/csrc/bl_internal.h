// bl_internal.h -- launchers shared between the kernel files and the C-ABI layer.
// Every launcher enqueues on `stream` and returns the cudaError_t of its launch.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

namespace bl {

// A named NVTX range around an entry point, so that a profiler's timeline shows which
// library call enqueued which kernels; without an attached tool it costs a test of one
// function pointer.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
#define BL_RANGE(name) ::bl::NvtxRange bl_nvtx_range_(name)

// Weight quantisation (absmean partial sums, ternarise + pack, pack of int8 codes).
// The absmean kernel never uses more than kAbsMaxParts blocks (fp64 partial sums).
constexpr int kAbsMaxParts = 148 * 8;
int absmean_num_partials(int64_t numel);
cudaError_t launch_absmean_partials(const float* W, int64_t numel, double* partials, int nparts,
                                    cudaStream_t stream);
// gamma from the partials (gamma_in == nullptr) or given (gamma_in != nullptr).
cudaError_t launch_ternarise_pack(const float* W, int64_t numel, const float* gamma_in,
                                  const double* partials, int nparts, float eps,
                                  float* gamma_out, uint8_t* packed, cudaStream_t stream);
cudaError_t launch_pack_codes(const int8_t* codes, int64_t numel, uint8_t* packed, int32_t* err,
                              cudaStream_t stream);

// Device index checks of a debugging build (BL_DEBUG_CHECKS=1; compute-sanitizer is not
// available on the GPUs this was built for): bl_check(cond, err) returns cond and, when it
// is false, ORs BL_ERRBIT_INDEX (0x4) into the error word, so that the caller skips the
// access instead of trapping.  In a normal build it is `true` and costs nothing.
#ifndef BL_DEBUG_CHECKS
#define BL_DEBUG_CHECKS 0
#endif
constexpr int kErrBitIndex = 0x4;
#ifdef __CUDACC__
__device__ __forceinline__ bool bl_check(bool cond, int32_t* err) {
#if BL_DEBUG_CHECKS
    if (!cond && err != nullptr) atomicOr(err, kErrBitIndex);
    return cond;
#else
    (void)cond;
    (void)err;
    return true;
#endif
}
// Bytes of dynamic shared memory of the running launch.
__device__ __forceinline__ uint32_t dynamic_smem_bytes() {
    uint32_t v;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(v));
    return v;
}
#endif

// Layouts of x_q (mirror bl_xq_layout).
enum XqLayout : int { kXqRowMajor = 0, kXqEvenOdd16 = 1, kXqStride4K16 = 2 };

// Per-token absmax int8 activation quantisation.
cudaError_t launch_quantize_act(const uint16_t* X, int64_t M, int64_t K, float eps, int8_t* xq,
                                float* s, int layout, cudaStream_t stream);

// RMSNorm (kind 0) or LayerNorm (kind 1), optional per-channel weight, then the per-token
// quantiser; K % 8 == 0 (K % 16 == 0 for the k16 layouts).
cudaError_t launch_norm_quantize_act(const uint16_t* X, const float* norm_weight, int64_t M, int64_t K, int kind,
                                     float norm_eps, float eps, int8_t* xq, float* s, int layout,
                                     cudaStream_t stream);

// Output kinds (mirror bl_dtype).
enum OutKind : int { kOutF32 = 0, kOutBF16 = 1, kOutI32 = 2 };
// The forward launchers' `kind` may also carry kGammaPerRow: gamma then points to N
// weight scales, one per output row, instead of one.
constexpr int kGammaPerRow = 0x100;
inline int out_kind_of(int kind) { return kind & 0xFF; }
inline int gamma_rows_of(int kind) { return (kind & kGammaPerRow) ? 1 : 0; }

// Decode GEMV: register unpack + mma.sync, any M (token groups of 16), K % 64 == 0.
// With x_q in the stride-4 k16 layout it runs the kernel fed by per-thread asynchronous
// copies (k_gemv_stream.cu) where gemv_stream_applicable accepts the shape, else the
// persistent TMA-fed kernel (k_gemv_tma.cu) where gemv_tma_applicable does.
cudaError_t launch_gemv(const int8_t* xq, const float* s, const uint8_t* packed,
                        const float* gamma, int64_t M, int64_t N, int64_t K, void* out, int kind,
                        int32_t* err, int layout, cudaStream_t stream);
bool gemv_tma_applicable(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemv_tma(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                            int64_t M, int64_t N, int64_t K, void* out, int kind, int32_t* err,
                            cudaStream_t stream);
// The GEMV fed by per-thread asynchronous copies (k_gemv_stream.cu), x_q in the
// stride-4 k16 layout; gemv_stream_applicable states its shape conditions.
bool gemv_stream_applicable(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemv_stream(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                               int64_t M, int64_t N, int64_t K, void* out, int kind, cudaStream_t stream);
// Plain fallback for K % 64 != 0 (one output per thread).
cudaError_t launch_gemv_generic(const int8_t* xq, const float* s, const uint8_t* packed,
                                const float* gamma, int64_t M, int64_t N, int64_t K, void* out,
                                int kind, int layout, cudaStream_t stream);

// Tiled tcgen05 kind::i8 paths (K % 64 == 0): launch_gemm_tc picks between the
// single-SM kernel (tc1) and the CTA-pair kernel (tc2).
cudaError_t launch_gemm_tc(const int8_t* xq, const float* s, const uint8_t* packed,
                           const float* gamma, int64_t M, int64_t N, int64_t K, void* out,
                           int kind, int32_t* err, int layout, cudaStream_t stream);
cudaError_t launch_gemm_tc1(const int8_t* xq, const float* s, const uint8_t* packed,
                            const float* gamma, int64_t M, int64_t N, int64_t K, void* out,
                            int kind, int32_t* err, int layout, cudaStream_t stream);
cudaError_t launch_gemm_tc2(const int8_t* xq, const float* s, const uint8_t* packed,
                            const float* gamma, int64_t M, int64_t N, int64_t K, void* out,
                            int kind, int32_t* err, int layout, cudaStream_t stream);

// Small-batch tcgen05 kernel (K split over a cluster when rows are few), K % 64 == 0, any
// M (token tiles of up to 128).
cudaError_t launch_gemv_tc(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma, int64_t M,
                           int64_t N, int64_t K, void* out, int kind, int32_t* err, int layout, cudaStream_t stream);

// The 1.6-bit (five codes per byte) weight format, K % 16 == 0 (k_tl5.cu).
int64_t tl5_row_bytes(int64_t K);
cudaError_t launch_tl5_pack(const int8_t* codes, int64_t N, int64_t K, uint8_t* out, int32_t* err,
                            cudaStream_t stream);
cudaError_t launch_tl5_repack(const uint8_t* packed, int64_t N, int64_t K, uint8_t* out, cudaStream_t stream);
cudaError_t launch_gemv_tl5(const int8_t* xq, const float* s, const uint8_t* w5, const float* gamma, int64_t M,
                            int64_t N, int64_t K, void* out, int kind, cudaStream_t stream);

// The straight-through backward (k_ste.cu): dX = gamma dY C, dW = gamma dY^T (x_q / s).
cudaError_t launch_ste_grad_input(const float* dY, const uint8_t* packed, const float* gamma, int64_t M, int64_t N,
                                  int64_t K, float* dX, cudaStream_t stream);
cudaError_t launch_ste_grad_weight(const float* dY, const int8_t* xq, const float* s, const float* gamma, int64_t M,
                                   int64_t N, int64_t K, float* dW, cudaStream_t stream);

// Keep a CUDA error code for bitlinear_last_cuda_error() on the calling thread.
void record_cuda_error(int code);

// Limits of the device-side waits of the TMA-fed forward kernels, as the launchers copy
// them into the kernel arguments.  Outside a call of bitlinear_forward_stall_test they
// are {2 s, -1}: every wait gives up after 2 s, and producers never stall.  That test
// entry point sets them on the calling thread for the duration of its call only: the
// waits give up after wait_ns, and each block's producer stops issuing loads after
// stall_after of them, so that the waits for the next load run out.
struct WaitTest {
    unsigned long long wait_ns;
    int stall_after;
};
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;
WaitTest wait_test();

// Identifier of the calling thread's current CUDA context, unique for the life of the
// process (a context created after cudaDeviceReset gets a new one); 0 if unknown.
unsigned long long current_context_id();

// Remembers, for up to kCtxSlots contexts, that a one-time set-up (a kernel attribute)
// was done in that context, so it is redone in a context that replaced a reset one.
struct PerContextOnce {
    static constexpr int kCtxSlots = 64;
    unsigned long long done[kCtxSlots] = {};
    // Runs set() unless it already succeeded in the current context.
    template <typename F>
    cudaError_t run(F set) {
        const unsigned long long id = current_context_id();
        if (id != 0)
            for (int i = 0; i < kCtxSlots; ++i)
                if (__atomic_load_n(&done[i], __ATOMIC_ACQUIRE) == id) return cudaSuccess;
        const cudaError_t e = set();
        if (e != cudaSuccess || id == 0) return e;
        for (int i = 0; i < kCtxSlots; ++i) {
            unsigned long long expect = 0;
            if (__atomic_compare_exchange_n(&done[i], &expect, id, false, __ATOMIC_ACQ_REL, __ATOMIC_ACQUIRE) ||
                expect == id)
                return cudaSuccess;
        }
        return cudaSuccess;  // every slot taken: set() simply runs again next time
    }
};

// Launch `kernel` on `stream` with programmatic stream serialisation allowed (the kernel
// calls pdl_wait_then_release() before touching global memory) and, when cluster.x > 0,
// a thread-block cluster of that shape.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       dim3 cluster, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster.x > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster.x;
        attr[n].val.clusterDim.y = cluster.y;
        attr[n].val.clusterDim.z = cluster.z;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}
constexpr unsigned kNoCluster = 0;

}  // namespace bl
