// k_ste.cu -- the straight-through backward of the BitLinear forward.
//
// "1-bit & Ternary LLMs (BitNet b1.58)", "Training: shadow weights + the straight-through
// estimator": the forward uses the ternary weights, and the backward treats the
// quantisation as the identity so the gradient reaches the full-precision shadow
// weights.  With this library's forward y[m,n] = (sum_k c[n,k] x_q[m,k]) gamma / s[m]
// and both quantisers passed straight through (d x_q / d x = s, gamma and s constant):
//   dX[m,k] = gamma sum_n dY[m,n] c[n,k]            (a ternary contraction over N)
//   dW[n,k] = gamma sum_m dY[m,n] x_q[m,k] / s[m]    (a contraction over the tokens)
// The next forward re-ternarises the updated shadow weights (the quantisation kernels).
//
// Both are output-stationary SIMT tiles: a 128 x 128 output tile per block of 256
// threads, 8 x 8 outputs per thread in fp32 registers (rows 4ty..4ty+3 and 64+4ty..,
// columns likewise, so the shared-memory reads of a warp are conflict-free float4s), the
// contraction in chunks of 16 staged through two shared-memory buffers: the next
// chunk's global loads are issued before the current chunk's products and stored into
// the other buffer after them.  Operands are expanded to fp32 on the way in (codes to
// -1/0/+1, x_q to its integer value, dY divided by s for dW).  The products with a code
// are exact and the sums round in fp32 in contraction order; gamma scales once.
#include <cuda_runtime.h>

#include <cstdint>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {
namespace {

constexpr int kTile = 128;  // output tile edge
constexpr int kChunk = 16;  // contraction chunk
constexpr int kThreads = 256;
constexpr int kPad = 4;

__device__ __forceinline__ float code_of(uint32_t byte, int i) {
    const uint32_t c = (byte >> (2 * i)) & 3u;
    return c == 1u ? 1.0f : (c == 2u ? -1.0f : 0.0f);  // 11 reads as 0
}

// acc[i][j] += A[c][row i] * B[c][col j] over one staged chunk; the thread's rows are
// 4ty + (0..3) and 64 + 4ty + (0..3), its columns 4tx + (0..3) and 64 + 4tx + (0..3).
__device__ __forceinline__ void chunk_fma(const float (*sA)[kTile + kPad], const float (*sB)[kTile + kPad], int ty,
                                          int tx, float (&acc)[8][8]) {
#pragma unroll
    for (int c = 0; c < kChunk; ++c) {
        const float4 a0 = *reinterpret_cast<const float4*>(&sA[c][4 * ty]);
        const float4 a1 = *reinterpret_cast<const float4*>(&sA[c][64 + 4 * ty]);
        const float4 b0 = *reinterpret_cast<const float4*>(&sB[c][4 * tx]);
        const float4 b1 = *reinterpret_cast<const float4*>(&sB[c][64 + 4 * tx]);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = __fmaf_rn(av[i], bv[j], acc[i][j]);
    }
}

__device__ __forceinline__ int out_index(int t, int h) { return h * 64 + 4 * t; }

// dX tile (tokens m0.., columns k0..): A = dY[m, n] staged as [n][m], B = codes[n, k].
// Per chunk a thread loads 8 dY values (e = tid + 256 u: token e / 16, n e % 16) and
// 2 packed bytes (e = tid + 256 u: row e / 32, byte e % 32).
__global__ void __launch_bounds__(kThreads) ste_grad_input_kernel(const float* __restrict__ dY,
                                                                 const uint8_t* __restrict__ packed,
                                                                 const float* __restrict__ gamma, int M, int N,
                                                                 int K, float* __restrict__ dX) {
    pdl_wait_then_release();
    __shared__ __align__(16) float sA[2][kChunk][kTile + kPad];
    __shared__ __align__(16) float sB[2][kChunk][kTile + kPad];
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const int m0 = blockIdx.y * kTile, k0 = blockIdx.x * kTile;
    const int KB = K / 4;
    float ra[8];
    uint32_t rb[2];
    auto load = [&](int n0) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = tid + kThreads * u;
            const int m = m0 + e / kChunk, n = n0 + e % kChunk;
            ra[u] = (m < M && n < N) ? __ldg(dY + static_cast<int64_t>(m) * N + n) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int e = tid + kThreads * u;
            const int n = n0 + e / (kTile / 4), kb = k0 / 4 + e % (kTile / 4);
            rb[u] = (n < N && kb < KB) ? __ldg(packed + static_cast<int64_t>(n) * KB + kb) : 0u;
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = tid + kThreads * u;
            sA[buf][e % kChunk][e / kChunk] = ra[u];
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int e = tid + kThreads * u;
            const int r = e / (kTile / 4), b = e % (kTile / 4);
            *reinterpret_cast<float4*>(&sB[buf][r][4 * b]) =
                make_float4(code_of(rb[u], 0), code_of(rb[u], 1), code_of(rb[u], 2), code_of(rb[u], 3));
        }
    };
    float acc[8][8] = {};
    load(0);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int n0 = 0; n0 < N; n0 += kChunk) {
        const bool more = n0 + kChunk < N;
        if (more) load(n0 + kChunk);
        chunk_fma(sA[buf], sB[buf], ty, tx, acc);
        if (more) store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
    const float g = *gamma;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int m = m0 + out_index(ty, i / 4) + i % 4;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int k = k0 + out_index(tx, j / 4) + j % 4;
            if (k < K) dX[static_cast<int64_t>(m) * K + k] = __fmul_rn(g, acc[i][j]);
        }
    }
}

// dW tile (rows n0.., columns k0..): A = dY[m, n] / s[m] staged as [m][n], B = x_q[m, k].
// Per chunk a thread loads 8 dY values and 8 x_q values (e = tid + 256 u: token e / 128,
// column e % 128).
__global__ void __launch_bounds__(kThreads) ste_grad_weight_kernel(const float* __restrict__ dY,
                                                                  const int8_t* __restrict__ xq,
                                                                  const float* __restrict__ s,
                                                                  const float* __restrict__ gamma, int M, int N,
                                                                  int K, float* __restrict__ dW) {
    pdl_wait_then_release();
    __shared__ __align__(16) float sA[2][kChunk][kTile + kPad];
    __shared__ __align__(16) float sB[2][kChunk][kTile + kPad];
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const int n0 = blockIdx.y * kTile, k0 = blockIdx.x * kTile;
    float ra[8], rb[8];
    auto load = [&](int mc) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = tid + kThreads * u;
            const int m = mc + e / kTile, c = e % kTile;
            const int n = n0 + c, k = k0 + c;
            ra[u] = (m < M && n < N) ? __fdiv_rn(__ldg(dY + static_cast<int64_t>(m) * N + n), __ldg(s + m)) : 0.0f;
            rb[u] = (m < M && k < K) ? static_cast<float>(__ldg(xq + static_cast<int64_t>(m) * K + k)) : 0.0f;
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = tid + kThreads * u;
            sA[buf][e / kTile][e % kTile] = ra[u];
            sB[buf][e / kTile][e % kTile] = rb[u];
        }
    };
    float acc[8][8] = {};
    load(0);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int mc = 0; mc < M; mc += kChunk) {
        const bool more = mc + kChunk < M;
        if (more) load(mc + kChunk);
        chunk_fma(sA[buf], sB[buf], ty, tx, acc);
        if (more) store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
    const float g = *gamma;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int n = n0 + out_index(ty, i / 4) + i % 4;
        if (n >= N) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int k = k0 + out_index(tx, j / 4) + j % 4;
            if (k < K) dW[static_cast<int64_t>(n) * K + k] = __fmul_rn(g, acc[i][j]);
        }
    }
}

}  // namespace

cudaError_t launch_ste_grad_input(const float* dY, const uint8_t* packed, const float* gamma, int64_t M, int64_t N,
                                  int64_t K, float* dX, cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>((K + kTile - 1) / kTile), static_cast<unsigned>((M + kTile - 1) / kTile));
    return launch_pdl(ste_grad_input_kernel, grid, dim3(kThreads), 0, stream, dim3(kNoCluster), dY, packed, gamma,
                      static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), dX);
}

cudaError_t launch_ste_grad_weight(const float* dY, const int8_t* xq, const float* s, const float* gamma, int64_t M,
                                   int64_t N, int64_t K, float* dW, cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>((K + kTile - 1) / kTile), static_cast<unsigned>((N + kTile - 1) / kTile));
    return launch_pdl(ste_grad_weight_kernel, grid, dim3(kThreads), 0, stream, dim3(kNoCluster), dY, xq, s, gamma,
                      static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), dW);
}

}  // namespace bl
