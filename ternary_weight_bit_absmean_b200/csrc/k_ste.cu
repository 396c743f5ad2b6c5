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
// Both are output-stationary SIMT tiles: a 64 x 64 output tile per block of 256
// threads, 4 x 4 outputs per thread in fp32 registers, the contraction in chunks of 32
// staged through shared memory (operands expanded to fp32 there: codes to -1/0/+1,
// x_q to its integer value, dY divided by s for dW).  The products with a code are exact
// and the sums round in fp32; the result is scaled by gamma once.
#include <cuda_runtime.h>

#include <cstdint>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {
namespace {

constexpr int kTile = 64;   // output tile edge
constexpr int kChunk = 32;  // contraction chunk
constexpr int kThreads = 256;

__device__ __forceinline__ float code_of(uint32_t byte, int i) {
    const uint32_t c = (byte >> (2 * i)) & 3u;
    return c == 1u ? 1.0f : (c == 2u ? -1.0f : 0.0f);  // 11 reads as 0
}

// dX tile (tokens m0.., columns k0..): A = dY[m, n] (staged transposed as [n][m]),
// B = codes[n, k] expanded from the 2-bit rows.
__global__ void __launch_bounds__(kThreads) ste_grad_input_kernel(const float* __restrict__ dY,
                                                                 const uint8_t* __restrict__ packed,
                                                                 const float* __restrict__ gamma, int M, int N,
                                                                 int K, float* __restrict__ dX) {
    pdl_wait_then_release();
    __shared__ __align__(16) float sA[kChunk][kTile + 4];
    __shared__ __align__(16) float sB[kChunk][kTile + 4];
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const int m0 = blockIdx.y * kTile, k0 = blockIdx.x * kTile;
    const int KB = K / 4;
    float acc[4][4] = {};
    for (int n0 = 0; n0 < N; n0 += kChunk) {
        // dY[m0 + r][n0 + c]: 64 x 32, c fastest (coalesced), stored transposed
        for (int e = tid; e < kTile * kChunk; e += kThreads) {
            const int r = e / kChunk, c = e % kChunk;
            const int m = m0 + r, n = n0 + c;
            sA[c][r] = (m < M && n < N) ? __ldg(dY + static_cast<int64_t>(m) * N + n) : 0.0f;
        }
        // codes of rows n0..n0+31, columns k0..k0+63: 16 packed bytes per row
        for (int e = tid; e < kChunk * (kTile / 4); e += kThreads) {
            const int r = e / (kTile / 4), b = e % (kTile / 4);
            const int n = n0 + r, kb = k0 / 4 + b;
            const uint32_t byte = (n < N && kb < KB) ? __ldg(packed + static_cast<int64_t>(n) * KB + kb) : 0u;
#pragma unroll
            for (int i = 0; i < 4; ++i) sB[r][4 * b + i] = code_of(byte, i);
        }
        __syncthreads();
#pragma unroll 8
        for (int c = 0; c < kChunk; ++c) {
            const float4 a = *reinterpret_cast<const float4*>(&sA[c][4 * ty]);
            const float4 b = *reinterpret_cast<const float4*>(&sB[c][4 * tx]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    const float g = *gamma;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + 4 * ty + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = k0 + 4 * tx + j;
            if (k < K) dX[static_cast<int64_t>(m) * K + k] = __fmul_rn(g, acc[i][j]);
        }
    }
}

// dW tile (rows n0.., columns k0..): A = dY[m, n] / s[m] (as [m][n]), B = x_q[m, k].
__global__ void __launch_bounds__(kThreads) ste_grad_weight_kernel(const float* __restrict__ dY,
                                                                  const int8_t* __restrict__ xq,
                                                                  const float* __restrict__ s,
                                                                  const float* __restrict__ gamma, int M, int N,
                                                                  int K, float* __restrict__ dW) {
    pdl_wait_then_release();
    __shared__ __align__(16) float sA[kChunk][kTile + 4];
    __shared__ __align__(16) float sB[kChunk][kTile + 4];
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const int n0 = blockIdx.y * kTile, k0 = blockIdx.x * kTile;
    float acc[4][4] = {};
    for (int mc = 0; mc < M; mc += kChunk) {
        for (int e = tid; e < kChunk * kTile; e += kThreads) {
            const int r = e / kTile, c = e % kTile;
            const int m = mc + r;
            const int n = n0 + c, k = k0 + c;
            sA[r][c] = (m < M && n < N) ? __fdiv_rn(__ldg(dY + static_cast<int64_t>(m) * N + n), __ldg(s + m)) : 0.0f;
            sB[r][c] = (m < M && k < K) ? static_cast<float>(__ldg(xq + static_cast<int64_t>(m) * K + k)) : 0.0f;
        }
        __syncthreads();
#pragma unroll 8
        for (int r = 0; r < kChunk; ++r) {
            const float4 a = *reinterpret_cast<const float4*>(&sA[r][4 * ty]);
            const float4 b = *reinterpret_cast<const float4*>(&sB[r][4 * tx]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    const float g = *gamma;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int n = n0 + 4 * ty + i;
        if (n >= N) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = k0 + 4 * tx + j;
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
