// k_tl5.cu -- the 1.6-bit weight format: five ternary codes per byte.
//
// "1-bit & Ternary LLMs (BitNet b1.58)", "What it is (the intuition)": a ternary weight
// carries log2(3) ~ 1.58 bits and packs to about 1.6 bits in practice; "What 1.58 Bits
// Actually Changes", "How the low-bit linear path works": several ternary values share
// a storage unit and are unpacked where they are used.  3^5 = 243 <= 256, so a byte
// holds five codes: 1.6 bits each, 20% fewer weight bytes than the 2-bit format.
//
// Format (uint8 [N, 16 * ceil(K / 80)], K % 16 == 0):
//   digit t = c + 1 in {0, 1, 2};  a row is cut into blocks of 80 codes, 16 bytes each;
//   byte j of block b holds the codes k = 80 b + 16 p + j (p = 0..4, "plane" p) as
//   v = sum_p t_p 3^(4-p), stored in 8-bit fixed point: B = ceil(256 v / 243).
//   Reading: v = floor(243 B / 256), defined for every byte value.  Codes past K (the
//   last block's missing planes) are written as 0 and never read.
//
// Decoding without a division.  With B = ceil(256 v / 243), h_p = floor(B 3^(p+1) / 256)
// equals floor(v / 3^(4-p)), the number formed by the first p + 1 digits, for every p
// (the error term B - 256 v / 243 < 1 grows by 3^(p+1) / 256 < 1 / 3^(4-p), too little
// to cross an integer).  So digit p is h_p - 3 h_(p-1).  For any byte value the same
// differences are floor(3a) - 3 floor(a) in {0, 1, 2} and sum to floor(243 B / 256),
// which is the reading above.  Four bytes are decoded at once: the even and odd bytes
// of a word are spread into 16-bit lanes (B 3^5 <= 61965 fits a lane), multiplied by
// 3^(p+1), and byte 1 of every lane (the floor by 256) is gathered back into one word
// with a byte permute.  h_p - 3 h_(p-1) over a whole word has no borrow (every byte's
// difference is in [0, 2]).  The digits t = c + 1 meet 4 bytes of x_q in one dp4a
// (unsigned by signed bytes), and each token's sum of x_q is subtracted once at the end.
// The four bytes of a word sit at k = 80 b + 16 p + 4 q .. + 3 for word q of the block,
// contiguous in a row-major x_q row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {
namespace {

constexpr int kTl5BlockCodes = 80;
constexpr int kTl5BlockBytes = 16;

// the stored byte of five digits t0..t4 (t0 most significant)
__device__ __forceinline__ uint32_t tl5_byte(uint32_t v) { return (v * 256u + 242u) / 243u; }

// digit of an int8 code; codes outside {-1, 0, +1} are written as 0 and flagged
__device__ __forceinline__ uint32_t tl5_digit(int c, bool& bad) {
    if (c < -1 || c > 1) {
        bad = true;
        return 1u;
    }
    return static_cast<uint32_t>(c + 1);
}

// One thread per output byte: its five codes sit 16 apart in the codes row.
__global__ void __launch_bounds__(256) tl5_pack_kernel(const int8_t* __restrict__ codes, int64_t N, int K,
                                                       int nblk, uint8_t* __restrict__ out,
                                                       int32_t* __restrict__ err) {
    pdl_wait_then_release();
    bool bad = false;
    const int64_t row_bytes = static_cast<int64_t>(nblk) * kTl5BlockBytes;
    const int64_t total = N * row_bytes;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t n = i / row_bytes;
        const int r = static_cast<int>(i - n * row_bytes);
        const int k0 = (r / kTl5BlockBytes) * kTl5BlockCodes + r % kTl5BlockBytes;
        const int8_t* cr = codes + n * K;
        uint32_t v = 0;
#pragma unroll
        for (int p = 0; p < 5; ++p) {
            const int k = k0 + 16 * p;
            v = 3u * v + (k < K ? tl5_digit(cr[k], bad) : 1u);
        }
        out[i] = static_cast<uint8_t>(tl5_byte(v));
    }
    if (bad && err != nullptr) atomicOr(err, kErrBitBadCode);
}

// The same from the 2-bit format (00 -> 0, 01 -> +1, 10 -> -1, 11 read as 0).
__global__ void __launch_bounds__(256) tl5_repack_kernel(const uint8_t* __restrict__ packed, int64_t N, int K,
                                                         int nblk, uint8_t* __restrict__ out) {
    pdl_wait_then_release();
    const int64_t row_bytes = static_cast<int64_t>(nblk) * kTl5BlockBytes;
    const int64_t total = N * row_bytes;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t n = i / row_bytes;
        const int r = static_cast<int>(i - n * row_bytes);
        const int k0 = (r / kTl5BlockBytes) * kTl5BlockCodes + r % kTl5BlockBytes;
        const uint8_t* pr = packed + n * (K / 4);
        uint32_t v = 0;
#pragma unroll
        for (int p = 0; p < 5; ++p) {
            const int k = k0 + 16 * p;
            uint32_t t = 1u;
            if (k < K) {
                const uint32_t c2 = (__ldg(pr + k / 4) >> (2 * (k % 4))) & 3u;
                t = c2 == 1u ? 2u : (c2 == 2u ? 0u : 1u);
            }
            v = 3u * v + t;
        }
        out[i] = static_cast<uint8_t>(tl5_byte(v));
    }
}

// Digits (0, 1, 2 per byte) of plane P for the four bytes whose even and odd bytes are
// spread into the 16-bit lanes of `even` and `odd`, given the previous plane's h (0
// before plane 0); h is updated.
template <int P>
__device__ __forceinline__ uint32_t tl5_digits(uint32_t even, uint32_t odd, uint32_t& h) {
    constexpr uint32_t kMul = P == 0 ? 3u : P == 1 ? 9u : P == 2 ? 27u : P == 3 ? 81u : 243u;
    const uint32_t hn = __byte_perm(even * kMul, odd * kMul, 0x7351);
    const uint32_t d = hn - 3u * h;  // no borrow: every byte's difference is in [0, 2]
    h = hn;
    return d;
}

// acc + sum of the four products of unsigned bytes a with signed bytes b
__device__ __forceinline__ uint32_t dp4a_us(uint32_t a, uint32_t b, uint32_t acc) {
    uint32_t d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(acc));
    return d;
}

__device__ __forceinline__ void tl5_store(void* out, int kind, int64_t idx, int acc, float fac) {
    if (kind == kOutI32) {
        static_cast<int*>(out)[idx] = acc;
        return;
    }
    const float y = __fmul_rn(__int2float_rn(acc), fac);
    if (kind == kOutF32)
        static_cast<float*>(out)[idx] = y;
    else
        static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(y);
}

// Decode GEMV: one warp per output row, lanes over the row's 16-byte blocks (kUnroll
// blocks in flight per lane), MT tokens per pass (blockIdx.y selects the group of MT
// tokens).  x_q row-major; its 16-byte pieces are read through L1, which every warp of
// the SM shares.
//
// The dot products use the digits t = c + 1 directly (unsigned bytes against the
// signed x_q bytes) and subtract each token's sum of x_q once at the end:
// sum_k c_k x_k = sum_k t_k x_k - sum_k x_k.  The block computes those sums first.  The
// sums are exact modulo 2^32 and the result's magnitude is at most 128 K < 2^31, so the
// wrapped unsigned arithmetic gives it exactly.  Only the last block of a row can miss
// planes (K % 80 != 0): it alone checks each plane against K and skips the missing ones.
constexpr int kTl5Warps = 8;
constexpr int kTl5Threads = 32 * kTl5Warps;
constexpr int kUnroll = 4;

template <int MT, bool PARTIAL>
__device__ __forceinline__ void tl5_block(const uint4 w, const int8_t* xb, int K, int kb, int mt,
                                          uint32_t (&acc)[MT]) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    uint32_t ev[4], od[4], h[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        ev[q] = __byte_perm(ww[q], 0u, 0x4240);  // bytes 0, 2 -> 16-bit lanes
        od[q] = __byte_perm(ww[q], 0u, 0x4341);  // bytes 1, 3
        h[q] = 0u;
    }
#pragma unroll
    for (int p = 0; p < 5; ++p) {
        if (PARTIAL && kb + 16 * p >= K) break;
        uint32_t d[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (p == 0) d[q] = tl5_digits<0>(ev[q], od[q], h[q]);
            if (p == 1) d[q] = tl5_digits<1>(ev[q], od[q], h[q]);
            if (p == 2) d[q] = tl5_digits<2>(ev[q], od[q], h[q]);
            if (p == 3) d[q] = tl5_digits<3>(ev[q], od[q], h[q]);
            if (p == 4) d[q] = tl5_digits<4>(ev[q], od[q], h[q]);
        }
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            if (j < mt) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xb + static_cast<int64_t>(j) * K + 16 * p));
                uint32_t a = acc[j];
                a = dp4a_us(d[0], xv.x, a);
                a = dp4a_us(d[1], xv.y, a);
                a = dp4a_us(d[2], xv.z, a);
                a = dp4a_us(d[3], xv.w, a);
                acc[j] = a;
            }
        }
    }
}

template <int MT>
__global__ void __launch_bounds__(kTl5Threads) gemv_tl5_kernel(const int8_t* __restrict__ xq,
                                                              const float* __restrict__ s,
                                                              const uint8_t* __restrict__ w5,
                                                              const float* __restrict__ gamma, int M, int N,
                                                              int K, int nblk, void* __restrict__ out,
                                                              int okind, int grow) {
    pdl_wait_then_release();
    __shared__ uint32_t xsum[MT];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * MT;
    const int mt = M - m0 < MT ? M - m0 : MT;
    const int8_t* x0 = xq + static_cast<int64_t>(m0) * K;

    // every token's sum of x_q, shared by the block's rows
    if (threadIdx.x < MT) xsum[threadIdx.x] = 0u;
    __syncthreads();
    for (int j = 0; j < mt; ++j) {
        uint32_t part = 0u;
        const uint4* xr = reinterpret_cast<const uint4*>(x0 + static_cast<int64_t>(j) * K);
        for (int i = threadIdx.x; i < K / 16; i += kTl5Threads) {
            const uint4 xv = __ldg(xr + i);
            part = dp4a_us(0x01010101u, xv.x, part);
            part = dp4a_us(0x01010101u, xv.y, part);
            part = dp4a_us(0x01010101u, xv.z, part);
            part = dp4a_us(0x01010101u, xv.w, part);
        }
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        if (lane == 0) atomicAdd(&xsum[j], part);
    }
    __syncthreads();

    const int64_t row = static_cast<int64_t>(blockIdx.x) * kTl5Warps + warp;
    if (row >= N) return;
    const uint4* wr = reinterpret_cast<const uint4*>(w5 + row * static_cast<int64_t>(nblk) * kTl5BlockBytes);
    const int nfull = K / kTl5BlockCodes;  // blocks with all five planes inside K

    uint32_t acc[MT];
#pragma unroll
    for (int j = 0; j < MT; ++j) acc[j] = 0u;

    for (int b0 = 0; b0 < nblk; b0 += 32 * kUnroll) {
        uint4 wv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int blk = b0 + lane + 32 * u;
            wv[u] = blk < nblk ? __ldcs(wr + blk) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int blk = b0 + lane + 32 * u;
            const int kb = blk * kTl5BlockCodes;
            if (blk < nfull)
                tl5_block<MT, false>(wv[u], x0 + kb, K, kb, mt, acc);
            else if (blk < nblk)
                tl5_block<MT, true>(wv[u], x0 + kb, K, kb, mt, acc);
        }
    }
#pragma unroll
    for (int j = 0; j < MT; ++j)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);

#pragma unroll
    for (int j = 0; j < MT; ++j) {
        if (lane == j && j < mt) {
            const int m = m0 + j;
            const int a = static_cast<int>(acc[j] - xsum[j]);
            float fac = 0.0f;
            if (okind != kOutI32) fac = __fdiv_rn(grow ? gamma[row] : *gamma, s[m]);
            tl5_store(out, okind, static_cast<int64_t>(m) * N + row, a, fac);
        }
    }
}

int tl5_blocks(int64_t K) { return static_cast<int>((K + kTl5BlockCodes - 1) / kTl5BlockCodes); }

dim3 tl5_elementwise_grid(int64_t total) {
    int64_t g = (total + 255) / 256;
    const int64_t cap = int64_t(148) * 32;
    return dim3(static_cast<unsigned>(g < 1 ? 1 : (g > cap ? cap : g)));
}

template <int MT>
cudaError_t launch_tl5_mt(const int8_t* xq, const float* s, const uint8_t* w5, const float* gamma, int64_t M,
                          int64_t N, int64_t K, void* out, int kind, cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>((N + kTl5Warps - 1) / kTl5Warps), static_cast<unsigned>((M + MT - 1) / MT));
    return launch_pdl(gemv_tl5_kernel<MT>, grid, dim3(kTl5Threads), 0, stream, dim3(kNoCluster), xq, s, w5,
                      gamma, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), tl5_blocks(K), out,
                      out_kind_of(kind), gamma_rows_of(kind));
}

}  // namespace

int64_t tl5_row_bytes(int64_t K) { return static_cast<int64_t>(tl5_blocks(K)) * kTl5BlockBytes; }

cudaError_t launch_tl5_pack(const int8_t* codes, int64_t N, int64_t K, uint8_t* out, int32_t* err,
                            cudaStream_t stream) {
    return launch_pdl(tl5_pack_kernel, tl5_elementwise_grid(N * tl5_row_bytes(K)), dim3(256), 0, stream,
                      dim3(kNoCluster), codes, N, static_cast<int>(K), tl5_blocks(K), out, err);
}

cudaError_t launch_tl5_repack(const uint8_t* packed, int64_t N, int64_t K, uint8_t* out, cudaStream_t stream) {
    return launch_pdl(tl5_repack_kernel, tl5_elementwise_grid(N * tl5_row_bytes(K)), dim3(256), 0, stream,
                      dim3(kNoCluster), packed, N, static_cast<int>(K), tl5_blocks(K), out);
}

cudaError_t launch_gemv_tl5(const int8_t* xq, const float* s, const uint8_t* w5, const float* gamma, int64_t M,
                            int64_t N, int64_t K, void* out, int kind, cudaStream_t stream) {
    if (M <= 1) return launch_tl5_mt<1>(xq, s, w5, gamma, M, N, K, out, kind, stream);
    if (M <= 2) return launch_tl5_mt<2>(xq, s, w5, gamma, M, N, K, out, kind, stream);
    if (M <= 4) return launch_tl5_mt<4>(xq, s, w5, gamma, M, N, K, out, kind, stream);
    if (M <= 8) return launch_tl5_mt<8>(xq, s, w5, gamma, M, N, K, out, kind, stream);
    return launch_tl5_mt<16>(xq, s, w5, gamma, M, N, K, out, kind, stream);
}

}  // namespace bl
