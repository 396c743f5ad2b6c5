// k_quant.cu -- the HBM-bound quantisation kernels of the BitLinear forward:
//   * absmean partial sums of |W| (fp64) and the fused gamma + ternarise + 2-bit pack,
//   * packing of caller-supplied int8 ternary codes,
//   * per-token absmax int8 activation quantisation.
//
// Definitions ("1-bit & Ternary LLMs (BitNet b1.58)", "How it works", block
// "BitNet b1.58 (Feb 2024)"): gamma = (1/nm) sum |W_ij| (+ eps),
// W~ = RoundClip(W / gamma, -1, 1).  Block "BitNet (Oct 2023)" and "What 1.58 Bits
// Actually Changes" ("How the low-bit linear path works"): activations scaled per token
// by their absmax to signed 8 bits with no zero point.
//
// Bit-exactness: every float step is the IEEE operation the definition names --
// __fdiv_rn for W / gamma and 127 / absmax, __fmul_rn for x * s, and a round half to
// even for round() (__float2int_rn for the weights, an exact add of 1.5 * 2^23 for the
// activations); nothing here is compiled with fast-math.
#include <cstdint>
#include <cuda_runtime.h>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {
namespace {

constexpr int kAbsThreads = 256;

// 2-bit code of round-half-even(t) clipped to [-1, 1]: 01 for +1, 10 for -1, 00 for 0.
__device__ __forceinline__ uint32_t code_of_ratio(float t) {
    const int q = __float2int_rn(t);
    return q >= 1 ? 1u : (q <= -1 ? 2u : 0u);
}

__device__ __forceinline__ uint32_t pack4_codes(float4 w, float gamma) {
    return code_of_ratio(__fdiv_rn(w.x, gamma)) | (code_of_ratio(__fdiv_rn(w.y, gamma)) << 2) |
           (code_of_ratio(__fdiv_rn(w.z, gamma)) << 4) | (code_of_ratio(__fdiv_rn(w.w, gamma)) << 6);
}

// ---------------------------------------------------------- absmean partials --
// Each block accumulates |W| over a grid-stride range of float4s in fp64 and writes
// one fp64 partial.  The partials are summed in a fixed order by the pack kernel.
__global__ void __launch_bounds__(kAbsThreads) absmean_partials_kernel(const float4* __restrict__ W4,
                                                                      int64_t n4,
                                                                      double* __restrict__ partials) {
    pdl_wait_then_release();
    double acc = 0.0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kAbsThreads;
    int64_t i = static_cast<int64_t>(blockIdx.x) * kAbsThreads + threadIdx.x;
    // four float4 loads in flight per thread, summed in the order of the plain loop
    for (; i + 3 * stride < n4; i += 4 * stride) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldg(W4 + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            acc += static_cast<double>(fabsf(v[u].x));
            acc += static_cast<double>(fabsf(v[u].y));
            acc += static_cast<double>(fabsf(v[u].z));
            acc += static_cast<double>(fabsf(v[u].w));
        }
    }
    for (; i < n4; i += stride) {
        const float4 v = __ldg(W4 + i);
        acc += static_cast<double>(fabsf(v.x));
        acc += static_cast<double>(fabsf(v.y));
        acc += static_cast<double>(fabsf(v.z));
        acc += static_cast<double>(fabsf(v.w));
    }
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    __shared__ double warp_sum[kAbsThreads / 32];
    if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < kAbsThreads / 32; ++w) t += warp_sum[w];
        partials[blockIdx.x] = t;
    }
}

// -------------------------------------------------------- ternarise + pack --
// Every block first forms gamma: from the caller's device scalar, or by summing the
// absmean partials in a fixed order (identical in every block), dividing by N*K in
// fp64, rounding to fp32 and adding eps in fp32.  Block 0 stores it.  Then each thread
// turns 16 weights (four float4) into one 32-bit word of packed codes.
__global__ void __launch_bounds__(256) ternarise_pack_kernel(
    const float4* __restrict__ W4, int64_t numel, const float* __restrict__ gamma_in,
    const double* __restrict__ partials, int nparts, float eps, float* __restrict__ gamma_out,
    uint8_t* __restrict__ packed) {
    pdl_wait_then_release();
    __shared__ float s_gamma;
    if (threadIdx.x < 32) {
        float g;
        if (gamma_in != nullptr) {
            g = *gamma_in;
        } else {
            double sum = 0.0;
            for (int i = threadIdx.x; i < nparts; i += 32) sum += partials[i];
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            g = __fadd_rn(__double2float_rn(sum / static_cast<double>(numel)), eps);
            if (blockIdx.x == 0 && threadIdx.x == 0) *gamma_out = g;
        }
        if (threadIdx.x == 0) s_gamma = g;
    }
    __syncthreads();
    const float gamma = s_gamma;

    const int64_t ngroups = numel / 16;
    uint32_t* packed32 = reinterpret_cast<uint32_t*>(packed);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < ngroups;
         i += stride) {
        const float4* src = W4 + 4 * i;
        const float4 a = __ldg(src), b = __ldg(src + 1), c = __ldg(src + 2), d = __ldg(src + 3);
        packed32[i] = pack4_codes(a, gamma) | (pack4_codes(b, gamma) << 8) |
                      (pack4_codes(c, gamma) << 16) | (pack4_codes(d, gamma) << 24);
    }
    // tail: numel % 16 weights (numel is a multiple of 4), one byte per float4
    const int64_t done4 = ngroups * 4, n4 = numel / 4;
    for (int64_t j = done4 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < n4;
         j += stride)
        packed[j] = static_cast<uint8_t>(pack4_codes(__ldg(W4 + j), gamma));
}

// -------------------------------------------------------------- pack codes --
__device__ __forceinline__ uint32_t encode_byte_code(uint32_t b, bool& bad) {
    if (b == 0x01u) return 1u;
    if (b == 0xFFu) return 2u;
    if (b != 0u) bad = true;
    return 0u;
}

// Four int8 codes (one per byte of w) -> one packed byte.  For valid bytes (0x00, 0x01,
// 0xFF) the "-1" flag is the sign bit and the "+1" flag the low bit without the sign;
// the flags of byte j sit at bits 8j and 8j+1 of x, and one multiply by
// 2^24 + 2^18 + 2^12 + 2^6 moves them to bits 24+2j (the other partial products land
// in disjoint fields below bit 24 or above bit 31, so nothing carries).  A word whose
// flags do not re-expand to itself holds an invalid code; it takes the per-byte path,
// which writes invalid codes as 00.
__device__ __forceinline__ uint32_t pack_word_codes(uint32_t w, bool& bad) {
    const uint32_t minus = (w >> 7) & 0x01010101u;
    const uint32_t plus = w & ~(w >> 7) & 0x01010101u;
    if ((plus | (minus * 0xFFu)) != w) {
        return encode_byte_code(w & 0xFFu, bad) | (encode_byte_code((w >> 8) & 0xFFu, bad) << 2) |
               (encode_byte_code((w >> 16) & 0xFFu, bad) << 4) | (encode_byte_code(w >> 24, bad) << 6);
    }
    const uint32_t x = plus | (minus << 1);
    return (x * 0x01041040u) >> 24;
}

__global__ void __launch_bounds__(256) pack_codes_kernel(const uint4* __restrict__ codes16,
                                                         int64_t numel,
                                                         uint8_t* __restrict__ packed,
                                                         int32_t* __restrict__ err) {
    pdl_wait_then_release();
    bool bad = false;
    const int64_t ngroups = numel / 16;  // 16 codes -> one 32-bit word
    uint32_t* packed32 = reinterpret_cast<uint32_t*>(packed);
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    // four groups per thread per step, all loads issued before any is used
    int64_t i = tid;
    for (; i + 3 * nthreads < ngroups; i += 4 * nthreads) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldg(codes16 + i + u * nthreads);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            packed32[i + u * nthreads] = pack_word_codes(v[u].x, bad) | (pack_word_codes(v[u].y, bad) << 8) |
                                         (pack_word_codes(v[u].z, bad) << 16) | (pack_word_codes(v[u].w, bad) << 24);
    }
    for (; i < ngroups; i += nthreads) {
        const uint4 v = __ldg(codes16 + i);
        packed32[i] = pack_word_codes(v.x, bad) | (pack_word_codes(v.y, bad) << 8) |
                      (pack_word_codes(v.z, bad) << 16) | (pack_word_codes(v.w, bad) << 24);
    }
    const uint32_t* codes4 = reinterpret_cast<const uint32_t*>(codes16);
    for (int64_t j = ngroups * 4 + tid; j < numel / 4; j += nthreads)
        packed[j] = static_cast<uint8_t>(pack_word_codes(__ldg(codes4 + j), bad));
    if (bad && err != nullptr) atomicOr(err, kErrBitBadCode);
}

// --------------------------------------------------- activation quantisation --
// round-half-even(x * s) as an int8 bit pattern in the low byte of the result.
// t = fl(x * s) satisfies |t| <= 127 (1 + 2^-23): s = fl(127 / max(a, eps)) with
// |x| <= a, or |x| <= a < eps.  Adding 1.5 * 2^23 to such a t rounds it to the nearest
// integer, ties to even, in one IEEE add, leaving that integer in the low mantissa
// bits; rint(t) is within [-127, 127], so the clip to [-128, 127] is never active.
__device__ __forceinline__ uint32_t q8_bits(float x, float s) {
    return __float_as_uint(__fadd_rn(__fmul_rn(x, s), 12582912.0f));
}

// 8 bf16 (one 16-byte vector) -> 8 int8 (8 bytes), in order.
__device__ __forceinline__ uint2 quant8(uint4 v, float s) {
    uint32_t q[8];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        q[2 * i] = q8_bits(__uint_as_float(w[i] << 16), s);
        q[2 * i + 1] = q8_bits(__uint_as_float(w[i] & 0xFFFF0000u), s);
    }
    uint2 r;
    r.x = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
    r.y = __byte_perm(__byte_perm(q[4], q[5], 0x0040), __byte_perm(q[6], q[7], 0x0040), 0x5410);
    return r;
}

// 16 bf16 (two 16-byte vectors) -> 16 int8 in the even/odd k16 layout: the group's
// elements 0,2,4,6 | 8,10,12,14 | 1,3,5,7 | 9,11,13,15.
__device__ __forceinline__ uint4 quant16_evenodd(uint4 a, uint4 b, float s) {
    uint32_t q[16];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        q[2 * i] = q8_bits(__uint_as_float(w[i] << 16), s);
        q[2 * i + 1] = q8_bits(__uint_as_float(w[i] & 0xFFFF0000u), s);
    }
    auto pack4 = [&](int e0, int e1, int e2, int e3) {
        return __byte_perm(__byte_perm(q[e0], q[e1], 0x0040), __byte_perm(q[e2], q[e3], 0x0040), 0x5410);
    };
    return make_uint4(pack4(0, 2, 4, 6), pack4(8, 10, 12, 14), pack4(1, 3, 5, 7), pack4(9, 11, 13, 15));
}

// 16 bf16 -> 16 int8 in the stride-4 k16 layout: word i of the group holds the
// elements i, i+4, i+8, i+12.
__device__ __forceinline__ uint4 quant16_stride4(uint4 a, uint4 b, float s) {
    uint32_t q[16];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        q[2 * i] = q8_bits(__uint_as_float(w[i] << 16), s);
        q[2 * i + 1] = q8_bits(__uint_as_float(w[i] & 0xFFFF0000u), s);
    }
    auto pack4 = [&](int e0, int e1, int e2, int e3) {
        return __byte_perm(__byte_perm(q[e0], q[e1], 0x0040), __byte_perm(q[e2], q[e3], 0x0040), 0x5410);
    };
    return make_uint4(pack4(0, 4, 8, 12), pack4(1, 5, 9, 13), pack4(2, 6, 10, 14), pack4(3, 7, 11, 15));
}

// |x| of two bf16 at once as unsigned 16-bit lanes; for finite values the integer
// order of |x| bit patterns is the float order.
__device__ __forceinline__ uint32_t absmax_vec(uint32_t m, uint4 v) {
    m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
    return m;
}

// A unit is the U 16-byte input vectors of one row that make one output store.  The
// output layout L (XqLayout) fixes U: 1 (8 elements, row-major) or 2 (16 elements, the
// even/odd or stride-4 k16 orders).
template <int L>
constexpr int kUnitVecs = L == kXqRowMajor ? 1 : 2;

template <int U>
struct Unit {
    uint4 v[U];
};

template <int U>
__device__ __forceinline__ Unit<U> load_unit(const uint4* xr, int idx) {
    Unit<U> u;
#pragma unroll
    for (int i = 0; i < U; ++i) u.v[i] = __ldg(xr + U * idx + i);
    return u;
}

template <int L, int U>
__device__ __forceinline__ void store_unit(uint8_t* qrow, int idx, const Unit<U>& u, float s) {
    if constexpr (L == kXqRowMajor)
        reinterpret_cast<uint2*>(qrow)[idx] = quant8(u.v[0], s);
    else if constexpr (L == kXqEvenOdd16)
        reinterpret_cast<uint4*>(qrow)[idx] = quant16_evenodd(u.v[0], u.v[1], s);
    else
        reinterpret_cast<uint4*>(qrow)[idx] = quant16_stride4(u.v[0], u.v[1], s);
}

// One group of G threads per token row; each thread keeps up to NV units of its row in
// registers between the absmax pass and the quantise pass (longer rows are re-read for
// the remainder).  Short rows (G = 32) give each warp R rows, whose loads are all issued
// before the first reduction.  Needs K % (8 U) == 0.
// VPT is the number of 16-byte vectors a thread keeps (NV = VPT / U units).
template <int G, int R, int L, int VPT>
__global__ void __launch_bounds__(G > 256 ? G : 256)
    act_quant_vec_kernel(const uint4* __restrict__ X, int64_t M, int K, float eps,
                         uint8_t* __restrict__ xq, float* __restrict__ s_out) {
    pdl_wait_then_release();
    constexpr int U = kUnitVecs<L>;
    constexpr int CTA = G > 256 ? G : 256;
    constexpr int RPC = CTA / G * R;  // rows per block
    constexpr int WPG = G / 32;       // warps per row group
    constexpr int NV = VPT / U;
    static_assert(R == 1 || G == 32, "several rows per group only for warp groups");
    __shared__ uint32_t red[CTA / 32];

    const int sub = threadIdx.x / G;
    const int j = threadIdx.x % G;
    const int nunit = K / (8 * U);
    const int64_t row_base = static_cast<int64_t>(blockIdx.x) * RPC + static_cast<int64_t>(sub) * R;

    Unit<U> v[R][NV];
    uint32_t m2[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t row = row_base + r;
        const bool active = row < M;
        const uint4* xr = X + (active ? row : 0) * (K / 8);
        m2[r] = 0;
#pragma unroll
        for (int u = 0; u < NV; ++u) {
            const int idx = j + u * G;
            if (active && idx < nunit) {
                v[r][u] = load_unit<U>(xr, idx);
            } else {
#pragma unroll
                for (int i = 0; i < U; ++i) v[r][u].v[i] = make_uint4(0, 0, 0, 0);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t row = row_base + r;
        const bool active = row < M;
        const uint4* xr = X + (active ? row : 0) * (K / 8);
#pragma unroll
        for (int u = 0; u < NV; ++u)
#pragma unroll
            for (int i = 0; i < U; ++i) m2[r] = absmax_vec(m2[r], v[r][u].v[i]);
        for (int idx = j + NV * G; active && idx < nunit; idx += G) {
            const Unit<U> t = load_unit<U>(xr, idx);
#pragma unroll
            for (int i = 0; i < U; ++i) m2[r] = absmax_vec(m2[r], t.v[i]);
        }

        uint32_t am = max(m2[r] & 0xFFFFu, m2[r] >> 16);
        for (int off = 16; off > 0; off >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, off));
        if constexpr (WPG > 1) {
            if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = am;
            __syncthreads();
            am = 0;
#pragma unroll
            for (int w = 0; w < WPG; ++w) am = max(am, red[sub * WPG + w]);
        }
        const float a = __uint_as_float(am << 16);
        const float s = __fdiv_rn(127.0f, fmaxf(a, eps));
        if (!active) continue;
        if (j == 0) s_out[row] = s;
        uint8_t* qrow = xq + row * K;
#pragma unroll
        for (int u = 0; u < NV; ++u) {
            const int idx = j + u * G;
            if (idx < nunit) store_unit<L>(qrow, idx, v[r][u], s);
        }
        for (int idx = j + NV * G; idx < nunit; idx += G) store_unit<L>(qrow, idx, load_unit<U>(xr, idx), s);
    }
}

// ------------------------------------ normalisation + activation quantisation --
// Quant(LN(x)) ("1-bit & Ternary LLMs (BitNet b1.58)", block "BitNet (Oct 2023)": the
// LayerNorm in front of the quantiser; the b1.58 models use RMSNorm):
//   kind 0 (RMSNorm): mu = 0;   kind 1 (LayerNorm): mu = sum(x) / K
//   v = sum((x - mu)^2) / K;  r = 1 / sqrt(v + norm_eps)      (fp64, then mu and r to fp32)
//   x_n = ((x - mu) * r) * w   (fp32, one IEEE rounding per operation)
//   s = 127 / max(max |x_n|, eps),  x_q = rint(x_n s).
// One group of G threads per row; each thread keeps its first units of the row in
// registers across the passes (mean, variance, absmax of x_n, quantise + store) and
// re-reads the rest through L1.  The norm weight w is shared by every row: for K up to
// kNormStageMaxK the block copies it once into shared memory, as the 16-byte chunks of
// each unit with an XOR swizzle so that a warp's float4 reads of consecutive units hit
// distinct bank groups (a direct read has the lanes a whole unit apart).  The sums run in fp64: a different order than a
// sequential sum changes them by ~1e-16 relative, which reaches mu or r only when they
// sit that close to an fp32 rounding boundary; the element-wise part has no order.

// bf16 element i (0 .. 8U-1) of a unit, as fp32 (exact)
template <int U>
__device__ __forceinline__ float unit_elem(const Unit<U>& u, int i) {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&u.v[0]);
    const uint32_t x = w[i >> 1];
    return __uint_as_float((i & 1) ? (x & 0xFFFF0000u) : (x << 16));
}

__device__ __forceinline__ uint32_t pack4_q(uint32_t q0, uint32_t q1, uint32_t q2, uint32_t q3) {
    return __byte_perm(__byte_perm(q0, q1, 0x0040), __byte_perm(q2, q3, 0x0040), 0x5410);
}

// int8 bit patterns (low bytes of q[]) of a unit's E elements, stored in layout L
template <int L>
__device__ __forceinline__ void store_q(uint8_t* qrow, int idx, const uint32_t (&q)[8 * kUnitVecs<L>]) {
    if constexpr (L == kXqRowMajor) {
        reinterpret_cast<uint2*>(qrow)[idx] = make_uint2(pack4_q(q[0], q[1], q[2], q[3]), pack4_q(q[4], q[5], q[6], q[7]));
    } else if constexpr (L == kXqEvenOdd16) {
        reinterpret_cast<uint4*>(qrow)[idx] =
            make_uint4(pack4_q(q[0], q[2], q[4], q[6]), pack4_q(q[8], q[10], q[12], q[14]),
                       pack4_q(q[1], q[3], q[5], q[7]), pack4_q(q[9], q[11], q[13], q[15]));
    } else {
        reinterpret_cast<uint4*>(qrow)[idx] =
            make_uint4(pack4_q(q[0], q[4], q[8], q[12]), pack4_q(q[1], q[5], q[9], q[13]),
                       pack4_q(q[2], q[6], q[10], q[14]), pack4_q(q[3], q[7], q[11], q[15]));
    }
}

constexpr int kNormStageMaxK = 8192;  // K fp32 weights = 32 KB of shared memory, within the default 48 KB

// position of 16-byte chunk c of unit idx in the staged weights (C chunks per unit):
// 8 lanes with consecutive idx land on the 8 distinct 16-byte bank groups of 128 bytes
template <int C>
__device__ __forceinline__ int norm_w_chunk(int idx, int c) {
    return idx * C + (c ^ ((idx / (8 / C)) & (C - 1)));
}

extern __shared__ float4 norm_w_sm[];

// VPT is the number of 16-byte vectors a thread keeps in registers (NV = VPT / U units).
template <int G, int L, int KIND, int VPT>
__global__ void __launch_bounds__(G > 256 ? G : 256)
    norm_act_quant_kernel(const uint4* __restrict__ X, const float* __restrict__ nw, int64_t M, int K,
                          float norm_eps, float eps, uint8_t* __restrict__ xq, float* __restrict__ s_out,
                          int stage_w) {
    pdl_wait_then_release();
    constexpr int U = kUnitVecs<L>;
    constexpr int E = 8 * U;  // elements per unit
    constexpr int C = E / 4;  // 16-byte weight chunks per unit
    constexpr int CTA = G > 256 ? G : 256;
    constexpr int RPC = CTA / G;  // rows per block
    constexpr int WPG = G / 32;   // warps per row group
    constexpr int NV = VPT / U;   // units kept in registers
    __shared__ double red_d[CTA / 32];
    __shared__ float red_f[CTA / 32];

    const int sub = threadIdx.x / G;
    const int j = threadIdx.x % G;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int nunit = K / E;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * RPC + sub;
    const bool active = row < M;
    const uint4* xr = X + (active ? row : 0) * (K / 8);

    Unit<U> v[NV];
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const int idx = j + u * G;
        if (active && idx < nunit) {
            v[u] = load_unit<U>(xr, idx);
        } else {
#pragma unroll
            for (int i = 0; i < U; ++i) v[u].v[i] = make_uint4(0, 0, 0, 0);
        }
    }
    if (stage_w) {
        // element e of w: chunk e / 4 (unit e / E, chunk (e % E) / 4), word e % 4
        float* ws = reinterpret_cast<float*>(norm_w_sm);
        for (int e = threadIdx.x; e < K; e += CTA)
            ws[4 * norm_w_chunk<C>(e / E, (e % E) / 4) + (e & 3)] = __ldg(nw + e);
        __syncthreads();
    }
    // every unit of this thread's share of the row: the cached ones, then the rest
    auto for_units = [&](auto&& fn) {
#pragma unroll
        for (int u = 0; u < NV; ++u)
            if (j + u * G < nunit) fn(j + u * G, v[u]);
        for (int idx = j + NV * G; active && idx < nunit; idx += G) fn(idx, load_unit<U>(xr, idx));
    };
    auto group_sum = [&](double x) {
        for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        if constexpr (WPG > 1) {
            __syncthreads();
            if (lane == 0) red_d[wid] = x;
            __syncthreads();
            x = 0.0;
#pragma unroll
            for (int w = 0; w < WPG; ++w) x += red_d[sub * WPG + w];
        }
        return x;
    };
    auto group_max = [&](float x) {
        for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
        if constexpr (WPG > 1) {
            __syncthreads();
            if (lane == 0) red_f[wid] = x;
            __syncthreads();
            x = 0.0f;
#pragma unroll
            for (int w = 0; w < WPG; ++w) x = fmaxf(x, red_f[sub * WPG + w]);
        }
        return x;
    };

    double mu = 0.0;
    if constexpr (KIND == 1) {
        double sx = 0.0;
        for_units([&](int, const Unit<U>& un) {
#pragma unroll
            for (int i = 0; i < E; ++i) sx += static_cast<double>(unit_elem(un, i));
        });
        mu = group_sum(sx) / static_cast<double>(K);
    }
    double sd = 0.0;
    for_units([&](int, const Unit<U>& un) {
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const double d = static_cast<double>(unit_elem(un, i)) - mu;
            sd += d * d;
        }
    });
    const double r = 1.0 / sqrt(group_sum(sd) / static_cast<double>(K) + static_cast<double>(norm_eps));
    const float mu32 = __double2float_rn(mu), r32 = __double2float_rn(r);
    // the norm weights of unit idx
    auto w_unit = [&](int idx, float (&wv)[E]) {
        if (stage_w) {
#pragma unroll
            for (int c = 0; c < C; ++c) {
                const float4 t = norm_w_sm[norm_w_chunk<C>(idx, c)];
                wv[4 * c] = t.x; wv[4 * c + 1] = t.y; wv[4 * c + 2] = t.z; wv[4 * c + 3] = t.w;
            }
        } else if (nw != nullptr) {
#pragma unroll
            for (int i = 0; i < E; ++i) wv[i] = __ldg(nw + idx * E + i);
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i) wv[i] = 1.0f;
        }
    };
    auto xn_of = [&](const Unit<U>& un, int i, const float (&wv)[E]) {
        return __fmul_rn(__fmul_rn(__fsub_rn(unit_elem(un, i), mu32), r32), wv[i]);
    };
    float am = 0.0f;
    for_units([&](int idx, const Unit<U>& un) {
        float wv[E];
        w_unit(idx, wv);
#pragma unroll
        for (int i = 0; i < E; ++i) am = fmaxf(am, fabsf(xn_of(un, i, wv)));
    });
    const float s = __fdiv_rn(127.0f, fmaxf(group_max(am), eps));
    if (!active) return;
    if (j == 0) s_out[row] = s;
    uint8_t* qrow = xq + row * K;
    for_units([&](int idx, const Unit<U>& un) {
        float wv[E];
        w_unit(idx, wv);
        uint32_t q[E];
#pragma unroll
        for (int i = 0; i < E; ++i) q[i] = q8_bits(xn_of(un, i, wv), s);
        store_q<L>(qrow, idx, q);
    });
}

// Any K: one warp per row, scalar loads.
__global__ void __launch_bounds__(256) act_quant_scalar_kernel(const uint16_t* __restrict__ X,
                                                              int64_t M, int64_t K, float eps,
                                                              int8_t* __restrict__ xq,
                                                              float* __restrict__ s_out) {
    pdl_wait_then_release();
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= M) return;
    const uint16_t* xr = X + row * K;
    uint32_t am = 0;
    for (int64_t k = lane; k < K; k += 32) am = max(am, static_cast<uint32_t>(xr[k] & 0x7FFFu));
    for (int off = 16; off > 0; off >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, off));
    const float s = __fdiv_rn(127.0f, fmaxf(__uint_as_float(am << 16), eps));
    if (lane == 0) s_out[row] = s;
    for (int64_t k = lane; k < K; k += 32) {
        int q = __float2int_rn(__fmul_rn(__uint_as_float(static_cast<uint32_t>(xr[k]) << 16), s));
        xq[row * K + k] = static_cast<int8_t>(max(-128, min(127, q)));
    }
}

int grid_for(int64_t work, int per_block, int cap) {
    int64_t g = (work + per_block - 1) / per_block;
    if (g < 1) g = 1;
    if (g > cap) g = cap;
    return static_cast<int>(g);
}

}  // namespace

int absmean_num_partials(int64_t numel) {
    const int64_t n4 = numel / 4;
    int64_t want = (n4 + kAbsThreads * 8 - 1) / (kAbsThreads * 8);
    if (want < 1) want = 1;
    if (want > kAbsMaxParts) want = kAbsMaxParts;
    return static_cast<int>(want);
}

cudaError_t launch_absmean_partials(const float* W, int64_t numel, double* partials, int nparts,
                                    cudaStream_t stream) {
    return launch_pdl(absmean_partials_kernel, dim3(nparts), dim3(kAbsThreads), 0, stream, dim3(kNoCluster),
                      reinterpret_cast<const float4*>(W), numel / 4, partials);
}

cudaError_t launch_ternarise_pack(const float* W, int64_t numel, const float* gamma_in,
                                  const double* partials, int nparts, float eps,
                                  float* gamma_out, uint8_t* packed, cudaStream_t stream) {
    const int grid = grid_for(numel / 16, 256 * 4, 148 * 16);
    return launch_pdl(ternarise_pack_kernel, dim3(grid), dim3(256), 0, stream, dim3(kNoCluster),
                      reinterpret_cast<const float4*>(W), numel, gamma_in, partials, nparts, eps, gamma_out, packed);
}

cudaError_t launch_pack_codes(const int8_t* codes, int64_t numel, uint8_t* packed, int32_t* err,
                              cudaStream_t stream) {
    const int grid = grid_for(numel / 16, 256 * 4, 148 * 16);
    return launch_pdl(pack_codes_kernel, dim3(grid), dim3(256), 0, stream, dim3(kNoCluster),
                      reinterpret_cast<const uint4*>(codes), numel, packed, err);
}

template <int G, int R, int L, int VPT = (R > 1 ? 4 : 8)>
static cudaError_t launch_act_g(const uint4* X4, int64_t M, int K, float eps, uint8_t* xq, float* s,
                                cudaStream_t stream) {
    constexpr int CTA = G > 256 ? G : 256;
    return launch_pdl(act_quant_vec_kernel<G, R, L, VPT>, dim3(grid_for(M, CTA / G * R, 1 << 30)), dim3(CTA), 0, stream,
                      dim3(kNoCluster), X4, M, K, eps, xq, s);
}

template <int L>
static cudaError_t launch_act_vec(const uint4* X4, int64_t M, int K, float eps, uint8_t* xq, float* s,
                                  cudaStream_t stream) {
    const int nvec = K / 8;
    if (nvec <= 32) return launch_act_g<32, 4, L>(X4, M, K, eps, xq, s, stream);
    if (nvec <= 128) return launch_act_g<32, 2, L>(X4, M, K, eps, xq, s, stream);
    // rows up to 4096 elements: one warp per row holding the whole row (16 vectors per
    // lane), so the reduction needs no block barrier and a block keeps 8 rows in flight
    if (nvec <= 512) return launch_act_g<32, 1, L, 16>(X4, M, K, eps, xq, s, stream);
    if (nvec <= 1024) return launch_act_g<256, 1, L>(X4, M, K, eps, xq, s, stream);
    return launch_act_g<512, 1, L>(X4, M, K, eps, xq, s, stream);
}

template <int G, int L, int VPT = 8>
static cudaError_t launch_norm_g(const uint4* X4, const float* nw, int64_t M, int K, int kind, float norm_eps,
                                 float eps, uint8_t* xq, float* s, cudaStream_t stream) {
    constexpr int CTA = G > 256 ? G : 256;
    const dim3 grid(grid_for(M, CTA / G, 1 << 30)), block(CTA);
    const int stage_w = nw != nullptr && K <= kNormStageMaxK ? 1 : 0;
    const size_t smem = stage_w ? static_cast<size_t>(K) * sizeof(float) : 0;
    if (kind == 1)
        return launch_pdl(norm_act_quant_kernel<G, L, 1, VPT>, grid, block, smem, stream, dim3(kNoCluster), X4, nw,
                          M, K, norm_eps, eps, xq, s, stage_w);
    return launch_pdl(norm_act_quant_kernel<G, L, 0, VPT>, grid, block, smem, stream, dim3(kNoCluster), X4, nw, M,
                      K, norm_eps, eps, xq, s, stage_w);
}

template <int L>
static cudaError_t launch_norm_l(const uint4* X4, const float* nw, int64_t M, int K, int kind, float norm_eps,
                                 float eps, uint8_t* xq, float* s, cudaStream_t stream) {
    const int nvec = K / 8;  // 16-byte vectors per row; a thread holds 8 of them
    if (nvec <= 8 * 32) return launch_norm_g<32, L>(X4, nw, M, K, kind, norm_eps, eps, xq, s, stream);
    // rows up to 4096 elements: one warp per row holding all of it, no block barriers
    if (nvec <= 16 * 32) return launch_norm_g<32, L, 16>(X4, nw, M, K, kind, norm_eps, eps, xq, s, stream);
    if (nvec <= 8 * 128) return launch_norm_g<128, L>(X4, nw, M, K, kind, norm_eps, eps, xq, s, stream);
    if (nvec <= 8 * 256) return launch_norm_g<256, L>(X4, nw, M, K, kind, norm_eps, eps, xq, s, stream);
    return launch_norm_g<512, L>(X4, nw, M, K, kind, norm_eps, eps, xq, s, stream);
}

cudaError_t launch_norm_quantize_act(const uint16_t* X, const float* norm_weight, int64_t M, int64_t K, int kind,
                                     float norm_eps, float eps, int8_t* xq, float* s, int layout,
                                     cudaStream_t stream) {
    uint8_t* q = reinterpret_cast<uint8_t*>(xq);
    const uint4* X4 = reinterpret_cast<const uint4*>(X);
    const int k = static_cast<int>(K);
    if (layout == kXqEvenOdd16) return launch_norm_l<kXqEvenOdd16>(X4, norm_weight, M, k, kind, norm_eps, eps, q, s, stream);
    if (layout == kXqStride4K16) return launch_norm_l<kXqStride4K16>(X4, norm_weight, M, k, kind, norm_eps, eps, q, s, stream);
    return launch_norm_l<kXqRowMajor>(X4, norm_weight, M, k, kind, norm_eps, eps, q, s, stream);
}

cudaError_t launch_quantize_act(const uint16_t* X, int64_t M, int64_t K, float eps, int8_t* xq,
                                float* s, int layout, cudaStream_t stream) {
    uint8_t* q = reinterpret_cast<uint8_t*>(xq);
    const uint4* X4 = reinterpret_cast<const uint4*>(X);
    // K % 16 == 0 for the k16 layouts is checked by the caller
    if (layout == kXqEvenOdd16) return launch_act_vec<kXqEvenOdd16>(X4, M, static_cast<int>(K), eps, q, s, stream);
    if (layout == kXqStride4K16) return launch_act_vec<kXqStride4K16>(X4, M, static_cast<int>(K), eps, q, s, stream);
    if (K % 8 != 0 || K > (int64_t(1) << 30))
        return launch_pdl(act_quant_scalar_kernel, dim3(grid_for(M, 8, 1 << 30)), dim3(256), 0, stream,
                          dim3(kNoCluster), X, M, K, eps, xq, s);
    return launch_act_vec<kXqRowMajor>(X4, M, static_cast<int>(K), eps, q, s, stream);
}

}  // namespace bl
