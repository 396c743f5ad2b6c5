// k_gemv_stream.cu -- decode-regime BitLinear forward for wide layers, fed by per-thread
// asynchronous copies at full occupancy instead of a TMA producer.
//
// Same arithmetic as the other decode kernels ("What 1.58 Bits Actually Changes", "How
// the low-bit linear path works": +1 adds, -1 subtracts, 0 skips; "1-bit & Ternary LLMs",
// block "BitNet (Oct 2023)": one float rescale at the end):
//   acc[m, n] = sum_k x_q[m, k] * c[n, k],   y[m, n] = acc[m, n] * gamma / s[m].
// The 2-bit codes are unpacked in registers by the stride-4 unpack (codes scaled by 64,
// the epilogue shifts the int32 sums back by 6) and multiplied on the tensor pipe with
// mma.sync m16n8k32 s8: the ternary operand is A (16 weight rows), the tokens are B.
//
// Why another decode kernel.  The TMA-fed GEMV keeps 14 busy warps per SM and its
// consumers wait on shared stage barriers, so each warp spends most of its time stalled
// and the weights stream at about a third of the copy rate.  Here every thread copies
// the bytes it will itself unpack (cp.async, 16 bytes, L1 bypassed, with a 256-byte L2
// prefetch so DRAM still sees long runs) into a private ring of stages in shared memory:
// no barrier between warps in the main loop, 24 warps per SM, and several kilobytes per
// warp in flight.
//
// Work split.  One block per SM owns a contiguous, balanced run of 16-row tiles over the
// whole of K.  A unit is one tile's 16 rows x one 256-code quarter of K (1 KB of packed
// weights).  The block's units are ordered quarter-major (all tiles of quarter 0, then
// quarter 1, ...) and cut into equal contiguous chunks, one per warp, so a warp holds one
// quarter's activations in registers for a run of tiles.  After each unit the warp adds
// its int32 partial tile into a shared-memory accumulator of the block with shared
// atomics (integer sums are exact in any order); after a block barrier the block scales
// and stores its rows, coalesced along N.
//
// Thread (g, t) of a warp (g = lane / 4, t = lane % 4) owns, in every unit, rows g and
// g + 8 of the tile at bytes 64 q + 16 t of the quarter q (16-groups 4 (4q + t) + i,
// i = 0..3), and the activations of tokens g (and g + 8 for 9..16 tokens) at the same
// 64 codes.  Rows past N and codes past K copy zeros (cp.async with source size 0).
#include <cuda_bf16.h>
#include <cstdint>
#include <cuda_runtime.h>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {

namespace {

constexpr int kWarps = 24;
constexpr int kThreads = 32 * kWarps;
constexpr int kStages = 4;                      // units in flight per warp
constexpr int kWarpStage = 1024;                // bytes per warp and stage: [row g | row g + 8][lane][16 B]
constexpr int kRingBytes = kWarps * kStages * kWarpStage;  // 96 KB
constexpr int kMaxTiles = 64;                   // 16-row tiles per block
constexpr int kTokStride = 20;                  // ints per token row of a tile's accumulator
constexpr int64_t kMaxK = int64_t(1) << 17;     // keeps 64 * 128 * K below 2^31

struct GsArgs {
    const uint8_t* packed;
    const int8_t* xq;
    const float* s;
    const float* gamma;
    int M, N, K;
    int ntiles;  // 16-row tiles in N
    int Q;       // 256-code quarters in K
    void* out;
    int kind;
    int grow;  // gamma holds one scale per output row
    S4Mul mul;
};

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

#define BL_MMA(D, A, B) "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 " D ", " A ", " B ", " D ";\n\t"

// One 16-group of the thread's two rows (words wg: row g, wh: row g + 8) against one
// token tile's activations b (16 bytes in stride-4 order): two MMAs into acc.
__device__ __forceinline__ void s4_group(int (&acc)[4], uint32_t wg, uint32_t wh, uint4 b, const S4Mul& k) {
    asm volatile(
        "{\n\t.reg .b32 ta, tx, ty, tv, tt;\n\t"
        ".reg .b32 p0,p1,p2,p3,q0,q1,q2,q3;\n\t"
        BL_S4_UNPACK("%4", "p0", "p1", "p2", "p3", "%10", "%11", "%12", "%13", "%14")
        BL_S4_UNPACK("%5", "q0", "q1", "q2", "q3", "%10", "%11", "%12", "%13", "%14")
        BL_MMA("{%0,%1,%2,%3}", "{p0,q0,p1,q1}", "{%6,%7}")
        BL_MMA("{%0,%1,%2,%3}", "{p2,q2,p3,q3}", "{%8,%9}")
        "}\n"
        : "+r"(acc[0]), "+r"(acc[1]), "+r"(acc[2]), "+r"(acc[3])
        : "r"(wg), "r"(wh), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w), "r"(k.hi1), "r"(k.two), "r"(k.m4), "r"(k.m16),
          "r"(k.m64));
}

// The same for two token tiles sharing the unpacked words (tokens 0-7 into acc, 8-15
// into acc2).
__device__ __forceinline__ void s4_group2(int (&acc)[4], int (&acc2)[4], uint32_t wg, uint32_t wh, uint4 b,
                                          uint4 bb, const S4Mul& k) {
    asm volatile(
        "{\n\t.reg .b32 ta, tx, ty, tv, tt;\n\t"
        ".reg .b32 p0,p1,p2,p3,q0,q1,q2,q3;\n\t"
        BL_S4_UNPACK("%8", "p0", "p1", "p2", "p3", "%18", "%19", "%20", "%21", "%22")
        BL_S4_UNPACK("%9", "q0", "q1", "q2", "q3", "%18", "%19", "%20", "%21", "%22")
        BL_MMA("{%0,%1,%2,%3}", "{p0,q0,p1,q1}", "{%10,%11}")
        BL_MMA("{%0,%1,%2,%3}", "{p2,q2,p3,q3}", "{%12,%13}")
        BL_MMA("{%4,%5,%6,%7}", "{p0,q0,p1,q1}", "{%14,%15}")
        BL_MMA("{%4,%5,%6,%7}", "{p2,q2,p3,q3}", "{%16,%17}")
        "}\n"
        : "+r"(acc[0]), "+r"(acc[1]), "+r"(acc[2]), "+r"(acc[3]), "+r"(acc2[0]), "+r"(acc2[1]), "+r"(acc2[2]),
          "+r"(acc2[3])
        : "r"(wg), "r"(wh), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w), "r"(bb.x), "r"(bb.y), "r"(bb.z), "r"(bb.w),
          "r"(k.hi1), "r"(k.two), "r"(k.m4), "r"(k.m16), "r"(k.m64));
}
#undef BL_MMA

__device__ __forceinline__ void store_y(void* out, int kind, int64_t idx, int acc, float fac) {
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

// Shared memory: the block accumulator [tile][token][kTokStride ints: 16 rows + 4 pad]
// (the pad puts the eight row groups and four token pairs of a warp's atomics in 32
// distinct banks), then the copy ring [warp][stage][row g, row g + 8][lane][16 B], so
// that each of a warp's two shared loads per unit reads 512 contiguous bytes.
template <int MT>
__global__ void __launch_bounds__(kThreads, 1) gemv_stream_kernel(const GsArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    constexpr int TOK = 8 * MT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int t_begin = static_cast<int>((static_cast<int64_t>(blockIdx.x) * a.ntiles) / gridDim.x);
    const int t_end = static_cast<int>((static_cast<int64_t>(blockIdx.x + 1) * a.ntiles) / gridDim.x);
    const int T = t_end - t_begin;
    int* red = reinterpret_cast<int*>(smem);
    const uint32_t red_bytes = static_cast<uint32_t>(kMaxTiles * TOK * kTokStride * sizeof(int));
    const uint32_t ring = smem_u32(smem) + red_bytes + static_cast<uint32_t>(warp * kStages * kWarpStage) +
                          static_cast<uint32_t>(16 * lane);

    for (int i = threadIdx.x; i < T * TOK * kTokStride; i += kThreads) red[i] = 0;
    pdl_wait_then_release();
    __syncthreads();

    const int U = T * a.Q;
    const int u0 = static_cast<int>((static_cast<int64_t>(warp) * U) / kWarps);
    const int u1 = static_cast<int>((static_cast<int64_t>(warp + 1) * U) / kWarps);
    const int64_t rs = a.K / 4;  // packed bytes per row
    const int rowg = 16 * t_begin + g;

    // unit (q, tile): copy rows g and g + 8 of the tile at bytes 64 q + 16 t
    auto issue = [&](int q, int tile, int stage) {
        const int off = 64 * q + 16 * t;
        const bool in_k = 4 * off < a.K;
        const int r0 = rowg + 16 * tile, r1 = r0 + 8;
        const bool v0 = in_k && r0 < a.N, v1 = in_k && r1 < a.N;
        const uint8_t* p0 = a.packed + (v0 ? static_cast<int64_t>(r0) * rs + off : 0);
        const uint8_t* p1 = a.packed + (v1 ? static_cast<int64_t>(r1) * rs + off : 0);
        const uint32_t dst = ring + static_cast<uint32_t>(stage * kWarpStage);
        cp_async_16(dst, p0, v0 ? 16u : 0u);
        cp_async_16(dst + kWarpStage / 2, p1, v1 ? 16u : 0u);
    };
    // unit u is (q, tile) = (u / T, u % T); the issue and compute positions advance by
    // one tile at a time
    int iq = u0 / T, itile = u0 - iq * T;
    const int cq0 = iq, ctile0 = itile;
    auto advance = [&](int& q, int& tile) {
        if (++tile == T) {
            tile = 0;
            ++q;
        }
    };
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
        if (u0 + s < u1) {
            issue(iq, itile, s);
            advance(iq, itile);
        }
        cp_async_commit();
    }

    // the unpack's multipliers, held in registers for the whole loop
    S4Mul mul;
    asm volatile("mov.b32 %0, %5;\n\tmov.b32 %1, %6;\n\tmov.b32 %2, %7;\n\tmov.b32 %3, %8;\n\tmov.b32 %4, %9;"
                 : "=r"(mul.hi1), "=r"(mul.two), "=r"(mul.m4), "=r"(mul.m16), "=r"(mul.m64)
                 : "r"(a.mul.hi1), "r"(a.mul.two), "r"(a.mul.m4), "r"(a.mul.m16), "r"(a.mul.m64));
    // activation rows of tokens g and g + 8; a token past M, or a quarter piece past K,
    // holds zeros (its products are never stored, or meet zero-filled weights)
    const int8_t* x0 = a.xq + static_cast<int64_t>(g) * a.K + 64 * t;
    const int8_t* x1 = a.xq + static_cast<int64_t>(g + 8) * a.K + 64 * t;
    uint4 b[4], bb[4];
    int qcur = -1;
    int acc[2][4], acc2[2][4];
    int stage = 0;
    int q = cq0, tile = ctile0;
    for (int u = u0; u < u1; ++u, advance(q, tile)) {
        if (q != qcur) {
            qcur = q;
            const bool in_k = 256 * q + 64 * t < a.K;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                b[i] = (in_k && g < a.M) ? __ldg(reinterpret_cast<const uint4*>(x0 + 256 * q + 16 * i))
                                         : make_uint4(0, 0, 0, 0);
                if constexpr (MT == 2)
                    bb[i] = (in_k && g + 8 < a.M) ? __ldg(reinterpret_cast<const uint4*>(x1 + 256 * q + 16 * i))
                                                  : make_uint4(0, 0, 0, 0);
            }
        }
        cp_async_wait<kStages - 1>();
        const uint32_t src = ring + static_cast<uint32_t>(stage * kWarpStage);
        uint4 wg, wh;
        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(wg.x), "=r"(wg.y), "=r"(wg.z), "=r"(wg.w) : "r"(src));
        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(wh.x), "=r"(wh.y), "=r"(wh.z), "=r"(wh.w)
                     : "r"(src + kWarpStage / 2));
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][e] = acc2[j][e] = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr (MT == 1)
                s4_group(acc[i & 1], word_of(wg, i), word_of(wh, i), b[i], mul);
            else
                s4_group2(acc[i & 1], acc2[i & 1], word_of(wg, i), word_of(wh, i), b[i], bb[i], mul);
        }
        // the MMAs have consumed the stage's words: refill it with the unit kStages ahead
        if (u + kStages < u1) {
            issue(iq, itile, stage);
            advance(iq, itile);
        }
        cp_async_commit();
        if (++stage == kStages) stage = 0;
        // fragment: rows g (e = 0, 1) and g + 8 (e = 2, 3), tokens 2t + (e & 1)
        int* rt = red + tile * TOK * kTokStride;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int idx = (2 * t + (e & 1)) * kTokStride + g + 8 * (e >> 1);
            atomicAdd(rt + idx, acc[0][e] + acc[1][e]);
            if constexpr (MT == 2) atomicAdd(rt + 8 * kTokStride + idx, acc2[0][e] + acc2[1][e]);
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // epilogue: consecutive threads take consecutive rows of one token
    const int rows = 16 * T;
    const int mt = a.M < TOK ? a.M : TOK;
    const float gamma = (a.kind == kOutI32 || a.grow) ? 0.0f : *a.gamma;
    for (int i = threadIdx.x; i < mt * rows; i += kThreads) {
        const int tok = i / rows, rl = i - tok * rows;
        const int64_t n = 16 * static_cast<int64_t>(t_begin) + rl;
        if (n >= a.N) continue;
        const int acc_v = red[((rl >> 4) * TOK + tok) * kTokStride + (rl & 15)] >> 6;
        float fac = 0.0f;
        if (a.kind != kOutI32) fac = __fdiv_rn(a.grow ? a.gamma[n] : gamma, a.s[tok]);
        store_y(a.out, a.kind, static_cast<int64_t>(tok) * a.N + n, acc_v, fac);
    }
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

size_t smem_bytes(int MT) { return static_cast<size_t>(kMaxTiles) * 8 * MT * kTokStride * sizeof(int) + kRingBytes; }

}  // namespace

// M <= 16, K % 64 == 0 (16-byte aligned packed rows), K <= 2^17, and between one and
// kMaxTiles 16-row tiles per SM.
bool gemv_stream_applicable(int64_t M, int64_t N, int64_t K) {
    if (M < 1 || M > 16 || K < 64 || K % 64 != 0 || K > kMaxK || N < 1) return false;
    const int64_t sms = sm_count();
    const int64_t ntiles = (N + 15) / 16;
    return ntiles >= sms && (ntiles + sms - 1) / sms <= kMaxTiles;
}

cudaError_t launch_gemv_stream(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                               int64_t M, int64_t N, int64_t K, void* out, int kind, cudaStream_t stream) {
    if (!gemv_stream_applicable(M, N, K)) return cudaErrorInvalidValue;
    const int sms = sm_count();
    const int MT = M <= 8 ? 1 : 2;
    GsArgs a{packed, xq, s, gamma, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
             static_cast<int>((N + 15) / 16), static_cast<int>((K + 255) / 256), out, out_kind_of(kind),
             gamma_rows_of(kind), s4_mul()};
    static PerContextOnce attr[2];
    cudaError_t e = attr[MT - 1].run([MT] {
        return MT == 1 ? cudaFuncSetAttribute(gemv_stream_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(smem_bytes(1)))
                       : cudaFuncSetAttribute(gemv_stream_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(smem_bytes(2)));
    });
    if (e != cudaSuccess) return e;
    if (MT == 1)
        return launch_pdl(gemv_stream_kernel<1>, dim3(sms), dim3(kThreads), smem_bytes(1), stream, dim3(kNoCluster), a);
    return launch_pdl(gemv_stream_kernel<2>, dim3(sms), dim3(kThreads), smem_bytes(2), stream, dim3(kNoCluster), a);
}

}  // namespace bl
