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
// no barrier between warps in the main loop, 24-32 warps per SM, and 96 KB per SM in
// flight.
//
// Work split.  One block per SM owns a contiguous, balanced run of 16-row tiles over the
// whole of K.  A unit is one tile's 16 rows x one 256-code quarter of K (1 KB of packed
// weights).  The block's units are ordered quarter-major (all tiles of quarter 0, then
// quarter 1, ...) and cut into equal contiguous chunks, one per warp, so a warp holds one
// quarter's activations in registers for a run of tiles (read from the block's copy of
// the activations in shared memory when they fit there, else from global memory).  After
// each unit the warp adds its int32 partial tile into a shared-memory accumulator of the
// block with shared atomics (integer sums are exact in any order); after a block barrier
// the block scales and stores its rows, coalesced along N.  (A tile-major order, each
// warp walking along K, was measured slower: it reloads the activations every unit.)
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

// Warps per block and units in flight per warp, per token-tile count: one token tile
// fits 64 registers, so 32 warps x 3 stages; two need more, so 24 warps x 4 stages
// (measured on the LLaMA-70B decode shapes).  Either way 96 KB of copies per SM.
template <int MT>
struct StreamCfg {
    static constexpr int W = MT == 1 ? 32 : 24;
    static constexpr int S = MT == 1 ? 3 : 4;
};
constexpr int kWarpStage = 1024;                // bytes per warp and stage: [row g | row g + 8][lane][16 B]
constexpr int kRingBytes = 96 * 1024;
static_assert(StreamCfg<1>::W * StreamCfg<1>::S * kWarpStage == kRingBytes, "ring size");
static_assert(StreamCfg<2>::W * StreamCfg<2>::S * kWarpStage == kRingBytes, "ring size");
constexpr int kMaxTiles = 64;                   // 16-row tiles per block
constexpr int kSmemLimit = 227 * 1024;
constexpr int kXPad = 16;                       // bytes after each staged activation row
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
    int tmax;  // the most tiles a block owns (sizes the accumulator)
    int xs;    // the activations are staged in shared memory (M rows of K + kXPad bytes)
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

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
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
// distinct banks), the copy ring [warp][stage][row g, row g + 8][lane][16 B] (each of a
// warp's two shared loads per unit reads 512 contiguous bytes), and, when they fit, the
// block's copy of the activations [token][K + kXPad bytes] (the pad spreads the tokens'
// rows over the banks).
__host__ __device__ constexpr uint32_t red_bytes_of(int tmax, int MT) {
    return (static_cast<uint32_t>(tmax) * 8 * MT * kTokStride * 4 + 15u) & ~15u;
}

template <int MT>
__global__ void __launch_bounds__(32 * StreamCfg<MT>::W, 1) gemv_stream_kernel(const GsArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    constexpr int TOK = 8 * MT;
    constexpr int kWarps = StreamCfg<MT>::W, kStages = StreamCfg<MT>::S, kThreads = 32 * kWarps;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int t_begin = static_cast<int>((static_cast<int64_t>(blockIdx.x) * a.ntiles) / gridDim.x);
    const int t_end = static_cast<int>((static_cast<int64_t>(blockIdx.x + 1) * a.ntiles) / gridDim.x);
    const int T = t_end - t_begin;
    int* red = reinterpret_cast<int*>(smem);
    const uint32_t red_bytes = red_bytes_of(a.tmax, MT);
    const uint32_t ring = smem_u32(smem) + red_bytes + static_cast<uint32_t>(warp * kStages * kWarpStage) +
                          static_cast<uint32_t>(16 * lane);
    const uint32_t xsm = smem_u32(smem) + red_bytes + kRingBytes;
    const int xstride = a.K + kXPad;

    for (int i = threadIdx.x; i < T * TOK * kTokStride; i += kThreads) red[i] = 0;
    pdl_wait_then_release();
    if (a.xs) {
        const int cpr = a.K / 16;  // 16-byte chunks per activation row
        for (int c = threadIdx.x; c < a.M * cpr; c += kThreads) {
            const int r = c / cpr, k = c - r * cpr;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.xq + static_cast<int64_t>(r) * a.K) + k);
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(xsm + r * xstride + 16 * k), "r"(v.x),
                         "r"(v.y), "r"(v.z), "r"(v.w)
                         : "memory");
        }
    }
    __syncthreads();

    const int U = T * a.Q;
    const int u0 = static_cast<int>((static_cast<int64_t>(warp) * U) / kWarps);
    const int u1 = static_cast<int>((static_cast<int64_t>(warp + 1) * U) / kWarps);
    const int64_t rs = a.K / 4;  // packed bytes per row
    const int rowg = 16 * t_begin + g;

    // unit u is (q, tile) = (u / T, u % T); the issue and compute positions advance by
    // one tile at a time.  The issue position keeps the byte offset of row g of its tile
    // at its quarter (row g + 8 is 8 rows further), moved by one tile (16 rows) per unit.
    int iq = u0 / T, itile = u0 - iq * T;
    const int cq0 = iq, ctile0 = itile;
    auto advance = [&](int& q, int& tile) {
        if (++tile == T) {
            tile = 0;
            ++q;
        }
    };
    const int64_t tile_bytes = 16 * rs;
    int64_t ioff = (rowg + 16 * static_cast<int64_t>(itile)) * rs + 64 * iq + 16 * t;
    bool iin_k = 256 * iq + 64 * t < a.K;
    // copy rows g and g + 8 of the issue position's unit into the stage, then advance it
    auto issue_next = [&](int stage) {
        const int r0 = rowg + 16 * itile;
        const bool v0 = iin_k && r0 < a.N, v1 = iin_k && r0 + 8 < a.N;
        const uint32_t dst = ring + static_cast<uint32_t>(stage * kWarpStage);
        cp_async_16(dst, a.packed + (v0 ? ioff : 0), v0 ? 16u : 0u);
        cp_async_16(dst + kWarpStage / 2, a.packed + (v1 ? ioff + 8 * rs : 0), v1 ? 16u : 0u);
        ioff += tile_bytes;
        if (++itile == T) {
            itile = 0;
            ++iq;
            ioff += 64 - T * tile_bytes;
            iin_k = 256 * iq + 64 * t < a.K;
        }
    };
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
        if (u0 + s < u1) issue_next(s);
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
                b[i] = bb[i] = make_uint4(0, 0, 0, 0);
                if (a.xs) {
                    if (in_k && g < a.M) b[i] = lds128(xsm + g * xstride + 256 * q + 64 * t + 16 * i);
                    if (MT == 2 && in_k && g + 8 < a.M)
                        bb[i] = lds128(xsm + (g + 8) * xstride + 256 * q + 64 * t + 16 * i);
                } else {
                    if (in_k && g < a.M) b[i] = __ldg(reinterpret_cast<const uint4*>(x0 + 256 * q + 16 * i));
                    if (MT == 2 && in_k && g + 8 < a.M)
                        bb[i] = __ldg(reinterpret_cast<const uint4*>(x1 + 256 * q + 16 * i));
                }
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
        if (u + kStages < u1) issue_next(stage);
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

// Shared memory of a launch, and whether the activations are staged in it.
size_t smem_bytes(int MT, int tmax, int64_t M, int64_t K, bool* xs) {
    const size_t base = red_bytes_of(tmax, MT) + static_cast<size_t>(kRingBytes);
    const size_t xbytes = static_cast<size_t>(M) * static_cast<size_t>(K + kXPad);
    *xs = base + xbytes <= static_cast<size_t>(kSmemLimit);
    return *xs ? base + xbytes : base;
}

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
    const int64_t ntiles = (N + 15) / 16;
    const int tmax = static_cast<int>((ntiles + sms - 1) / sms);
    bool xs = false;
    const size_t smem = smem_bytes(MT, tmax, M, K, &xs);
    GsArgs a{packed, xq, s, gamma, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
             static_cast<int>(ntiles), static_cast<int>((K + 255) / 256), out, out_kind_of(kind),
             gamma_rows_of(kind), tmax, xs ? 1 : 0, s4_mul()};
    static PerContextOnce attr[2];
    cudaError_t e = attr[MT - 1].run([MT] {
        return MT == 1 ? cudaFuncSetAttribute(gemv_stream_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              kSmemLimit)
                       : cudaFuncSetAttribute(gemv_stream_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              kSmemLimit);
    });
    if (e != cudaSuccess) return e;
    if (MT == 1)
        return launch_pdl(gemv_stream_kernel<1>, dim3(sms), dim3(32 * StreamCfg<1>::W), smem, stream,
                          dim3(kNoCluster), a);
    return launch_pdl(gemv_stream_kernel<2>, dim3(sms), dim3(32 * StreamCfg<2>::W), smem, stream, dim3(kNoCluster),
                      a);
}

}  // namespace bl
