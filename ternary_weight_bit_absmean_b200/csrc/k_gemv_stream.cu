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
// whole of K (a layer with fewer tiles than SMs gives each tile to a cluster of 2 to 8
// blocks that split its K and add their partial sums through distributed shared memory).  A unit is one tile's 16 rows x one 256-code quarter of K (1 KB of packed
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

// Warps per block and units in flight per warp, per token-tile count MT (tiles of 8
// tokens): one token tile fits 64 registers, so 32 warps x 3 stages; two need more, so 24
// warps x 4 stages (measured on the LLaMA-70B decode shapes); four hold 64 activation
// registers, so 16 warps x 6 stages.  Either way 96 KB of copies per SM.  NS accumulator
// sets alternate between the 16-groups of a unit (two independent MMA chains) where the
// registers allow.  A block takes at most kMaxTiles 16-row tiles (fewer with four token
// tiles, whose accumulator is larger).
template <int MT>
struct StreamCfg {
    static constexpr int W = MT == 1 ? 32 : MT == 2 ? 24 : 16;
    static constexpr int S = MT == 1 ? 3 : MT == 2 ? 4 : 6;
    static constexpr int NS = MT == 4 ? 1 : 2;
    static constexpr int kMaxTiles = MT == 4 ? 48 : 64;
};
constexpr int kWarpStage = 1024;                // bytes per warp and stage: [row g | row g + 8][lane][16 B]
constexpr int kRingBytes = 96 * 1024;
static_assert(StreamCfg<1>::W * StreamCfg<1>::S * kWarpStage == kRingBytes, "ring size");
static_assert(StreamCfg<2>::W * StreamCfg<2>::S * kWarpStage == kRingBytes, "ring size");
static_assert(StreamCfg<4>::W * StreamCfg<4>::S * kWarpStage == kRingBytes, "ring size");
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
    int ksplit;  // blocks (a cluster) sharing each run of tiles, splitting its K
    int xs;    // the block's tokens' activations are staged in shared memory (K + kXPad bytes a row)
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

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// One 16-group of the thread's two rows (words wg: row g, wh: row g + 8) unpacked into
// the A fragments of two MMAs, {p0, q0, p1, q1} and {p2, q2, p3, q3}.
__device__ __forceinline__ void unpack_pair(uint32_t wg, uint32_t wh, uint32_t (&p)[4], uint32_t (&q)[4],
                                            const S4Mul& k) {
    asm("{\n\t.reg .b32 ta, tx, ty, tv, tt;\n\t"
        BL_S4_UNPACK("%8", "%0", "%1", "%2", "%3", "%10", "%11", "%12", "%13", "%14")
        BL_S4_UNPACK("%9", "%4", "%5", "%6", "%7", "%10", "%11", "%12", "%13", "%14")
        "}\n"
        : "=&r"(p[0]), "=&r"(p[1]), "=&r"(p[2]), "=&r"(p[3]), "=&r"(q[0]), "=&r"(q[1]), "=&r"(q[2]), "=&r"(q[3])
        : "r"(wg), "r"(wh), "r"(k.hi1), "r"(k.two), "r"(k.m4), "r"(k.m16), "r"(k.m64));
}

// d += A (16 rows x 32 codes) * B (32 codes x 8 tokens), s8 x s8 -> s32.
__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

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

// grid: x = one block per SM (a run of 16-row tiles each) or, for layers with fewer tiles
// than SMs, a cluster of a.ksplit blocks per tile (SPLIT); y = groups of 8 MT tokens.
template <int MT, bool SPLIT>
__global__ void __launch_bounds__(32 * StreamCfg<MT>::W, 1) gemv_stream_kernel(const GsArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    constexpr int TOK = 8 * MT;
    constexpr int kWarps = StreamCfg<MT>::W, kStages = StreamCfg<MT>::S, NS = StreamCfg<MT>::NS;
    constexpr int kThreads = 32 * kWarps;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    // a.ksplit blocks (one cluster when more than one) own the same run of tiles, each a
    // contiguous share of its units (a range of K, the units being quarter-major)
    const int S = SPLIT ? a.ksplit : 1;
    const int rank = SPLIT ? static_cast<int>(cluster_ctarank()) : 0;
    const int cid = blockIdx.x / S, ncl = gridDim.x / S;
    const int t_begin = static_cast<int>((static_cast<int64_t>(cid) * a.ntiles) / ncl);
    const int t_end = static_cast<int>((static_cast<int64_t>(cid + 1) * a.ntiles) / ncl);
    const int T = t_end - t_begin;
    // this block's tokens: m0 .. m0 + Mg - 1
    const int m0 = TOK * static_cast<int>(blockIdx.y);
    const int Mg = a.M - m0 < TOK ? a.M - m0 : TOK;
    int* red = reinterpret_cast<int*>(smem);
    const uint32_t red_bytes = red_bytes_of(a.tmax, MT);
    const uint32_t ring = smem_u32(smem) + red_bytes + static_cast<uint32_t>(warp * kStages * kWarpStage) +
                          static_cast<uint32_t>(16 * lane);
    const uint32_t xsm = smem_u32(smem) + red_bytes + kRingBytes;
    const int xstride = a.K + kXPad;
    const int8_t* xblk = a.xq + static_cast<int64_t>(m0) * a.K;

    for (int i = threadIdx.x; i < T * TOK * kTokStride; i += kThreads) red[i] = 0;
    pdl_wait_then_release();
    if (a.xs) {
        const int cpr = a.K / 16;  // 16-byte chunks per activation row
        for (int c = threadIdx.x; c < Mg * cpr; c += kThreads) {
            const int r = c / cpr, k = c - r * cpr;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(xblk + static_cast<int64_t>(r) * a.K) + k);
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(xsm + r * xstride + 16 * k), "r"(v.x),
                         "r"(v.y), "r"(v.z), "r"(v.w)
                         : "memory");
        }
    }
    __syncthreads();

    const int U = T * a.Q;
    const int bu0 = static_cast<int>((static_cast<int64_t>(rank) * U) / S);
    const int bu1 = static_cast<int>((static_cast<int64_t>(rank + 1) * U) / S);
    const int u0 = bu0 + static_cast<int>((static_cast<int64_t>(warp) * (bu1 - bu0)) / kWarps);
    const int u1 = bu0 + static_cast<int>((static_cast<int64_t>(warp + 1) * (bu1 - bu0)) / kWarps);
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
    // b[m][i]: the activations of token g + 8 m of the group at the thread's 16-group i of
    // the current quarter; a token past the group, or a piece past K, holds zeros (its
    // products are never stored, or meet zero-filled weights)
    uint4 b[MT][4];
    int qcur = -1;
    int acc[NS][MT][4];
    int stage = 0;
    int q = cq0, tile = ctile0;
    for (int u = u0; u < u1; ++u, advance(q, tile)) {
        if (q != qcur) {
            qcur = q;
            const bool in_k = 256 * q + 64 * t < a.K;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const bool ok = in_k && g + 8 * m < Mg;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int off = 256 * q + 64 * t + 16 * i;
                    b[m][i] = !ok ? make_uint4(0, 0, 0, 0)
                              : a.xs ? lds128(xsm + (g + 8 * m) * xstride + off)
                                     : __ldg(reinterpret_cast<const uint4*>(
                                           xblk + static_cast<int64_t>(g + 8 * m) * a.K + off));
                }
            }
        }
        cp_async_wait<kStages - 1>();
        const uint32_t src = ring + static_cast<uint32_t>(stage * kWarpStage);
        const uint4 wg = lds128(src), wh = lds128(src + kWarpStage / 2);
#pragma unroll
        for (int j = 0; j < NS; ++j)
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[j][m][e] = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t pa[4], qa[4];
            unpack_pair(word_of(wg, i), word_of(wh, i), pa, qa, mul);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                mma_s8(acc[i % NS][m], pa[0], qa[0], pa[1], qa[1], b[m][i].x, b[m][i].y);
                mma_s8(acc[i % NS][m], pa[2], qa[2], pa[3], qa[3], b[m][i].z, b[m][i].w);
            }
        }
        // the MMAs have consumed the stage's words: refill it with the unit kStages ahead
        if (u + kStages < u1) issue_next(stage);
        cp_async_commit();
        if (++stage == kStages) stage = 0;
        // fragment: rows g (e = 0, 1) and g + 8 (e = 2, 3), tokens 8 m + 2t + (e & 1)
        int* rt = red + tile * TOK * kTokStride;
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int idx = (8 * m + 2 * t + (e & 1)) * kTokStride + g + 8 * (e >> 1);
                int v = acc[0][m][e];
                if constexpr (NS == 2) v += acc[NS - 1][m][e];
                atomicAdd(rt + idx, v);
            }
    }
    cp_async_wait<0>();
    __syncthreads();
    // with a K split, every block's partial sums are complete and visible across the
    // cluster after this barrier; each block then finishes its share of the rows, adding
    // all blocks' partials through distributed shared memory in rank order (integer sums:
    // exact in any order), and the second barrier keeps each block's shared memory alive
    // until the others have read it
    if constexpr (SPLIT) cluster_sync_all();

    // epilogue: consecutive threads take consecutive rows of one token
    const int rows = 16 * T;
    const int r_begin = (rows * rank) / S, nr = (rows * (rank + 1)) / S - r_begin;
    const float gamma = (a.kind == kOutI32 || a.grow) ? 0.0f : *a.gamma;
    const uint32_t red_addr = smem_u32(red);
    for (int i = threadIdx.x; i < Mg * nr; i += kThreads) {
        const int tok = i / nr, rl = r_begin + (i - tok * nr);
        const int64_t n = 16 * static_cast<int64_t>(t_begin) + rl;
        if (n >= a.N) continue;
        const int idx = ((rl >> 4) * TOK + tok) * kTokStride + (rl & 15);
        int sum = red[idx];
        if constexpr (SPLIT)
            for (int b = 0; b < S; ++b)
                if (b != rank) sum += static_cast<int>(ld_cluster_u32(mapa_shared(red_addr + 4u * idx, b)));
        const int acc_v = sum >> 6;
        float fac = 0.0f;
        if (a.kind != kOutI32) fac = __fdiv_rn(a.grow ? a.gamma[n] : gamma, a.s[m0 + tok]);
        store_y(a.out, a.kind, static_cast<int64_t>(m0 + tok) * a.N + n, acc_v, fac);
    }
    if constexpr (SPLIT) cluster_sync_all();
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// Shared memory of a launch with token groups of mg tokens, and whether the activations
// are staged in it.
size_t smem_bytes(int MT, int tmax, int64_t mg, int64_t K, bool* xs) {
    const size_t base = red_bytes_of(tmax, MT) + static_cast<size_t>(kRingBytes);
    const size_t xbytes = static_cast<size_t>(mg) * static_cast<size_t>(K + kXPad);
    *xs = base + xbytes <= static_cast<size_t>(kSmemLimit);
    return *xs ? base + xbytes : base;
}

// Token tiles of 8 per block: 1 or 2 up to 16 tokens, else groups of 32 tokens (4 tiles).
int token_tiles(int64_t M) { return M <= 8 ? 1 : M <= 16 ? 2 : 4; }

int max_tiles(int MT) {
    return MT == 1 ? StreamCfg<1>::kMaxTiles : MT == 2 ? StreamCfg<2>::kMaxTiles : StreamCfg<4>::kMaxTiles;
}

template <int MT, bool SPLIT>
cudaError_t launch_split(const GsArgs& a, int blocks, int groups, size_t smem, cudaStream_t stream) {
    static PerContextOnce attr;
    const cudaError_t e = attr.run([] {
        return cudaFuncSetAttribute(gemv_stream_kernel<MT, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kSmemLimit);
    });
    if (e != cudaSuccess) return e;
    return launch_pdl(gemv_stream_kernel<MT, SPLIT>, dim3(blocks, groups), dim3(32 * StreamCfg<MT>::W), smem, stream,
                      SPLIT ? dim3(a.ksplit, 1, 1) : dim3(kNoCluster), a);
}

template <int MT>
cudaError_t launch_mt(const GsArgs& a, int blocks, int groups, size_t smem, cudaStream_t stream) {
    return a.ksplit > 1 ? launch_split<MT, true>(a, blocks, groups, smem, stream)
                        : launch_split<MT, false>(a, blocks, groups, smem, stream);
}

// Work split: with at least one 16-row tile per SM, one block per SM over a balanced run
// of tiles; with fewer tiles, one tile per run and K split over a cluster of S blocks (a
// power of two up to 8, S x tiles <= SMs, at most one 256-code quarter per block less).
struct StreamPlan {
    int blocks, ksplit, tmax;
};
StreamPlan plan_stream(int64_t ntiles, int64_t K, int sms) {
    if (ntiles >= sms) return {sms, 1, static_cast<int>((ntiles + sms - 1) / sms)};
    const int64_t Q = (K + 255) / 256;
    int S = 1;
    while (S < 8 && 2 * S * ntiles <= sms && 2 * S <= Q) S *= 2;
    return {static_cast<int>(S * ntiles), S, 1};
}

}  // namespace

// M <= 64 (token groups of up to 32), K % 64 == 0 (16-byte aligned packed rows),
// K <= 2^17, and at most 64 (48 above 16 tokens) 16-row tiles per SM.
bool gemv_stream_applicable(int64_t M, int64_t N, int64_t K) {
    if (M < 1 || M > 64 || K < 64 || K % 64 != 0 || K > kMaxK || N < 1) return false;
    const int64_t sms = sm_count();
    const int64_t ntiles = (N + 15) / 16;
    return (ntiles + sms - 1) / sms <= max_tiles(token_tiles(M));
}

cudaError_t launch_gemv_stream(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                               int64_t M, int64_t N, int64_t K, void* out, int kind, cudaStream_t stream) {
    if (!gemv_stream_applicable(M, N, K)) return cudaErrorInvalidValue;
    const int sms = sm_count();
    const int MT = token_tiles(M);
    const int groups = static_cast<int>((M + 8 * MT - 1) / (8 * MT));
    const int64_t ntiles = (N + 15) / 16;
    const StreamPlan p = plan_stream(ntiles, K, sms);
    bool xs = false;
    const size_t smem = smem_bytes(MT, p.tmax, M < 8 * MT ? M : 8 * MT, K, &xs);
    const GsArgs a{packed, xq, s, gamma, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
                   static_cast<int>(ntiles), static_cast<int>((K + 255) / 256), out, out_kind_of(kind),
                   gamma_rows_of(kind), p.tmax, p.ksplit, xs ? 1 : 0, s4_mul()};
    if (MT == 1) return launch_mt<1>(a, p.blocks, groups, smem, stream);
    if (MT == 2) return launch_mt<2>(a, p.blocks, groups, smem, stream);
    return launch_mt<4>(a, p.blocks, groups, smem, stream);
}

}  // namespace bl
