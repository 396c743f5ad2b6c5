// k_ste.cu -- the straight-through backward of the BitLinear forward, on the 5th-generation
// tensor cores (tcgen05.mma kind::f16, fp32 accumulators in tensor memory).
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
// Both are one GEMM shape, D[i][j] = sum_c A[i][c] B[j][c], written out as
// out[i][j] = gamma D[i][j]:
//   dX: i = token m, j = column k, c = n;  A[m][n] = dY[m][n],        B[k][n] = c[n][k]
//   dW: i = row n,   j = column k, c = m;  A[n][m] = dY[m][n] / s[m], B[k][m] = x_q[m][k]
// B is exact in bf16 (codes are -1/0/+1; |x_q| <= 128 needs 8 significant bits).  The
// fp32 operand A is split into two bf16 parts, A = hi + lo + d with hi = bf16(A),
// lo = bf16(A - hi) (A - hi is exact in fp32) and |d| <= 2^-16 |A|; both parts are
// multiplied by the same B tile into one fp32 accumulator, so each product hi*b and lo*b
// is exact and the result carries the fp32 accumulation error plus 2^-16 relative per
// term -- near the precision of an fp32 contraction, at the bf16 tensor-core rate (two
// MMAs per K step).  For dW, A = dY * (1 / s[m]) with the reciprocal rounded to fp32
// (2^-23 relative per term more).
//
// Tile: 128 rows i (MMA M, TMEM lanes) x BJ columns j (MMA N, BJ = 128 or 256), the
// contraction in stages of 64 (one 128-byte swizzled bf16 row).  No operand is in a
// layout TMA could load directly (dY must be split; the codes and x_q must be transposed
// to put the contraction index innermost), so every operand is written by threads:
//   warp 0 (one lane)  MMA issuer: per stage, for each 16-wide K step, one MMA with A_hi
//                      and one with A_lo against B; tcgen05.commit frees the stage;
//   warps 1-4          A producers: load fp32 dY, scale by 1/s for dW, split, and write
//                      A_hi and A_lo in the 128-byte-swizzled K-major layout;
//   warps 5-12         B producers: expand 2-bit codes (dX) or int8 x_q (dW) to bf16,
//                      transposed into the same layout;
//   warps 13-16        epilogue: tcgen05.ld of the finished accumulator (one row i per
//                      thread, 32 columns at a time), times gamma, row-contiguous stores.
// Two TMEM accumulators let the epilogue of one tile overlap the main loop of the next
// (persistent blocks, one per SM).  Rows, columns and contraction entries past the
// matrix edges are written as zeros.  Every wait is bounded (BL_ERRBIT_TIMEOUT is not
// reported here: the backward has no error word, so a timed-out launch returns early and
// leaves its output incomplete).
#include <cuda_bf16.h>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {

bool encode_tmap_u8_2d(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                       uint32_t box_outer, bool swizzle128);
bool encode_tmap_f32_2d(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                        uint32_t box_outer);

namespace {

constexpr int kBI = 128;           // rows per tile (MMA M)
constexpr int kBC = 64;            // contraction elements per stage (128 bytes of bf16)
constexpr int kRowBytes = 128;     // one swizzled K-major row
constexpr int kThreads = 544;      // 17 warps
constexpr int kWarpMma = 0, kWarpA = 1, kWarpB = 5, kWarpEpi = 13;
constexpr int kAWarps = kWarpB - kWarpA, kBWarps = kWarpEpi - kWarpB, kEpiWarps = 4;
constexpr int kSmemBudget = 200 * 1024;
constexpr unsigned long long kDrainNs = 200000000ull;  // 0.2 s

enum SteKind : int { kDX = 0, kDW = 1 };

template <int BJ>
struct SteCfg {
    static_assert(BJ == 128 || BJ == 256, "column tile");
    static constexpr int kATile = kBI * kRowBytes;  // one bf16 part of A
    static constexpr int kBTile = BJ * kRowBytes;
    static constexpr int kStageBytes = 2 * kATile + kBTile;
    static constexpr int kStages = kSmemBudget / kStageBytes;
    static constexpr int kTmemCols = 2 * BJ;
    static constexpr int kBarBytes = 8 * (2 * kStages + 5) + 16;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBarBytes;
    static_assert(kStages >= 2, "stages");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct SteArgs {
    const float* dY;        // [M, N]
    const uint8_t* packed;  // dX: [N, K/4]
    const int8_t* xq;       // dW: [M, K]
    const float* s;         // dW: [M]
    const float* gamma;
    float* out;             // dX [M, K] or dW [N, K]
    int M, N, K;
    int I, J, C;            // rows, columns and contraction length of D
    int tiles_i, num_tiles;
};

// Instruction descriptor: kind::f16 with A and B bf16, K-major, D fp32, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4)                                // D format: F32
           | (1u << 7)                              // A format: BF16
           | (1u << 10)                             // B format: BF16
           | (static_cast<uint32_t>(N >> 3) << 17)  // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24); // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 x bf16 -> fp32, issued by one thread.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mbar_drain_ste(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kDrainNs) return;
    }
}

// Byte offset of 16-byte chunk `ch` of row `r` in a 128-byte-swizzled K-major tile.
__device__ __forceinline__ uint32_t sw128(int r, int ch) {
    return static_cast<uint32_t>(r) * kRowBytes + (static_cast<uint32_t>(ch ^ (r & 7)) << 4);
}

// Split 8 fp32 values into bf16 hi and lo parts (x = hi + lo + d, |d| <= 2^-16 |x|),
// each as one 16-byte chunk (element e in the low half of word e / 2 when e is even).
__device__ __forceinline__ void split8(const float (&x)[8], uint4& hi, uint4& lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const __nv_bfloat162 hb = __floats2bfloat162_rn(x[2 * p], x[2 * p + 1]);
        const uint32_t hw = *reinterpret_cast<const uint32_t*>(&hb);
        const float r0 = __fsub_rn(x[2 * p], __uint_as_float(hw << 16));          // exact
        const float r1 = __fsub_rn(x[2 * p + 1], __uint_as_float(hw & 0xFFFF0000u));  // exact
        const __nv_bfloat162 lb = __floats2bfloat162_rn(r0, r1);
        h[p] = hw;
        l[p] = *reinterpret_cast<const uint32_t*>(&lb);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Byte table for the code expansion: for a 2-bit code c, byte c of kLoTab and byte c of
// kHiTab are the low and high bytes of bf16(c): 00 -> 0, 01 -> +1 (0x3F80), 10 -> -1
// (0xBF80), 11 -> 0.
constexpr uint32_t kLoTab = 0x00808000u;
constexpr uint32_t kHiTab = 0x00BF3F00u;

// Four codes, one per byte of x (bits 0..1 of each byte), to four bf16 values: the two
// words (bf16 of byte 0 | bf16 of byte 1 << 16) and (byte 2 | byte 3 << 16).
__device__ __forceinline__ void codes4_to_bf16(uint32_t x, uint32_t& w01, uint32_t& w23) {
    // selector nibbles c and 4 + c per byte: c * 0x11 + 0x40, no carries (c <= 3)
    const uint32_t y = x * 0x11u + 0x40404040u;
    w01 = __byte_perm(kLoTab, kHiTab, y);
    w23 = __byte_perm(kLoTab, kHiTab, y >> 16);
}

__device__ __forceinline__ uint32_t bf16x2_of_s8(uint32_t a, uint32_t b) {
    // a, b: int8 values in the low byte; exact in bf16
    const __nv_bfloat162 v = __floats2bfloat162_rn(static_cast<float>(static_cast<int8_t>(a & 0xFFu)),
                                                   static_cast<float>(static_cast<int8_t>(b & 0xFFu)));
    return *reinterpret_cast<const uint32_t*>(&v);
}

template <int KIND, int BJ>
__global__ void __launch_bounds__(kThreads, 1) ste_tc_kernel(const SteArgs a) {
    using Cfg = SteCfg<BJ>;
    constexpr int ST = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    auto sAhi = [&](int s) { return static_cast<uint32_t>(s * Cfg::kStageBytes); };
    auto sAlo = [&](int s) { return static_cast<uint32_t>(s * Cfg::kStageBytes + Cfg::kATile); };
    auto sB = [&](int s) { return static_cast<uint32_t>(s * Cfg::kStageBytes + 2 * Cfg::kATile); };
    const uint32_t sBar = base + ST * Cfg::kStageBytes;
    auto full = [&](int s) { return sBar + 8u * s; };
    auto empty = [&](int s) { return sBar + 8u * (ST + s); };
    auto tfull = [&](int b) { return sBar + 8u * (2 * ST + b); };
    auto tempty = [&](int b) { return sBar + 8u * (2 * ST + 2 + b); };
    const uint32_t drain_bar = sBar + 8u * (2 * ST + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + ST * Cfg::kStageBytes + 8 * (2 * ST + 5));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(full(s), kAWarps + kBWarps);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull(b), 1);
            mbar_init(tempty(b), kEpiWarps);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    pdl_wait_then_release();
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int nC = (a.C + kBC - 1) / kBC;

    if (warp == kWarpMma) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer --
            constexpr uint32_t idesc = idesc_bf16(kBI, BJ);
            int stage = 0, buf = 0;
            uint32_t phase = 0, bphase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x) {
                if (!mbar_wait_bounded(tempty(buf), bphase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BJ);
                for (int kc = 0; kc < nC; ++kc) {
                    if (!mbar_wait_bounded(full(stage), phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kBC / 16; ++kk) {
                        const uint64_t bd = smem_desc_sw128(base + sB(stage) + 32 * kk);
                        tc_mma_bf16(d_tmem, smem_desc_sw128(base + sAhi(stage) + 32 * kk), bd, idesc,
                                    (kc | kk) != 0 ? 1u : 0u);
                        tc_mma_bf16(d_tmem, smem_desc_sw128(base + sAlo(stage) + 32 * kk), bd, idesc, 1u);
                    }
                    tc_commit(empty(stage));
                    if (++stage == ST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(tfull(buf));
                if (++buf == 2) {
                    buf = 0;
                    bphase ^= 1u;
                }
            }
            if (!ok) {
                // let every MMA already issued finish before TMEM is released
                tc_commit(drain_bar);
                mbar_drain_ste(drain_bar, 0);
            }
        }
    } else if (warp < kWarpB) {
        // ------------------------------------------------------------ A producers --
        // Every global load of a stage is issued before the wait for the stage to be
        // free, so the load latency overlaps that wait; the conversion follows.
        const int t = threadIdx.x - 32 * kWarpA;  // 0 .. 127
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x) {
            const int i0 = (tile % a.tiles_i) * kBI;
            for (int kc = 0; kc < nC; ++kc) {
                const int c0 = kc * kBC;
                if constexpr (KIND == kDX) {
                    // A[m][n] = dY[m][n]: eight threads per row, each eight consecutive n;
                    // the 16 rows of a pass are 16 apart, eight passes per stage
                    const int r_off = t >> 3, ch = t & 7;
                    const int n = c0 + 8 * ch;
                    const bool vec = (a.N & 3) == 0 && n + 8 <= a.N;
                    float x[kBI / 16][8];
#pragma unroll
                    for (int p = 0; p < kBI / 16; ++p) {
                        const int m = i0 + 16 * p + r_off;
                        if (m < a.M && vec) {
                            const float4* src = reinterpret_cast<const float4*>(a.dY + static_cast<int64_t>(m) * a.N + n);
                            const float4 u = __ldg(src), v = __ldg(src + 1);
                            x[p][0] = u.x; x[p][1] = u.y; x[p][2] = u.z; x[p][3] = u.w;
                            x[p][4] = v.x; x[p][5] = v.y; x[p][6] = v.z; x[p][7] = v.w;
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                x[p][e] = (m < a.M && n + e < a.N) ? __ldg(a.dY + static_cast<int64_t>(m) * a.N + n + e)
                                                                   : 0.0f;
                        }
                    }
                    if (!mbar_wait_bounded(empty(stage), phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* ahi = gbase + sAhi(stage);
                    uint8_t* alo = gbase + sAlo(stage);
#pragma unroll
                    for (int p = 0; p < kBI / 16; ++p) {
                        const int r = 16 * p + r_off;
                        uint4 hi, lo;
                        split8(x[p], hi, lo);
                        *reinterpret_cast<uint4*>(ahi + sw128(r, ch)) = hi;
                        *reinterpret_cast<uint4*>(alo + sw128(r, ch)) = lo;
                    }
                } else {
                    // A[n][m] = dY[m][n] / s[m]: one thread per row n, the stage's 64 tokens.
                    // Each warp forms the 64 reciprocals itself (two per lane) and hands them
                    // round by shuffles, so the producer warps never wait on one another.
                    const int mA = c0 + lane, mB = c0 + 32 + lane;
                    const float rA = mA < a.M ? __frcp_rn(__ldg(a.s + mA)) : 0.0f;
                    const float rB = mB < a.M ? __frcp_rn(__ldg(a.s + mB)) : 0.0f;
                    const int n = i0 + t;
                    const bool row_ok = n < a.N;
                    float x[kBC];
#pragma unroll
                    for (int e = 0; e < kBC; ++e) {
                        const int m = c0 + e;
                        x[e] = (row_ok && m < a.M) ? __ldg(a.dY + static_cast<int64_t>(m) * a.N + n) : 0.0f;
                    }
#pragma unroll
                    for (int e = 0; e < kBC; ++e)
                        x[e] = __fmul_rn(x[e], __shfl_sync(0xffffffffu, e < 32 ? rA : rB, e & 31));
                    if (!mbar_wait_bounded(empty(stage), phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* ahi = gbase + sAhi(stage);
                    uint8_t* alo = gbase + sAlo(stage);
#pragma unroll
                    for (int ch = 0; ch < kBC / 8; ++ch) {
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = x[8 * ch + e];
                        uint4 hi, lo;
                        split8(y, hi, lo);
                        *reinterpret_cast<uint4*>(ahi + sw128(t, ch)) = hi;
                        *reinterpret_cast<uint4*>(alo + sw128(t, ch)) = lo;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(full(stage));
                if (++stage == ST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp < kWarpEpi) {
        // ------------------------------------------------------------ B producers --
        // loads first, then the wait for the stage, then the conversion (as above)
        const int t = threadIdx.x - 32 * kWarpB;  // 0 .. 255
        constexpr int kUnits = KIND == kDX ? (BJ / 8) * 8 : (BJ / 4) * 8;  // units per stage
        constexpr int kPer = (kUnits + 32 * kBWarps - 1) / (32 * kBWarps);   // units per thread
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x) {
            const int j0 = (tile / a.tiles_i) * BJ;
            for (int kc = 0; kc < nC; ++kc) {
                const int c0 = kc * kBC;
                uint32_t w[kPer][8];
                if constexpr (KIND == kDX) {
                    // B[k][n] = c[n][k]: a unit is 8 consecutive k (two packed bytes per n)
                    // x 8 consecutive n; the warp's lanes take consecutive k groups of one
                    // n chunk, so each load of a warp reads one packed row contiguously
                    const int KB = a.K >> 2;
#pragma unroll
                    for (int v = 0; v < kPer; ++v) {
                        const int u = t + 32 * kBWarps * v;
                        const int kg = u % (BJ / 8), nch = u / (BJ / 8);
                        const int k = j0 + 8 * kg, n = c0 + 8 * nch;
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            w[v][q] = 0;
                            if (u < kUnits && n + q < a.N) {
                                const uint8_t* row = a.packed + static_cast<int64_t>(n + q) * KB;
                                if (k + 8 <= a.K && (KB & 1) == 0) {
                                    w[v][q] = __ldg(reinterpret_cast<const uint16_t*>(row + (k >> 2)));
                                } else {
                                    if (k < a.K) w[v][q] = __ldg(row + (k >> 2));
                                    if (k + 4 < a.K) w[v][q] |= static_cast<uint32_t>(__ldg(row + (k >> 2) + 1)) << 8;
                                }
                            }
                        }
                    }
                } else {
                    // B[k][m] = x_q[m][k]: a unit is 4 consecutive k (one word per token) x 8
                    // consecutive m; lanes take consecutive k words of one m chunk
#pragma unroll
                    for (int v = 0; v < kPer; ++v) {
                        const int u = t + 32 * kBWarps * v;
                        const int kw = u % (BJ / 4), mch = u / (BJ / 4);
                        const int k = j0 + 4 * kw, m = c0 + 8 * mch;
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            w[v][q] = (u < kUnits && m + q < a.M && k < a.K)
                                          ? __ldg(reinterpret_cast<const uint32_t*>(a.xq + static_cast<int64_t>(m + q) * a.K + k))
                                          : 0u;
                    }
                }
                if (!mbar_wait_bounded(empty(stage), phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t* bt = gbase + sB(stage);
#pragma unroll
                for (int v = 0; v < kPer; ++v) {
                    const int u = t + 32 * kBWarps * v;
                    if (u >= kUnits) continue;
                    if constexpr (KIND == kDX) {
                        const int kg = u % (BJ / 8), nch = u / (BJ / 8);
                        // gather byte b (k rows 4b .. 4b + 3) of n = q into byte q % 4 of
                        // g[b][q / 4]
                        uint32_t g[2][2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t t01 = __byte_perm(w[v][4 * h], w[v][4 * h + 1], 0x5140);
                            const uint32_t t23 = __byte_perm(w[v][4 * h + 2], w[v][4 * h + 3], 0x5140);
                            g[0][h] = __byte_perm(t01, t23, 0x5410);
                            g[1][h] = __byte_perm(t01, t23, 0x7632);
                        }
#pragma unroll
                        for (int kr = 0; kr < 8; ++kr) {
                            const int b = kr >> 2, sh = 2 * (kr & 3);
                            uint4 o;
                            codes4_to_bf16((g[b][0] >> sh) & 0x03030303u, o.x, o.y);
                            codes4_to_bf16((g[b][1] >> sh) & 0x03030303u, o.z, o.w);
                            *reinterpret_cast<uint4*>(bt + sw128(8 * kg + kr, nch)) = o;
                        }
                    } else {
                        const int kw = u % (BJ / 4), mch = u / (BJ / 4);
#pragma unroll
                        for (int kr = 0; kr < 4; ++kr) {
                            uint4 o;
                            o.x = bf16x2_of_s8(w[v][0] >> (8 * kr), w[v][1] >> (8 * kr));
                            o.y = bf16x2_of_s8(w[v][2] >> (8 * kr), w[v][3] >> (8 * kr));
                            o.z = bf16x2_of_s8(w[v][4] >> (8 * kr), w[v][5] >> (8 * kr));
                            o.w = bf16x2_of_s8(w[v][6] >> (8 * kr), w[v][7] >> (8 * kr));
                            *reinterpret_cast<uint4*>(bt + sw128(4 * kw + kr, mch)) = o;
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(full(stage));
                if (++stage == ST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // -------------------------------------------------------------- epilogue --
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const float g = *a.gamma;
        const bool vec = (a.J & 3) == 0;
        int buf = 0;
        uint32_t bphase = 0;
        for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
            const int i0 = (tile % a.tiles_i) * kBI, j0 = (tile / a.tiles_i) * BJ;
            if (!mbar_wait_bounded(tfull(buf), bphase, abort_flag)) break;
            tc_fence_after();
            const int i = i0 + 32 * q + lane;
            float* orow = a.out + static_cast<int64_t>(i) * a.J;
#pragma unroll 1
            for (int c0 = 0; c0 < BJ; c0 += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                                       static_cast<uint32_t>(buf * BJ + c0),
                                   r);
                tmem_ld_wait();
                if (i >= a.I) continue;
                const int j = j0 + c0;
                if (vec && j + 32 <= a.J) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(orow + j + e) =
                            make_float4(__fmul_rn(g, __uint_as_float(r[e])), __fmul_rn(g, __uint_as_float(r[e + 1])),
                                        __fmul_rn(g, __uint_as_float(r[e + 2])),
                                        __fmul_rn(g, __uint_as_float(r[e + 3])));
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (j + e < a.J) orow[j + e] = __fmul_rn(g, __uint_as_float(r[e]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty(buf));
            if (++buf == 2) {
                buf = 0;
                bphase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

// ---------------------------------------------------------------------------------
// The same GEMM with the raw operands staged by TMA (shapes whose rows are 16-byte
// aligned: N % 4 == 0, and K % 64 == 0 for dX / K % 16 == 0 for dW).  One thread loads
// each stage's raw tiles -- dY as fp32 and the packed codes (dX) or x_q (dW) as bytes --
// into a ring of raw stages, several stages ahead; the converter warps turn a raw stage
// into the bf16 operand tiles of a converted stage (shared to shared, no global latency
// on their path) and release the raw stage; the MMA issuer consumes converted stages as
// before.
//   warp 0 (one lane)  TMA producer;  warp 1 (one lane)  MMA issuer;
//   warps 2-5          A converters;  warps 6-13  B converters;  warps 14-17  epilogue.
constexpr int kThreadsT = 576;  // 18 warps
constexpr int kWarpTmaT = 0, kWarpMmaT = 1, kWarpAT = 2, kWarpBT = 6, kWarpEpiT = 14;
constexpr int kAWarpsT = kWarpBT - kWarpAT, kBWarpsT = kWarpEpiT - kWarpBT;

template <int KIND, int BJ>
struct SteTCfg {
    static constexpr int kATile = kBI * kRowBytes;
    static constexpr int kBTile = BJ * kRowBytes;
    static constexpr int kConvBytes = 2 * kATile + kBTile;
    static constexpr int kRawA = kBI * kBC * 4;                          // 128 x 64 fp32 either way
    static constexpr int kRawB = KIND == kDX ? kBC * (BJ / 4) : kBC * BJ;  // 64 rows of codes or x_q
    static constexpr int kRawBytes = kRawA + kRawB;
    static constexpr int kCS = 2;  // converted stages
    static constexpr int kRSRaw = (227 * 1024 - 1024 - 512 - kCS * kConvBytes) / kRawBytes;
    static constexpr int kRS = kRSRaw > 4 ? 4 : kRSRaw;  // raw stages
    static constexpr int kTmemCols = 2 * BJ;
    static constexpr int kBarCount = 2 * kRS + 2 * kCS + 5;
    static constexpr int kSmemBytes = 1024 + kCS * kConvBytes + kRS * kRawBytes + 8 * kBarCount + 16;
    static_assert(kRS >= 2, "raw stages");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

template <int KIND, int BJ>
__global__ void __launch_bounds__(kThreadsT, 1)
    ste_tma_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                   const SteArgs a) {
    using Cfg = SteTCfg<KIND, BJ>;
    constexpr int CS = Cfg::kCS, RS = Cfg::kRS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw0 = smem_u32(smem_raw);
    const uint32_t base = (raw0 + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw0);
    // converted stages first (1024-aligned swizzled tiles), then the raw stages
    auto cAhi = [&](int c) { return static_cast<uint32_t>(c * Cfg::kConvBytes); };
    auto cAlo = [&](int c) { return static_cast<uint32_t>(c * Cfg::kConvBytes + Cfg::kATile); };
    auto cB = [&](int c) { return static_cast<uint32_t>(c * Cfg::kConvBytes + 2 * Cfg::kATile); };
    auto rA = [&](int r) { return static_cast<uint32_t>(CS * Cfg::kConvBytes + r * Cfg::kRawBytes); };
    auto rB = [&](int r) { return static_cast<uint32_t>(CS * Cfg::kConvBytes + r * Cfg::kRawBytes + Cfg::kRawA); };
    const uint32_t sBar = base + CS * Cfg::kConvBytes + RS * Cfg::kRawBytes;
    auto rfull = [&](int r) { return sBar + 8u * r; };
    auto rempty = [&](int r) { return sBar + 8u * (RS + r); };
    auto cfull = [&](int c) { return sBar + 8u * (2 * RS + c); };
    auto cempty = [&](int c) { return sBar + 8u * (2 * RS + CS + c); };
    auto tfull = [&](int b) { return sBar + 8u * (2 * RS + 2 * CS + b); };
    auto tempty = [&](int b) { return sBar + 8u * (2 * RS + 2 * CS + 2 + b); };
    const uint32_t drain_bar = sBar + 8u * (2 * RS + 2 * CS + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + (sBar - base) + 8 * Cfg::kBarCount);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int r = 0; r < RS; ++r) {
            mbar_init(rfull(r), 1);
            mbar_init(rempty(r), kAWarpsT + kBWarpsT);
        }
        for (int c = 0; c < CS; ++c) {
            mbar_init(cfull(c), kAWarpsT + kBWarpsT);
            mbar_init(cempty(c), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull(b), 1);
            mbar_init(tempty(b), kEpiWarps);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        mbar_fence_init();
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_b);
    }
    pdl_wait_then_release();
    if (warp == kWarpMmaT) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int nC = (a.C + kBC - 1) / kBC;
    const int my_tiles = a.num_tiles > static_cast<int>(blockIdx.x)
                             ? (a.num_tiles - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x
                             : 0;
    const int total = my_tiles * nC;  // stages this block runs, across its tiles

    if (warp == kWarpTmaT) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer --
            int r = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x) {
                const int i0 = (tile % a.tiles_i) * kBI, j0 = (tile / a.tiles_i) * BJ;
                for (int kc = 0; kc < nC; ++kc) {
                    const int c0 = kc * kBC;
                    if (!mbar_wait_bounded(rempty(r), phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(rfull(r), Cfg::kRawBytes);
                    if constexpr (KIND == kDX) {
                        tma_load_2d(base + rA(r), &tmap_a, rfull(r), c0, i0);       // dY[i0 .., c0 ..]
                        tma_load_2d(base + rB(r), &tmap_b, rfull(r), j0 / 4, c0);   // packed[c0 .., j0/4 ..]
                    } else {
                        tma_load_2d(base + rA(r), &tmap_a, rfull(r), i0, c0);       // dY[c0 .., i0 ..]
                        tma_load_2d(base + rB(r), &tmap_b, rfull(r), j0, c0);       // x_q[c0 .., j0 ..]
                    }
                    ++issued;
                    if (++r == RS) {
                        r = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                for (int q = 0; q < RS; ++q) {
                    const long long fills = (issued - q + RS - 1) / RS;
                    if (fills > 0) mbar_drain_ste(rfull(q), static_cast<uint32_t>((fills - 1) & 1));
                }
            }
        }
    } else if (warp == kWarpMmaT) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer --
            constexpr uint32_t idesc = idesc_bf16(kBI, BJ);
            int c = 0, buf = 0;
            uint32_t phase = 0, bphase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x) {
                if (!mbar_wait_bounded(tempty(buf), bphase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BJ);
                for (int kc = 0; kc < nC; ++kc) {
                    if (!mbar_wait_bounded(cfull(c), phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kBC / 16; ++kk) {
                        const uint64_t bd = smem_desc_sw128(base + cB(c) + 32 * kk);
                        tc_mma_bf16(d_tmem, smem_desc_sw128(base + cAhi(c) + 32 * kk), bd, idesc,
                                    (kc | kk) != 0 ? 1u : 0u);
                        tc_mma_bf16(d_tmem, smem_desc_sw128(base + cAlo(c) + 32 * kk), bd, idesc, 1u);
                    }
                    tc_commit(cempty(c));
                    if (++c == CS) {
                        c = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(tfull(buf));
                if (++buf == 2) {
                    buf = 0;
                    bphase ^= 1u;
                }
            }
            if (!ok) {
                tc_commit(drain_bar);
                mbar_drain_ste(drain_bar, 0);
            }
        }
    } else if (warp < kWarpEpiT) {
        // ------------------------------------------------------------- converters --
        // every converter warp takes part in every stage: wait for its raw stage and a
        // free converted stage, convert its share, release the raw stage, then mark the
        // converted stage full
        const bool is_a = warp < kWarpBT;
        const int t = is_a ? threadIdx.x - 32 * kWarpAT : threadIdx.x - 32 * kWarpBT;
        for (int i = 0; i < total; ++i) {
            const int r = i % RS, c = i % CS;
            const uint32_t rph = static_cast<uint32_t>((i / RS) & 1), cph = static_cast<uint32_t>((i / CS) & 1);
            const int kc = i % nC;
            const int c0 = kc * kBC;
            // dW: the stage's 64 reciprocals 1/s_m (two per lane), fetched before the waits
            float rA_ = 0.0f, rB_ = 0.0f;
            if constexpr (KIND == kDW) {
                if (is_a) {
                    const int mA = c0 + lane, mB = c0 + 32 + lane;
                    rA_ = mA < a.M ? __frcp_rn(__ldg(a.s + mA)) : 0.0f;
                    rB_ = mB < a.M ? __frcp_rn(__ldg(a.s + mB)) : 0.0f;
                }
            }
            if (!mbar_wait_bounded(rfull(r), rph, abort_flag) || !mbar_wait_bounded(cempty(c), cph ^ 1u, abort_flag))
                break;
            const uint8_t* ra = gbase + rA(r);
            const uint8_t* rb = gbase + rB(r);
            if (is_a) {
                uint8_t* ahi = gbase + cAhi(c);
                uint8_t* alo = gbase + cAlo(c);
                if constexpr (KIND == kDX) {
                    // raw [128 tokens][64 n] fp32 -> A[m][n]: eight threads per row
                    const int r_off = t >> 3, ch = t & 7;
#pragma unroll
                    for (int p = 0; p < kBI / 16; ++p) {
                        const int row = 16 * p + r_off;
                        const float4* src = reinterpret_cast<const float4*>(ra + row * (kBC * 4) + ch * 32);
                        const float4 u = src[0], v = src[1];
                        const float x[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
                        uint4 hi, lo;
                        split8(x, hi, lo);
                        *reinterpret_cast<uint4*>(ahi + sw128(row, ch)) = hi;
                        *reinterpret_cast<uint4*>(alo + sw128(row, ch)) = lo;
                    }
                } else {
                    // raw [64 tokens][128 n] fp32 -> A[n][m] = dY[m][n] / s[m]: thread = row n
                    const float* rf = reinterpret_cast<const float*>(ra);
#pragma unroll
                    for (int ch = 0; ch < kBC / 8; ++ch) {
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int m = 8 * ch + e;
                            x[e] = __fmul_rn(rf[m * kBI + t], __shfl_sync(0xffffffffu, m < 32 ? rA_ : rB_, m & 31));
                        }
                        uint4 hi, lo;
                        split8(x, hi, lo);
                        *reinterpret_cast<uint4*>(ahi + sw128(t, ch)) = hi;
                        *reinterpret_cast<uint4*>(alo + sw128(t, ch)) = lo;
                    }
                }
            } else {
                uint8_t* bt = gbase + cB(c);
                if constexpr (KIND == kDX) {
                    // raw packed [64 n][BJ/4 bytes] -> B[k][n]: units of 8 k x 8 n
                    constexpr int kUnits = (BJ / 8) * 8;
                    for (int u = t; u < kUnits; u += 32 * kBWarpsT) {
                        const int kg = u % (BJ / 8), nch = u / (BJ / 8);
                        uint32_t w[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            w[q] = *reinterpret_cast<const uint16_t*>(rb + (8 * nch + q) * (BJ / 4) + 2 * kg);
                        uint32_t g[2][2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t t01 = __byte_perm(w[4 * h], w[4 * h + 1], 0x5140);
                            const uint32_t t23 = __byte_perm(w[4 * h + 2], w[4 * h + 3], 0x5140);
                            g[0][h] = __byte_perm(t01, t23, 0x5410);
                            g[1][h] = __byte_perm(t01, t23, 0x7632);
                        }
#pragma unroll
                        for (int kr = 0; kr < 8; ++kr) {
                            const int b = kr >> 2, sh = 2 * (kr & 3);
                            uint4 o;
                            codes4_to_bf16((g[b][0] >> sh) & 0x03030303u, o.x, o.y);
                            codes4_to_bf16((g[b][1] >> sh) & 0x03030303u, o.z, o.w);
                            *reinterpret_cast<uint4*>(bt + sw128(8 * kg + kr, nch)) = o;
                        }
                    }
                } else {
                    // raw x_q [64 tokens][BJ bytes] -> B[k][m]: units of 4 k x 8 m
                    constexpr int kUnits = (BJ / 4) * 8;
                    for (int u = t; u < kUnits; u += 32 * kBWarpsT) {
                        const int kw = u % (BJ / 4), mch = u / (BJ / 4);
                        uint32_t w[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            w[q] = *reinterpret_cast<const uint32_t*>(rb + (8 * mch + q) * BJ + 4 * kw);
#pragma unroll
                        for (int kr = 0; kr < 4; ++kr) {
                            uint4 o;
                            o.x = bf16x2_of_s8(w[0] >> (8 * kr), w[1] >> (8 * kr));
                            o.y = bf16x2_of_s8(w[2] >> (8 * kr), w[3] >> (8 * kr));
                            o.z = bf16x2_of_s8(w[4] >> (8 * kr), w[5] >> (8 * kr));
                            o.w = bf16x2_of_s8(w[6] >> (8 * kr), w[7] >> (8 * kr));
                            *reinterpret_cast<uint4*>(bt + sw128(4 * kw + kr, mch)) = o;
                        }
                    }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(rempty(r));
                mbar_arrive(cfull(c));
            }
        }
    } else {
        // -------------------------------------------------------------- epilogue --
        const int q = warp & 3;
        const float g = *a.gamma;
        const bool vec = (a.J & 3) == 0;
        int buf = 0;
        uint32_t bphase = 0;
        for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
            const int i0 = (tile % a.tiles_i) * kBI, j0 = (tile / a.tiles_i) * BJ;
            if (!mbar_wait_bounded(tfull(buf), bphase, abort_flag)) break;
            tc_fence_after();
            const int i = i0 + 32 * q + lane;
            float* orow = a.out + static_cast<int64_t>(i) * a.J;
#pragma unroll 1
            for (int c0 = 0; c0 < BJ; c0 += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                                       static_cast<uint32_t>(buf * BJ + c0),
                                   r);
                tmem_ld_wait();
                if (i >= a.I) continue;
                const int j = j0 + c0;
                if (vec && j + 32 <= a.J) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(orow + j + e) =
                            make_float4(__fmul_rn(g, __uint_as_float(r[e])), __fmul_rn(g, __uint_as_float(r[e + 1])),
                                        __fmul_rn(g, __uint_as_float(r[e + 2])),
                                        __fmul_rn(g, __uint_as_float(r[e + 3])));
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (j + e < a.J) orow[j + e] = __fmul_rn(g, __uint_as_float(r[e]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty(buf));
            if (++buf == 2) {
                buf = 0;
                bphase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMmaT) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

int sm_count_ste() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// Column tile: the one with fewer waves x columns per tile (a tile's time is about
// proportional to its columns once the producers keep up); ties go to 256.
int ste_tile(int64_t I, int64_t J, int sms) {
    const int64_t ti = (I + kBI - 1) / kBI;
    int best = 256;
    int64_t best_cost = -1;
    for (int bj : {256, 128}) {
        const int64_t tiles = ti * ((J + bj - 1) / bj);
        const int64_t cost = (tiles + sms - 1) / sms * bj;
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = bj;
        }
    }
    return best;
}

template <int KIND, int BJ>
cudaError_t launch_ste_bj(SteArgs a, int sms, cudaStream_t stream) {
    using Cfg = SteCfg<BJ>;
    static PerContextOnce attr;
    cudaError_t e = attr.run([] {
        return cudaFuncSetAttribute(ste_tc_kernel<KIND, BJ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Cfg::kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    a.tiles_i = (a.I + kBI - 1) / kBI;
    a.num_tiles = a.tiles_i * ((a.J + BJ - 1) / BJ);
    const int grid = a.num_tiles < sms ? a.num_tiles : sms;
    return launch_pdl(ste_tc_kernel<KIND, BJ>, dim3(grid), dim3(kThreads), Cfg::kSmemBytes, stream,
                      dim3(kNoCluster), a);
}

template <int KIND, int BJ>
cudaError_t launch_ste_tma_bj(SteArgs a, int sms, cudaStream_t stream) {
    using Cfg = SteTCfg<KIND, BJ>;
    CUtensorMap ta, tb;
    // dY is [M, N] fp32 for both; the raw box is 64 x 128 (dX: n-inner) or 128 x 64 (dW)
    const bool ok_a = KIND == kDX
                          ? encode_tmap_f32_2d(&ta, a.dY, static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.M), kBC, kBI)
                          : encode_tmap_f32_2d(&ta, a.dY, static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.M), kBI, kBC);
    const bool ok_b = KIND == kDX
                          ? encode_tmap_u8_2d(&tb, a.packed, static_cast<uint64_t>(a.K / 4), static_cast<uint64_t>(a.N),
                                              BJ / 4, kBC, false)
                          : encode_tmap_u8_2d(&tb, a.xq, static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M), BJ, kBC,
                                              false);
    if (!ok_a || !ok_b) return cudaErrorInvalidValue;
    static PerContextOnce attr;
    cudaError_t e = attr.run([] {
        return cudaFuncSetAttribute(ste_tma_kernel<KIND, BJ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Cfg::kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    a.tiles_i = (a.I + kBI - 1) / kBI;
    a.num_tiles = a.tiles_i * ((a.J + BJ - 1) / BJ);
    const int grid = a.num_tiles < sms ? a.num_tiles : sms;
    return launch_pdl(ste_tma_kernel<KIND, BJ>, dim3(grid), dim3(kThreadsT), Cfg::kSmemBytes, stream,
                      dim3(kNoCluster), ta, tb, a);
}

template <int KIND>
cudaError_t launch_ste(SteArgs a, cudaStream_t stream) {
    const int sms = sm_count_ste();
    const int bj = ste_tile(a.I, a.J, sms);
    // TMA needs 16-byte row pitches: dY rows (N % 4), packed rows (K % 64) or x_q rows (K % 16)
    const bool staged = (a.N % 4) == 0 && (KIND == kDX ? a.K % 64 == 0 : a.K % 16 == 0);
    if (staged) return bj == 256 ? launch_ste_tma_bj<KIND, 256>(a, sms, stream) : launch_ste_tma_bj<KIND, 128>(a, sms, stream);
    if (bj == 256) return launch_ste_bj<KIND, 256>(a, sms, stream);
    return launch_ste_bj<KIND, 128>(a, sms, stream);
}

}  // namespace

cudaError_t launch_ste_grad_input(const float* dY, const uint8_t* packed, const float* gamma, int64_t M, int64_t N,
                                  int64_t K, float* dX, cudaStream_t stream) {
    SteArgs a{dY, packed, nullptr, nullptr, gamma, dX, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
              static_cast<int>(M), static_cast<int>(K), static_cast<int>(N), 0, 0};
    return launch_ste<kDX>(a, stream);
}

cudaError_t launch_ste_grad_weight(const float* dY, const int8_t* xq, const float* s, const float* gamma, int64_t M,
                                   int64_t N, int64_t K, float* dW, cudaStream_t stream) {
    SteArgs a{dY, nullptr, xq, s, gamma, dW, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
              static_cast<int>(N), static_cast<int>(K), static_cast<int>(M), 0, 0};
    return launch_ste<kDW>(a, stream);
}

}  // namespace bl
