// k_gemv_tma.cu -- decode-regime BitLinear forward for wide layers: a persistent GEMV
// fed by TMA, with the shortest unpack of the 2-bit codes.
//
// Same arithmetic as k_gemv.cu ("What 1.58 Bits Actually Changes", "How the low-bit
// linear path works": +1 adds, -1 subtracts, 0 skips; one float rescale at the end):
//   acc[m, n] = sum_k x_q[m, k] * c[n, k],   y[m, n] = acc[m, n] * gamma / s[m].
//
// Unpack.  The 2-bit fields of a packed word are first rewritten as 2-bit two's
// complement (00 -> 00, 01 -> 01, 10 -> 11, and the unused 11 -> 00) with two 3-input
// logic ops and one multiply-add; each of the four output words is then one left shift
// (a multiply, on the FMA pipe) and one mask that keeps bits 6..7 of every byte.  Byte j
// of output word i is thus 64 * code(4j + i): the codes come out in stride-4 order
// (i, i+4, i+8, i+12) and scaled by 64.  The activations are read in the matching
// stride-4 k16 layout, the int32 sums are 64 times the true sums (exact while
// 64 * 128 * K < 2^31) and the epilogue shifts them back by 6, exactly.
//
// Work split.  One block per SM owns a contiguous, balanced run of 16-row tiles over
// the whole of K.  The block's warps are grouped per pair of tiles; when a block has
// few tiles, several warps share a pair, each taking part of every stage's K range, and
// they add their partial sums through shared memory at the end.  A producer lane
// streams the weights, per stage and per 1024 codes of K, as one TMA box of 16 rows x
// 256 bytes per tile (256 contiguous bytes per row keep the DRAM reads long; 128-byte
// boxes measured a third slower).  The activations, a few kilobytes per stage shared by
// every warp, are read by the warps themselves through L1, issued before each wait for
// the weights.  K tails and rows past N read the TMA's zero fill.  Every wait is
// bounded.
#include <cuda_bf16.h>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {

bool encode_tmap_u8_2d(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                       uint32_t box_outer, bool swizzle128);

namespace {

constexpr int kConsumerWarps = 16;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kUnitCodes = 1024;      // K codes per weight box: 256 packed bytes per row
constexpr int kTileBytes = 16 * 256;  // one 16-row weight box
constexpr int kMaxTilesPerBlock = 2 * kConsumerWarps;
constexpr int kMaxPairs = kMaxTilesPerBlock / 2;
constexpr int64_t kMaxK = int64_t(1) << 17;  // keeps 64 * 128 * K below 2^31
constexpr int kSmemLimit = 227 * 1024;

struct GtArgs {
    const int8_t* xq;
    const float* s;
    const float* gamma;
    int M, N, K;
    int ntiles;      // 16-row tiles in N
    int nstages;     // shared-memory stages
    int tile_slots;  // tiles per unit buffer (even, >= the most tiles any block owns)
    int units;       // 1024-code units per stage
    int wpp;         // warps per tile pair (a power of two)
    void* out;
    int kind;
    int32_t* err;
    S4Mul mul;
    int grow;  // gamma holds one scale per output row
    unsigned long long wait_ns;  // limit of every wait (2 s outside the bounded-wait test)
    int stall_after;             // the producer stops after this many stages (< 0: never)
};

__device__ __forceinline__ void store_y1(void* out, int kind, int64_t idx, int acc, float fac) {
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

#define BL_MMA(D, A, B) "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 " D ", " A ", " B ", " D ";\n\t"

// One K step of 16 codes for the thread's four rows (words w0: tile 0 row g, w1: tile 0
// row g + 8, w2/w3: the same rows of tile 1), against token tile 0 (B = b) and, with
// MT == 2, token tile 1 (B = bb).  Each row pair takes two MMAs (m16n8k32): unpacked
// words 0/1 against activation words 0/1, then words 2/3 against words 2/3.
template <int MT>
__device__ __forceinline__ void s4_step(int (&acc)[2][MT][4], uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                        uint4 b, uint4 bb, const S4Mul& k) {
    if constexpr (MT == 1) {
        // %0-%7 accumulators, %8-%11 words, %12-%15 activations, %16-%20 multipliers
        asm volatile(
            "{\n\t.reg .b32 ta, tx, ty, tv, tt;\n\t"
            ".reg .b32 p0,p1,p2,p3,q0,q1,q2,q3,r0,r1,r2,r3,u0,u1,u2,u3;\n\t"
            BL_S4_UNPACK("%8", "p0", "p1", "p2", "p3", "%16", "%17", "%18", "%19", "%20")
            BL_S4_UNPACK("%9", "q0", "q1", "q2", "q3", "%16", "%17", "%18", "%19", "%20")
            BL_MMA("{%0,%1,%2,%3}", "{p0,q0,p1,q1}", "{%12,%13}")
            BL_MMA("{%0,%1,%2,%3}", "{p2,q2,p3,q3}", "{%14,%15}")
            BL_S4_UNPACK("%10", "r0", "r1", "r2", "r3", "%16", "%17", "%18", "%19", "%20")
            BL_S4_UNPACK("%11", "u0", "u1", "u2", "u3", "%16", "%17", "%18", "%19", "%20")
            BL_MMA("{%4,%5,%6,%7}", "{r0,u0,r1,u1}", "{%12,%13}")
            BL_MMA("{%4,%5,%6,%7}", "{r2,u2,r3,u3}", "{%14,%15}")
            "}\n"
            : "+r"(acc[0][0][0]), "+r"(acc[0][0][1]), "+r"(acc[0][0][2]), "+r"(acc[0][0][3]),
              "+r"(acc[1][0][0]), "+r"(acc[1][0][1]), "+r"(acc[1][0][2]), "+r"(acc[1][0][3])
            : "r"(w0), "r"(w1), "r"(w2), "r"(w3), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w), "r"(k.hi1), "r"(k.two),
              "r"(k.m4), "r"(k.m16), "r"(k.m64));
    } else {
        // %0-%15 accumulators, %16-%19 words, %20-%27 activations, %28-%32 multipliers
        asm volatile(
            "{\n\t.reg .b32 ta, tx, ty, tv, tt;\n\t"
            ".reg .b32 p0,p1,p2,p3,q0,q1,q2,q3,r0,r1,r2,r3,u0,u1,u2,u3;\n\t"
            BL_S4_UNPACK("%16", "p0", "p1", "p2", "p3", "%28", "%29", "%30", "%31", "%32")
            BL_S4_UNPACK("%17", "q0", "q1", "q2", "q3", "%28", "%29", "%30", "%31", "%32")
            BL_MMA("{%0,%1,%2,%3}", "{p0,q0,p1,q1}", "{%20,%21}")
            BL_MMA("{%0,%1,%2,%3}", "{p2,q2,p3,q3}", "{%22,%23}")
            BL_MMA("{%8,%9,%10,%11}", "{p0,q0,p1,q1}", "{%24,%25}")
            BL_MMA("{%8,%9,%10,%11}", "{p2,q2,p3,q3}", "{%26,%27}")
            BL_S4_UNPACK("%18", "r0", "r1", "r2", "r3", "%28", "%29", "%30", "%31", "%32")
            BL_S4_UNPACK("%19", "u0", "u1", "u2", "u3", "%28", "%29", "%30", "%31", "%32")
            BL_MMA("{%4,%5,%6,%7}", "{r0,u0,r1,u1}", "{%20,%21}")
            BL_MMA("{%4,%5,%6,%7}", "{r2,u2,r3,u3}", "{%22,%23}")
            BL_MMA("{%12,%13,%14,%15}", "{r0,u0,r1,u1}", "{%24,%25}")
            BL_MMA("{%12,%13,%14,%15}", "{r2,u2,r3,u3}", "{%26,%27}")
            "}\n"
            : "+r"(acc[0][0][0]), "+r"(acc[0][0][1]), "+r"(acc[0][0][2]), "+r"(acc[0][0][3]),
              "+r"(acc[1][0][0]), "+r"(acc[1][0][1]), "+r"(acc[1][0][2]), "+r"(acc[1][0][3]),
              "+r"(acc[0][MT - 1][0]), "+r"(acc[0][MT - 1][1]), "+r"(acc[0][MT - 1][2]), "+r"(acc[0][MT - 1][3]),
              "+r"(acc[1][MT - 1][0]), "+r"(acc[1][MT - 1][1]), "+r"(acc[1][MT - 1][2]), "+r"(acc[1][MT - 1][3])
            : "r"(w0), "r"(w1), "r"(w2), "r"(w3), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w), "r"(bb.x), "r"(bb.y),
              "r"(bb.z), "r"(bb.w), "r"(k.hi1), "r"(k.two), "r"(k.m4), "r"(k.m16), "r"(k.m64));
    }
}
#undef BL_MMA

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Shared memory (1024-byte aligned): per stage and per 1024-code unit, the weight boxes
// [tile slot][16 rows][256 B]; after the stages one full barrier per (stage, tile pair),
// one empty barrier per stage, and the abort flag.  A stage streams every tile of the
// block at the same K offset (long, regular DRAM reads), but each pair of tiles has its
// own full barrier, so a warp starts on its tiles as soon as their boxes land.  Warps
// that share a tile pair add their partial sums through the stage memory once every
// stage has been consumed.
//
// Quarter c of a unit (256 codes) gives thread t of a quad weight piece P = 4c + t of its
// rows (16-groups 4P + i, i = 0..3).  Those weight reads, 256 bytes apart per row, are
// 2-way bank conflicted.  The thread reads the matching 16 activation bytes of its
// tokens straight from global memory (the stride-4 layout keeps a 16-group contiguous):
// every warp of the block reads the same few kilobytes per stage, which stay in L1.
template <int MT>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_tma_kernel(const __grid_constant__ CUtensorMap tmap_w, const GtArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
    uint8_t* gbase = smem_raw + pad;
    const uint32_t base = raw + pad;
    const int ST = a.nstages, U = a.units, R = a.wpp;
    const uint32_t w_unit = static_cast<uint32_t>(a.tile_slots) * kTileBytes;
    const uint32_t stage_bytes = static_cast<uint32_t>(U) * w_unit;
    const uint32_t off_bar = static_cast<uint32_t>(ST) * stage_bytes;
    const uint32_t sBar = base + off_bar;
    auto full = [&](int s, int pr) { return sBar + 8u * (s * kMaxPairs + pr); };
    auto empty = [&](int s) { return sBar + 8u * (ST * kMaxPairs + s); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + off_bar + 8 * ST * (kMaxPairs + 1));
    int* red = reinterpret_cast<int*>(gbase);  // aliases the stages once they are all consumed

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t_begin = static_cast<int>((static_cast<int64_t>(blockIdx.x) * a.ntiles) / gridDim.x);
    const int t_end = static_cast<int>((static_cast<int64_t>(blockIdx.x + 1) * a.ntiles) / gridDim.x);
    const int nt = t_end - t_begin;
    const int npairs = (nt + 1) / 2;
    const int kunits = (a.K + kUnitCodes - 1) / kUnitCodes;  // 1024-code units in K
    const int nstep = (kunits + U - 1) / U;

    if (threadIdx.x == 0) {
        // only the warps that own a tile pair consume (and release) stages: a warp with no
        // pair must not arrive, or its arrivals would run ahead into later phases and
        // release a stage that a slower pair is still reading
        for (int s = 0; s < ST; ++s) {
            for (int pr = 0; pr < npairs; ++pr) mbar_init(full(s, pr), 1);
            mbar_init(empty(s), npairs * R);
        }
        *abort_flag = 0;
        mbar_fence_init();
        tma_prefetch_desc(&tmap_w);
    }
    pdl_wait_then_release();
    __syncthreads();

    if (warp == kConsumerWarps) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer --
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int kt = 0; kt < nstep; ++kt) {
                if (!mbar_wait_bounded(empty(stage), phase ^ 1u, abort_flag, a.wait_ns)) {
                    ok = false;
                    break;
                }
                if (issued == a.stall_after) {  // the bounded-wait test: stop issuing
                    stall_until_abort(abort_flag, 4 * a.wait_ns);
                    ok = false;
                    break;
                }
                // units past the end of K are neither loaded nor read
                const int u0 = kt * U;
                const int uk = kunits - u0 < U ? kunits - u0 : U;
                const uint32_t sw = base + stage * stage_bytes;
                for (int pr = 0; pr < npairs; ++pr) {
                    const int tn = nt - 2 * pr < 2 ? nt - 2 * pr : 2;
                    mbar_arrive_expect_tx(full(stage, pr), static_cast<uint32_t>(uk * tn) * kTileBytes);
                    for (int u = 0; u < uk; ++u)
                        for (int t = 2 * pr; t < 2 * pr + tn; ++t)
                            tma_load_2d(sw + u * w_unit + t * kTileBytes, &tmap_w, full(stage, pr), (u0 + u) * 256,
                                        16 * (t_begin + t));
                }
                ++issued;
                if (++stage == ST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) {
                // let every issued copy land before the block exits
                for (int s = 0; s < ST; ++s) {
                    const long long fills = (issued - s + ST - 1) / ST;
                    for (int pr = 0; fills > 0 && pr < npairs; ++pr) {
                        const unsigned long long t0 = globaltimer_ns();
                        while (!mbar_try_wait(full(s, pr), static_cast<uint32_t>((fills - 1) & 1)) &&
                               globaltimer_ns() - t0 < 200000000ull) {
                        }
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ consumers --
        const int g = lane >> 2, t = lane & 3;
        const int pair = warp / R, part = warp % R;
        const bool active = pair < npairs;
        // the unpack's multipliers, held in registers for the whole loop
        S4Mul mul;
        asm volatile("mov.b32 %0, %5;\n\tmov.b32 %1, %6;\n\tmov.b32 %2, %7;\n\tmov.b32 %3, %8;\n\tmov.b32 %4, %9;"
                     : "=r"(mul.hi1), "=r"(mul.two), "=r"(mul.m4), "=r"(mul.m16), "=r"(mul.m64)
                     : "r"(a.mul.hi1), "r"(a.mul.two), "r"(a.mul.m4), "r"(a.mul.m16), "r"(a.mul.m64));
        int acc[2][MT][4];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int j = 0; j < MT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][j][e] = 0;
        // byte offsets in a unit's weight buffer of rows g and g + 8 of the pair's tiles,
        // at this thread's piece of quarter 0
        const uint32_t tb = static_cast<uint32_t>(2 * pair) * kTileBytes + 16u * t;
        const uint32_t woff[4] = {tb + g * 256u, tb + (g + 8) * 256u, tb + kTileBytes + g * 256u,
                                  tb + kTileBytes + (g + 8) * 256u};
        // this thread's activation rows, tokens g and g + 8.  A padding token (>= M) reads
        // token 0's row: it only feeds MMA columns whose outputs are never stored.  A
        // 16-group past K reads the row's start: its weights are the TMA's zero fill.
        // So every load is unconditional, on an in-bounds address.
        const int8_t* xrow0 = a.xq + static_cast<int64_t>(g < a.M ? g : 0) * a.K + 64 * t;
        const int8_t* xrow1 = a.xq + static_cast<int64_t>(g + 8 < a.M ? g + 8 : 0) * a.K + 64 * t;
        // the activations of 256-code quarter q (global index) for this thread
        auto load_x = [&](int q, uint4 (&b)[4], uint4 (&bb)[4]) {
            // K % 128 == 0: this thread's 64 codes are all inside K or all past it
            const int k0 = q * 256 + 64 * t < a.K ? q * 256 : 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                b[i] = __ldg(reinterpret_cast<const uint4*>(xrow0 + k0 + 16 * i));
                if constexpr (MT > 1)
                    bb[i] = __ldg(reinterpret_cast<const uint4*>(xrow1 + k0 + 16 * i));
                else
                    bb[i] = b[i];
            }
        };
        int stage = 0;
        uint32_t phase = 0;
        for (int kt = 0; kt < nstep; ++kt) {
            const int uk = kunits - kt * U < U ? kunits - kt * U : U;
            // the first quarter's activations are requested before the wait for the weights;
            // with one token tile (registers to spare) each later quarter's are requested
            // while the previous quarter computes
            uint4 b[4], bb[4];
            if (active && part < 4 * uk) load_x(4 * kt * U + part, b, bb);
            if (active && !mbar_wait_bounded(full(stage, pair), phase, abort_flag, a.wait_ns)) break;
            if (active) {
                const uint8_t* sw = gbase + stage * stage_bytes;
                for (int c = part; c < 4 * uk; c += R) {
                    uint4 nb[4], nbb[4];
                    if constexpr (MT == 1) {
                        if (c + R < 4 * uk) load_x(4 * kt * U + c + R, nb, nbb);
                    } else {
                        if (c != part) load_x(4 * kt * U + c, b, bb);
                    }
                    const uint8_t* wq = sw + (c >> 2) * w_unit + (c & 3) * 64;
                    uint4 w[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) w[r] = *reinterpret_cast<const uint4*>(wq + woff[r]);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        s4_step<MT>(acc, word_of(w[0], i), word_of(w[1], i), word_of(w[2], i), word_of(w[3], i),
                                    b[i], bb[i], mul);
                    if constexpr (MT == 1) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) b[i] = nb[i];
                    }
                }
            }
            __syncwarp();
            if (active && lane == 0) mbar_arrive(empty(stage));
            if (++stage == ST) {
                stage = 0;
                phase ^= 1u;
            }
        }
        // warps that share a pair add their partial sums into the pair's first warp, in
        // the stage memory: every consumer has left the loop, and every issued copy was
        // waited for, before the first write
        if (R > 1) {
            asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumerWarps) : "memory");
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int j = 0; j < MT; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        red[(warp * (8 * MT) + (i * MT + j) * 4 + e) * 32 + lane] = acc[i][j][e];
            asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumerWarps) : "memory");
            if (part == 0) {
                for (int q = 1; q < R; ++q) {
#pragma unroll
                    for (int i = 0; i < 2; ++i)
#pragma unroll
                        for (int j = 0; j < MT; ++j)
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                acc[i][j][e] += red[((warp + q) * (8 * MT) + (i * MT + j) * 4 + e) * 32 + lane];
                }
            }
        }
        if (active && part == 0 && !*abort_flag) {
            const float gamma = (a.kind == kOutI32) ? 0.0f : *a.gamma;
            const int64_t row0 = 16 * static_cast<int64_t>(t_begin + 2 * pair);
            // fragment (tile, j): rows row0 + 16 tile + g (+8), tokens 8 j + 2 t (+1)
#pragma unroll
            for (int j = 0; j < MT; ++j) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tok = 8 * j + 2 * t + e;
                    if (tok >= a.M) continue;
                    const float fac = (a.kind == kOutI32) ? 0.0f : __fdiv_rn(gamma, a.s[tok]);
#pragma unroll
                    for (int tile = 0; tile < 2; ++tile) {
                        if (2 * pair + tile >= nt) continue;
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int64_t row = row0 + 16 * tile + g + 8 * hh;
                            if (row >= a.N) continue;
                            const float f =
                                (a.grow && a.kind != kOutI32) ? __fdiv_rn(a.gamma[row], a.s[tok]) : fac;
                            store_y1(a.out, a.kind, static_cast<int64_t>(tok) * a.N + row,
                                     acc[tile][j][2 * hh + e] >> 6, f);
                        }
                    }
                }
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag && a.err != nullptr) atomicOr(a.err, kErrBitTimeout);
}

struct GtPlan {
    int grid, tile_slots, units, wpp, stages;
    size_t smem;
};

// Launch plan, or false when the shape is outside this kernel's range: M <= 16,
// K % 128 == 0, K <= 2^17, at least one 16-row tile per SM and at most 32 per SM.
bool plan_gemv_tma(int64_t M, int64_t N, int64_t K, int sms, GtPlan* p) {
    if (M < 1 || M > 16 || K < 128 || K % 128 != 0 || K > kMaxK || sms < 1) return false;
    const int MT = M <= 8 ? 1 : 2;
    const int64_t ntiles = (N + 15) / 16;
    if (ntiles < sms) return false;
    int slots = static_cast<int>((ntiles + sms - 1) / sms);
    if (slots > kMaxTilesPerBlock) return false;
    slots += slots & 1;
    const int npairs = slots / 2;
    int wpp = 1;
    while (2 * wpp * npairs <= kConsumerWarps) wpp *= 2;
    const int kunits = static_cast<int>((K + kUnitCodes - 1) / kUnitCodes);
    int units = wpp / 4 > 1 ? wpp / 4 : 1;  // a unit gives four warps a quarter each
    if (units > kunits) units = kunits;
    const size_t red = static_cast<size_t>(kConsumerWarps) * 32 * 8 * MT * sizeof(int);
    const size_t fixed = 1024 + 16 + 64;
    for (;;) {
        const size_t stage = static_cast<size_t>(units) * static_cast<size_t>(slots) * kTileBytes;
        int stages = static_cast<int>((kSmemLimit - fixed) / (stage + 8 * (kMaxPairs + 1)));
        if (stages > 8) stages = 8;
        if (stages >= 2 && static_cast<size_t>(stages) * stage >= red) {
            p->grid = sms;
            p->tile_slots = slots;
            p->units = units;
            p->wpp = wpp;
            p->stages = stages;
            p->smem = fixed + static_cast<size_t>(stages) * (stage + 8 * (kMaxPairs + 1));
            return true;
        }
        if (units == 1) return false;
        units /= 2;
    }
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

}  // namespace

bool gemv_tma_applicable(int64_t M, int64_t N, int64_t K) {
    GtPlan p;
    return plan_gemv_tma(M, N, K, sm_count(), &p);
}

cudaError_t launch_gemv_tma(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                            int64_t M, int64_t N, int64_t K, void* out, int kind, int32_t* err,
                            cudaStream_t stream) {
    GtPlan p;
    if (!plan_gemv_tma(M, N, K, sm_count(), &p)) return cudaErrorInvalidValue;
    const int MT = M <= 8 ? 1 : 2;
    CUtensorMap tw;
    if (!encode_tmap_u8_2d(&tw, packed, static_cast<uint64_t>(K / 4), static_cast<uint64_t>(N), 256, 16, false))
        return cudaErrorInvalidValue;
    const int64_t ntiles = (N + 15) / 16;
    const WaitTest wt = wait_test();
    GtArgs a{xq, s, gamma, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), static_cast<int>(ntiles),
             p.stages, p.tile_slots, p.units, p.wpp, out, out_kind_of(kind), err, s4_mul(), gamma_rows_of(kind),
             wt.wait_ns, wt.stall_after};
    static PerContextOnce attr[2];
    cudaError_t e = attr[MT - 1].run([MT] {
        return MT == 1 ? cudaFuncSetAttribute(gemv_tma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              kSmemLimit)
                       : cudaFuncSetAttribute(gemv_tma_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              kSmemLimit);
    });
    if (e != cudaSuccess) return e;
    if (MT == 1) return launch_pdl(gemv_tma_kernel<1>, dim3(p.grid), dim3(kThreads), p.smem, stream, dim3(kNoCluster), tw, a);
    return launch_pdl(gemv_tma_kernel<2>, dim3(p.grid), dim3(kThreads), p.smem, stream, dim3(kNoCluster), tw, a);
}

}  // namespace bl
