// k_gemm_tm.cu -- prefill-regime BitLinear forward on tcgen05 with the expanded weights in
// tensor memory: the tiled, persistent counterpart of k_gemv_tc.cu.
//
// Same arithmetic as k_gemm_tc.cu ("1-bit & Ternary LLMs (BitNet b1.58)", block
// "BitNet (Oct 2023)": an integer product and one float rescale; "1.58 bits: what BitNet
// promised and what it required", "What you get on today's hardware": on GPUs the
// packed weights are unpacked and then multiplied):
//   acc[m, n] = sum_k x_q[m, k] * c[n, k],   y[m, n] = acc[m, n] * gamma / s[m].
//
// Why.  The shared-memory kernels (k_gemm_tc.cu) write every expanded weight byte into
// shared memory and the tensor core reads it back: per 128-code stage of a 128-row tile
// that is 32 KB of shared-memory traffic on top of the activation tile, which keeps the
// tensor pipe near half busy.  Here the expanders store the int8 codes into tensor
// memory (tcgen05.st) and the MMA takes its A operand from there, so shared memory
// carries only the packed weights and the activation tile.
//
// Tile: 128 output features (MMA M, TMEM lanes) x BT tokens (MMA N) x K in stages of 128
// codes; persistent blocks, one per SM, static round-robin over tiles.  Roles:
//   warp 0 (one lane)   TMA: x_q tile [BT x 128 B] (128-byte swizzle) and packed weights
//                       [128 rows x 32 B] per stage, one mbarrier;
//   warps 2-17          expanders, four groups of four warps (one per TMEM lane quarter);
//                       the stages of the block's whole sequence go to the groups in
//                       turn; each thread unpacks its row's 128 codes and stores 32 TMEM
//                       columns of that stage's slot, then one lane per warp arrives;
//   warp 1 (one lane)   MMA issuer: four tcgen05.mma kind::i8 (K = 32) per stage, A from
//                       the stage's TMEM slot, B from shared memory, into one of two TMEM
//                       accumulators; tcgen05.commit frees the stage (smem and TMEM slot);
//   warps 18-25         epilogue: tcgen05.ld of the finished accumulator (one feature row
//                       per thread, two warps per lane quarter taking alternate 32-token
//                       chunks), y = acc * (gamma / s_m), stores coalesced along N.
// Two accumulators overlap one tile's epilogue with the next tile's main loop.  Ragged
// edges come from TMA zero fill.  Every wait is bounded as in the other kernels.
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

constexpr int kBN = 128;                    // output features per tile (MMA M)
constexpr int kBK = 128;                    // K codes per stage
constexpr int kPBytes = kBN * (kBK / 4);    // packed weights per stage: 4 KB
constexpr int kACols = kBK / 4;             // TMEM columns of one expanded stage
constexpr int kThreads = 832;               // 26 warps
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpExp = 2, kWarpEpi = 18;
constexpr int kExpGroups = 4;
constexpr int kEpiWarps = 8;
constexpr unsigned long long kDrainNs = 200000000ull;  // 0.2 s

template <int BT>
struct TmCfg {
    static_assert(BT % 32 == 0 && BT >= 64 && BT <= 192, "token tile");
    static constexpr int kXBytes = BT * kBK;
    static constexpr int kStageBytes = kXBytes + kPBytes;
    // two accumulators of BT columns plus the expanded stages fill the 512 columns
    static constexpr int kStages = (512 - 2 * BT) / kACols < 8 ? (512 - 2 * BT) / kACols : 8;
    static constexpr int kTmemCols = 512;
    static constexpr int kBarBytes = 8 * (3 * kStages + 5) + 16;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBarBytes;
    // keep a second block off the SM: the block owns all 512 TMEM columns
    static constexpr int kSmemLaunch = kSmemBytes > 116 * 1024 ? kSmemBytes : 116 * 1024;
    static_assert(kStages >= 4, "stages");
    static_assert(kSmemLaunch <= 227 * 1024, "shared memory");
};

struct TmArgs {
    const float* s;
    const float* gamma;
    int M, N, K;
    int n_tiles_n, num_tiles;
    void* out;
    int kind;
    int32_t* err;
    S4Mul mul;
    int grow;                    // gamma holds one scale per output row
    unsigned long long wait_ns;  // limit of every wait (2 s outside the bounded-wait test)
    int stall_after;             // the producer stops after this many loads (< 0: never)
};

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

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kDrainNs) return;
    }
}

template <int BT, int LAY>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_p,
                   const TmArgs a) {
    using C = TmCfg<BT>;
    constexpr int ST = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t sX = base;  // x tiles first: 1024-aligned for the swizzle
    const uint32_t sP = sX + ST * C::kXBytes;
    const uint32_t sBar = sP + ST * kPBytes;
    auto full = [&](int s) { return sBar + 8u * s; };
    auto afull = [&](int s) { return sBar + 8u * (ST + s); };
    auto empty = [&](int s) { return sBar + 8u * (2 * ST + s); };
    auto tfull = [&](int b) { return sBar + 8u * (3 * ST + b); };
    auto tempty = [&](int b) { return sBar + 8u * (3 * ST + 2 + b); };
    const uint32_t drain_bar = sBar + 8u * (3 * ST + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + (sBar - base) + 8 * (3 * ST + 5));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(full(s), 1);
            mbar_init(afull(s), 4);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull(b), 1);
            mbar_init(tempty(b), kEpiWarps);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        mbar_fence_init();
        tma_prefetch_desc(&tmap_x);
        tma_prefetch_desc(&tmap_p);
    }
    pdl_wait_then_release();
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t acc_col0 = static_cast<uint32_t>(ST * kACols);  // accumulators after the A slots
    const int nK = (a.K + kBK - 1) / kBK;
    const int my_tiles = a.num_tiles > static_cast<int>(blockIdx.x)
                             ? (a.num_tiles - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x
                             : 0;
    const int total = my_tiles * nK;  // stages this block runs, across its tiles

    if (warp == kWarpTma) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer --
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x) {
                const int n0 = (tile % a.n_tiles_n) * kBN;
                const int t0 = (tile / a.n_tiles_n) * BT;
                for (int kt = 0; kt < nK; ++kt) {
                    if (!mbar_wait_bounded(empty(stage), phase ^ 1u, abort_flag, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    if (issued == a.stall_after) {  // the bounded-wait test: stop issuing
                        stall_until_abort(abort_flag, 4 * a.wait_ns);
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full(stage), C::kXBytes + kPBytes);
                    tma_load_2d(sX + stage * C::kXBytes, &tmap_x, full(stage), kt * kBK, t0);
                    tma_load_2d(sP + stage * kPBytes, &tmap_p, full(stage), kt * (kBK / 4), n0);
                    ++issued;
                    if (++stage == ST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                for (int s = 0; s < ST; ++s) {
                    const long long fills = (issued - s + ST - 1) / ST;
                    if (fills > 0) drain_wait(full(s), static_cast<uint32_t>((fills - 1) & 1));
                }
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer --
            constexpr uint32_t idesc = idesc_i8(kBN, BT);
            int stage = 0, buf = 0;
            uint32_t phase = 0, bphase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x) {
                if (!mbar_wait_bounded(tempty(buf), bphase ^ 1u, abort_flag, a.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc_col0 + static_cast<uint32_t>(buf * BT);
                for (int kt = 0; kt < nK; ++kt) {
                    if (!mbar_wait_bounded(full(stage), phase, abort_flag, a.wait_ns) ||
                        !mbar_wait_bounded(afull(stage), phase, abort_flag, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_tmem = tmem_base + static_cast<uint32_t>(stage * kACols);
                    const uint32_t b_addr = sX + stage * C::kXBytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 32; ++kk)
                        tc_mma_i8_tmem_a(d_tmem, a_tmem + 8 * kk, smem_desc_sw128(b_addr + 32 * kk), idesc,
                                         (kt | kk) != 0 ? 1u : 0u);
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
                tc_commit(drain_bar);
                drain_wait(drain_bar, 0);
            }
        }
    } else if (warp < kWarpEpi) {
        // ------------------------------------------------------------- expanders --
        // group g expands the block's stages g, g + 4, g + 8, ... (counted across tiles);
        // its thread owns weight row r (its TMEM lane) and the row's 128 codes
        const int q = warp & 3, grp = (warp - kWarpExp) >> 2;
        const int r = 32 * q + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
        for (int i = grp; i < total; i += kExpGroups) {
            const int stage = i % ST;
            const uint32_t phase = static_cast<uint32_t>((i / ST) & 1);
            if (!mbar_wait_bounded(full(stage), phase, abort_flag, a.wait_ns)) break;
            const uint8_t* prow = gbase + (sP - base) + stage * kPBytes + r * (kBK / 4);
            const uint4 p0 = *reinterpret_cast<const uint4*>(prow);
            const uint4 p1 = *reinterpret_cast<const uint4*>(prow + 16);
            const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
            uint32_t v[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                if constexpr (LAY == kXqEvenOdd16)
                    unpack16_evenodd(words[c], v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                else if constexpr (LAY == kXqStride4K16)
                    unpack16_stride4_x64(words[c], a.mul, v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                else
                    unpack16_natural(words[c], v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            }
            tmem_st_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(stage * kACols), v);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(afull(stage));
        }
    } else {
        // -------------------------------------------------------------- epilogue --
        // the stride-4 unpack feeds 64 * code: its sums are exact multiples of 64
        constexpr int kAccShift = LAY == kXqStride4K16 ? 6 : 0;
        const int q = warp & 3;
        const int first = 32 * ((warp - kWarpEpi) >> 2);  // this warp's first column chunk
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
        const float gamma = (a.kind == kOutI32) ? 0.0f : *a.gamma;
        int buf = 0;
        uint32_t bphase = 0;
        for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
            const int n0 = (tile % a.n_tiles_n) * kBN;
            const int t0 = (tile / a.n_tiles_n) * BT;
            float s_next = (a.kind != kOutI32 && t0 + first + lane < a.M) ? __ldg(a.s + t0 + first + lane) : 1.0f;
            if (!mbar_wait_bounded(tfull(buf), bphase, abort_flag, a.wait_ns)) break;
            tc_fence_after();
            const int row = n0 + 32 * q + lane;
            const bool row_ok = row < a.N;
            const float grow_gamma = (a.grow && a.kind != kOutI32 && row_ok) ? __ldg(a.gamma + row) : 0.0f;
#pragma unroll 1
            for (int c0 = first; c0 < BT; c0 += 64) {
                const float s_cur = s_next;
                const float fac = __fdiv_rn(gamma, s_cur);
                const int tk = t0 + c0 + 64 + lane;
                if (c0 + 64 < BT) s_next = (a.kind != kOutI32 && tk < a.M) ? __ldg(a.s + tk) : 1.0f;
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + lane_addr + acc_col0 + static_cast<uint32_t>(buf * BT + c0), r);
                tmem_ld_wait();
                if (a.grow) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float fj = __fdiv_rn(grow_gamma, __shfl_sync(0xffffffffu, s_cur, j));
                        const int tok = t0 + c0 + j;
                        if (tok < a.M && row_ok)
                            store_y(a.out, a.kind, static_cast<int64_t>(tok) * a.N + row,
                                    static_cast<int>(r[j]) >> kAccShift, fj);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float fj = __shfl_sync(0xffffffffu, fac, j);
                        const int tok = t0 + c0 + j;
                        if (tok < a.M && row_ok)
                            store_y(a.out, a.kind, static_cast<int64_t>(tok) * a.N + row,
                                    static_cast<int>(r[j]) >> kAccShift, fj);
                    }
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
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
    if (threadIdx.x == 0 && *abort_flag && a.err != nullptr) atomicOr(a.err, kErrBitTimeout);
}

template <int BT, int LAY>
cudaError_t launch_bt(const int8_t* xq, const uint8_t* packed, TmArgs a, int sms, cudaStream_t stream) {
    using C = TmCfg<BT>;
    CUtensorMap tx, tp;
    if (!encode_tmap_u8_2d(&tx, xq, static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M), kBK, BT, true) ||
        !encode_tmap_u8_2d(&tp, packed, static_cast<uint64_t>(a.K / 4), static_cast<uint64_t>(a.N), kBK / 4, kBN,
                           false))
        return cudaErrorInvalidValue;
    static PerContextOnce attr;
    cudaError_t e = attr.run([] {
        return cudaFuncSetAttribute(gemm_tm_kernel<BT, LAY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmemLaunch);
    });
    if (e != cudaSuccess) return e;
    a.num_tiles = a.n_tiles_n * static_cast<int>((a.M + BT - 1) / BT);
    const int grid = a.num_tiles < sms ? a.num_tiles : sms;
    return launch_pdl(gemm_tm_kernel<BT, LAY>, dim3(grid), dim3(kThreads), C::kSmemLaunch, stream,
                      dim3(kNoCluster), tx, tp, a);
}

template <int LAY>
cudaError_t launch_layout(int bt, const int8_t* xq, const uint8_t* packed, const TmArgs& a, int sms,
                          cudaStream_t stream) {
    switch (bt) {
        case 64: return launch_bt<64, LAY>(xq, packed, a, sms, stream);
        case 96: return launch_bt<96, LAY>(xq, packed, a, sms, stream);
        case 128: return launch_bt<128, LAY>(xq, packed, a, sms, stream);
        case 160: return launch_bt<160, LAY>(xq, packed, a, sms, stream);
        default: return launch_bt<192, LAY>(xq, packed, a, sms, stream);
    }
}

}  // namespace

// Token tile: among 64 ... 192 in steps of 32, the one with the fewest waves x per-tile
// cycles, a tile's stage costing about max(MMA, shared-memory traffic) ~ 40 + 2.1 BT
// cycles plus an epilogue share the next tile hides (ties: the larger tile).
int gemm_tm_tile(int64_t M, int64_t N, int64_t K, int sms) {
    const int64_t nN = (N + kBN - 1) / kBN;
    const int64_t nK = (K + kBK - 1) / kBK;
    int best = 192;
    int64_t best_cost = -1;
    for (int b = 192; b >= 64; b -= 32) {
        const int64_t tiles = nN * ((M + b - 1) / b);
        const int64_t waves = (tiles + sms - 1) / sms;
        const int64_t c = waves * nK * (40 + 21 * b / 10);
        if (best_cost < 0 || c < best_cost) {
            best_cost = c;
            best = b;
        }
    }
    return best;
}

cudaError_t launch_gemm_tm(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma, int64_t M,
                           int64_t N, int64_t K, void* out, int kind, int32_t* err, int layout, cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int bt = gemm_tm_tile(M, N, K, sms);
    const WaitTest wt = wait_test();
    TmArgs a{s, gamma, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
             static_cast<int>((N + kBN - 1) / kBN), 0, out, out_kind_of(kind), err, s4_mul(), gamma_rows_of(kind),
             wt.wait_ns, wt.stall_after};
    switch (layout) {
        case kXqEvenOdd16: return launch_layout<kXqEvenOdd16>(bt, xq, packed, a, sms, stream);
        case kXqStride4K16: return launch_layout<kXqStride4K16>(bt, xq, packed, a, sms, stream);
        default: return launch_layout<kXqRowMajor>(bt, xq, packed, a, sms, stream);
    }
}

}  // namespace bl
