// k_gemv_tc.cu -- BitLinear forward for small and middling token counts (decode and small
// batches, up to 128 tokens) on the tcgen05 tensor cores, with K split over a
// thread-block cluster so that a layer with few 128-row tiles still fills the GPU.
//
// What is computed ("What 1.58 Bits Actually Changes", "How the low-bit linear path
// works": +1 adds, -1 subtracts, 0 skips; "1-bit & Ternary LLMs", block "BitNet (Oct
// 2023)": one float rescale at the end):
//   acc[m, n] = sum_k x_q[m, k] * c[n, k],   y[m, n] = acc[m, n] * gamma / s[m].
//
// With few tokens the path is bound by streaming the packed weights: per 128-code stage
// of a 128-row tile, 4 KB of packed codes are expanded into 16 KB of int8 A operand.
// The expansion goes through shared memory in the 128-byte-swizzled K-major layout the
// MMA descriptor reads (as in the prefill kernels); keeping the expanded codes in tensor
// memory instead (tcgen05.st, A operand from TMEM) was built and measured slower here:
// the tensor-memory stores of 16 KB per stage capped the stream near 1.2 TB/s.
//
// Tile: 128 weight rows (MMA M, TMEM lanes) x BT tokens (MMA N; 16 to 128) x a slice of
// K in stages of 128 codes.  Per stage:
//   warp 0 (one lane)   TMA: the x_q tile [BT x 128 B] (128-byte swizzle) per stage,
//                       and the packed weights of eight stages at a time [128 rows x
//                       256 B] into a two-slot ring with its own mbarriers;
//   warps 2-17          expanders, two groups of eight warps taking alternate stages: two
//                       threads per weight row, each unpacking 64 codes in the order of
//                       the x_q layout into the swizzled A tile; fence.proxy.async, then
//                       one lane per warp arrives;
//   warp 1 (one lane)   MMA issuer: four tcgen05.mma kind::i8 (K = 32) per stage into the
//                       TMEM accumulator; tcgen05.commit frees the stage.
// After the last stage the expander warps read the int32 accumulator back (one weight
// row per thread).  When rows are few, K is split over the blocks of a cluster: each
// block writes its partial sums to its shared memory and the blocks add them through
// distributed shared memory, each finishing a share of the tokens.  Integer sums are
// exact, so the split changes nothing.  Rows and tokens past the edges read the TMA's
// zero fill and are not stored.  Every wait is bounded; a block that gives up drains its
// copies and MMAs, sets BL_ERRBIT_TIMEOUT and still takes part in the cluster barriers,
// so no block waits forever.
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

constexpr int kRows = 128;       // weight rows per tile (MMA M)
constexpr int kBK = 128;         // K codes per stage
constexpr int kABytes = kRows * kBK;        // expanded weights per stage: 16 KB
// The packed weights come in super-tiles of 8 stages: 128 rows x 256 bytes per TMA box,
// so every row is read in 256-byte runs (a 32-byte box per row and stage reads DRAM in
// short scattered pieces), into a ring of two slots.
constexpr int kSuper = 8;
constexpr int kPSBytes = kRows * (kSuper * kBK / 4);  // 32 KB
constexpr int kPS = 2;
constexpr int kThreads = 576;    // 18 warps
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpExp = 2;
constexpr int kExpGroups = 2;    // expander groups of eight warps, alternate stages
constexpr int kMaxCluster = 8;
constexpr unsigned long long kDrainNs = 200000000ull;  // 0.2 s

template <int BT>
struct GvCfg {
    static_assert(BT % 16 == 0 && BT >= 16 && BT <= 128, "token tile");
    static constexpr int kXBytes = BT * kBK;
    static constexpr int kStageBytes = kXBytes + kABytes;
    static constexpr int kStagesRaw = (200 * 1024 - kPS * kPSBytes) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kTmemCols = BT <= 32 ? 32 : BT;  // the accumulator (a power of two >= 32)
    static constexpr int kRedBytes = BT * kRows * 4;      // partial sums, aliasing the stages
    static constexpr int kBarBytes = 8 * (3 * kStages + 2 * kPS + 2) + 16;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kPS * kPSBytes + kBarBytes;
    static_assert(kStages >= 4, "stages");
    static_assert(BT != 48 && BT != 80 && BT != 96 && BT != 112, "power-of-two token tiles");
    static_assert(kRedBytes <= kStages * kStageBytes + kPS * kPSBytes, "reduction buffer");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct GvArgs {
    const float* s;
    const float* gamma;
    int M, N, K;
    int stages_per_split;  // K stages of each block of a cluster (the last one takes the rest)
    int nstages;           // K stages in all
    void* out;
    int kind;
    int32_t* err;
    S4Mul mul;
    int grow;              // gamma holds one scale per output row
    unsigned long long wait_ns;  // limit of every wait (2 s outside the bounded-wait test)
    int stall_after;             // the producer stops after this many loads (< 0: never)
};

__device__ __forceinline__ void store_out(void* out, int kind, int64_t idx, int acc, float fac) {
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

__device__ __forceinline__ uint32_t ld_shared_cluster_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// grid: x = the K split (the blocks of one cluster), y = 128-row weight tiles, z = token
// tiles of BT.
template <int BT, int LAY>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_p,
                   const GvArgs a) {
    using C = GvCfg<BT>;
    constexpr int ST = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t sX = base;  // swizzled tiles first: 1024-aligned
    const uint32_t sA = sX + ST * C::kXBytes;
    const uint32_t sP = sA + ST * kABytes;
    const uint32_t sBar = sP + kPS * kPSBytes;
    auto full = [&](int s) { return sBar + 8u * s; };                // x tile landed
    auto afull = [&](int s) { return sBar + 8u * (ST + s); };        // A tile expanded
    auto empty = [&](int s) { return sBar + 8u * (2 * ST + s); };    // stage read by the MMA
    auto pfull = [&](int p) { return sBar + 8u * (3 * ST + p); };    // packed super-tile landed
    auto pempty = [&](int p) { return sBar + 8u * (3 * ST + kPS + p); };  // super-tile expanded
    const uint32_t done_bar = sBar + 8u * (3 * ST + 2 * kPS);
    const uint32_t drain_bar = sBar + 8u * (3 * ST + 2 * kPS + 1);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + (sBar - base) + 8 * (3 * ST + 2 * kPS + 2));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* red = reinterpret_cast<int*>(gbase);  // [BT][128] partial sums, after the main loop

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, nsplit = gridDim.x;
    const int n0 = blockIdx.y * kRows;
    const int t0 = blockIdx.z * BT;
    const int kt_begin = split * a.stages_per_split;
    const int kt_end = split + 1 == nsplit ? a.nstages : kt_begin + a.stages_per_split;
    const int nk = kt_end - kt_begin;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(full(s), 1);
            mbar_init(afull(s), 8);
            mbar_init(empty(s), 1);
        }
        for (int p = 0; p < kPS; ++p) {
            mbar_init(pfull(p), 1);
            mbar_init(pempty(p), 8 * kExpGroups);
        }
        mbar_init(done_bar, 1);
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

    if (warp == kWarpTma) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer --
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0, issued_p = 0;
            bool ok = true;
            for (int i = 0; i < nk; ++i) {
                const int kt = kt_begin + i;
                if (i % kSuper == 0) {  // the next packed super-tile
                    const int j = i / kSuper, p = j % kPS;
                    if (!mbar_wait_bounded(pempty(p), static_cast<uint32_t>(((j / kPS) & 1) ^ 1), abort_flag,
                                           a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(pfull(p), kPSBytes);
                    tma_load_2d(sP + p * kPSBytes, &tmap_p, pfull(p), kt * (kBK / 4), n0);
                    ++issued_p;
                }
                if (!mbar_wait_bounded(empty(stage), phase ^ 1u, abort_flag, a.wait_ns)) {
                    ok = false;
                    break;
                }
                if (issued == a.stall_after) {  // the bounded-wait test: stop issuing
                    stall_until_abort(abort_flag, 4 * a.wait_ns);
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(full(stage), C::kXBytes);
                tma_load_2d(sX + stage * C::kXBytes, &tmap_x, full(stage), kt * kBK, t0);
                ++issued;
                if (++stage == ST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) {
                // wait for every load still in flight before the block may go on
                for (int q = 0; q < ST; ++q) {
                    const long long fills = (issued - q + ST - 1) / ST;
                    if (fills > 0) drain_wait(full(q), static_cast<uint32_t>((fills - 1) & 1));
                }
                for (int q = 0; q < kPS; ++q) {
                    const long long fills = (issued_p - q + kPS - 1) / kPS;
                    if (fills > 0) drain_wait(pfull(q), static_cast<uint32_t>((fills - 1) & 1));
                }
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer --
            constexpr uint32_t idesc = idesc_i8(kRows, BT);
            const uint32_t d_tmem = tmem_base;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int i = 0; i < nk; ++i) {
                if (!mbar_wait_bounded(full(stage), phase, abort_flag, a.wait_ns) ||
                    !mbar_wait_bounded(afull(stage), phase, abort_flag, a.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = sA + stage * kABytes;
                const uint32_t b_addr = sX + stage * C::kXBytes;
#pragma unroll
                for (int kk = 0; kk < kBK / 32; ++kk)
                    tc_mma_i8(d_tmem, smem_desc_sw128(a_addr + 32 * kk), smem_desc_sw128(b_addr + 32 * kk), idesc,
                              (i | kk) != 0 ? 1u : 0u);
                tc_commit(empty(stage));
                if (++stage == ST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            // the accumulator is complete (or, after an abort, no MMA is in flight) when
            // this arrives
            tc_commit(ok ? done_bar : drain_bar);
            if (!ok) {
                drain_wait(drain_bar, 0);
                mbar_arrive(done_bar);  // let the expander warps leave their wait
            }
        }
    } else {
        // ------------------------------------------------------------- expanders --
        // Group g (eight warps) expands the stages of iterations g, g + 2, ...: thread e
        // of the group owns half `half` (64 codes, 16 packed bytes) of weight row `erow`;
        // neighbouring lanes read neighbouring 16-byte pieces and write neighbouring
        // swizzled chunks, free of bank conflicts.
        const int grp = (warp - kWarpExp) >> 3;
        const int e = threadIdx.x - 32 * kWarpExp - 256 * grp;  // 0 .. 255
        const int erow = e >> 1, half = e & 1;
        const uint32_t sw = static_cast<uint32_t>(erow & 7);
        for (int i = grp; i < nk; i += kExpGroups) {
            const int stage = i % ST;
            const uint32_t phase = static_cast<uint32_t>((i / ST) & 1);
            const int j = i / kSuper, pslot = j % kPS;
            // the packed super-tile has landed, and the MMA is done with this stage's A tile
            if (!mbar_wait_bounded(pfull(pslot), static_cast<uint32_t>((j / kPS) & 1), abort_flag, a.wait_ns) ||
                !mbar_wait_bounded(empty(stage), phase ^ 1u, abort_flag, a.wait_ns))
                break;
            const uint8_t* pp = gbase + (sP - base) + pslot * kPSBytes + erow * (kSuper * kBK / 4) +
                                (i % kSuper) * (kBK / 4) + 16 * half;
            uint8_t* ap = gbase + (sA - base) + stage * kABytes + erow * kBK;
            // a debugging build checks that the piece read and the row written lie in the
            // launch's shared memory
            const uint32_t dyn = dynamic_smem_bytes();
            const bool ok_p = bl_check(pp + 16 <= smem_raw + dyn, a.err);
            const bool ok_a = bl_check(ap + kBK <= smem_raw + dyn, a.err);
            const uint4 p = ok_p ? *reinterpret_cast<const uint4*>(pp) : make_uint4(0, 0, 0, 0);
            const uint32_t words[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                // 16 codes -> 16 int8 in the order of the x_q layout (natural, even/odd,
                // or stride-4 as 64 * code)
                uint4 u;
                if constexpr (LAY == kXqEvenOdd16)
                    unpack16_evenodd(words[c], u.x, u.y, u.z, u.w);
                else if constexpr (LAY == kXqStride4K16)
                    unpack16_stride4_x64(words[c], a.mul, u.x, u.y, u.z, u.w);
                else
                    unpack16_natural(words[c], u.x, u.y, u.z, u.w);
                const uint32_t chunk = static_cast<uint32_t>(4 * half + c);
                if (ok_a) *reinterpret_cast<uint4*>(ap + ((chunk ^ sw) << 4)) = u;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(afull(stage));
                // the group's last stage of this super-tile frees the slot
                if (i + kExpGroups >= (j + 1) * kSuper || i + kExpGroups >= nk) mbar_arrive(pempty(pslot));
            }
        }
        // ------------------------------------------------------------- epilogue --
        // the four warps of a lane quarter read 16-token column chunks in turn; thread:
        // weight row r of the tile (its TMEM lane)
        constexpr int kAccShift = LAY == kXqStride4K16 ? 6 : 0;
        const int q = warp & 3, eg = (warp - kWarpExp) >> 2;  // lane quarter, its warp index 0..3
        const int r = 32 * q + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
        const bool got = mbar_wait_bounded(done_bar, 0, abort_flag, a.wait_ns);
        tc_fence_after();
        const int row = n0 + r;
        const float gamma = (a.kind == kOutI32) ? 0.0f : *a.gamma;
        const float grow_gamma = (a.grow && a.kind != kOutI32 && row < a.N) ? __ldg(a.gamma + row) : 0.0f;
#pragma unroll 1
        for (int c0 = 16 * eg; c0 < BT; c0 += 64) {
            uint32_t acc[16];
            tmem_ld_32x32b_x16(tmem_base + lane_addr + static_cast<uint32_t>(c0), acc);
            tmem_ld_wait();
            if (!got) continue;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int v = static_cast<int>(acc[j]) >> kAccShift;
                if (nsplit > 1) {
                    if (bl_check((c0 + j) * kRows + r < BT * kRows, a.err)) red[(c0 + j) * kRows + r] = v;
                } else {
                    const int tok = t0 + c0 + j;
                    if (tok < a.M && row < a.N) {
                        const float sv = a.kind == kOutI32 ? 1.0f : __ldg(a.s + tok);
                        const float fac = a.kind == kOutI32 ? 0.0f : __fdiv_rn(a.grow ? grow_gamma : gamma, sv);
                        store_out(a.out, a.kind, static_cast<int64_t>(tok) * a.N + row, v, fac);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (nsplit > 1) {
        // every block's partial sums are in its shared memory: each block adds, for the
        // tokens t with t % nsplit == split, the partials of all blocks (fixed order)
        cluster_sync_all();
        const int tid = threadIdx.x;
        const int rr = tid & (kRows - 1);
        const int row = n0 + rr;
        const float gamma = (a.kind == kOutI32 || row >= a.N) ? 0.0f : (a.grow ? __ldg(a.gamma + row) : *a.gamma);
        const uint32_t red_addr = smem_u32(red);
        for (int tt = split + nsplit * (tid / kRows); tid < 2 * kRows && tt < BT; tt += 2 * nsplit) {
            const int tok = t0 + tt;
            if (tok >= a.M || row >= a.N) continue;
            int sum = 0;
            if (!bl_check(tt * kRows + rr < BT * kRows, a.err)) continue;
            for (int b = 0; b < nsplit; ++b)
                sum += static_cast<int>(ld_shared_cluster_u32(mapa_shared(red_addr + 4u * (tt * kRows + rr), b)));
            const float fac = a.kind == kOutI32 ? 0.0f : __fdiv_rn(gamma, __ldg(a.s + tok));
            store_out(a.out, a.kind, static_cast<int64_t>(tok) * a.N + row, sum, fac);
        }
        // no block leaves while another may still read its shared memory
        cluster_sync_all();
    }
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
    if (threadIdx.x == 0 && *abort_flag && a.err != nullptr) atomicOr(a.err, kErrBitTimeout);
}

int sm_count_gtc() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <int BT, int LAY>
cudaError_t launch_bt(const CUtensorMap& tx, const CUtensorMap& tp, const GvArgs& a, dim3 grid, cudaStream_t stream) {
    using C = GvCfg<BT>;
    static PerContextOnce attr;
    cudaError_t e = attr.run([] {
        return cudaFuncSetAttribute(gemv_tc_kernel<BT, LAY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    return launch_pdl(gemv_tc_kernel<BT, LAY>, grid, dim3(kThreads), C::kSmemBytes, stream,
                      grid.x > 1 ? dim3(grid.x, 1, 1) : dim3(kNoCluster), tx, tp, a);
}

template <int LAY>
cudaError_t launch_layout(int bt, const CUtensorMap& tx, const CUtensorMap& tp, const GvArgs& a, dim3 grid,
                          cudaStream_t stream) {
    switch (bt) {
        case 16: return launch_bt<16, LAY>(tx, tp, a, grid, stream);
        case 32: return launch_bt<32, LAY>(tx, tp, a, grid, stream);
        case 64: return launch_bt<64, LAY>(tx, tp, a, grid, stream);
        default: return launch_bt<128, LAY>(tx, tp, a, grid, stream);
    }
}

}  // namespace

// Token tile for M tokens: the smallest of 16, 32, 64, 128 that holds them (M > 128 runs
// several token tiles, each streaming the weights again).
int gemv_tc_token_tile(int64_t M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

cudaError_t launch_gemv_tc(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma, int64_t M,
                           int64_t N, int64_t K, void* out, int kind, int32_t* err, int layout, cudaStream_t stream) {
    const int bt = gemv_tc_token_tile(M);
    const int sms = sm_count_gtc();
    const int64_t row_tiles = (N + kRows - 1) / kRows;
    const int64_t tok_tiles = (M + bt - 1) / bt;
    const int nstages = static_cast<int>((K + kBK - 1) / kBK);
    // split K over a cluster of up to 8 blocks (one block per SM): the split with the
    // fewest waves x (stages per block + a block's fixed cost, about 16 stages: start,
    // pipeline fill and the reduction), at least two stages per block (ties: fewer blocks)
    const int64_t tiles = row_tiles * tok_tiles;
    int64_t split = 1, best = -1;
    for (int64_t sp = 1; sp <= kMaxCluster && (sp == 1 || sp <= nstages / 2); ++sp) {
        const int64_t waves = (tiles * sp + sms - 1) / sms;
        const int64_t per = nstages - (sp - 1) * (nstages / sp);  // the last block's stages
        const int64_t cost = waves * (per + 16);
        if (best < 0 || cost < best) {
            best = cost;
            split = sp;
        }
    }
    // blocks start on packed super-tile boundaries where that keeps the split (a super-tile
    // that runs past a block's K range would load bytes the block never reads)
    int64_t sps = (nstages + split - 1) / split;
    if (sps >= kSuper) sps = (sps + kSuper - 1) / kSuper * kSuper;
    split = (nstages + sps - 1) / sps;
    if (row_tiles > 65535 || tok_tiles > 65535) return cudaErrorInvalidValue;
    CUtensorMap tx, tp;
    if (!encode_tmap_u8_2d(&tx, xq, static_cast<uint64_t>(K), static_cast<uint64_t>(M), kBK, bt, true) ||
        !encode_tmap_u8_2d(&tp, packed, static_cast<uint64_t>(K / 4), static_cast<uint64_t>(N), kSuper * kBK / 4,
                           kRows, false))
        return cudaErrorInvalidValue;
    const WaitTest wt = wait_test();
    GvArgs a{s, gamma, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
             static_cast<int>(sps), nstages, out, out_kind_of(kind), err, s4_mul(), gamma_rows_of(kind),
             wt.wait_ns, wt.stall_after};
    const dim3 grid(static_cast<unsigned>(split), static_cast<unsigned>(row_tiles), static_cast<unsigned>(tok_tiles));
    switch (layout) {
        case kXqEvenOdd16: return launch_layout<kXqEvenOdd16>(bt, tx, tp, a, grid, stream);
        case kXqStride4K16: return launch_layout<kXqStride4K16>(bt, tx, tp, a, grid, stream);
        default: return launch_layout<kXqRowMajor>(bt, tx, tp, a, grid, stream);
    }
}

}  // namespace bl
