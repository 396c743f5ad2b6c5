// k_gemm_tc.cu -- prefill-regime BitLinear forward on the 5th-generation tensor cores
// (tcgen05.mma kind::i8, int32 accumulators in tensor memory).
//
// What is computed ("1-bit & Ternary LLMs (BitNet b1.58)", block "BitNet (Oct 2023)":
// y = W~ . Quant(x) . scale, an integer product and one float rescale; block
// "BitNet b1.58 (Feb 2024)": W~ in {-1, 0, +1}; "1.58 bits: what BitNet promised and what
// it required", "What you get on today's hardware": on GPUs the packed weights are
// unpacked and then multiplied):
//   acc[m, n] = sum_k x_q[m, k] * c[n, k]   (int32, exact)
//   y[m, n]   = acc[m, n] * gamma / s[m]
//
// Tile: 128 output features (MMA M, TMEM lanes) x BT tokens (MMA N, TMEM columns), K in
// stages of 128 bytes.  The weights are the A operand so that the expansion work per
// MMA is 128 x 32 codes whatever the token tile, and each expanded code is reused by BT
// tokens.  Per stage:
//   warp 0 (one lane)  TMA: x_q tile [BT x 128 B] (128-byte swizzle) and the packed
//                      weight tile [128 x 32 B] into shared memory, one mbarrier;
//   warps 2-9          expanders: two threads per packed row, each unpacking 64 codes
//                      into int8 and writing them in the same 128-byte-swizzled K-major
//                      layout (two expander warps per SM sub-partition keep the
//                      unpack off the critical path of a stage);
//   warp 1 (one lane)  MMA issuer: four tcgen05.mma (K = 32 each) per stage into a TMEM
//                      accumulator, tcgen05.commit frees the stage;
//   warps 10-17        epilogue: tcgen05.ld of the finished accumulator (one feature row
//                      per thread, two warps per lane quarter taking alternate 32-column
//                      chunks), y = acc * (gamma / s_m), coalesced stores along N.
// Two TMEM accumulators let the epilogue of one tile overlap the main loop of the next
// (persistent blocks, one per SM, static round-robin over tiles).  Ragged M, N and K
// edges come from TMA zero fill: a zero packed byte is four zero codes.
//
// Every wait is bounded: a role that waits longer than kWaitTimeoutNs raises an abort
// flag, the other roles leave their loops, outstanding TMA loads and MMAs are drained,
// TMEM is freed and BL_ERRBIT_TIMEOUT is OR-ed into the caller's error word.
#include <cuda_bf16.h>
#include <cstdint>
#include <mutex>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {
namespace {

constexpr int kBN = 128;          // output features per tile (MMA M)
constexpr int kBK = 128;          // K bytes per stage (one 128-byte swizzle row)
constexpr int kThreads = 576;     // 18 warps
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpExp = 2, kWarpEpi = 10;
constexpr int kExpWarps = kWarpEpi - kWarpExp;
constexpr int kEpiWarps = 8;      // two per TMEM lane quarter, alternating 32-column chunks
constexpr unsigned long long kDrainTimeoutNs = 200000000ull;  // 0.2 s

constexpr int pow2_at_least(int v) { return v <= 32 ? 32 : 2 * pow2_at_least((v + 1) / 2); }

template <int BT>
struct TcCfg {
    // the epilogue reads the accumulator in 32-column chunks
    static_assert(BT % 32 == 0 && BT >= 32 && BT <= 256, "token tile");
    static constexpr int kXBytes = BT * kBK;
    static constexpr int kABytes = kBN * kBK;
    static constexpr int kPBytes = kBN * (kBK / 4);
    static constexpr int kStageBytes = kXBytes + kABytes + kPBytes;
    static constexpr int kStagesRaw = (220 * 1024) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kTmemCols = pow2_at_least(2 * BT);  // TMEM is allocated in powers of two
    static constexpr int kBarBytes = 8 * (3 * kStages + 5) + 16;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBarBytes;
    static_assert(kStages >= 2, "stages");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct TcArgs {
    const float* s;
    const float* gamma;
    int M, N, K;
    int n_tiles_n, num_tiles;
    void* out;
    int kind;
    int32_t* err;
    S4Mul mul;
    int grow;  // gamma holds one scale per output row
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

// Wait for the given phase parity of `bar`, giving up after `limit_ns` regardless of
// the abort flag (used only to drain after an abort).
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kDrainTimeoutNs) return;
    }
}

template <int BT, int LAY>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_p,
                   const TcArgs a) {
    using C = TcCfg<BT>;
    constexpr int ST = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t sX = base;
    const uint32_t sA = sX + ST * C::kXBytes;
    const uint32_t sP = sA + ST * C::kABytes;
    const uint32_t sBar = sP + ST * C::kPBytes;
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
            mbar_init(afull(s), kExpWarps);
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
    const int nK = (a.K + kBK - 1) / kBK;

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
                    mbar_arrive_expect_tx(full(stage), C::kXBytes + C::kPBytes);
                    tma_load_2d(sX + stage * C::kXBytes, &tmap_x, full(stage), kt * kBK, t0);
                    tma_load_2d(sP + stage * C::kPBytes, &tmap_p, full(stage), kt * (kBK / 4), n0);
                    ++issued;
                    if (++stage == ST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // wait for every load still in flight before the block may exit
                for (int s = 0; s < ST; ++s) {
                    const long long fills = (issued - s + ST - 1) / ST;  // loads issued into stage s
                    if (fills > 0) mbar_drain(full(s), static_cast<uint32_t>((fills - 1) & 1));
                }
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer --
            constexpr uint32_t idesc = idesc_i8(kBN, BT);
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x) {
                if (!mbar_wait_bounded(tempty(buf), bphase ^ 1u, abort_flag, a.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BT);
                for (int kt = 0; kt < nK; ++kt) {
                    if (!mbar_wait_bounded(full(stage), phase, abort_flag, a.wait_ns) ||
                        !mbar_wait_bounded(afull(stage), phase, abort_flag, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = sA + stage * C::kABytes;
                    const uint32_t b_addr = sX + stage * C::kXBytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 32; ++kk)
                        tc_mma_i8(d_tmem, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32),
                                  idesc, (kt | kk) != 0 ? 1u : 0u);
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
                mbar_drain(drain_bar, 0);
            }
        }
    } else if (warp < kWarpEpi) {
        // ------------------------------------------------------------- expanders --
        // Thread e owns half `half` (64 codes = 16 packed bytes) of weight row `row`;
        // neighbouring lanes read neighbouring 16-byte pieces, so both the packed reads
        // and the swizzled writes are free of bank conflicts.
        const int e = threadIdx.x - 32 * kWarpExp;  // 0 .. 32 * kExpWarps - 1
        const int row = e >> 1, half = e & 1;
        const uint32_t sw = static_cast<uint32_t>(row & 7);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x) {
            for (int kt = 0; kt < nK; ++kt) {
                if (!mbar_wait_bounded(full(stage), phase, abort_flag, a.wait_ns)) {
                    ok = false;
                    break;
                }
                const uint8_t* pp = gbase + (sP - base) + stage * C::kPBytes + row * (kBK / 4) + half * 16;
                const uint4 p0 = *reinterpret_cast<const uint4*>(pp);
                uint8_t* ap = gbase + (sA - base) + stage * C::kABytes + row * kBK;
                const uint32_t words[4] = {p0.x, p0.y, p0.z, p0.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    // 16 codes -> 16 int8 in the order of the x_q layout: natural, the
                    // even/odd k16 order (codes 0,2,4,6 | 8,..,14 | 1,3,5,7 | 9,..,15) or
                    // the stride-4 k16 order (0,4,8,12 | 1,5,9,13 | ..), the last as
                    // 64 * code
                    uint4 u;
                    if constexpr (LAY == kXqEvenOdd16)
                        unpack16_evenodd(words[c], u.x, u.y, u.z, u.w);
                    else if constexpr (LAY == kXqStride4K16)
                        unpack16_stride4_x64(words[c], a.mul, u.x, u.y, u.z, u.w);
                    else
                        unpack16_natural(words[c], u.x, u.y, u.z, u.w);
                    const uint32_t chunk = static_cast<uint32_t>(4 * half + c);
                    *reinterpret_cast<uint4*>(ap + ((chunk ^ sw) << 4)) = u;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(afull(stage));
                if (++stage == ST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // -------------------------------------------------------------- epilogue --
        // the stride-4 unpack feeds 64 * code: its sums are exact multiples of 64
        constexpr int kAccShift = LAY == kXqStride4K16 ? 6 : 0;
        const int q = warp & 3;                   // TMEM lane quarter this warp may access
        const int first = 32 * ((warp - kWarpEpi) >> 2);  // this warp's first column chunk
        const float gamma = (a.kind == kOutI32) ? 0.0f : *a.gamma;
        int buf = 0;
        uint32_t bphase = 0;
        for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
            const int n0 = (tile % a.n_tiles_n) * kBN;
            const int t0 = (tile / a.n_tiles_n) * BT;
            // s of the first chunk's tokens is fetched before the accumulator is ready;
            // each chunk then fetches the next chunk's while it converts and stores
            float s_next = (a.kind != kOutI32 && t0 + first + lane < a.M) ? __ldg(a.s + t0 + first + lane) : 1.0f;
            if (!mbar_wait_bounded(tfull(buf), bphase, abort_flag, a.wait_ns)) break;
            tc_fence_after();
            const int row = n0 + 32 * q + lane;
            const bool row_ok = row < a.N;
            // with one scale per output row, this thread's row scale
            const float grow_gamma = (a.grow && a.kind != kOutI32 && row_ok) ? __ldg(a.gamma + row) : 0.0f;
#pragma unroll 1
            for (int c0 = first; c0 < BT; c0 += 64) {
                const float s_cur = s_next;
                const float fac = __fdiv_rn(gamma, s_cur);
                const int tk = t0 + c0 + 64 + lane;
                if (c0 + 64 < BT) s_next = (a.kind != kOutI32 && tk < a.M) ? __ldg(a.s + tk) : 1.0f;
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                                       static_cast<uint32_t>(buf * BT + c0),
                                   r);
                tmem_ld_wait();
                if (a.grow) {
                    // one scale per output row: this row's gamma over each token's s
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

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

}  // namespace

// 2-D uint8 tensor map over a row-major [outer, inner] byte matrix with a
// [box_outer, box_inner] box; 128-byte swizzle or none.
namespace {

// Encoded tensor maps of recent calls.  A map is a pure function of the arguments that
// describe it (address, element type, extents, box, swizzle), so a stored copy is valid
// for any later call with the same arguments, whatever the memory holds; repeated calls
// on the same buffers (a decode loop) then skip the driver's encoding.
struct TmapKey {
    const void* ptr;
    uint64_t inner, outer;
    uint32_t box_inner, box_outer, kind;  // kind: element type and swizzle
    bool operator==(const TmapKey& o) const {
        return ptr == o.ptr && inner == o.inner && outer == o.outer && box_inner == o.box_inner &&
               box_outer == o.box_outer && kind == o.kind;
    }
};
constexpr int kTmapCacheSlots = 64;
struct TmapEntry {
    TmapKey key;
    CUtensorMap map;
    bool used;
};
std::mutex g_tmap_mu;
TmapEntry g_tmap_cache[kTmapCacheSlots];

int tmap_slot(const TmapKey& k) {
    uint64_t h = reinterpret_cast<uint64_t>(k.ptr) ^ (k.inner * 0x9E3779B97F4A7C15ull) ^ (k.outer << 17) ^
                 (static_cast<uint64_t>(k.box_inner) << 40) ^ (static_cast<uint64_t>(k.box_outer) << 28) ^ k.kind;
    h ^= h >> 29;
    h *= 0xBF58476D1CE4E5B9ull;
    h ^= h >> 32;
    return static_cast<int>(h % kTmapCacheSlots);
}

// Looks the map up, else encodes it with `encode` and stores it.
template <typename F>
bool cached_tmap(CUtensorMap* map, const TmapKey& key, F encode) {
    const int slot = tmap_slot(key);
    {
        std::lock_guard<std::mutex> lock(g_tmap_mu);
        const TmapEntry& e = g_tmap_cache[slot];
        if (e.used && e.key == key) {
            *map = e.map;
            return true;
        }
    }
    if (!encode(map)) return false;
    std::lock_guard<std::mutex> lock(g_tmap_mu);
    g_tmap_cache[slot] = TmapEntry{key, *map, true};
    return true;
}

}  // namespace

bool encode_tmap_u8_2d(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                       uint32_t box_outer, bool swizzle128) {
    const TmapKey key{ptr, inner, outer, box_inner, box_outer, swizzle128 ? 1u : 0u};
    return cached_tmap(map, key, [&](CUtensorMap* m) {
        PFN_cuTensorMapEncodeTiled_v12000 fn = get_encode_fn();
        if (fn == nullptr) return false;
        const cuuint64_t dims[2] = {inner, outer};
        const cuuint64_t strides[1] = {inner};
        const cuuint32_t box[2] = {box_inner, box_outer};
        const cuuint32_t estr[2] = {1, 1};
        return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    });
}

// 2-D tensor map over a row-major [outer, inner] matrix of 4-byte elements (fp32), no
// swizzle, zero fill outside the matrix.
bool encode_tmap_f32_2d(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                        uint32_t box_outer) {
    const TmapKey key{ptr, inner, outer, box_inner, box_outer, 2u};
    return cached_tmap(map, key, [&](CUtensorMap* m) {
        PFN_cuTensorMapEncodeTiled_v12000 fn = get_encode_fn();
        if (fn == nullptr) return false;
        const cuuint64_t dims[2] = {inner, outer};
        const cuuint64_t strides[1] = {inner * 4};
        const cuuint32_t box[2] = {box_inner, box_outer};
        const cuuint32_t estr[2] = {1, 1};
        return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    });
}

namespace {

template <int BT, int LAY>
cudaError_t launch_bt(const int8_t* xq, const uint8_t* packed, TcArgs a, int sms, cudaStream_t stream) {
    using C = TcCfg<BT>;
    CUtensorMap tx, tp;
    if (!encode_tmap_u8_2d(&tx, xq, static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M), kBK, BT, true) ||
        !encode_tmap_u8_2d(&tp, packed, static_cast<uint64_t>(a.K / 4), static_cast<uint64_t>(a.N), kBK / 4, kBN,
                           false))
        return cudaErrorInvalidValue;
    static PerContextOnce attr;
    cudaError_t e = attr.run([] {
        return cudaFuncSetAttribute(gemm_tc_kernel<BT, LAY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    const int grid = a.num_tiles < sms ? a.num_tiles : sms;
    return launch_pdl(gemm_tc_kernel<BT, LAY>, dim3(grid), dim3(kThreads), C::kSmemBytes, stream, dim3(kNoCluster),
                      tx, tp, a);
}

}  // namespace

template <int LAY>
static cudaError_t launch_bt_layout(int bt, const int8_t* xq, const uint8_t* packed, const TcArgs& a, int sms,
                                   cudaStream_t stream) {
    switch (bt) {
        case 32: return launch_bt<32, LAY>(xq, packed, a, sms, stream);
        case 64: return launch_bt<64, LAY>(xq, packed, a, sms, stream);
        case 96: return launch_bt<96, LAY>(xq, packed, a, sms, stream);
        case 128: return launch_bt<128, LAY>(xq, packed, a, sms, stream);
        case 160: return launch_bt<160, LAY>(xq, packed, a, sms, stream);
        case 192: return launch_bt<192, LAY>(xq, packed, a, sms, stream);
        case 224: return launch_bt<224, LAY>(xq, packed, a, sms, stream);
        default: return launch_bt<256, LAY>(xq, packed, a, sms, stream);
    }
}

// Token tile of the single-SM kernel and its cost (cycles of the busiest SM, up to a
// constant).  A 128-byte K stage's MMAs take ~2.9 BT cycles at the int8 peak, but its
// shared-memory traffic (the activation tile written by TMA and read by the MMA, the
// expanded weights written and read, the packed codes) takes ~320 + 2 BT cycles at 128
// bytes per cycle and dominates; the epilogue of a tile adds ~8 BT cycles that the next
// tile's main loop does not hide (its outputs leave as 2-byte stores).  Among token
// tiles in steps of 32, the one with the fewest waves x tile cycles wins (ties: the
// smaller).
static int tc1_tile(int64_t M, int64_t N, int64_t K, int sms, int64_t* cost) {
    const int64_t nN = (N + kBN - 1) / kBN;
    const int64_t nK = (K + kBK - 1) / kBK;
    int best = 32;
    int64_t best_cost = -1;
    for (int b = 32; b <= 256; b += 32) {
        const int64_t tiles = nN * ((M + b - 1) / b);
        const int64_t waves = (tiles + sms - 1) / sms;
        const int64_t c = waves * (nK * (320 + 2 * b) + 8 * b);
        if (best_cost < 0 || c < best_cost) {
            best_cost = c;
            best = b;
        }
    }
    *cost = best_cost;
    return best;
}

cudaError_t launch_gemm_tc1(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                            int64_t M, int64_t N, int64_t K, void* out, int kind, int32_t* err, int layout,
                            cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t nN = (N + kBN - 1) / kBN;
    int64_t cost = 0;
    const int bt = tc1_tile(M, N, K, sms, &cost);
    const WaitTest wt = wait_test();
    TcArgs a{s, gamma, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), static_cast<int>(nN),
             0, out, out_kind_of(kind), err, s4_mul(), gamma_rows_of(kind), wt.wait_ns, wt.stall_after};
    a.num_tiles = static_cast<int>(nN * ((M + bt - 1) / bt));
    switch (layout) {
        case kXqEvenOdd16: return launch_bt_layout<kXqEvenOdd16>(bt, xq, packed, a, sms, stream);
        case kXqStride4K16: return launch_bt_layout<kXqStride4K16>(bt, xq, packed, a, sms, stream);
        default: return launch_bt_layout<kXqRowMajor>(bt, xq, packed, a, sms, stream);
    }
}

// The pair kernel moves half the activation bytes per SM and stores 16-byte vectors; the
// two kernels are compared with the cost model of tc1_tile.
cudaError_t launch_gemm_tc(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                           int64_t M, int64_t N, int64_t K, void* out, int kind, int32_t* err, int layout,
                           cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t cost1 = 0;
    tc1_tile(M, N, K, sms, &cost1);
    // a pair tile (256 x 256) costs ~918 cycles per stage in the same units, its vector-
    // store epilogue hidden behind the next tile (fitted to the measured times of both
    // kernels on ten prefill shapes, M = 512 to 8192)
    const int64_t tiles2 = ((N + 255) / 256) * ((M + 255) / 256);
    const int64_t pairs = sms / 2;
    const int64_t cost2 = (tiles2 + pairs - 1) / pairs * ((K + kBK - 1) / kBK) * 918;
    if (M > 128 && cost2 <= cost1)
        return launch_gemm_tc2(xq, s, packed, gamma, M, N, K, out, kind, err, layout, stream);
    return launch_gemm_tc1(xq, s, packed, gamma, M, N, K, out, kind, err, layout, stream);
}

}  // namespace bl
