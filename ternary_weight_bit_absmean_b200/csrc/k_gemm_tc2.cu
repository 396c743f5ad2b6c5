// k_gemm_tc2.cu -- prefill-regime BitLinear forward on a pair of SMs
// (tcgen05.mma.cta_group::2 kind::i8, int32 accumulators in tensor memory).
//
// Same arithmetic as k_gemm_tc.cu ("1-bit & Ternary LLMs (BitNet b1.58)", block
// "BitNet (Oct 2023)": an integer product and one float rescale; "1.58 bits: what BitNet
// promised and what it required", "What you get on today's hardware": on GPUs the
// packed weights are unpacked and then multiplied):
//   acc[m, n] = sum_k x_q[m, k] * c[n, k],   y[m, n] = acc[m, n] * gamma / s[m].
//
// A cluster of two CTAs computes a 256-token x 256-feature tile with one pair MMA per 32
// K bytes (M = 256 tokens, N = 256 features).  CTA r holds tokens [128 r, 128 r + 128)
// of the tile (its half of A) and expands features [128 r, 128 r + 128) (its half of B);
// the tensor cores of the pair exchange the B halves, so each SM loads half the
// activation bytes and expands half the weight codes a single-SM 256 x 256 tile would
// need.  The accumulator of CTA r holds its 128 tokens x all 256 features, one token per
// TMEM lane: an epilogue thread owns one token, computes gamma / s once per tile and
// writes 32 consecutive outputs per TMEM load as 16-byte stores.
//
// Roles per CTA (22 warps): warp 0 lane 0 issues the TMA loads (its x half, signalled on
// the even CTA's barrier; its packed rows, signalled locally); warps 2-17 expand the
// packed rows (four threads per row, natural code order, 128-byte-swizzled K-major) and
// arrive on the even CTA's barrier; warp 1 lane 0 of the even CTA issues the pair MMAs
// and multicasts the commits to both CTAs; warps 18-21 run the epilogue and arrive on
// the even CTA's accumulator-free barrier.  Two 256-column TMEM accumulators overlap the
// epilogue of one tile with the main loop of the next.  All waits are bounded as in
// k_gemm_tc.cu.  No load uses multicast.
#include <cuda_bf16.h>
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {
namespace {

constexpr int kTok = 128;                 // tokens per CTA (pair MMA M = 256)
constexpr int kFeat = 128;                // feature rows expanded per CTA (pair MMA N = 256)
constexpr int kBK = 128;                  // K bytes per stage
constexpr int kThreads = 704;             // 22 warps
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpExp = 2, kWarpEpi = 18;
constexpr int kExpWarps = kWarpEpi - kWarpExp;  // 16: four threads per packed row
constexpr int kEpiWarps = 4;              // one per TMEM lane quarter
constexpr int kXBytes = kTok * kBK;       // 16 KB
constexpr int kBBytes = kFeat * kBK;      // 16 KB
constexpr int kPBytes = kFeat * (kBK / 4);  // 4 KB
constexpr int kStageBytes = kXBytes + kBBytes + kPBytes;
constexpr int kStages = 6;
constexpr int kTmemCols = 512;            // two accumulators of 256 columns
constexpr int kBarCount = 5 * kStages + 5;
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 8 * kBarCount + 16;
constexpr unsigned long long kDrainTimeoutNs = 200000000ull;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

struct Tc2Args {
    const float* s;
    const float* gamma;
    int M, N, K;
    int n_tiles_n, num_tiles;
    void* out;
    int kind;
    int32_t* err;
    S4Mul mul;
    int grow;  // gamma holds one scale per output row
};

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait_cluster(bar, parity)) {
        if (globaltimer_ns() - t0 > kDrainTimeoutNs) return;
    }
}

// 32 accumulators of one token (features f .. f+31) -> y, 16-byte stores when the row
// segment is aligned and inside N, element stores otherwise.
__device__ __forceinline__ void store_row32(void* out, int kind, int64_t row_off, int f, int N,
                                            const uint32_t (&r)[32], float fac, bool vec_ok) {
    if (vec_ok && f + 32 <= N) {
        if (kind == kOutBF16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + row_off + f);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                uint32_t w[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float lo = __fmul_rn(__int2float_rn(static_cast<int>(r[8 * v + 2 * h])), fac);
                    const float hi = __fmul_rn(__int2float_rn(static_cast<int>(r[8 * v + 2 * h + 1])), fac);
                    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
                    w[h] = *reinterpret_cast<const uint32_t*>(&p);
                }
                dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
            }
        } else if (kind == kOutF32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + row_off + f);
#pragma unroll
            for (int v = 0; v < 8; ++v)
                dst[v] = make_float4(__fmul_rn(__int2float_rn(static_cast<int>(r[4 * v])), fac),
                                     __fmul_rn(__int2float_rn(static_cast<int>(r[4 * v + 1])), fac),
                                     __fmul_rn(__int2float_rn(static_cast<int>(r[4 * v + 2])), fac),
                                     __fmul_rn(__int2float_rn(static_cast<int>(r[4 * v + 3])), fac));
        } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<int*>(out) + row_off + f);
#pragma unroll
            for (int v = 0; v < 8; ++v) dst[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
        }
        return;
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        if (f + j >= N) break;
        const int acc = static_cast<int>(r[j]);
        if (kind == kOutI32) {
            static_cast<int*>(out)[row_off + f + j] = acc;
        } else {
            const float y = __fmul_rn(__int2float_rn(acc), fac);
            if (kind == kOutF32)
                static_cast<float*>(out)[row_off + f + j] = y;
            else
                static_cast<__nv_bfloat16*>(out)[row_off + f + j] = __float2bfloat16_rn(y);
        }
    }
}

template <int LAY>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_p,
                    const Tc2Args a) {
    constexpr int ST = kStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t sX = base;
    const uint32_t sB = sX + ST * kXBytes;
    const uint32_t sP = sB + ST * kBBytes;
    const uint32_t sBar = sP + ST * kPBytes;
    auto xfull = [&](int s) { return sBar + 8u * s; };               // even CTA: x halves of both CTAs
    auto pfull = [&](int s) { return sBar + 8u * (ST + s); };        // local: packed rows
    auto bfull = [&](int s) { return sBar + 8u * (2 * ST + s); };    // even CTA: expanded B of both
    auto empty = [&](int s) { return sBar + 8u * (3 * ST + s); };    // local: stage free (MMA done)
    auto tfull = [&](int b) { return sBar + 8u * (4 * ST + b); };    // local: accumulator ready
    auto tempty = [&](int b) { return sBar + 8u * (4 * ST + 2 + b); };  // even CTA: accumulator read
    const uint32_t drain_bar = sBar + 8u * (4 * ST + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + (sBar - base) + 8 * kBarCount);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster_id = blockIdx.x >> 1;
    const int num_clusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(xfull(s), 1);
            mbar_init(pfull(s), 1);
            mbar_init(bfull(s), 2 * kExpWarps);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull(b), 1);
            mbar_init(tempty(b), 2 * kEpiWarps);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        mbar_fence_init();
        tma_prefetch_desc(&tmap_x);
        tma_prefetch_desc(&tmap_p);
    }
    pdl_wait_then_release();
    if (warp == kWarpMma) {
        tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers exist before either signals the other
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
            for (int tile = cluster_id; ok && tile < a.num_tiles; tile += num_clusters) {
                const int n0 = (tile % a.n_tiles_n) * (2 * kFeat);
                const int t0 = (tile / a.n_tiles_n) * (2 * kTok);
                for (int kt = 0; kt < nK; ++kt) {
                    if (!mbar_wait_cluster_bounded(empty(stage), phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (leader) mbar_arrive_expect_tx(xfull(stage), 2 * kXBytes);
                    tma_load_2d_pair(sX + stage * kXBytes, &tmap_x, mapa_shared(xfull(stage), 0), kt * kBK,
                                     t0 + kTok * static_cast<int>(rank));
                    mbar_arrive_expect_tx(pfull(stage), kPBytes);
                    tma_load_2d(sP + stage * kPBytes, &tmap_p, pfull(stage), kt * (kBK / 4),
                                n0 + kFeat * static_cast<int>(rank));
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
                    if (fills > 0) {
                        drain_wait(pfull(s), static_cast<uint32_t>((fills - 1) & 1));
                        if (leader) drain_wait(xfull(s), static_cast<uint32_t>((fills - 1) & 1));
                    }
                }
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0 && leader) {
            // ---------------------------------------------------------- MMA issuer --
            constexpr uint32_t idesc = idesc_i8(2 * kTok, 2 * kFeat);
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            bool ok = true;
            for (int tile = cluster_id; ok && tile < a.num_tiles; tile += num_clusters) {
                if (!mbar_wait_cluster_bounded(tempty(buf), bphase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * 2 * kFeat);
                for (int kt = 0; kt < nK; ++kt) {
                    if (!mbar_wait_cluster_bounded(xfull(stage), phase, abort_flag) ||
                        !mbar_wait_cluster_bounded(bfull(stage), phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = sX + stage * kXBytes;
                    const uint32_t b_addr = sB + stage * kBBytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 32; ++kk)
                        tc_mma_i8_pair(d_tmem, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32),
                                       idesc, (kt | kk) != 0 ? 1u : 0u);
                    tc_commit_pair_multicast(empty(stage), 0x3);
                    if (++stage == ST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit_pair_multicast(tfull(buf), 0x3);
                if (++buf == 2) {
                    buf = 0;
                    bphase ^= 1u;
                }
            }
            if (!ok) {
                tc_commit_pair_multicast(drain_bar, 0x1);
                drain_wait(drain_bar, 0);
            }
        }
    } else if (warp < kWarpEpi) {
        // ------------------------------------------------------------- expanders --
        // thread e owns quarter `part` (32 codes = 8 packed bytes) of weight row `row`
        const int e = threadIdx.x - 32 * kWarpExp;
        const int row = e >> 2, part = e & 3;
        const uint32_t sw = static_cast<uint32_t>(row & 7);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = cluster_id; ok && tile < a.num_tiles; tile += num_clusters) {
            for (int kt = 0; kt < nK; ++kt) {
                if (!mbar_wait_cluster_bounded(pfull(stage), phase, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint8_t* pp = gbase + (sP - base) + stage * kPBytes + row * (kBK / 4) + part * 8;
                const uint2 p0 = *reinterpret_cast<const uint2*>(pp);
                uint8_t* bp = gbase + (sB - base) + stage * kBBytes + row * kBK;
                const uint32_t words[2] = {p0.x, p0.y};
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    // natural order, or the even/odd or stride-4 k16 order of the x_q
                    // layout (the last as 64 * code)
                    uint4 u;
                    if constexpr (LAY == kXqEvenOdd16)
                        unpack16_evenodd(words[c], u.x, u.y, u.z, u.w);
                    else if constexpr (LAY == kXqStride4K16)
                        unpack16_stride4_x64(words[c], a.mul, u.x, u.y, u.z, u.w);
                    else
                        unpack16_natural(words[c], u.x, u.y, u.z, u.w);
                    const uint32_t chunk = static_cast<uint32_t>(2 * part + c);
                    *reinterpret_cast<uint4*>(bp + ((chunk ^ sw) << 4)) = u;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(bfull(stage), 0));
                if (++stage == ST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // -------------------------------------------------------------- epilogue --
        const int q = warp & 3;
        const int first = 32 * ((warp - kWarpEpi) >> 2);  // this warp's first column chunk
        constexpr int kChunkStep = 32 * (kEpiWarps / 4);
        const float gamma = (a.kind == kOutI32) ? 0.0f : *a.gamma;
        const bool vec_ok = (a.kind == kOutBF16) ? (a.N % 8 == 0) : (a.N % 4 == 0);
        int buf = 0;
        uint32_t bphase = 0;
        for (int tile = cluster_id; tile < a.num_tiles; tile += num_clusters) {
            const int n0 = (tile % a.n_tiles_n) * (2 * kFeat);
            const int t0 = (tile / a.n_tiles_n) * (2 * kTok);
            const int tok = t0 + kTok * static_cast<int>(rank) + 32 * q + lane;
            const bool tok_ok = tok < a.M;
            const float fac = (a.kind != kOutI32 && tok_ok) ? __fdiv_rn(gamma, __ldg(a.s + tok)) : 0.0f;
            if (!mbar_wait_cluster_bounded(tfull(buf), bphase, abort_flag)) break;
            tc_fence_after();
            const int64_t row_off = static_cast<int64_t>(tok) * a.N;
#pragma unroll 1
            for (int c0 = first; c0 < 2 * kFeat; c0 += kChunkStep) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                                       static_cast<uint32_t>(buf * 2 * kFeat + c0),
                                   r);
                tmem_ld_wait();
                if constexpr (LAY == kXqStride4K16) {
                    // the stride-4 unpack feeds 64 * code: the sums are exact multiples of 64
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = static_cast<uint32_t>(static_cast<int>(r[j]) >> 6);
                }
                if (!tok_ok || n0 + c0 >= a.N) {
                    // nothing of this chunk to store for this lane
                } else if (a.grow && a.kind != kOutI32) {
                    // one scale per output row: y = acc * (gamma_f / s), element stores
                    const float st = __ldg(a.s + tok);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int f = n0 + c0 + j;
                        if (f >= a.N) break;
                        const float y = __fmul_rn(__int2float_rn(static_cast<int>(r[j])), __fdiv_rn(__ldg(a.gamma + f), st));
                        if (a.kind == kOutF32)
                            static_cast<float*>(a.out)[row_off + f] = y;
                        else
                            static_cast<__nv_bfloat16*>(a.out)[row_off + f] = __float2bfloat16_rn(y);
                    }
                } else {
                    store_row32(a.out, a.kind, row_off, n0 + c0, a.N, r, fac, vec_ok);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty(buf), 0));
            if (++buf == 2) {
                buf = 0;
                bphase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // no CTA leaves while its peer may still signal its barriers
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
    if (threadIdx.x == 0 && *abort_flag && a.err != nullptr) atomicOr(a.err, kErrBitTimeout);
}

}  // namespace

bool encode_tmap_u8_2d(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                       uint32_t box_outer, bool swizzle128);

int gemm_tc2_clusters(int64_t M, int64_t N, int sms) {
    const int64_t tiles = ((N + 255) / 256) * ((M + 255) / 256);
    const int64_t pairs = sms / 2;
    return static_cast<int>(tiles < pairs ? tiles : pairs);
}

template <int LAY>
static cudaError_t launch_tc2_layout(const CUtensorMap& tx, const CUtensorMap& tp, const Tc2Args& a, int clusters,
                                 cudaStream_t stream) {
    static PerContextOnce attr;
    cudaError_t e = attr.run([] {
        return cudaFuncSetAttribute(gemm_tc2_kernel<LAY>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    return launch_pdl(gemm_tc2_kernel<LAY>, dim3(static_cast<unsigned>(2 * clusters)), dim3(kThreads), kSmemBytes,
                      stream, dim3(2, 1, 1), tx, tp, a);
}

cudaError_t launch_gemm_tc2(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                            int64_t M, int64_t N, int64_t K, void* out, int kind, int32_t* err, int layout,
                            cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    CUtensorMap tx, tp;
    if (!encode_tmap_u8_2d(&tx, xq, static_cast<uint64_t>(K), static_cast<uint64_t>(M), kBK, kTok, true) ||
        !encode_tmap_u8_2d(&tp, packed, static_cast<uint64_t>(K / 4), static_cast<uint64_t>(N), kBK / 4, kFeat,
                           false))
        return cudaErrorInvalidValue;
    Tc2Args a{s, gamma, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
              static_cast<int>((N + 255) / 256), static_cast<int>(((N + 255) / 256) * ((M + 255) / 256)),
              out, out_kind_of(kind), err, s4_mul(), gamma_rows_of(kind)};
    const int clusters = gemm_tc2_clusters(M, N, sms);
    switch (layout) {
        case kXqEvenOdd16: return launch_tc2_layout<kXqEvenOdd16>(tx, tp, a, clusters, stream);
        case kXqStride4K16: return launch_tc2_layout<kXqStride4K16>(tx, tp, a, clusters, stream);
        default: return launch_tc2_layout<kXqRowMajor>(tx, tp, a, clusters, stream);
    }
}

}  // namespace bl
