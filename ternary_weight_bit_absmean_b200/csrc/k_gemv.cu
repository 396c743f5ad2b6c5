// k_gemv.cu -- decode-regime BitLinear forward (small M): stream the packed ternary
// weights from HBM once, unpack them in registers, and accumulate exactly in int32.
//
// What is computed ("What 1.58 Bits Actually Changes", "How the low-bit linear path
// works": +1 adds the activation, -1 subtracts it, 0 skips; "1-bit & Ternary LLMs",
// block "BitNet (Oct 2023)": one float rescale at the end):
//   acc[m, n] = sum_k x_q[m, k] * c[n, k],   y[m, n] = acc[m, n] * gamma / s[m].
//
// How: the products of a ternary code and an int8 activation are formed and summed by
// the tensor cores' legacy warp-level int8 MMA (m16n8k32, int32 accumulate), so the
// integer pipes only have to unpack.  Each weight code is unpacked once, into the A
// fragment (16 output rows x 32 K) in registers; the activations of up to 16 tokens are
// the B fragment (8 tokens per MMA).  The unpack writes codes in even/odd order within
// each group of 16 (fewer instructions than natural order); the activations are staged
// in shared memory with the same permutation, so every integer dot product is
// unchanged.
//
// Work split: a block owns 256 output rows (8 warps x 32 rows) and one slice of K.  The
// slices of one row block form a thread-block cluster; their int32 partial sums are
// added through distributed shared memory by the cluster's blocks, each reducing and
// storing a share of the outputs.  Integer sums are exact, so the split changes nothing.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <cuda_runtime.h>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace cg = cooperative_groups;

namespace bl {
namespace {

constexpr int kGvWarps = 8;
constexpr int kGvThreads = 32 * kGvWarps;
constexpr int kGvRows = 32 * kGvWarps;  // output rows per block
constexpr int kChunk = 256;             // K codes per main-loop step (64 packed bytes per row)
constexpr int kWindow = 4096;           // K codes of activations staged in shared memory at once
constexpr int kMaxCluster = 8;

struct GemvArgs {
    const int8_t* xq;
    const float* s;
    const uint8_t* packed;
    const float* gamma;
    int64_t M, N;
    int K;
    int Kc;        // K codes per slice (multiple of kChunk)
    int xs_bytes;  // shared bytes reserved for staged activations (the reduction buffer follows)
    void* out;
    int kind;
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

template <int MT>
__global__ void __launch_bounds__(kGvThreads) gemv_kernel(GemvArgs a) {
    constexpr int MP = 8 * MT;  // tokens per block (padded)
    extern __shared__ __align__(16) uint8_t smem[];
    // xs: for window chunk c, word i (0..3), token m, thread-in-group t: 16 permuted bytes
    // at (((c * 4 + i) * MP + m) * 4 + t) * 16.  red (clusters only): int32 [MP][kGvRows].
    uint8_t* xs = smem;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kGvRows + warp * 32;
    const int k_begin = blockIdx.y * a.Kc;
    const int k_end = min(a.K, k_begin + a.Kc);
    const int64_t m0 = static_cast<int64_t>(blockIdx.z) * MP;
    const int64_t KB = a.K / 4;

    const uint8_t* wrow[4];
    bool wok[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int64_t row = row0 + g + 8 * r;
        wok[r] = row < a.N;
        wrow[r] = a.packed + (wok[r] ? row : 0) * KB;
    }

    int acc[2][MT][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < MT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0;

    for (int kw = k_begin; kw < k_end; kw += kWindow) {
        const int kw_end = min(k_end, kw + kWindow);
        const int nch = (kw_end - kw + kChunk - 1) / kChunk;

        // weights of chunk c of this window for this thread: 64 codes of each of its 4 rows
        auto load_chunk = [&](uint4 (&buf)[4], int c) {
            const int k = kw + c * kChunk + 64 * t;
            const bool ok = c < nch && k < kw_end;
#pragma unroll
            for (int r = 0; r < 4; ++r)
                buf[r] = (ok && wok[r]) ? ldg_stream_v4(wrow[r] + (k >> 2)) : make_uint4(0, 0, 0, 0);
        };
        auto compute_chunk = [&](const uint4 (&buf)[4], int c) {
            if (c >= nch) return;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t e0[4], e1[4], o0[4], o1[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const uint32_t w = i == 0 ? buf[r].x : i == 1 ? buf[r].y : i == 2 ? buf[r].z : buf[r].w;
                    unpack16_evenodd(w, e0[r], e1[r], o0[r], o1[r]);
                }
#pragma unroll
                for (int j = 0; j < MT; ++j) {
                    const uint4 b = *reinterpret_cast<const uint4*>(
                        xs + ((((c * 4 + i) * MP) + 8 * j + g) * 4 + t) * 16);
#pragma unroll
                    for (int tile = 0; tile < 2; ++tile) {
                        mma_m16n8k32_s8(acc[tile][j], e0[2 * tile], e0[2 * tile + 1], o0[2 * tile],
                                        o0[2 * tile + 1], b.x, b.y);
                        mma_m16n8k32_s8(acc[tile][j], e1[2 * tile], e1[2 * tile + 1], o1[2 * tile],
                                        o1[2 * tile + 1], b.z, b.w);
                    }
                }
            }
        };

        uint4 bufA[4], bufB[4], bufC[4];
        load_chunk(bufA, 0);
        load_chunk(bufB, 1);

        // stage this window's activations, permuted to match the even/odd unpack
        __syncthreads();
        const int groups = nch * 16;  // 16-byte groups per token row in the window
        for (int idx = threadIdx.x; idx < groups * MP; idx += kGvThreads) {
            const int m = idx / groups, q = idx % groups;
            const int k = kw + 16 * q;
            const int64_t tok = m0 + m;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (tok < a.M && k < kw_end)
                v = __ldg(reinterpret_cast<const uint4*>(a.xq + tok * a.K + k));
            const int c = q >> 4, tt = (q >> 2) & 3, i = q & 3;
            *reinterpret_cast<uint4*>(xs + ((((c * 4 + i) * MP) + m) * 4 + tt) * 16) =
                permute16_evenodd(v);
        }
        __syncthreads();

        for (int c = 0; c < nch; c += 3) {
            load_chunk(bufC, c + 2);
            compute_chunk(bufA, c);
            load_chunk(bufA, c + 3);
            compute_chunk(bufB, c + 1);
            load_chunk(bufB, c + 4);
            compute_chunk(bufC, c + 2);
        }
    }

    const float gamma = (a.kind == kOutI32) ? 0.0f : *a.gamma;
    if (gridDim.y == 1) {
        // fragment (tile, j): rows row0 + 16 tile + g (+8), tokens m0 + 8 j + 2 t (+1)
#pragma unroll
        for (int j = 0; j < MT; ++j) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int64_t tok = m0 + 8 * j + 2 * t + e;
                if (tok >= a.M) continue;
                const float fac = (a.kind == kOutI32) ? 0.0f : __fdiv_rn(gamma, a.s[tok]);
#pragma unroll
                for (int tile = 0; tile < 2; ++tile) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int64_t row = row0 + 16 * tile + g + 8 * h;
                        if (row < a.N) store_y(a.out, a.kind, tok * a.N + row, acc[tile][j][2 * h + e], fac);
                    }
                }
            }
        }
        return;
    }

    // cluster reduction of the K-slice partial sums through distributed shared memory
    int* red = reinterpret_cast<int*>(smem + a.xs_bytes);
#pragma unroll
    for (int j = 0; j < MT; ++j)
#pragma unroll
        for (int tile = 0; tile < 2; ++tile)
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int e = 0; e < 2; ++e)
                    red[(8 * j + 2 * t + e) * kGvRows + warp * 32 + 16 * tile + g + 8 * h] =
                        acc[tile][j][2 * h + e];
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int S = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int items = MP * kGvRows;
    const int per = (items + S - 1) / S;
    const int lo = rank * per, hi = min(items, lo + per);
    for (int idx = lo + threadIdx.x; idx < hi; idx += kGvThreads) {
        int sum = 0;
        for (int q = 0; q < S; ++q) sum += cluster.map_shared_rank(red, q)[idx];
        const int64_t tok = m0 + idx / kGvRows;
        const int64_t row = static_cast<int64_t>(blockIdx.x) * kGvRows + idx % kGvRows;
        if (tok < a.M && row < a.N) {
            const float fac = (a.kind == kOutI32) ? 0.0f : __fdiv_rn(gamma, a.s[tok]);
            store_y(a.out, a.kind, tok * a.N + row, sum, fac);
        }
    }
    cluster.sync();
}

// One output per thread, any K % 4 == 0 (rows of packed bytes need not be aligned).
__global__ void __launch_bounds__(256) gemv_generic_kernel(GemvArgs a) {
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= a.M * a.N) return;
    const int64_t m = idx / a.N, n = idx % a.N;
    const int64_t KB = a.K / 4;
    const uint8_t* w = a.packed + n * KB;
    const int8_t* x = a.xq + m * a.K;
    int acc = 0;
    for (int64_t j = 0; j < KB; ++j) {
        const uint32_t b = w[j];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t c = (b >> (2 * i)) & 3u;
            const int xv = x[4 * j + i];
            acc += c == 1u ? xv : (c == 2u ? -xv : 0);
        }
    }
    const float fac = (a.kind == kOutI32) ? 0.0f : __fdiv_rn(*a.gamma, a.s[m]);
    store_y(a.out, a.kind, idx, acc, fac);
}

template <int MT>
cudaError_t launch_gemv_mt(GemvArgs a, int S, int64_t row_blocks, int64_t token_blocks,
                           cudaStream_t stream) {
    constexpr int MP = 8 * MT;
    const int win = a.Kc < kWindow ? a.Kc : kWindow;
    a.xs_bytes = win * MP;
    const size_t smem = static_cast<size_t>(a.xs_bytes) +
                        (S > 1 ? static_cast<size_t>(MP) * kGvRows * sizeof(int) : 0);
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gemv_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kWindow * MP + MP * kGvRows * static_cast<int>(sizeof(int)));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(row_blocks), static_cast<unsigned>(S),
                       static_cast<unsigned>(token_blocks));
    cfg.blockDim = dim3(kGvThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (S > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = S;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, gemv_kernel<MT>, a);
}

}  // namespace

cudaError_t launch_gemv(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                        int64_t M, int64_t N, int64_t K, void* out, int kind,
                        cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t row_blocks = (N + kGvRows - 1) / kGvRows;
    const int MT = M <= 8 ? 1 : 2;
    const int64_t token_blocks = (M + 8 * MT - 1) / (8 * MT);
    // K slices: enough blocks for ~2 per SM, at least one chunk per slice, at most 8.
    const int64_t kchunks = (K + kChunk - 1) / kChunk;
    int64_t S = (2 * sms + row_blocks * token_blocks - 1) / (row_blocks * token_blocks);
    if (S < 1) S = 1;
    if (S > kMaxCluster) S = kMaxCluster;
    if (S > kchunks) S = kchunks;
    int64_t Kc = ((K + S - 1) / S + kChunk - 1) / kChunk * kChunk;
    S = (K + Kc - 1) / Kc;
    GemvArgs a{xq, s, packed, gamma, M, N, static_cast<int>(K), static_cast<int>(Kc), 0, out, kind};
    if (MT == 1) return launch_gemv_mt<1>(a, static_cast<int>(S), row_blocks, token_blocks, stream);
    return launch_gemv_mt<2>(a, static_cast<int>(S), row_blocks, token_blocks, stream);
}

cudaError_t launch_gemv_generic(const int8_t* xq, const float* s, const uint8_t* packed,
                                const float* gamma, int64_t M, int64_t N, int64_t K, void* out,
                                int kind, cudaStream_t stream) {
    GemvArgs a{xq, s, packed, gamma, M, N, static_cast<int>(K), static_cast<int>(K), 0, out, kind};
    const int64_t total = M * N;
    gemv_generic_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace bl
