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
    uint32_t mul2, mul16;  // 2^30 and 2^16: right shifts by 2 and 16 as high-half multiplies
    int layout;            // XqLayout of x_q
    int grow;              // gamma holds one scale per output row
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

// One K step of 16 codes per row for the thread's four rows (word w_r of each row):
// the even/odd unpack of the four words (masks on the ALU pipe, shifts as high-half
// multiplies on the FMA pipe, one prmt table lookup per output register) feeding the
// warp MMAs of both 16-row tiles directly, written as one block so that the unpacked
// registers are the MMA operands.  acc0/acc1: tiles 0/1 against token tile 0 (B = b0..b3);
// with MT == 2 also acc2/acc3 against token tile 1 (B = c0..c3).
// One K step of 16 codes per row for the thread's four rows (word w_r of each row):
// the even/odd unpack of the four words (masks on the ALU pipe, shifts as high-half
// multiplies on the FMA pipe, one prmt table lookup per output register) feeding the
// warp MMAs of both 16-row tiles directly, written as one block so that the unpacked
// registers are the MMA operands.  acc[0]/acc[1]: the two 16-row tiles; token tile 0
// uses B = b, token tile 1 (MT == 2) uses B = bb.
template <int MT>
__device__ __forceinline__ void gemv_step(int (&acc)[2][MT][4], uint32_t w0, uint32_t w1, uint32_t w2,
                                          uint32_t w3, uint4 b, uint4 bb, uint32_t mul2, uint32_t mul16) {
    if constexpr (MT == 1) {
        asm volatile(
            "{\n\t.reg .b32 sa0,sa1,sa2,sa3,sb0,sb1,sb2,sb3,tt0,tt1,tt2,tt3,ha0,ha1,ha2,ha3,hb0,hb1,hb2,hb3;\n\t"
            ".reg .b32 e00,e01,e02,e03,e10,e11,e12,e13,o00,o01,o02,o03,o10,o11,o12,o13;\n\t"
            "and.b32 sa0, %8, 0x33333333;\n\t"
            "mul.hi.u32 tt0, %8, %16;\n\t"
            "and.b32 sb0, tt0, 0x33333333;\n\t"
            "mul.hi.u32 ha0, sa0, %17;\n\t"
            "mul.hi.u32 hb0, sb0, %17;\n\t"
            "prmt.b32 e00, %18, 0, sa0;\n\t"
            "prmt.b32 e10, %18, 0, ha0;\n\t"
            "prmt.b32 o00, %18, 0, sb0;\n\t"
            "prmt.b32 o10, %18, 0, hb0;\n\t"
            "and.b32 sa1, %9, 0x33333333;\n\t"
            "mul.hi.u32 tt1, %9, %16;\n\t"
            "and.b32 sb1, tt1, 0x33333333;\n\t"
            "mul.hi.u32 ha1, sa1, %17;\n\t"
            "mul.hi.u32 hb1, sb1, %17;\n\t"
            "prmt.b32 e01, %18, 0, sa1;\n\t"
            "prmt.b32 e11, %18, 0, ha1;\n\t"
            "prmt.b32 o01, %18, 0, sb1;\n\t"
            "prmt.b32 o11, %18, 0, hb1;\n\t"
            "and.b32 sa2, %10, 0x33333333;\n\t"
            "mul.hi.u32 tt2, %10, %16;\n\t"
            "and.b32 sb2, tt2, 0x33333333;\n\t"
            "mul.hi.u32 ha2, sa2, %17;\n\t"
            "mul.hi.u32 hb2, sb2, %17;\n\t"
            "prmt.b32 e02, %18, 0, sa2;\n\t"
            "prmt.b32 e12, %18, 0, ha2;\n\t"
            "prmt.b32 o02, %18, 0, sb2;\n\t"
            "prmt.b32 o12, %18, 0, hb2;\n\t"
            "and.b32 sa3, %11, 0x33333333;\n\t"
            "mul.hi.u32 tt3, %11, %16;\n\t"
            "and.b32 sb3, tt3, 0x33333333;\n\t"
            "mul.hi.u32 ha3, sa3, %17;\n\t"
            "mul.hi.u32 hb3, sb3, %17;\n\t"
            "prmt.b32 e03, %18, 0, sa3;\n\t"
            "prmt.b32 e13, %18, 0, ha3;\n\t"
            "prmt.b32 o03, %18, 0, sb3;\n\t"
            "prmt.b32 o13, %18, 0, hb3;\n\t"
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {e00,e01,o00,o01}, {%12,%13}, {%0,%1,%2,%3};\n\t"
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {e10,e11,o10,o11}, {%14,%15}, {%0,%1,%2,%3};\n\t"
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%4,%5,%6,%7}, {e02,e03,o02,o03}, {%12,%13}, {%4,%5,%6,%7};\n\t"
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%4,%5,%6,%7}, {e12,e13,o12,o13}, {%14,%15}, {%4,%5,%6,%7};\n\t"
            "}\n"
            : "+r"(acc[0][0][0]), "+r"(acc[0][0][1]), "+r"(acc[0][0][2]), "+r"(acc[0][0][3]),
              "+r"(acc[1][0][0]), "+r"(acc[1][0][1]), "+r"(acc[1][0][2]), "+r"(acc[1][0][3])
            : "r"(w0), "r"(w1), "r"(w2), "r"(w3), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w),
              "r"(mul2), "r"(mul16), "r"(kCodeTable));
    } else {
        asm volatile(
            "{\n\t.reg .b32 sa0,sa1,sa2,sa3,sb0,sb1,sb2,sb3,tt0,tt1,tt2,tt3,ha0,ha1,ha2,ha3,hb0,hb1,hb2,hb3;\n\t"
            ".reg .b32 e00,e01,e02,e03,e10,e11,e12,e13,o00,o01,o02,o03,o10,o11,o12,o13;\n\t"
            "and.b32 sa0, %16, 0x33333333;\n\t"
            "mul.hi.u32 tt0, %16, %28;\n\t"
            "and.b32 sb0, tt0, 0x33333333;\n\t"
            "mul.hi.u32 ha0, sa0, %29;\n\t"
            "mul.hi.u32 hb0, sb0, %29;\n\t"
            "prmt.b32 e00, %30, 0, sa0;\n\t"
            "prmt.b32 e10, %30, 0, ha0;\n\t"
            "prmt.b32 o00, %30, 0, sb0;\n\t"
            "prmt.b32 o10, %30, 0, hb0;\n\t"
            "and.b32 sa1, %17, 0x33333333;\n\t"
            "mul.hi.u32 tt1, %17, %28;\n\t"
            "and.b32 sb1, tt1, 0x33333333;\n\t"
            "mul.hi.u32 ha1, sa1, %29;\n\t"
            "mul.hi.u32 hb1, sb1, %29;\n\t"
            "prmt.b32 e01, %30, 0, sa1;\n\t"
            "prmt.b32 e11, %30, 0, ha1;\n\t"
            "prmt.b32 o01, %30, 0, sb1;\n\t"
            "prmt.b32 o11, %30, 0, hb1;\n\t"
            "and.b32 sa2, %18, 0x33333333;\n\t"
            "mul.hi.u32 tt2, %18, %28;\n\t"
            "and.b32 sb2, tt2, 0x33333333;\n\t"
            "mul.hi.u32 ha2, sa2, %29;\n\t"
            "mul.hi.u32 hb2, sb2, %29;\n\t"
            "prmt.b32 e02, %30, 0, sa2;\n\t"
            "prmt.b32 e12, %30, 0, ha2;\n\t"
            "prmt.b32 o02, %30, 0, sb2;\n\t"
            "prmt.b32 o12, %30, 0, hb2;\n\t"
            "and.b32 sa3, %19, 0x33333333;\n\t"
            "mul.hi.u32 tt3, %19, %28;\n\t"
            "and.b32 sb3, tt3, 0x33333333;\n\t"
            "mul.hi.u32 ha3, sa3, %29;\n\t"
            "mul.hi.u32 hb3, sb3, %29;\n\t"
            "prmt.b32 e03, %30, 0, sa3;\n\t"
            "prmt.b32 e13, %30, 0, ha3;\n\t"
            "prmt.b32 o03, %30, 0, sb3;\n\t"
            "prmt.b32 o13, %30, 0, hb3;\n\t"
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {e00,e01,o00,o01}, {%20,%21}, {%0,%1,%2,%3};\n\t"
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {e10,e11,o10,o11}, {%22,%23}, {%0,%1,%2,%3};\n\t"
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%4,%5,%6,%7}, {e02,e03,o02,o03}, {%20,%21}, {%4,%5,%6,%7};\n\t"
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%4,%5,%6,%7}, {e12,e13,o12,o13}, {%22,%23}, {%4,%5,%6,%7};\n\t"
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%8,%9,%10,%11}, {e00,e01,o00,o01}, {%24,%25}, {%8,%9,%10,%11};\n\t"
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%8,%9,%10,%11}, {e10,e11,o10,o11}, {%26,%27}, {%8,%9,%10,%11};\n\t"
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%12,%13,%14,%15}, {e02,e03,o02,o03}, {%24,%25}, {%12,%13,%14,%15};\n\t"
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%12,%13,%14,%15}, {e12,e13,o12,o13}, {%26,%27}, {%12,%13,%14,%15};\n\t"
            "}\n"
            : "+r"(acc[0][0][0]), "+r"(acc[0][0][1]), "+r"(acc[0][0][2]), "+r"(acc[0][0][3]),
              "+r"(acc[1][0][0]), "+r"(acc[1][0][1]), "+r"(acc[1][0][2]), "+r"(acc[1][0][3]),
              "+r"(acc[0][MT - 1][0]), "+r"(acc[0][MT - 1][1]), "+r"(acc[0][MT - 1][2]), "+r"(acc[0][MT - 1][3]),
              "+r"(acc[1][MT - 1][0]), "+r"(acc[1][MT - 1][1]), "+r"(acc[1][MT - 1][2]), "+r"(acc[1][MT - 1][3])
            : "r"(w0), "r"(w1), "r"(w2), "r"(w3), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w), "r"(bb.x), "r"(bb.y), "r"(bb.z), "r"(bb.w),
              "r"(mul2), "r"(mul16), "r"(kCodeTable));
    }
}

template <int MT, int LAY>
__global__ void __launch_bounds__(kGvThreads, 2) gemv_kernel(GemvArgs a) {
    pdl_wait_then_release();
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
    const uint32_t mul2 = a.mul2, mul16 = a.mul16;

    // Rows past N read the last row (always valid memory); their sums are never stored.
    const uint8_t* wrow[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int64_t row = row0 + g + 8 * r;
        wrow[r] = a.packed + (row < a.N ? row : a.N - 1) * KB + 16 * t;
    }

    int acc[2][MT][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < MT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0;

    auto compute_chunk = [&](const uint4 (&buf)[4], int c) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint8_t* xb = xs + ((((c * 4 + i) * MP) + g) * 4 + t) * 16;
            const uint4 b = *reinterpret_cast<const uint4*>(xb);
            const uint4 bb = MT > 1 ? *reinterpret_cast<const uint4*>(xb + 8 * 4 * 16) : b;
#define BL_W(R) (i == 0 ? buf[R].x : i == 1 ? buf[R].y : i == 2 ? buf[R].z : buf[R].w)
            gemv_step<MT>(acc, BL_W(0), BL_W(1), BL_W(2), BL_W(3), b, bb, mul2, mul16);
#undef BL_W
        }
    };

    for (int kw = k_begin; kw < k_end; kw += kWindow) {
        const int kw_end = min(k_end, kw + kWindow);
        const int nfull = (kw_end - kw) / kChunk;        // chunks of 256 codes
        const int tail = (kw_end - kw) - nfull * kChunk;  // 0, 64, 128 or 192 codes
        const int nch = nfull + (tail ? 1 : 0);
        const int64_t kb = kw / 4;  // packed byte offset of the window in each row

        // weights of full chunk c of this window: 64 codes of each of this thread's 4 rows
        auto load_full = [&](uint4 (&buf)[4], int c) {
#pragma unroll
            for (int r = 0; r < 4; ++r) buf[r] = ldg_stream_v4(wrow[r] + kb + c * (kChunk / 4));
        };

        uint4 bufA[4], bufB[4], bufC[4];
        if (nfull > 0) load_full(bufA, 0);
        if (nfull > 1) load_full(bufB, 1);

        // stage this window's activations in the order of the even/odd unpack
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
            // words wanted per 16-group: {0,2,4,6}, {1,3,5,7}, {8,..,14}, {9,..,15}; the
            // even/odd k16 layout already holds them, as words 0, 2, 1, 3; the stride-4
            // layout holds {0,4,8,12}, {1,5,9,13}, {2,6,10,14}, {3,7,11,15}
            uint4 o;
            if constexpr (LAY == kXqEvenOdd16) {
                o = make_uint4(v.x, v.z, v.y, v.w);
            } else if constexpr (LAY == kXqStride4K16) {
                o = make_uint4(__byte_perm(v.x, v.z, 0x5140), __byte_perm(v.y, v.w, 0x5140),
                               __byte_perm(v.x, v.z, 0x7362), __byte_perm(v.y, v.w, 0x7362));
            } else {
                o = permute16_evenodd(v);
            }
            *reinterpret_cast<uint4*>(xs + ((((c * 4 + i) * MP) + m) * 4 + tt) * 16) = o;
        }
        __syncthreads();

        // full chunks: loads two chunks ahead, no per-load predicates
        for (int c = 0; c < nfull; c += 3) {
            if (c + 2 < nfull) load_full(bufC, c + 2);
            compute_chunk(bufA, c);
            if (c + 1 >= nfull) break;
            if (c + 3 < nfull) load_full(bufA, c + 3);
            compute_chunk(bufB, c + 1);
            if (c + 2 >= nfull) break;
            if (c + 4 < nfull) load_full(bufB, c + 4);
            compute_chunk(bufC, c + 2);
        }
        if (tail) {
            // last partial chunk: thread t holds codes [64 t, 64 t + 64) of it
            const bool ok = 64 * t < tail;
#pragma unroll
            for (int r = 0; r < 4; ++r)
                bufA[r] = ok ? ldg_stream_v4(wrow[r] + kb + nfull * (kChunk / 4)) : make_uint4(0, 0, 0, 0);
            compute_chunk(bufA, nfull);
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
                        if (row >= a.N) continue;
                        const float f = (a.grow && a.kind != kOutI32) ? __fdiv_rn(a.gamma[row], a.s[tok]) : fac;
                        store_y(a.out, a.kind, tok * a.N + row, acc[tile][j][2 * h + e], f);
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
            const float fac = (a.kind == kOutI32) ? 0.0f : __fdiv_rn(a.grow ? a.gamma[row] : gamma, a.s[tok]);
            store_y(a.out, a.kind, tok * a.N + row, sum, fac);
        }
    }
    cluster.sync();
}

// One output per thread, any K % 4 == 0 (rows of packed bytes need not be aligned).
__global__ void __launch_bounds__(256) gemv_generic_kernel(GemvArgs a) {
    pdl_wait_then_release();
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
            const int64_t k = 4 * j + i;
            // position of element k: itself, or its slot in a k16 layout
            int64_t pos = k;
            if (a.layout == kXqEvenOdd16)
                pos = (k & ~int64_t(15)) | ((k & 1) * 8 + ((k >> 3) & 1) * 4 + ((k & 7) >> 1));
            else if (a.layout == kXqStride4K16)
                pos = (k & ~int64_t(15)) | ((k & 3) * 4 + ((k & 15) >> 2));
            const int xv = x[pos];
            acc += c == 1u ? xv : (c == 2u ? -xv : 0);
        }
    }
    const float fac = (a.kind == kOutI32) ? 0.0f : __fdiv_rn(a.grow ? a.gamma[n] : *a.gamma, a.s[m]);
    store_y(a.out, a.kind, idx, acc, fac);
}

template <int MT, int LAY>
cudaError_t launch_gemv_mt(GemvArgs a, int S, int64_t row_blocks, int64_t token_blocks,
                           cudaStream_t stream) {
    constexpr int MP = 8 * MT;
    const int win = a.Kc < kWindow ? a.Kc : kWindow;
    a.xs_bytes = win * MP;
    const size_t smem = static_cast<size_t>(a.xs_bytes) +
                        (S > 1 ? static_cast<size_t>(MP) * kGvRows * sizeof(int) : 0);
    static PerContextOnce attr;
    cudaError_t e = attr.run([] {
        return cudaFuncSetAttribute(gemv_kernel<MT, LAY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kWindow * MP + MP * kGvRows * static_cast<int>(sizeof(int)));
    });
    if (e != cudaSuccess) return e;
    return launch_pdl(gemv_kernel<MT, LAY>,
                      dim3(static_cast<unsigned>(row_blocks), static_cast<unsigned>(S), static_cast<unsigned>(token_blocks)),
                      dim3(kGvThreads), smem, stream, S > 1 ? dim3(1, S, 1) : dim3(kNoCluster), a);
}

}  // namespace

cudaError_t launch_gemv(const int8_t* xq, const float* s, const uint8_t* packed, const float* gamma,
                        int64_t M, int64_t N, int64_t K, void* out, int kind, int32_t* err, int layout,
                        cudaStream_t stream) {
    if (layout == kXqStride4K16 && gemv_stream_applicable(M, N, K))
        return launch_gemv_stream(xq, s, packed, gamma, M, N, K, out, kind, stream);
    if (layout == kXqStride4K16 && gemv_tma_applicable(M, N, K))
        return launch_gemv_tma(xq, s, packed, gamma, M, N, K, out, kind, err, stream);
    const int grow = gamma_rows_of(kind);
    kind = out_kind_of(kind);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t row_blocks = (N + kGvRows - 1) / kGvRows;
    const int MT = M <= 8 ? 1 : 2;
    const int64_t token_blocks = (M + 8 * MT - 1) / (8 * MT);
    // K slices (the cluster size S <= 8, at least one chunk per slice): pick the S whose
    // block count fills the resident slots (2 blocks per SM) in the most even waves,
    // preferring more blocks among near ties.
    const int64_t kchunks = (K + kChunk - 1) / kChunk;
    const int64_t slots = 2 * static_cast<int64_t>(sms);
    int64_t S = 1;
    double best = -1.0;
    for (int64_t cand = 1; cand <= kMaxCluster && cand <= kchunks; ++cand) {
        const int64_t kc = ((K + cand - 1) / cand + kChunk - 1) / kChunk * kChunk;
        if ((K + kc - 1) / kc != cand) continue;  // that split leaves an empty slice
        const int64_t blocks = row_blocks * token_blocks * cand;
        const int64_t waves = (blocks + slots - 1) / slots;
        const double eff = static_cast<double>(blocks) / static_cast<double>(waves * slots);
        if (eff > best + 0.02) {
            best = eff;
            S = cand;
        } else if (eff > best - 0.02 && waves == 1) {
            S = cand;  // a single, fuller wave with more, shorter blocks
            best = eff > best ? eff : best;
        }
    }
    int64_t Kc = ((K + S - 1) / S + kChunk - 1) / kChunk * kChunk;
    S = (K + Kc - 1) / Kc;
    GemvArgs a{xq, s, packed, gamma, M, N, static_cast<int>(K), static_cast<int>(Kc), 0, out, kind, 1u << 30, 1u << 16,
               layout, grow};
    const int Si = static_cast<int>(S);
    if (MT == 1) {
        if (layout == kXqEvenOdd16) return launch_gemv_mt<1, kXqEvenOdd16>(a, Si, row_blocks, token_blocks, stream);
        if (layout == kXqStride4K16) return launch_gemv_mt<1, kXqStride4K16>(a, Si, row_blocks, token_blocks, stream);
        return launch_gemv_mt<1, kXqRowMajor>(a, Si, row_blocks, token_blocks, stream);
    }
    if (layout == kXqEvenOdd16) return launch_gemv_mt<2, kXqEvenOdd16>(a, Si, row_blocks, token_blocks, stream);
    if (layout == kXqStride4K16) return launch_gemv_mt<2, kXqStride4K16>(a, Si, row_blocks, token_blocks, stream);
    return launch_gemv_mt<2, kXqRowMajor>(a, Si, row_blocks, token_blocks, stream);
}

cudaError_t launch_gemv_generic(const int8_t* xq, const float* s, const uint8_t* packed,
                                const float* gamma, int64_t M, int64_t N, int64_t K, void* out,
                                int kind, int layout, cudaStream_t stream) {
    GemvArgs a{xq, s, packed, gamma, M, N, static_cast<int>(K), static_cast<int>(K), 0, out, out_kind_of(kind),
               1u << 30, 1u << 16, layout, gamma_rows_of(kind)};
    const int64_t total = M * N;
    return launch_pdl(gemv_generic_kernel, dim3(static_cast<unsigned>((total + 255) / 256)), dim3(256), 0, stream,
                      dim3(kNoCluster), a);
}

}  // namespace bl
