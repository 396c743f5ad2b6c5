// bl_device.cuh -- device-side building blocks shared by the libbitlinear kernels:
// inline-PTX wrappers for mbarriers, TMA tensor loads, tcgen05 (TMEM allocation, MMA,
// commit, loads), programmatic dependent launch, bounded waits, streaming loads, and
// the three 2-bit -> int8 unpack routines (natural, even/odd and stride-4 order).
// Written for sm_100a only.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace bl {

// Bits OR-ed into the optional device error word (mirrors BL_ERRBIT_* in bitlinear.h).
constexpr int kErrBitBadCode = 0x1;
constexpr int kErrBitTimeout = 0x2;

// Every spin-wait in this library gives up after this long and reports a timeout.
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ mbarrier --

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that lets the hardware suspend the warp (up to `hint_ns`) until the phase
// completes, instead of spinning and taking issue slots from the working warps.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// How a blocked role waits: with a suspend-time hint (the hardware parks the warp until
// the phase completes or the hint runs out), or with the plain try_wait, whose own
// suspension the hardware bounds; the abort flag and the clock are read every
// kWaitCheckEvery polls.
#ifndef BL_WAIT_HINT_NS
#define BL_WAIT_HINT_NS 200000
#endif
#ifndef BL_WAIT_CHECK_EVERY
#define BL_WAIT_CHECK_EVERY 1
#endif
constexpr uint32_t kSuspendHintNs = BL_WAIT_HINT_NS;
constexpr uint32_t kWaitCheckEvery = BL_WAIT_CHECK_EVERY;

// Wait until the phase with parity `parity` of `bar` has completed.  Gives up after
// limit_ns, or as soon as another role of the CTA has raised *abort; returns false then
// (and raises *abort itself on a timeout).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort,
                                                  unsigned long long limit_ns = kWaitTimeoutNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    const uint32_t hint = limit_ns < kSuspendHintNs ? static_cast<uint32_t>(limit_ns) : kSuspendHintNs;
    for (uint32_t it = 1;; ++it) {
        if (kSuspendHintNs > 0 ? mbar_try_wait_sleep(bar, parity, hint) : mbar_try_wait(bar, parity)) return true;
        if (it % kWaitCheckEvery != 0) continue;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            *abort = 1;
            return false;
        }
    }
}

// The stall of the bounded-wait test: a producer that has stopped issuing loads spins
// here until another role of the block gives up waiting for them (raising *abort), or
// for at most limit_ns, then raises *abort itself.
__device__ __forceinline__ void stall_until_abort(volatile int* abort, unsigned long long limit_ns) {
    const unsigned long long t0 = globaltimer_ns();
    while (!*abort && globaltimer_ns() - t0 <= limit_ns) {
    }
    *abort = 1;
}

// ------------------------------------------------ programmatic dependent launch --

// Every kernel of the library is launched with programmatic stream serialisation
// allowed, so that its launch and prologue can overlap the tail of the previous kernel
// on the stream.  It calls this before its first access to global memory: wait until
// the previous kernel has completed and its writes are visible (a no-op when there is
// none), then let the next kernel on the stream launch.
__device__ __forceinline__ void pdl_wait_then_release() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ----------------------------------------------------------------------- TMA --

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled bulk tensor load global -> shared::cta, completion counted on `bar`.
// c0 is the innermost (contiguous) coordinate in elements.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async proxy
// (the tensor core reads its operands through it).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------- tcgen05 --

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, int8 x int8 -> int32, issued by one thread.
__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns; each thread receives its lane's 32 values.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 16 consecutive 32-bit columns; each thread receives its lane's 16 values.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile stored in the canonical
// 128-byte-swizzled layout: rows of 128 bytes, 8-row groups of 1024 bytes, the 16-byte
// chunk index of each row XOR-ed with (row % 8).  The tile base must be 1024-aligned;
// `addr` may be advanced by a multiple of 32 bytes inside the row to step along K.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);  // start address
    d |= static_cast<uint64_t>(1u) << 16;                // leading byte offset (unused for swizzled K-major)
    d |= static_cast<uint64_t>(1024u >> 4) << 32;        // stride byte offset: next 8-row group
    d |= static_cast<uint64_t>(1u) << 46;                // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2u) << 61;                // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::i8, A and B signed 8-bit, K-major, D int32, shape M x N.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
    return (2u << 4)                                   // D format: S32
           | (1u << 7)                                 // A format: signed 8-bit
           | (1u << 10)                                // B format: signed 8-bit
           | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// ----------------------------------------------------- CTA pairs (cta_group::2) --

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address, in the shared::cluster window, of the variable at CTA-local shared address
// `addr` in the CTA of the cluster with rank `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Arrive on an mbarrier that may live in another CTA of the cluster (default
// semantics: release at CTA scope; a cluster-scope release costs a full fence).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    return mbar_try_wait(bar, parity);
}

// As mbar_wait_bounded, for barriers that also receive arrivals from the peer CTA.
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint32_t bar, uint32_t parity, volatile int* abort,
                                                          unsigned long long limit_ns = kWaitTimeoutNs) {
    return mbar_wait_bounded(bar, parity, abort, limit_ns);
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// 2-D tiled TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (`bar_cluster` is a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// D[tmem of both CTAs] (+)= A * B^T over a CTA pair: A's rows and B's rows are split
// between the two CTAs' shared memory at the same offsets.  Issued by one thread of the
// even CTA.
__device__ __forceinline__ void tc_mma_i8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the mbarrier at shared offset `bar` in every CTA of `cta_mask` when all
// pair MMAs issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit_pair_multicast(uint32_t bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"(cta_mask)
        : "memory");
}

// ------------------------------------------------------------- global loads --

// Streaming 16-byte load that bypasses L1 (each packed weight byte is read once).
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// --------------------------------------------------------------- 2-bit unpack --

// Byte table indexed by a 2-bit code: 00 -> 0, 01 -> +1, 10 -> -1 (0xFF), 11 -> 0.
constexpr uint32_t kCodeTable = 0x00FF0100u;

// Unpack 16 codes (one 32-bit word, code i at bits 2i..2i+1) into 16 int8 in natural
// order: w0 = codes 0..3, w1 = 4..7, w2 = 8..11, w3 = 12..15.  The codes of each byte
// are spread into nibbles (one per code) and each nibble selects a table byte.
__device__ __forceinline__ void unpack16_natural(uint32_t p, uint32_t& w0, uint32_t& w1,
                                                 uint32_t& w2, uint32_t& w3) {
    uint32_t lo = __byte_perm(p, 0u, 0x4140);  // [b0, 0, b1, 0]
    uint32_t hi = __byte_perm(p, 0u, 0x4342);  // [b2, 0, b3, 0]
    lo = (lo | (lo << 4)) & 0x0F0F0F0Fu;
    hi = (hi | (hi << 4)) & 0x0F0F0F0Fu;
    lo = (lo | (lo << 2)) & 0x33333333u;
    hi = (hi | (hi << 2)) & 0x33333333u;
    w0 = __byte_perm(kCodeTable, 0u, lo);
    w1 = __byte_perm(kCodeTable, 0u, lo >> 16);
    w2 = __byte_perm(kCodeTable, 0u, hi);
    w3 = __byte_perm(kCodeTable, 0u, hi >> 16);
}

// Unpack 16 codes into 16 int8 in even/odd order, which needs fewer instructions:
// e0 = codes {0,2,4,6}, e1 = {8,10,12,14}, o0 = {1,3,5,7}, o1 = {9,11,13,15}.
// The activations fed against these words are permuted the same way, which leaves
// every integer dot product unchanged.
__device__ __forceinline__ void unpack16_evenodd(uint32_t p, uint32_t& e0, uint32_t& e1,
                                                 uint32_t& o0, uint32_t& o1) {
    const uint32_t sa = p & 0x33333333u;
    const uint32_t sb = (p >> 2) & 0x33333333u;
    e0 = __byte_perm(kCodeTable, 0u, sa);
    e1 = __byte_perm(kCodeTable, 0u, sa >> 16);
    o0 = __byte_perm(kCodeTable, 0u, sb);
    o1 = __byte_perm(kCodeTable, 0u, sb >> 16);
}

// Runtime multipliers of the stride-4 unpack: passed in as values so that the shifts
// stay multiplies (FMA pipe) and leave the integer ALU pipe to the logic ops.
struct S4Mul {
    uint32_t hi1;                // 2^31: a right shift by 1 as a high-half multiply
    uint32_t two, m4, m16, m64;  // left shifts by 1, 2, 4, 6
};
__host__ __device__ constexpr S4Mul s4_mul() { return S4Mul{1u << 31, 2u, 4u, 16u, 64u}; }

// PTX of the stride-4 unpack of one packed word W (16 codes) into O0..O3, with scratch
// registers ta, tx, ty, tv, tt; HI1, TWO, M4, M16, M64 name the operands holding the
// S4Mul values.  The fields are first rewritten as 2-bit two's complement (00 -> 00,
// 01 -> 01, 10 -> 11, the unused 11 -> 00): low bit l ^ h, high bit h & ~l, from two
// 3-input logic ops and one multiply-add; output word i is then the word shifted left by
// 6 - 2i and masked to bits 6..7 of every byte.  Byte j of Oi is 64 * code(4j + i).
#define BL_S4_UNPACK(W, O0, O1, O2, O3, HI1, TWO, M4, M16, M64)                     \
    "mul.hi.u32 ta, " W ", " HI1 ";\n\t"                                           \
    "lop3.b32 tx, " W ", ta, 0x55555555, 0x28;\n\t" /* (w ^ (w >> 1)) & 0x55.. */  \
    "lop3.b32 ty, ta, " W ", 0x55555555, 0x20;\n\t" /* (w >> 1) & ~w & 0x55.. */   \
    "mad.lo.u32 tv, ty, " TWO ", tx;\n\t"                                          \
    "and.b32 " O3 ", tv, 0xC0C0C0C0;\n\t"                                          \
    "mul.lo.u32 tt, tv, " M4 ";\n\t"                                               \
    "and.b32 " O2 ", tt, 0xC0C0C0C0;\n\t"                                          \
    "mul.lo.u32 tt, tv, " M16 ";\n\t"                                              \
    "and.b32 " O1 ", tt, 0xC0C0C0C0;\n\t"                                          \
    "mul.lo.u32 tt, tv, " M64 ";\n\t"                                              \
    "and.b32 " O0 ", tt, 0xC0C0C0C0;\n\t"

// Unpack 16 codes into 16 int8 equal to 64 * code, in stride-4 order: o0 = codes
// {0,4,8,12}, o1 = {1,5,9,13}, o2 = {2,6,10,14}, o3 = {3,7,11,15}.  Matched against
// activations in the same order, the integer dot products come out 64 times the true
// ones (exact while they fit in int32), and an arithmetic shift right by 6 restores them.
__device__ __forceinline__ void unpack16_stride4_x64(uint32_t p, const S4Mul& k, uint32_t& o0, uint32_t& o1,
                                                     uint32_t& o2, uint32_t& o3) {
    asm("{\n\t.reg .b32 ta, tx, ty, tv, tt;\n\t"
        BL_S4_UNPACK("%4", "%0", "%1", "%2", "%3", "%5", "%6", "%7", "%8", "%9")
        "}\n"
        : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
        : "r"(p), "r"(k.hi1), "r"(k.two), "r"(k.m4), "r"(k.m16), "r"(k.m64));
}

// The matching permutation of 16 activation bytes (v = bytes 0..15 little-endian):
// returns {0,2,4,6}, {1,3,5,7}, {8,10,12,14}, {9,11,13,15}.
__device__ __forceinline__ uint4 permute16_evenodd(uint4 v) {
    uint4 r;
    r.x = __byte_perm(v.x, v.y, 0x6420);
    r.y = __byte_perm(v.x, v.y, 0x7531);
    r.z = __byte_perm(v.z, v.w, 0x6420);
    r.w = __byte_perm(v.z, v.w, 0x7531);
    return r;
}

}  // namespace bl
