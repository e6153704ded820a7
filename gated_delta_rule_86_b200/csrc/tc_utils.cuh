// Thin inline-PTX wrappers for the sm_100a features the chunk kernel uses:
// mbarriers, the async-proxy fence, Tensor Memory (TMEM) allocation and loads,
// tcgen05.mma with shared-memory operand descriptors, and tcgen05.commit.
//
// Operand layouts used throughout (bf16, 128-byte swizzle, "SW128"): a tile is
// stored as 8-row groups of 128-byte rows; inside a group, row r's 16-byte
// chunk c lives at chunk position c ^ (r % 8).  Groups are 1024 bytes apart and
// every group is 1024-byte aligned.  A [rows x 64] bf16 block therefore takes
// rows * 128 bytes; wider tiles are stored as consecutive 64-column blocks.
// The same bytes serve as a K-major operand (rows = M or N, columns = K) or as
// an MN-major operand (rows = K, columns = M or N); only the descriptor
// differs.  SW64 is the 64-byte-row analogue (32 bf16 columns, 512-byte groups,
// chunk position c ^ ((r / 2) % 4)).
#pragma once

#include <stdint.h>

#include "kda_common.cuh"

namespace kda {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ---------------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, at most kSpinLimit
// polls.  On timeout records the error word, sets *abort (shared) and returns
// false; also returns false at once if *abort is already set.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
    }
    record_device_error(kDevErrTimeout);
    *abort = 1;
    return false;
}

// Barrier over a subset of the CTA's warps (ids 1..15; id 0 is __syncthreads).
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Same, returning whether any participating thread passed pred = true.
__device__ __forceinline__ bool named_sync_or(uint32_t id, uint32_t nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Make generic-proxy shared-memory writes visible to the async proxy (the
// tensor cores read operands through it).
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- bulk copies ------------------------------------------------------------------------------

// Orders this thread's earlier generic-proxy accesses to global memory before its later
// asynchronous-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// ---- flags in global memory (progress signals between CTAs of one grid) -----------------------

__device__ __forceinline__ void st_release_gpu(int *p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Plain (relaxed, GPU scope) store: a progress signal that orders none of the caller's earlier
// accesses, so it does not wait for them.
__device__ __forceinline__ void st_relaxed_gpu(int *p, int v) {
    asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Longest wait on a global flag before the kernel gives up (a healthy grid waits microseconds).
constexpr uint64_t kFlagWaitNs = 2000000000ull;
__device__ __forceinline__ int ld_relaxed_gpu(const int *p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Launch-wide limits of the waits on global flags, and the launch's abort word (in the workspace,
// zeroed before each launch): a CTA whose wait runs out sets it, and every other CTA's flag waits
// see it within a few microseconds and give up too, so that one timeout ends the whole grid
// quickly instead of one wait limit per dependent CTA.
struct FlagWait {
    uint64_t limit_ns;
    int *abort_all;
};
// Wait until *p >= v; same contract as mbar_wait (records the error word and sets *abort on
// timeout, returns false at once once *abort is set).  The flags are progress counters released
// by their writers (st.release.gpu after the data they announce is complete in global memory);
// every poll is an acquire load, so the waiting thread's later accesses, including the bulk copies
// it issues after a proxy fence, are ordered after the announced data.
__device__ __forceinline__ bool flag_wait_ge(const int *p, int v, volatile int *abort, const FlagWait &fw) {
    if (ld_acquire_gpu(p) >= v) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0;; ++i) {
        __nanosleep(32);
        if (ld_acquire_gpu(p) >= v) return true;
        if (*abort) return false;
        if ((i & 255u) == 255u) {
            if (ld_relaxed_gpu(fw.abort_all) != 0) {   // another CTA gave up: leave as well
                *abort = 1;
                return false;
            }
            if (global_ns() - t0 > fw.limit_ns) break;
        }
    }
    record_device_error(kDevErrTimeout);
    *abort = 1;
    st_relaxed_gpu(fw.abort_all, 1);
    return false;
}

// Bulk copy global -> this CTA's shared memory; completes `bytes` of transaction on `bar`.
__device__ __forceinline__ void bulk_load(void *sdst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(sdst)),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Bulk copy shared -> global, added to the current bulk group (close it with bulk_commit).
__device__ __forceinline__ void bulk_store_nc(void *gdst, const void *ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(ssrc)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk store of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until at most the newest committed bulk group of this thread is still reading shared memory.
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// Wait until every committed bulk store of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Tiled TMA load of one box of a 3-D tensor map at coordinates (c0, c1, c2) (innermost first) into
// this CTA's shared memory; completes the box's bytes of transaction on `bar`.
__device__ __forceinline__ void tma_load_3d(void *sdst, const void *tmap, int c0, int c1, int c2, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(sdst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// Tiled TMA store of one box of a 3-D tensor map at coordinates (c0, c1, c2) from this CTA's shared
// memory, in the current bulk group (close it with bulk_commit).
__device__ __forceinline__ void tma_store_3d(const void *tmap, int c0, int c1, int c2, const void *ssrc) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(ssrc))
                 : "memory");
}

// ---- TMEM -------------------------------------------------------------------------------------

// Whole-warp operations.  `dst` receives the TMEM base address.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Load 32 lanes x 16 consecutive 32-bit columns: thread i of the warp receives
// lane (warp's lane base + i), columns [col, col + 16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
    uint32_t *u = reinterpret_cast<uint32_t *>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]),
          "=r"(u[15])
        : "r"(taddr));
}

// Same for 32 consecutive columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&r)[32]) {
    uint32_t *u = reinterpret_cast<uint32_t *>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]),
          "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]),
          "=r"(u[22]), "=r"(u[23]), "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]),
          "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
        : "r"(taddr));
}

// Store 32 lanes x 16 consecutive 32-bit columns: thread i of the warp writes lane (warp's lane
// base + i), columns [col, col + 16).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&u)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]),
        "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15])
        : "memory");
}
// Same for 8 consecutive columns.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&u)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(u[0]),
                 "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Lane field of a TMEM address for the 32-lane subpartition a warp may access.
__device__ __forceinline__ uint32_t tmem_lane_base(int warp) { return static_cast<uint32_t>((warp & 3) * 32) << 16; }

// ---- descriptors ------------------------------------------------------------------------------

enum Swz : uint32_t { kSwzNone = 0, kSwz128 = 2, kSwz64 = 4, kSwz32 = 6 };

// Shared-memory matrix descriptor (sm_100 format): start address, leading- and
// stride-dimension byte offsets (all >> 4), version 1 at bit 46, swizzle mode
// at bits 61-63.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                               uint32_t swz) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(swz & 7) << 61;
    return d;
}

// Instruction descriptor for kind::f16 or kind::tf32 with an fp32 accumulator.
// `fmt` selects the operand type of both A and B (kF16 or kBF16 for kind::f16:
// one tcgen05.mma never mixes them; kTF32 for kind::tf32); a_mn / b_mn select
// MN-major operands; neg_a negates A.
enum OpFmt : uint32_t { kF16 = 0, kBF16 = 1, kTF32 = 2 };
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, uint32_t fmt, bool a_mn, bool b_mn,
                                                  bool neg_a = false) {
    return (1u << 4)                       // D format: f32
           | (fmt << 7)                    // A format
           | (fmt << 10)                   // B format
           | ((neg_a ? 1u : 0u) << 13)     // negate A
           | ((a_mn ? 1u : 0u) << 15)      // A major
           | ((b_mn ? 1u : 0u) << 16)      // B major
           | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N, bool a_mn, bool b_mn, bool neg_a = false) {
    return make_idesc(M, N, kBF16, a_mn, b_mn, neg_a);
}

// D[tmem] (+)= A[smem] * B[smem] (kind::f16: fp16 or bf16 operands); issued by one thread.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem] (kind::tf32: fp32 operands, read as tf32; K = 8 per
// instruction, i.e. the same 32 bytes of an operand row as a kind::f16 k-step); one thread.
__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem] (kind::f16).  A is M x K with row m in TMEM lane m and two
// consecutive K elements per 32-bit column, so k-step kk (16 elements) starts at column
// a_tmem + 8 kk; issued by one thread.
__device__ __forceinline__ void mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

// Arrive once on `bar` when all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// ---- swizzled byte offsets --------------------------------------------------------------------

// Byte offset of (row, 16-byte chunk) inside a SW128 block of 128-byte rows.
__host__ __device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}
// Byte offset of (row, 16-byte chunk) inside a SW64 block of 64-byte rows.
__host__ __device__ __forceinline__ uint32_t sw64(uint32_t row, uint32_t chunk) {
    return row * 64u + ((chunk ^ ((row >> 1) & 3u)) << 4);
}

}  // namespace tc
}  // namespace kda
