// Device helpers for the sm_100a kernels: mbarriers with bounded waits,
// bulk and 16-byte asynchronous copies, tcgen05 (TMEM allocation, MMA,
// commit, loads) and the shared-memory matrix descriptor of a K-major
// operand in the 128-byte swizzled layout.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe.h"

namespace moe {

// A device-side wait gives up after this long (nanoseconds of %globaltimer)
// and reports MOE_ERR_DEVICE_TIMEOUT in the status word; no correct run
// waits anywhere near this long.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

// status word layout in the workspace: [0] = moe_status_t code, [1] = detail
__device__ __forceinline__ void report_error(int32_t* status, int code, int detail) {
    if (status != nullptr && atomicCAS(status, 0, code) == 0) {
        atomicExch(status + 1, detail);
    }
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
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

// Non-blocking test: has the phase of `parity` completed?  The result is a
// register the caller may consume later, so the barrier read can overlap
// other work issued in between.
__device__ __forceinline__ uint32_t mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok;
}

// Wait until the phase of `parity` has completed.  Returns false if the
// CTA's abort flag is raised or the wait exceeds `limit_ns` (kWaitTimeoutNs
// unless a test shortens it); the caller then stops its role.  `abort_flag`
// lives in shared memory.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns = kWaitTimeoutNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 63u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > limit_ns) return false;
        }
    }
}

// ---------------------------------------------------------------------------
// asynchronous copies
// ---------------------------------------------------------------------------
// 1-D bulk copy global -> shared (TMA engine), completion counted in bytes on
// the mbarrier.  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                              uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// 2-D tiled tensor copy global -> shared (TMA), box and swizzle from the map;
// c0 is the inner (column) coordinate, c1 the row coordinate.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int c0, int c1,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

// 16-byte copy global -> shared; src_bytes = 0 writes zeros and reads nothing.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

// 4-byte copy global -> shared (cp.async, completion by cp.async.wait_group).
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// Order this thread's generic-proxy view of shared memory before its later
// async-proxy operations (tcgen05.mma operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// One lane of a converged warp (elect.sync): the warp keeps computing
// warp-uniform values (descriptors, ring indices) and only the elected lane
// issues the single-thread instructions.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b32 r;\n\t"
        "elect.sync r|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// ---------------------------------------------------------------------------
// tcgen05
// ---------------------------------------------------------------------------
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

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so
// far has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// 16 TMEM lanes x 32 fp32 columns in the m16n8 accumulator fragment layout:
// register i of thread t holds lane base + t/4 (+ 8 when i & 2) and column
// 8*(i/4) + 2*(t%4) + (i & 1).  taddr: lane base (a multiple of 16 inside the
// warp's 32-lane quadrant) << 16 | first column.
__device__ __forceinline__ void tmem_ld_16x256b_x4(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// Store four 8x8 bf16 matrices transposed: register m of thread t holds row
// t/4, columns 2*(t%4) and 2*(t%4)+1 (low half first) of matrix m; column c
// of matrix m is written as 16 bytes at the address given by thread 8m + c.
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t addr, uint32_t r0, uint32_t r1,
                                                  uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                 "r"(r0), "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory descriptor of a K-major bf16 operand stored as rows of 128
// bytes (64 elements) with the 128-byte swizzle: 16-byte chunk c of row r sits
// at r*128 + ((c ^ (r % 8)) * 16); groups of 8 rows are 1024 bytes apart.
// The tile base must be 1024-byte aligned.  Advancing K by 16 elements
// (32 bytes) adds 2 to the descriptor.
__device__ __forceinline__ uint64_t make_sw128_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);  // start address
    d |= static_cast<uint64_t>(1) << 16;                       // leading offset (unused)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;               // stride offset: 8 rows
    d |= static_cast<uint64_t>(1) << 46;                       // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;                       // 128-byte swizzle
    return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, both operands K-major, M x N.
__host__ __device__ __forceinline__ uint32_t make_idesc_bf16(int M, int N) {
    return (1u << 4)                                   // D format fp32
           | (1u << 7)                                 // A format bf16
           | (1u << 10)                                // B format bf16
           | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// ---------------------------------------------------------------------------
// programmatic dependent launch
// ---------------------------------------------------------------------------
// Lets the next kernel in the stream be scheduled once every CTA of this one
// has started (its CTAs then wait in pdl_wait).
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Waits until the preceding kernel in the stream has completed and its memory
// is visible (returns at once when launched without the attribute).  Every
// kernel calls it before its first access to global data that another kernel
// of the layer reads or writes.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------
// int4 -> bf16 expansion of the prepacked weights (shared by the grouped GEMM
// and the small-batch path, so both produce the same bf16 weights)
// ---------------------------------------------------------------------------
union BF2 {
    uint32_t u;
    __nv_bfloat162 h;
};

// Expand one 32-bit word of 8 nibbles into 8 bf16 weights (16 bytes).  The
// word holds K positions 2i (bits 4i..4i+3) and 2i+1 (bits 16+4i..) for
// i = 0..3, so masking with 0x000F000F and or-ing the bf16 pattern of 128
// yields the pair (128 + q_2i, 128 + q_2i+1) exactly; subtracting 128 is exact
// and the fused multiply-add q*s + b rounds once.
// Nibble pair i of a packed word as bf16x2 (128 + q_lo, 128 + q_hi):
// ((w >> 4i) & 0x000F000F) | 0x43004300.  For i > 0 the shift and the or run
// as one integer multiply-add on the FMA pipe, ((w & mask_i) * 2^(32-4i)) >> 32
// + 0x43004300 (the masked bits and the pattern share no bit), so the
// half-rate logic pipe takes one operation per pair instead of two.
__device__ __forceinline__ uint32_t nibble_pair_bf16(uint32_t w, int i) {
    if (i == 0) return (w & 0x000F000Fu) | 0x43004300u;
    uint32_t d;
    asm("mad.hi.u32 %0, %1, %2, %3;"
        : "=r"(d)
        : "r"(w & (0x000F000Fu << (4 * i))), "r"(1u << (32 - 4 * i)), "r"(0x43004300u));
    return d;
}

__device__ __forceinline__ uint4 expand8(uint32_t w, __nv_bfloat162 s2, __nv_bfloat162 b2) {
    BF2 k128;
    k128.u = 0x43004300u;
    uint32_t r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        BF2 v, o;
        v.u = nibble_pair_bf16(w, i);
        const __nv_bfloat162 q = __hsub2(v.h, k128.h);
        o.h = __hfma2(q, s2, b2);
        r[i] = o.u;
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

}  // namespace moe
