// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA tile loads, and the
// tcgen05 (5th-generation tensor core) allocation, MMA, commit and TMEM loads.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define AUT_DEV __device__ __forceinline__

namespace aut {

// Status codes written by kernels into a device status word (same values as
// aut_status in include/aut.h).
constexpr int kDevTimeout = 5;
constexpr int kDevBounds = 6;

// Debug builds (-DAUT_DEBUG_BOUNDS, libaut_debug.so) check the computed global
// addresses of the kernels that do not go through TMA: a failed check writes
// AUT_ERR_BOUNDS to the status word and the access is skipped, nothing traps.
// Release builds compile the checks away.
#ifdef AUT_DEBUG_BOUNDS
#define AUT_IN_BOUNDS(cond, status) ::aut::bounds_ok((cond), (status))
#else
#define AUT_IN_BOUNDS(cond, status) ((void)sizeof(cond), true)  // cond is not evaluated
#endif
__device__ __forceinline__ bool bounds_ok(bool ok, int *status) {
    if (!ok && status) atomicCAS(status, 0, kDevBounds);
    return ok;
}

AUT_DEV uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

AUT_DEV uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier --
AUT_DEV void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}
AUT_DEV void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
AUT_DEV void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}
AUT_DEV void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// A waiting thread is suspended (up to kWaitSuspendNs, or until the phase
// completes) instead of polling: a polling warp takes issue slots from the
// warps on its scheduler that have work, such as a GEMM's MMA issuer and
// epilogue.
constexpr uint32_t kWaitSuspendNs = 2000;
AUT_DEV bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(kWaitSuspendNs)
        : "memory");
    return ok != 0;
}

// Waits until the phase with the given parity has completed.  Gives up (and
// returns false) when *abort becomes non-zero (abort may be null) or after
// limit_ns nanoseconds.
AUT_DEV bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (abort && *abort) return false;
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
}

// Non-blocking: whether the phase with the given parity has completed
// (acquire semantics, as a successful wait).
AUT_DEV bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred q;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 q, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// mbar_wait for a whole converged warp, with one answer for every lane: each
// lane polls on its own, so near a time-out or an abort some lanes could see
// the phase complete and others give up; the vote makes the warp leave (or
// carry on) together, as the warp-wide tcgen05 operations after it require.
AUT_DEV bool mbar_wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort, uint64_t limit_ns) {
    const bool ok = mbar_wait(bar, parity, abort, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

// Completes `bytes` of the current phase's expected transaction count without
// a copy (for bytes that will never arrive).
AUT_DEV void mbar_complete_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.complete_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// mbar_wait with acquire at cluster scope: data another CTA of the cluster
// stored before its release-arrive on `bar` is visible once this returns true.
AUT_DEV bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = global_timer_ns();
    while (true) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(smem_addr(bar)), "r"(parity), "r"(kWaitSuspendNs)
            : "memory");
        if (ok) return true;
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
}

// -------------------------------------------------------------------- TMA --
AUT_DEV void tma_prefetch_desc(const CUtensorMap *m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
AUT_DEV void tma_load_2d(void *dst, const CUtensorMap *m, uint64_t *bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_addr(bar)), "r"(c0), "r"(c1)
        : "memory");
}
// Tile store shared -> global (bulk async-group completion; rows and columns
// outside the tensor are not written).  The source must be visible to the
// async proxy (fence_proxy_async_smem) before the call.
AUT_DEV void tma_store_2d(const CUtensorMap *m, const void *src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(smem_addr(src)), "r"(c0), "r"(c1)
                 : "memory");
}
AUT_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Every committed bulk store of this thread has finished reading shared memory.
AUT_DEV void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Every committed bulk store of this thread but the most recent has finished
// reading shared memory.
AUT_DEV void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// Every committed bulk store of this thread has completed.
AUT_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
AUT_DEV void prefetch_l1(const void *p) {
    asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}

AUT_DEV void tma_load_3d(void *dst, const CUtensorMap *m, uint64_t *bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
AUT_DEV void tma_load_4d(void *dst, const CUtensorMap *m, uint64_t *bar, int c0, int c1, int c2,
                         int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3)
        : "memory");
}

// ---------------------------------------------------------------- tcgen05 --
AUT_DEV void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
AUT_DEV void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
AUT_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
AUT_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
AUT_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrives on `bar` once every tcgen05 operation this thread issued before has
// completed.
AUT_DEV void tc_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_addr(bar))
        : "memory");
}

// D(tmem) (+)= A(smem) * B(smem)^T, bf16 inputs, fp32 accumulate.
AUT_DEV void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

AUT_DEV void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Loads 16 consecutive fp32 columns of this thread's TMEM lane (warp w of a
// warpgroup reads lanes [32 (w % 4), 32 (w % 4) + 32)).
AUT_DEV void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Loads 32 consecutive fp32 columns of this thread's TMEM lane.
AUT_DEV void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

AUT_DEV void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Stores 16 consecutive fp32 columns into this thread's TMEM lane.
AUT_DEV void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 128 bytes (64 bf16 of K), 8-row swizzle
// atoms 1024 bytes apart.  Fields: start address >> 4 (bits 0-13), leading
// byte offset >> 4 (bits 16-29, unused for this layout), stride byte offset >> 4
// (bits 32-45) = 1024 >> 4, descriptor version 1 (bits 46-47), layout type
// 2 = 128-byte swizzle (bits 61-63).
AUT_DEV uint64_t smem_desc_sw128(const void *tile) {
    const uint64_t addr = smem_addr(tile);
    return ((addr & 0x3FFFFull) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
           (2ull << 61);
}

// Descriptor for an MN-major operand tile (the N, or M, index contiguous) with
// 128-byte swizzling: rows of 128 bytes hold 64 bf16 of N for one K index;
// groups of 8 K rows (1024-byte swizzle atoms) follow at the stride byte offset
// 1024 >> 4.  The tile here is exactly 64 wide in N, so the leading byte
// offset (between 64-wide N groups) is never used.
AUT_DEV uint64_t smem_desc_sw128_mn(const void *tile) {
    const uint64_t addr = smem_addr(tile);
    return ((addr & 0x3FFFFull) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
           (2ull << 61);
}

// Fence making this thread's generic-proxy shared-memory writes visible to the
// async proxy (TMA, tcgen05.mma) after a subsequent barrier.
AUT_DEV void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Instruction descriptor for kind::f16 with bf16 A and B, fp32 accumulator,
// both operands K-major: c_format F32 (bit 4), a_format BF16 (bits 7-9),
// b_format BF16 (bits 10-12), N >> 3 (bits 17-22), M >> 4 (bits 24-28).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// The same for fp16 A and B (a_format = b_format = 0).
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Two floats to fp16x2 (round to nearest; beyond fp16's range clamps to
// +-65504 instead of becoming infinite); `a` lands at the lower address.
AUT_DEV uint32_t pack_f16x2_sat(float a, float b) {
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
    return r;
}

// Programmatic dependent launch: let the next kernel in the stream start its
// launch and set-up now; and wait until the previous kernel has completed and
// its memory is visible.  Every kernel of the forward waits before its first
// global-memory access, so stream order is kept for all data.
AUT_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
AUT_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// GELU(x) = x * Phi(x) = x (1 + erf(x / sqrt 2)) / 2, the exact form, with one
// exp2 per value.  For a = min(|x|, 6):
//   Phi(-a) = exp2(S(a) - a^2 log2(e) / 2),
// where S is a degree-7 polynomial least-squares fitted to
// log2 Phi(-a) + a^2 log2(e) / 2 on [0, 6] (gen_gelu_poly.py beside this file
// regenerates the coefficients).  Evaluated in fp32 the GELU is off by at most
// 5e-7 in absolute terms, far below the bf16 rounding of every GELU output;
// Phi(-6) ~ 1e-9 bounds what the clamp leaves out.
// Then GELU(x) = x (1 - Phi(-a)) for x >= 0 and x Phi(-a) for x < 0.
constexpr float kHalfLog2e = 0.72134752044448170f;  // log2(e) / 2

AUT_DEV float ex2_approx(float t) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(t));
    return r;
}

AUT_DEV float gelu_fast(float x) {
    const float a = fminf(fabsf(x), 6.0f);
    float s = -1.944917813e-06f;
    s = fmaf(s, a, 6.386046880e-05f);
    s = fmaf(s, a, -9.488704964e-04f);
    s = fmaf(s, a, 8.582371287e-03f);
    s = fmaf(s, a, -5.411831290e-02f);
    s = fmaf(s, a, 2.630500793e-01f);
    s = fmaf(s, a, -1.151324630e+00f);
    s = fmaf(s, a, -9.999869466e-01f);
    const float h = ex2_approx(fmaf(-kHalfLog2e * a, a, s));  // Phi(-a)
    return x * (x >= 0.0f ? 1.0f - h : h);
}

// Packed fp32x2 arithmetic (two lanes per instruction).
AUT_DEV unsigned long long f2_bits(float2 v) { return *reinterpret_cast<unsigned long long *>(&v); }
AUT_DEV float2 f2_from(unsigned long long b) { return *reinterpret_cast<float2 *>(&b); }
AUT_DEV float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
    return f2_from(d);
}
AUT_DEV float2 fmul2(float2 a, float2 b) {
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return f2_from(d);
}

AUT_DEV float2 fadd2(float2 a, float2 b) {
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return f2_from(d);
}
AUT_DEV float2 fsub2(float2 a, float2 b) {
    unsigned long long d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return f2_from(d);
}
// max(a, b, c) in one instruction.
AUT_DEV float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// gelu_fast on two values, the polynomial and scaling in packed fp32x2.
AUT_DEV float2 gelu_fast2(float2 x) {
    const float2 a = make_float2(fminf(fabsf(x.x), 6.0f), fminf(fabsf(x.y), 6.0f));
    float2 s = make_float2(-1.944917813e-06f, -1.944917813e-06f);
    s = ffma2(s, a, make_float2(6.386046880e-05f, 6.386046880e-05f));
    s = ffma2(s, a, make_float2(-9.488704964e-04f, -9.488704964e-04f));
    s = ffma2(s, a, make_float2(8.582371287e-03f, 8.582371287e-03f));
    s = ffma2(s, a, make_float2(-5.411831290e-02f, -5.411831290e-02f));
    s = ffma2(s, a, make_float2(2.630500793e-01f, 2.630500793e-01f));
    s = ffma2(s, a, make_float2(-1.151324630e+00f, -1.151324630e+00f));
    s = ffma2(s, a, make_float2(-9.999869466e-01f, -9.999869466e-01f));
    const float2 t = ffma2(fmul2(make_float2(-kHalfLog2e, -kHalfLog2e), a), a, s);
    const float h0 = ex2_approx(t.x), h1 = ex2_approx(t.y);  // Phi(-a)
    return fmul2(x, make_float2(x.x >= 0.0f ? 1.0f - h0 : h0, x.y >= 0.0f ? 1.0f - h1 : h1));
}

AUT_DEV uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

}  // namespace aut

// ------------------------------------------------ CTA pairs (cta_group::2) --
namespace aut {

AUT_DEV uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
AUT_DEV void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
// Address of the same shared-memory variable in CTA `rank` of the cluster.
AUT_DEV uint32_t map_to_rank(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}
AUT_DEV void st_shared_cluster_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
AUT_DEV void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
// TMA tile loads of one CTA of a pair whose completion is counted on an
// mbarrier that may live in the other CTA (cluster address).
AUT_DEV void tma_load_2d_pair(void *dst, const CUtensorMap *m, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}
AUT_DEV void tma_load_3d_pair(void *dst, const CUtensorMap *m, uint32_t bar, int c0, int c1,
                              int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
AUT_DEV void tma_load_4d_pair(void *dst, const CUtensorMap *m, uint32_t bar, int c0, int c1,
                              int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
AUT_DEV void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
AUT_DEV void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
AUT_DEV void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
// D(tmem of both CTAs) (+)= A(smem of both CTAs, 128 rows each) * B^T (smem of
// both CTAs, N/2 rows each); issued by one thread of the even CTA.
AUT_DEV void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives on the mbarrier at the same offset in every CTA of `mask` once the
// pair's earlier tcgen05 operations issued by this thread have completed.
AUT_DEV void tc_commit_pair(uint64_t *bar, uint16_t mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_addr(bar)),
        "h"(mask)
        : "memory");
}

}  // namespace aut
