// Device helpers shared by the W4A16 kernels (sm_100a only).
//
// Dequantization arithmetic ("推理优化中“用精度换性能“的核心技术：量化",
// §2.3: x̂ = (x_int − z) × s), done on bf16 pairs:
//   a 4-bit code q placed in the low mantissa bits of the bf16 pattern 0x4300
//   (the value 128) gives the bf16 value 128 + q exactly; subtracting the bf16
//   value 128 + z gives q − z exactly (an integer of magnitude ≤ 15); one
//   bf16 multiply by s then rounds (q − z)·s to bf16 once.  The result is
//   bit-identical to bf16_rn((q − z)·s).  Symmetric codes (4-bit two's
//   complement) are mapped to q + 8 by flipping bit 3, and 136 = 128 + 8 is
//   subtracted instead.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace w4a16 {

// Error word written by a kernel that gives up a bounded wait.
__device__ int g_device_error;

constexpr int kErrMbarTimeout = 1;
constexpr unsigned long long kWaitTimeoutNs = 1000000000ull;   // one second per wait

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void report_error(int code) { atomicCAS(&g_device_error, 0, code); }

// ------------------------------------------------------------------ loads
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    // Streaming read of data used once: bypass L1 allocation.
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ldg_cached(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint16_t ldg_u16(const uint16_t* p) {
    unsigned short v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// ------------------------------------------------------------------ bf16 bits
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ uint32_t f32_to_bf16_bits_rn(float f) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
    return r;
}

__device__ __forceinline__ uint32_t dup16(uint32_t b) { return (b & 0xFFFFu) * 0x00010001u; }

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t bf16x2_add(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// bf16x2 holding (128 + z, 128 + z) for an asymmetric zero point stored as bf16
// bits (an integer 0..15), or (136, 136) for symmetric codes.
template <bool SYM>
__device__ __forceinline__ uint32_t zero_pair(uint32_t z_bits) {
    if (SYM) return 0x43084308u;
    uint32_t z = (uint32_t)__float2int_rn(bf16_bits_to_f32(z_bits));
    return (0x4300u | (z & 0xFu)) * 0x00010001u;
}

// (a & mask) | magic  (asym)  or  (a & mask) ^ magic  (sym), as one LOP3.
template <bool SYM>
__device__ __forceinline__ uint32_t isolate_magic(uint32_t a, uint32_t mask) {
    uint32_t d;
    if (SYM) {
        asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(mask), "n"(0x43084308));
    } else {
        asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "n"(0x43004300));
    }
    return d;
}

// One bf16x2 of bf16_rn((q − z)·s) from codes isolated into the low nibble of
// each 16-bit half of `a` (the other bits of `a` are masked off).
template <bool SYM>
__device__ __forceinline__ uint32_t dq_pair(uint32_t a, uint32_t zz, uint32_t ss) {
    return bf16x2_mul(bf16x2_sub(isolate_magic<SYM>(a, 0x000F000Fu), zz), ss);
}

// A constant the compiler cannot see through: it is materialized once into a
// register and kept there, rather than re-created next to every use.
__device__ __forceinline__ uint32_t opaque_u32(uint32_t v) {
    uint32_t r;
    asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v));
    return r;
}

// dq_pair with the nibble mask (0x000F000F) supplied by the caller in a register.
template <bool SYM>
__device__ __forceinline__ uint32_t dq_pair_m(uint32_t a, uint32_t mask, uint32_t zz, uint32_t ss) {
    return bf16x2_mul(bf16x2_sub(isolate_magic<SYM>(a, mask), zz), ss);
}

// Eight codes of one 32-bit word (code i in nibble i) -> four bf16x2 values of
// bf16_rn((q − z)·s), in INTERLEAVED order: (q0,q4) (q1,q5) (q2,q6) (q3,q7).
template <bool SYM>
__device__ __forceinline__ void dequant8_interleaved(uint32_t w, uint32_t zz, uint32_t ss,
                                                     uint32_t out[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) out[j] = dq_pair<SYM>(w >> (4 * j), zz, ss);
}

// Same values in NATURAL order: (q0,q1) (q2,q3) (q4,q5) (q6,q7).
template <bool SYM>
__device__ __forceinline__ void dequant8_natural(uint32_t w, uint32_t zz, uint32_t ss,
                                                 uint32_t out[4]) {
    const uint32_t lo = w & 0x0F0F0F0Fu;          // q0 q2 q4 q6, one per byte
    const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;   // q1 q3 q5 q7
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // bytes: [lo.j, 0, hi.j, 0] — selector 8|x replicates the (zero) sign bit
        const uint32_t sel = (uint32_t)j | 0x80u | ((uint32_t)(4 + j) << 8) | 0xC000u;
        out[j] = dq_pair<SYM>(__byte_perm(lo, hi, sel), zz, ss);
    }
}

// ------------------------------------------------------------------ warp MMA (decode path)
// D[16x8] += A[16x16] · B[16x8], bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same MMA as a plain (non-volatile) asm statement: it only reads and writes
// registers, so the compiler may schedule it freely among the shared-memory
// loads that feed it.
__device__ __forceinline__ void mma_bf16_16816_nv(float c[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                  uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------ shared memory / mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint4 lds128(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ uint32_t lds_u16(const void* p) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ uint32_t lds_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ void sts_u32(void* p, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
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

// try_wait that lets the hardware suspend the thread until the phase completes
// (or about `hint_ns` pass), so that waiting warps take no issue slots.
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

// Wait for the phase with the given parity to complete; give up after about a
// second, record the error and return false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (global_timer_ns() - t0 > kWaitTimeoutNs) {
            report_error(kErrMbarTimeout);
            return false;
        }
    }
}

// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for a phase, polling with exponentially growing sleeps (32 ns up to
// max_sleep_ns) so that a warp that waits takes almost no issue slots from the
// warps that compute.  For roles off the critical path (a producer refilling a
// deep ring, a helper preparing data ahead).  Bounded like mbar_wait.
__device__ __forceinline__ bool mbar_wait_backoff(uint32_t bar, uint32_t parity, uint32_t max_sleep_ns) {
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    uint32_t ns = 32;
    while (true) {
        __nanosleep(ns);
        if (mbar_test_wait(bar, parity)) return true;
        ns = ns < max_sleep_ns ? 2 * ns : max_sleep_ns;
        if (global_timer_ns() - t0 > kWaitTimeoutNs) {
            report_error(kErrMbarTimeout);
            return false;
        }
    }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t c0,
                                            int32_t c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------ programmatic dependent launch
// Wait until the preceding grid on the stream has completed and its writes are visible.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Let the next grid on the stream (launched with programmatic serialization) start.
__device__ __forceinline__ void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05 / TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t holder_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     holder_smem),
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

// Shared-memory matrix descriptor for a K-major operand in the 128-byte swizzle
// layout: rows of 64 bf16 (128 B), 8-row groups 1024 B apart; the tile base
// must be 1024-byte aligned, the start address may advance by 32 B per K=16 step.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);        // start address
    d |= (uint64_t)(16u >> 4) << 16;                      // leading byte offset (unused here)
    d |= (uint64_t)(1024u >> 4) << 32;                    // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;                               // descriptor version for sm_100
    d |= (uint64_t)2 << 61;                               // 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::f16 with bf16 A and B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int mma_m, int mma_n) {
    return (1u << 4)                          // D = f32
           | (1u << 7)                        // A = bf16
           | (1u << 10)                       // B = bf16
           | ((uint32_t)(mma_n >> 3) << 17)   // N / 8
           | ((uint32_t)(mma_m >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void tc_mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05 ops of this thread complete.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t r[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

}  // namespace w4a16
