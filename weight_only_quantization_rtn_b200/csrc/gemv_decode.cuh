// Decode-path fused W4A16 GEMM for small M (M ≤ 16): persistent, stream-K,
// TMA-fed, one kernel per call.
//
// Decode is bound by reading the weights once from HBM ("推理优化中“用精度换性能“
// 的核心技术：量化", §1 and §3.2; "大模型推理中 Weight-only、W8A8 和 FP8 量化有什么
// 区别？如何选型？", §二: the cost is re-reading large weights for a single token).
// What limits a kernel that streams at HBM rate is the instruction issue of the
// dequantization, so the design spends as few instructions per weight as it can
// outside the core sequence (LOP3 nibble isolation, one bf16x2 subtract of the
// zero point, one bf16x2 multiply by the scale, one mma.sync per 8 codes a thread):
//
//  * Work unit = 256 weight rows x 256 K (32 KB of packed codes, one TMA box of
//    256 rows x 128 bytes with the 128-byte swizzle).  Units, in row-block-major
//    order, are split evenly over a persistent grid of one CTA per SM
//    (stream-K): every SM streams the same number of bytes whatever N and K are.
//    One CTA per SM, not two smaller ones: when the SM is issue bound the warp
//    schedulers favour the older CTA's warps, so a second CTA on an SM fell
//    about 17% behind the first and became the tail; the warps of one CTA are
//    held together by its stage ring instead.
//  * Warp 16 (producer): one lane issues, per unit, the TMA loads of the codes
//    tile and of the X slice (M rows x 256 bf16), completing on the stage's
//    "full" barrier.  Scales and zero points: when a scale row is 16-byte
//    aligned they come by TMA in slabs of 8 groups x 256 rows (one slab serves
//    8/GU consecutive units of a row block), into a ring of slab slots of their
//    own, loaded once per slab rather than once per unit — each slab row is a
//    separate 16-byte request, so re-loading it per unit would triple the
//    requests of the stream; otherwise the 32 lanes copy the unit's groups into
//    the stage with cp.async (plain loads when the rows are misaligned).  When
//    the caller states that the previous grid on the stream does not write the
//    weights, the codes and scales of the first ring's worth of units are
//    requested before the dependency wait, while that grid drains; X follows
//    after the wait.
//  * Warp 17 (helper): once a stage has landed, rewrites its X slice into
//    MMA-fragment order (the pairs (x_j, x_{j+4}) the nibble isolation below
//    produces) in a separate area, and signals "xf".  One warp does this once
//    per stage instead of every consumer thread permuting its own copy.  With a
//    per-input-channel activation scale a[K] (the activation half of the
//    equivalent scaling (X·diag(a))·(diag(a)⁻¹·W) of "推理优化中“用精度换性能“的
//    核心技术：量化", §5.2 and §6.2), the helper also forms x' = bf16_rn(x·a[k])
//    here, one rounding of the exact product, before permuting.
//  * Warps 0..15 (consumers): warp w owns rows 16w .. 16w+15 of every unit, so
//    its accumulators hold whole output rows across the K blocks of a row block
//    and no warp ever waits for another.  Lane (g, q) — g = lane/4, q = lane%4 —
//    reads 16 bytes (32 codes) of rows g and g+8 from 16-byte chunks 2q and
//    2q+1 (with the swizzle these loads hit 32 distinct banks per quarter warp),
//    turns them into bf16 pairs in registers and feeds them as the A operand of
//    m16n8k16 bf16 MMAs with fp32 accumulation; X (B operand) comes from the
//    fragment-ordered area with one 16-byte load per two MMAs.  The MMA reduces
//    over K in fragment order, so the nibble pairs are used in the order the
//    isolation yields them — (q0,q4)(q1,q5)(q2,q6)(q3,q7) — and the helper has
//    permuted X to match.  Two accumulator sets break the MMA dependency chain.
//  * A row block owned entirely by one CTA is rounded and written to Y by each
//    warp for its 16 rows.  A row block that the stream-K partition splits
//    between CTAs c_first .. c_last: every owner but c_first writes its fp32
//    part (per warp, in fragment layout) to the workspace and then a ready flag;
//    c_first — which reaches its part of that row block last, because every CTA
//    visits the row block it shares with its predecessor first and the one it
//    shares with its successor second — waits for the flags (bounded), adds the
//    parts to its own in CTA order and writes Y.  The sum order is fixed, so the
//    result is deterministic, and no second kernel is launched.
//  * Programmatic dependent launch lets the next kernel on the stream start
//    while this one drains; nothing but those static weights is read, and
//    nothing is written, before griddepcontrol.wait.
#pragma once

#include "common.cuh"

namespace w4a16 {

constexpr int kDecRows = 256;                   // weight rows per unit (16 warps x 16)
constexpr int kDecUnitRowBytes = 128;          // code bytes of one row per unit (one TMA box row)
constexpr int kDecPBytes = kDecRows * kDecUnitRowBytes; // code bytes per unit (32 KB)
// K per unit: 256 four-bit or 128 eight-bit codes per 128-byte row
template <int BITS> __host__ __device__ constexpr int dec_block_k() { return kDecUnitRowBytes * 8 / BITS; }
constexpr int kDecConsumers = 16;
constexpr int kDecProducerWarp = kDecConsumers;
constexpr int kDecHelperWarp = kDecConsumers + 1;
constexpr int kDecThreads = (kDecConsumers + 2) * 32;
constexpr int kDecMaxStages = 8;
// X rows of a unit: natural order (BK bf16), and in fragment order padded to
// 64 mod 128 bytes (576 B for 4-bit codes, 320 B for 8-bit codes)
template <int BITS> __host__ __device__ constexpr int dec_x_row_bytes() { return dec_block_k<BITS>() * 2; }
template <int BITS> __host__ __device__ constexpr int dec_xf_row_bytes() { return dec_block_k<BITS>() * 2 + 64; }
constexpr int kDecZeroBytes = 512;              // zero B fragments for columns m >= M
constexpr int kDecMaxSlabs = 8;
constexpr int kDecSlabArrayBytes = kDecRows * 8 * 2;    // 8 groups x 256 rows of bf16
constexpr int kDecSlabBytes = 2 * kDecSlabArrayBytes;   // scales and zeros
// Ready flag of a published part: a signalling-NaN bit pattern, which no
// floating-point arithmetic produces, so stale partial sums are never mistaken
// for it.
constexpr uint32_t kDecFlagReady = 0x7F8A5C3Du;
// Longest sleep between polls of a waiting producer / helper: the ring holds
// several microseconds of data, so a late wake-up costs nothing, while polling
// in a tight loop would take issue slots from the consumer warps.
constexpr uint32_t kDecProducerSleepNs = 256;
constexpr uint32_t kDecHelperSleepNs = 128;

// Unit u -> CTA that owns it under the even split u_c = floor(c·U/C).
__device__ __forceinline__ int64_t owner_of(int64_t u, int64_t U, int64_t C) {
    return ((u + 1) * C - 1) / U;
}

// Order in which a CTA visits its units [u0, u1): the partial row block at the
// start of the range (shared with the previous CTA, which finishes that row
// block), then the row block at its end (shared with the next CTA; this CTA
// finishes it), then the whole row blocks in between.
struct UnitWalk {
    int rb, kb;          // current unit (row block, K block)
    int kbn;             // K blocks per row block
    int rb_first, rb_last, kb_last_end;
    int phase;           // 0: first segment, 1: last segment, 2: middle row blocks
    bool two;            // the range touches more than one row block

    __device__ __forceinline__ void init(int64_t u0, int64_t u1, int kbn_) {
        kbn = kbn_;
        rb_first = (int)(u0 / kbn);
        rb = rb_first;
        kb = (int)(u0 - (int64_t)rb_first * kbn);
        rb_last = (int)((u1 - 1) / kbn);
        kb_last_end = (int)((u1 - 1) - (int64_t)rb_last * kbn) + 1;
        two = rb_last != rb_first;
        phase = 0;
    }
    // True when the current unit is the last of its row block within this CTA.
    __device__ __forceinline__ bool segment_end() const {
        if (phase == 0) return two ? kb == kbn - 1 : kb == kb_last_end - 1;
        if (phase == 1) return kb == kb_last_end - 1;
        return kb == kbn - 1;
    }
    __device__ __forceinline__ void advance() {
        if (phase == 0 && two && kb == kbn - 1) {
            phase = 1;
            rb = rb_last;
            kb = 0;
        } else if (phase == 1 && kb == kb_last_end - 1) {
            phase = 2;
            rb = rb_first + 1;
            kb = 0;
        } else if (phase == 2 && kb == kbn - 1) {
            ++rb;
            kb = 0;
        } else {
            ++kb;
        }
    }
};

struct DecodeArgs {
    const uint16_t* scales;
    const uint16_t* zeros;
    uint16_t* Y;
    const uint16_t* act_scale;   // bf16 [K] per-input-channel activation scale, or null
    uint32_t* ws_flag;    // [(RB + C) slots][16 warps] ready flags
    float* ws_part;       // [(RB + C) slots][16 warps][32 lanes][4·MB] fp32 parts
    int M;
    int N;
    int K;
    int RB;               // row blocks of 256 rows
    int KBn;              // K blocks of 256
    int Gtot;             // scale groups per row (1 for per-channel)
    int stages;
    int stage_bytes;      // multiple of 1024
    int xf_off;           // fragment-ordered X inside a stage
    int sz_off;           // without TMA slabs: scales then zeros in a stage, [2][256 rows][GU] bf16
    int sz_tma;           // 1: scales by TMA into the slab ring
    int slab_off;         // slab ring: `slabs` slots of [2][256 rows][8] bf16 (8 KB each)
    int slabs;
    int sz_copy;          // without TMA: bytes per scale copy, 16, 8 or 4 (cp.async), 2 (plain);
                          // 3: one group per unit, copied as the 4-byte aligned pair holding it
    int early;            // 1: the previous grid does not write the weights; stream them before the dependency wait
    int64_t U;            // units = RB · KBn
};

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, uint32_t src_bytes) {
    // 4-byte async copy global -> shared; bytes beyond src_bytes (0 or 4) are zero-filled.
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async_8(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
    // 16-byte async copy global -> shared; bytes beyond src_bytes (0..16) are zero-filled.
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    // Arrive on the barrier once this thread's earlier cp.async copies have landed.
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint4 lds128_u32addr(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_relaxed_u32(uint32_t* p, uint32_t v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ float4 ld_cg_f4(const float* p) {
    float4 v;
    asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

// Wait until another CTA has published its part (bounded: about one second,
// then the error is recorded and false returned).
__device__ __forceinline__ bool wait_flag(const uint32_t* flag) {
    if (ld_acquire_u32(flag) == kDecFlagReady) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        __nanosleep(64);
        if (ld_acquire_u32(flag) == kDecFlagReady) return true;
        if (global_timer_ns() - t0 > kWaitTimeoutNs) {
            report_error(kErrMbarTimeout);
            return false;
        }
    }
}

// The producer's cp.async copies of a unit's scales (and zeros) when their rows
// are not 16-byte aligned: per array and row, GU·2 bytes as copies of CS bytes,
// lane l taking rows l, l + 32, ... (no integer division in the loop).
template <int GU, int CS>
__device__ __forceinline__ void copy_scale_rows(const DecodeArgs& a, uint32_t sz, int sz_array, int rb,
                                                int g0, int arrays, int lane) {
    constexpr int kPerRow = (GU * 2 + CS - 1) / CS;
    for (int arr = 0; arr < arrays; ++arr) {
        const uint16_t* base = arr == 0 ? a.scales : a.zeros;
#pragma unroll 1
        for (int r = lane; r < kDecRows; r += 32) {
            const int n = rb * kDecRows + r;
            const uint32_t dst = sz + arr * sz_array + r * GU * 2;
#pragma unroll
            for (int t = 0; t < kPerRow; ++t) {
                const int gi = g0 + t * (CS / 2);
                const bool in = n < a.N && gi < a.Gtot;
                const uint16_t* src = base + (in ? (int64_t)n * a.Gtot + gi : 0);
                const uint32_t nb = in ? (uint32_t)CS : 0u;
                if (CS == 16) cp_async_16(dst + t * CS, src, nb);
                else if (CS == 8) cp_async_8(dst + t * CS, src, nb);
                else cp_async_4(dst + t * CS, src, nb);
            }
        }
    }
}

// Rounds a warp's finished 16-row tile to bf16 and stores it: lane (g, q) holds
// D[row g][col 2q, 2q+1] and D[row g+8][col 2q, 2q+1] of each 8-column block.
template <int MB>
__device__ __forceinline__ void decode_store_y(const DecodeArgs& a, const float (&d)[MB][4], int rb,
                                               int w, int g, int q) {
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int m = 8 * mb + 2 * q + (j & 1);
            const int n = rb * kDecRows + 16 * w + g + 8 * (j >> 1);
            if (m < a.M && n < a.N) a.Y[(int64_t)m * a.N + n] = (uint16_t)f32_to_bf16_bits_rn(d[mb][j]);
        }
}

// Four 8-bit codes of a word -> (q0, q1) and (q2, q3) as bf16 pairs of
// bf16_rn((q − z)·s).  The byte placed in a binary32 mantissa gives 2^23 + q
// exactly; subtracting zoff = 2^23 + z leaves q − z (exact), the product with s
// is exact (8-bit by 8-bit significands), and cvt.rn.bf16x2 rounds once.
// Symmetric words are XORed with 0x80808080 by the caller (offset-128 codes,
// zoff = 2^23 + 128).
__device__ __forceinline__ void dq_word8(uint32_t w, float s, float zoff, uint32_t& lo, uint32_t& hi) {
    float f[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        f[i] = (__uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u + (uint32_t)i)) - zoff) * s;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(lo) : "f"(f[1]), "f"(f[0]));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(hi) : "f"(f[3]), "f"(f[2]));
}

template <int MB, bool SYM, int G, int BITS>
__global__ void __launch_bounds__(kDecThreads, 1)
    gemv_decode_kernel(const __grid_constant__ CUtensorMap tmP,
                       const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmS,
                       const __grid_constant__ CUtensorMap tmZ, const DecodeArgs a) {
    // G == 0: per-channel granularity, one scale (and zero) per row for all of K.
    constexpr int BK = dec_block_k<BITS>();            // K per unit
    constexpr int XRB = dec_x_row_bytes<BITS>();
    constexpr int XFRB = dec_xf_row_bytes<BITS>();
    constexpr int GU = G == 0 ? 1 : BK / G;            // scale groups per row per unit
    // Groups per staged scale row: a TMA slab of 8 (16 bytes), else the unit's GU.
    const int SW = a.sz_tma ? 8 : (a.sz_copy == 3 ? 2 : GU);
    const int kSzArray = kDecRows * SW * 2;            // bytes of one scale (or zero) array

    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base (128-byte swizzle atoms), formed by offsetting the
    // shared array itself so that every derived pointer stays in the shared
    // address space and compiles to 32-bit shared loads.
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int S = a.stages;
    const uint32_t stages_u32 = smem_u32(smem);
    const uint8_t* slab_base = smem + a.slab_off;        // 1024-aligned, a.slabs x 4 KB
    const int SL = a.slabs;
    uint8_t* fixed = smem + a.slab_off + SL * kDecSlabBytes;   // 1024-aligned
    const uint8_t* zero_ptr = fixed + 64;              // 64 mod 128: see the consumers' X loads
    const uint32_t zero_u32 = smem_u32(zero_ptr);
    uint64_t* full = reinterpret_cast<uint64_t*>(fixed + 64 + kDecZeroBytes + 64);
    uint64_t* xfb = full + kDecMaxStages;
    uint64_t* empty = xfb + kDecMaxStages;
    uint64_t* sfull = empty + kDecMaxStages;           // slab slot landed
    uint64_t* sempty = sfull + kDecMaxSlabs;           // consumers done with the slab slot
    volatile int* abort_flag = reinterpret_cast<int*>(sempty + kDecMaxSlabs);   // a wait was given up

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t C = gridDim.x;
    const int64_t cta = blockIdx.x;
    const int64_t u0 = cta * a.U / C;
    const int64_t u1 = (cta + 1) * a.U / C;
    const int nunits = (int)(u1 - u0);
    const int M = a.M;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            // TMA expect_tx arrive (+ 32 scale-copying lanes without TMA slabs)
            mbar_init(smem_u32(&full[s]), a.sz_tma ? 1 : 1 + 32);
            mbar_init(smem_u32(&xfb[s]), 1);
            mbar_init(smem_u32(&empty[s]), kDecConsumers);
        }
        for (int t = 0; t < SL; ++t) {
            mbar_init(smem_u32(&sfull[t]), 1);
            mbar_init(smem_u32(&sempty[t]), kDecConsumers);
        }
        *abort_flag = 0;
        fence_mbar_init();
        grid_launch_dependents();            // the next kernel may start as this one drains
    }
    if (warp == kDecHelperWarp) {
        for (int i = lane; i < kDecZeroBytes / 16; i += 32) sts128(zero_u32 + 16 * i, make_uint4(0, 0, 0, 0));
    }
    __syncthreads();

    if (warp == kDecProducerWarp) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&tmP);
            prefetch_tensormap(&tmX);
            if (a.sz_tma) {
                prefetch_tensormap(&tmS);
                if (!SYM) prefetch_tensormap(&tmZ);
            }
        }
        const uint32_t tx = (uint32_t)kDecPBytes + (uint32_t)M * XRB;
        const int arrays = SYM ? 1 : 2;
        int slab_t = -1, slab_rb = -1, slab_j = -1;   // slabs requested so far - 1, current slab
        int slab_slot = SL - 1;                       // slab_t mod SL
        uint32_t slab_ph = 1u;                        // parity of slab_t's use of its slot
        // True when unit (rb, kb) reads a slab other than the last one requested.
        auto new_slab = [&](int rb, int kb) {
            return G != 0 && a.sz_tma && (rb != slab_rb || ((kb * GU) >> 3) != slab_j);
        };
        // Request the slab of unit (rb, kb) (groups kb·GU .. kb·GU + GU − 1; GU divides
        // 8) into the next slot, once the consumers have released that slot.
        auto request_slab = [&](int rb, int kb) -> bool {
            const int j = (kb * GU) >> 3;
            ++slab_t;
            if (++slab_slot == SL) {
                slab_slot = 0;
                slab_ph ^= 1u;
            }
            bool ok = true;
            if (lane == 0) ok = mbar_wait_backoff(smem_u32(&sempty[slab_slot]), slab_ph ^ 1u, kDecProducerSleepNs);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) return false;
            if (lane == 0) {
                const uint32_t sb = smem_u32(&sfull[slab_slot]);
                const uint32_t dst = smem_u32(slab_base + slab_slot * kDecSlabBytes);
                mbar_arrive_expect_tx(sb, (uint32_t)((SYM ? 1 : 2) * kDecSlabArrayBytes));
                tma_load_2d(dst, &tmS, 8 * j, rb * kDecRows, sb);
                if (!SYM) tma_load_2d(dst + kDecSlabArrayBytes, &tmZ, 8 * j, rb * kDecRows, sb);
            }
            slab_rb = rb;
            slab_j = j;
            return true;
        };
        // The weights of unit (rb, kb) into stage s: the codes tile by TMA (the
        // stage's "full" barrier expects the codes and the X slice), and — without
        // TMA slabs — the unit's scales (and zeros), [array][row][GU] bf16.
        auto load_weights = [&](int rb, int kb, int s) {
            const uint32_t st = stages_u32 + (uint32_t)(s * a.stage_bytes);
            const uint32_t bar = smem_u32(&full[s]);
            if (lane == 0) {
                mbar_arrive_expect_tx(bar, tx);
                tma_load_2d(st, &tmP, kb * kDecUnitRowBytes, rb * kDecRows, bar);
            }
            const uint32_t sz = st + (uint32_t)a.sz_off;
            if (G != 0 && a.sz_tma) {
                // scales come with the slab ring
            } else if constexpr (G == 0) {
                // per-channel: the row block's contiguous, 16-byte aligned scales (and zeros)
                for (int e = lane; e < (kDecRows / 8) * arrays; e += 32) {
                    const int arr = e / (kDecRows / 8), j = e % (kDecRows / 8);
                    const int n = rb * kDecRows + 8 * j;
                    const int valid = min(max(a.N - n, 0), 8);
                    const uint16_t* src = (arr == 0 ? a.scales : a.zeros) + (valid > 0 ? n : 0);
                    cp_async_16(sz + arr * kSzArray + 16 * j, src, 2u * (uint32_t)valid);
                }
                cp_async_arrive_noinc(bar);
            } else {
                const int g0 = kb * GU;
                const int cs = a.sz_copy;
                if (cs >= 4) {
                    // per row, GU·2 bytes as copies of cs bytes; Gtot·2 and g0·2 are multiples
                    // of cs, so a copy never straddles the end of a scale row
                    // (the host picks cs ≤ GU·2; instances with larger copies are never built)
                    if constexpr (GU * 2 >= 16) {
                        if (cs == 16) copy_scale_rows<GU, 16>(a, sz, kSzArray, rb, g0, arrays, lane);
                    }
                    if constexpr (GU * 2 >= 8) {
                        if (cs == 8) copy_scale_rows<GU, 8>(a, sz, kSzArray, rb, g0, arrays, lane);
                    }
                    if (cs == 4) copy_scale_rows<GU, 4>(a, sz, kSzArray, rb, g0, arrays, lane);
                    cp_async_arrive_noinc(bar);
                } else if (cs == 3) {
                    // one group per unit (8-bit codes at g = 128) and an even number of
                    // groups per row: the 4-byte aligned pair of groups holding g0, per row
                    // (the consumers read its half g0 mod 2)
                    if constexpr (GU == 1) {
                        const int gp = g0 & ~1;
                        for (int arr = 0; arr < arrays; ++arr) {
                            const uint16_t* base = arr == 0 ? a.scales : a.zeros;
#pragma unroll 4
                            for (int r = lane; r < kDecRows; r += 32) {
                                const int n = rb * kDecRows + r;
                                const bool in = n < a.N && gp < a.Gtot;
                                cp_async_4(sz + arr * kSzArray + r * 4, base + (in ? (int64_t)n * a.Gtot + gp : 0),
                                           in ? 4u : 0u);
                            }
                        }
                    }
                    cp_async_arrive_noinc(bar);
                } else {
                    // odd scale rows: two bytes at a time, eight loads in flight per lane
                    const int total = kDecRows * GU * arrays;
#pragma unroll 1
                    for (int e0 = lane; e0 < total; e0 += 32 * 8) {
                        uint16_t v[8];
#pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            const int e = e0 + 32 * t;
                            v[t] = 0;
                            if (e < total) {
                                const int arr = e / (kDecRows * GU);
                                const int rem = e - arr * (kDecRows * GU);
                                const int r = rem / GU, j = rem - r * GU;
                                const int n = rb * kDecRows + r;
                                const uint16_t* src = arr == 0 ? a.scales : a.zeros;
                                if (n < a.N && g0 + j < a.Gtot) v[t] = ldg_u16(src + (int64_t)n * a.Gtot + g0 + j);
                            }
                        }
#pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            const int e = e0 + 32 * t;
                            if (e < total) {
                                const int arr = e / (kDecRows * GU);
                                const int rem = e - arr * (kDecRows * GU);
                                const int r = rem / GU, j = rem - r * GU;
                                asm volatile("st.shared.u16 [%0], %1;" ::"r"(sz + arr * kSzArray + (r * SW + j) * 2),
                                             "h"(v[t])
                                             : "memory");
                            }
                        }
                    }
                    mbar_arrive(bar);
                }
            }
        };
        auto load_x = [&](int kb, int s) {
            if (lane == 0)
                tma_load_2d(stages_u32 + (uint32_t)(s * a.stage_bytes) + kDecPBytes, &tmX, kb * BK, 0,
                            smem_u32(&full[s]));
        };

        UnitWalk wk;
        wk.init(u0, u1, a.KBn);
        // With weights that the previous grid on the stream does not write, the
        // first ring's worth of units (as far as their slabs fit the slab ring
        // without waiting for a release) is requested before the dependency
        // wait, so the weight stream starts while the previous grid drains; only
        // X waits.  Otherwise nothing is read before the wait.
        int P = 0;
        bool ok = true;
        if (a.early) {
            const int pmax = min(S, nunits);
            for (; P < pmax; ++P) {
                UnitWalk nx = wk;
                if (P > 0) nx.advance();
                if (new_slab(nx.rb, nx.kb)) {
                    if (slab_t + 1 >= SL) break;
                    if (!request_slab(nx.rb, nx.kb)) {   // a fresh slot: no wait
                        ok = false;
                        break;
                    }
                }
                wk = nx;
                load_weights(wk.rb, wk.kb, P);
            }
        }
        grid_dependency_wait();              // X (and, without `early`, the weights) may be the previous grid's output
        if (P > 0) {
            UnitWalk xw;
            xw.init(u0, u1, a.KBn);
            for (int i = 0; i < P; ++i) {
                if (i > 0) xw.advance();
                load_x(xw.kb, i);
            }
        }
        int issued = P;
        int s = P > 0 ? P - 1 : 0;
        uint32_t ph = 0;
        for (int i = P; i < nunits && ok; ++i) {
            if (i > 0) {
                wk.advance();
                if (++s == S) { s = 0; ph ^= 1u; }
            }
            const int rb = wk.rb, kb = wk.kb;
            if (lane == 0) ok = mbar_wait_backoff(smem_u32(&empty[s]), ph ^ 1u, kDecProducerSleepNs);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                ok = false;
                break;
            }
            if (new_slab(rb, kb) && !request_slab(rb, kb)) {
                ok = false;
                break;
            }
            load_weights(rb, kb, s);
            load_x(kb, s);
            ++issued;
        }
        if (!ok) *abort_flag = 1;
        // Do not leave while copies into this CTA's shared memory are in flight.
        if (lane == 0) {
            for (int i = (issued > S ? issued - S : 0); i < issued; ++i) {
                if (!mbar_wait(smem_u32(&full[i % S]), (uint32_t)(i / S) & 1u)) break;
            }
            const int nslab = slab_t + 1;
            for (int t = (nslab > SL ? nslab - SL : 0); t < nslab; ++t) {
                if (!mbar_wait(smem_u32(&sfull[t % SL]), (uint32_t)(t / SL) & 1u)) break;
            }
        }
        return;
    }

    if (warp == kDecHelperWarp) {
        // ---------------------------------------------------------------- helper
        // X slice of each landed stage, natural order [m][BK] -> fragment order.
        // 4-bit codes: 16-byte chunk c = 8q + i of row m (elements x0..x7) becomes
        // ((x0,x4),(x1,x5),(x2,x6),(x3,x7)) at row m, slot i, lane-group q.
        // 8-bit codes: chunk c = 4q + i moves unchanged to slot i, lane-group q.
        int s = 0;
        uint32_t ph = 0;
        UnitWalk wk;
        wk.init(u0, u1, a.KBn);
        const uint16_t* act = a.act_scale;
        if (act != nullptr) grid_dependency_wait();   // the scales may be the previous grid's output
        for (int i = 0; i < nunits; ++i) {
            if (i > 0) {
                wk.advance();
                if (++s == S) { s = 0; ph ^= 1u; }
            }
            bool ok = mbar_test_wait(smem_u32(&full[s]), ph);
            if (!ok && *abort_flag == 0) ok = mbar_wait_backoff(smem_u32(&full[s]), ph, kDecHelperSleepNs);
            if (!ok) {
                *abort_flag = 1;
                break;
            }
            const uint32_t st = stages_u32 + (uint32_t)(s * a.stage_bytes);
            const uint32_t xn = st + kDecPBytes;
            const uint32_t xf = st + (uint32_t)a.xf_off;
#pragma unroll 1
            for (int it = lane; it < M * (BK / 8); it += 32) {
                constexpr int kShift = BITS == 4 ? 5 : 4;    // chunks of 8 per X row: 32 or 16
                const int m = it >> kShift, c = it & ((1 << kShift) - 1);
                uint4 v = lds128_u32addr(xn + m * XRB + c * 16);
                if (act != nullptr) {
                    // x' = bf16_rn(x·a): the chunk's 8 scales (K is a multiple of 32, so a
                    // chunk is wholly inside or wholly past the end of X, where x = 0)
                    const int k0 = wk.kb * BK + 8 * c;
                    const uint4 av = k0 < a.K ? ldg_cached(act + k0) : make_uint4(0, 0, 0, 0);
                    v.x = bf16x2_mul(v.x, av.x);
                    v.y = bf16x2_mul(v.y, av.y);
                    v.z = bf16x2_mul(v.z, av.z);
                    v.w = bf16x2_mul(v.w, av.w);
                }
                if constexpr (BITS == 4) {
                    uint4 o;
                    o.x = __byte_perm(v.x, v.z, 0x5410);   // (x0, x4)
                    o.y = __byte_perm(v.x, v.z, 0x7632);   // (x1, x5)
                    o.z = __byte_perm(v.y, v.w, 0x5410);   // (x2, x6)
                    o.w = __byte_perm(v.y, v.w, 0x7632);   // (x3, x7)
                    sts128(xf + m * XFRB + (c & 7) * 64 + (c >> 3) * 16, o);
                } else {
                    sts128(xf + m * XFRB + (c & 3) * 64 + (c >> 2) * 16, v);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&xfb[s]));
        }
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int w = warp;                     // rows 16w .. 16w+15 of every unit
    const int g = lane >> 2;
    const int q = lane & 3;
    // Codes of rows r0 = 16w + g and r0 + 8 (1024 bytes further), chunk 2q + h:
    // the 128-byte swizzle puts logical chunk c of row r at chunk c ^ (r % 8).
    const uint32_t a_off0 = (uint32_t)((16 * w + g) * 128 + (((2 * q) ^ g) * 16));
    const uint32_t a_off1 = (uint32_t)((16 * w + g) * 128 + (((2 * q + 1) ^ g) * 16));
    // This lane's B fragments: fragment-ordered X row g (and g + 8), or zeros for
    // columns beyond M.
    const bool col0 = g < M;
    const bool col1 = MB > 1 && g + 8 < M;
    const int xf0 = a.xf_off + g * XFRB + q * 16;
    const int xf1 = a.xf_off + (g + 8) * XFRB + q * 16;
    const uint4* zero_lane = reinterpret_cast<const uint4*>(zero_ptr) + q;
    // Scale (and zero) byte offsets of rows r0 and r0 + 8 for the groups of this
    // lane's two chunks (4-bit: K = 64q + 32h within the unit; 8-bit: K = 32q +
    // 16h, one group for both as g ≥ 32).
    constexpr int kG = G == 0 ? 1 : G;
    const int sgrp0 = G == 0 ? 0 : ((BITS == 4 ? 64 : 32) * q) / kG;
    const int sgrp1 = G == 0 ? 0 : ((BITS == 4 ? 64 : 32) * q + (BITS == 4 ? 32 : 16)) / kG;
    const int srow0 = (16 * w + g) * SW * 2;         // within the stage's scale area or a slab
    const int srow8 = 8 * SW * 2;                     // row r0 + 8
    const bool tma_slab = G != 0 && a.sz_tma;
    int slab_rb = -1, slab_j = -1;                   // the slab the consumers read
    int slab_slot = -1;                              // its slot (-1: none yet)
    uint32_t slab_ph = 1u;                           // parity of its use of the slot
    const uint8_t* slab_ptr = slab_base;
    const uint32_t nib = opaque_u32(0x000F000Fu);     // nibble-pair mask, held in a register
    const uint32_t zz_sym = opaque_u32(0x43084308u);  // 128 + 8 for symmetric codes

    float acc[2][MB][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[t][mb][j] = 0.0f;

    grid_dependency_wait();                 // Y and the workspace may be in use by the previous grid
    // Segments of this CTA's units in visiting order (see UnitWalk): the first
    // row block's part, the last row block's part, then the whole row blocks.
    const int rb_first = (int)(u0 / a.KBn);
    const int rb_last = (int)((u1 - 1) / a.KBn);
    const int kb_first = (int)(u0 - (int64_t)rb_first * a.KBn);
    const int kb_last_end = (int)((u1 - 1) - (int64_t)rb_last * a.KBn) + 1;
    const bool two = rb_last != rb_first;
    const int nseg = two ? 2 + (rb_last - rb_first - 1) : 1;
    int s = 0;
    uint32_t ph = 0;
    const uint8_t* stp = smem;
    for (int sg = 0; sg < nseg; ++sg) {
        int rb, kb0, kb1;
        if (sg == 0) {
            rb = rb_first; kb0 = kb_first; kb1 = two ? a.KBn : kb_last_end;
        } else if (sg == 1) {
            rb = rb_last; kb0 = 0; kb1 = kb_last_end;
        } else {
            rb = rb_first + sg - 1; kb0 = 0; kb1 = a.KBn;
        }
        for (int kb = kb0; kb < kb1; ++kb) {
            // Once any wait has been given up, skip the remaining work; every
            // role still runs its loop to the end, so the CTA exits.  The helper
            // signals xf only after the stage's copies landed, so this one wait
            // also orders the reads of the codes and scales after them.
            bool have = mbar_try_wait(smem_u32(&xfb[s]), ph);
            if (!have && *abort_flag == 0) {
                have = mbar_wait(smem_u32(&xfb[s]), ph);
                if (!have) *abort_flag = 1;
            }
            if (have) {
                const uint4* xp0 = col0 ? reinterpret_cast<const uint4*>(stp + xf0) : zero_lane;
                const uint4* xp1 = col1 ? reinterpret_cast<const uint4*>(stp + xf1) : zero_lane;
                const uint8_t* sb;
                if (tma_slab) {
                    // move to the unit's slab when it changes: release the old slot, wait for the new
                    const int j = (kb * GU) >> 3;
                    if (rb != slab_rb || j != slab_j) {
                        if (slab_slot >= 0) {
                            __syncwarp();
                            if (lane == 0) mbar_arrive(smem_u32(&sempty[slab_slot]));
                        }
                        if (++slab_slot == SL) slab_slot = 0;
                        if (slab_slot == 0) slab_ph ^= 1u;
                        if (!mbar_wait(smem_u32(&sfull[slab_slot]), slab_ph)) {
                            *abort_flag = 1;
                            have = false;
                        }
                        slab_ptr = slab_base + slab_slot * kDecSlabBytes;
                        slab_rb = rb;
                        slab_j = j;
                    }
                    // the unit's groups start at (kb·GU) mod 8 within a slab row
                    sb = slab_ptr + srow0 + ((kb * GU) & 7) * 2;
                } else {
                    // (pair copies: the unit's group is the half g0 mod 2 of its 4 bytes)
                    sb = stp + a.sz_off + srow0 + (a.sz_copy == 3 ? ((kb * GU) & 1) * 2 : 0);
                }
                if (have) {
                if constexpr (BITS == 4) {
                // scale and zero pairs of rows r0, r0 + 8 for chunk h = 0 (and h = 1 when
                // the two chunks lie in different groups)
                uint32_t ss[2][2], zz[2][2];
#pragma unroll
                for (int h = 0; h < (G == 32 ? 2 : 1); ++h) {
                    const uint8_t* sh = sb + (h == 0 ? sgrp0 : sgrp1) * 2;
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const uint8_t* sr = sh + hr * srow8;
                        ss[h][hr] = __byte_perm((uint32_t)*reinterpret_cast<const uint16_t*>(sr), 0, 0x1010);
                        zz[h][hr] = SYM ? zz_sym
                                        : bf16x2_add(__byte_perm((uint32_t)*reinterpret_cast<const uint16_t*>(
                                                                     sr + (tma_slab ? kDecSlabArrayBytes : kSzArray)),
                                                                 0, 0x1010),
                                                     0x43004300u);
                    }
                }
                if (G != 32) {
                    ss[1][0] = ss[0][0]; ss[1][1] = ss[0][1];
                    zz[1][0] = zz[0][0]; zz[1][1] = zz[0][1];
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint8_t* ap = stp + (h == 0 ? a_off0 : a_off1);
                    const uint4 va = *reinterpret_cast<const uint4*>(ap);
                    const uint4 vb = *reinterpret_cast<const uint4*>(ap + 1024);
                    const uint32_t w0[4] = {va.x, va.y, va.z, va.w};
                    const uint32_t w1[4] = {vb.x, vb.y, vb.z, vb.w};
                    uint4 xv0[4], xv1[4];
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii) {
                        xv0[ii] = xp0[(4 * h + ii) * 4];
                        xv1[ii] = MB > 1 ? xp1[(4 * h + ii) * 4] : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii) {
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            // fragment registers in the order the MMA reads them:
                            // (row g, k-pair lo) (row g+8, lo) (row g, hi) (row g+8, hi)
                            const uint32_t f0 = dq_pair_m<SYM>(w0[ii] >> (8 * hh), nib, zz[h][0], ss[h][0]);
                            const uint32_t f1 = dq_pair_m<SYM>(w1[ii] >> (8 * hh), nib, zz[h][1], ss[h][1]);
                            const uint32_t f2 = dq_pair_m<SYM>(w0[ii] >> (8 * hh + 4), nib, zz[h][0], ss[h][0]);
                            const uint32_t f3 = dq_pair_m<SYM>(w1[ii] >> (8 * hh + 4), nib, zz[h][1], ss[h][1]);
                            const uint32_t b0 = hh == 0 ? xv0[ii].x : xv0[ii].z;
                            const uint32_t b1 = hh == 0 ? xv0[ii].y : xv0[ii].w;
                            mma_bf16_16816_nv(acc[hh][0], f0, f1, f2, f3, b0, b1);
                            if (MB > 1) {
                                const uint32_t c0 = hh == 0 ? xv1[ii].x : xv1[ii].z;
                                const uint32_t c1 = hh == 0 ? xv1[ii].y : xv1[ii].w;
                                mma_bf16_16816_nv(acc[hh][MB - 1], f0, f1, f2, f3, c0, c1);
                            }
                        }
                    }
                }
                } else {
                    // 8-bit codes: one scale group per lane and unit; s and 2^23 + z in binary32
                    float sf[2], zf[2];
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const uint8_t* sr = sb + sgrp0 * 2 + hr * srow8;
                        sf[hr] = bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(sr));
                        zf[hr] = SYM ? 8388736.0f
                                     : 8388608.0f + bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(
                                                        sr + (tma_slab ? kDecSlabArrayBytes : kSzArray)));
                    }
                    const uint32_t flip = SYM ? 0x80808080u : 0u;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint8_t* ap = stp + (h == 0 ? a_off0 : a_off1);
                        const uint4 va = *reinterpret_cast<const uint4*>(ap);
                        const uint4 vb = *reinterpret_cast<const uint4*>(ap + 1024);
                        const uint32_t w0[4] = {va.x ^ flip, va.y ^ flip, va.z ^ flip, va.w ^ flip};
                        const uint32_t w1[4] = {vb.x ^ flip, vb.y ^ flip, vb.z ^ flip, vb.w ^ flip};
                        // X of this lane's chunk: 16 values at slots 2h, 2h + 1
                        uint4 xv0[2], xv1[2];
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            xv0[j] = xp0[(2 * h + j) * 4];
                            xv1[j] = MB > 1 ? xp1[(2 * h + j) * 4] : make_uint4(0, 0, 0, 0);
                        }
#pragma unroll
                        for (int ii = 0; ii < 4; ++ii) {
                            // word ii = codes K .. K+3: (q0,q1) as the low k pair, (q2,q3) high
                            uint32_t f0, f1, f2, f3;
                            dq_word8(w0[ii], sf[0], zf[0], f0, f2);
                            dq_word8(w1[ii], sf[1], zf[1], f1, f3);
                            const uint4 xa = xv0[ii >> 1];
                            mma_bf16_16816_nv(acc[ii & 1][0], f0, f1, f2, f3, (ii & 1) ? xa.z : xa.x,
                                              (ii & 1) ? xa.w : xa.y);
                            if (MB > 1) {
                                const uint4 xb = xv1[ii >> 1];
                                mma_bf16_16816_nv(acc[ii & 1][MB - 1], f0, f1, f2, f3, (ii & 1) ? xb.z : xb.x,
                                                  (ii & 1) ? xb.w : xb.y);
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
                }
            }
            if (++s == S) {
                s = 0;
                ph ^= 1u;
                stp = smem;
            } else {
                stp += a.stage_bytes;
            }
        }

        // ---------------------------------------------------------------- row block done
        float d[MB][4];
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                d[mb][j] = acc[0][mb][j] + acc[1][mb][j];
                acc[0][mb][j] = 0.0f;
                acc[1][mb][j] = 0.0f;
            }
        if (*abort_flag != 0) continue;
        // The row block is whole here iff all its units lie in this CTA's range.
        const int64_t first_u = (int64_t)rb * a.KBn;
        const bool whole = first_u >= u0 && first_u + a.KBn <= u1;
        if (whole) {
            decode_store_y<MB>(a, d, rb, w, g, q);
            continue;
        }
        const int64_t c_first = owner_of(first_u, a.U, C);
        const int64_t c_last = owner_of(first_u + a.KBn - 1, a.U, C);
        if (cta != c_first) {
            // publish this CTA's part, then its ready flag
            const int64_t slot = rb + cta;
            float* part = a.ws_part + ((slot * kDecConsumers + w) * 32 + lane) * (4 * MB);
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
                *reinterpret_cast<float4*>(part + 4 * mb) = make_float4(d[mb][0], d[mb][1], d[mb][2], d[mb][3]);
            __threadfence();                                 // every lane's part, before the flag
            __syncwarp();
            if (lane == 0) st_relaxed_u32(a.ws_flag + slot * kDecConsumers + w, kDecFlagReady);
            continue;
        }
        // first owner: wait until every other owner has published (each lane
        // acquires the flags itself, so its reads of the parts follow them), load
        // the parts eight at a time, four with two column blocks (one round trip
        // for most row blocks), and add them in CTA order, then write Y
        bool ok = true;
        for (int64_t p = c_first + 1; p <= c_last && ok; ++p)
            ok = wait_flag(a.ws_flag + (rb + p) * kDecConsumers + w);
        if (!__all_sync(0xffffffffu, ok ? 1 : 0)) {
            *abort_flag = 1;
            continue;
        }
        constexpr int PB = 8 / MB;           // parts per round trip, within the register budget
        for (int64_t p0 = c_first + 1; p0 <= c_last; p0 += PB) {
            float4 v[PB][MB];
#pragma unroll
            for (int k = 0; k < PB; ++k)
#pragma unroll
                for (int mb = 0; mb < MB; ++mb)
                    v[k][mb] = p0 + k <= c_last
                                   ? ld_cg_f4(a.ws_part + (((rb + p0 + k) * kDecConsumers + w) * 32 + lane) *
                                                              (4 * MB) + 4 * mb)
                                   : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
            for (int k = 0; k < PB; ++k) {
                if (p0 + k > c_last) break;
#pragma unroll
                for (int mb = 0; mb < MB; ++mb) {
                    d[mb][0] += v[k][mb].x; d[mb][1] += v[k][mb].y;
                    d[mb][2] += v[k][mb].z; d[mb][3] += v[k][mb].w;
                }
            }
        }
        __syncwarp();
        if (lane == 0)                                        // consumed: the slots are free again
            for (int64_t p = c_first + 1; p <= c_last; ++p)
                st_relaxed_u32(a.ws_flag + (rb + p) * kDecConsumers + w, 0u);
        decode_store_y<MB>(a, d, rb, w, g, q);
    }
}

}  // namespace w4a16
