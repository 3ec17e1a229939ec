// Decode-path fused W4A16 GEMM for small M (M ≤ 16): persistent, stream-K,
// TMA-fed.
//
// Decode is bound by reading the weights once from HBM (qwbw.cn,
// "推理优化中“用精度换性能“的核心技术：量化", §1 and §3.2; aigcbaba selection page
// §二: the bottleneck is re-reading large weights for a single token).  The
// kernel keeps HBM busy with deep asynchronous copies and spends as few
// instructions as possible per weight:
//
//  * Work unit = 32 weight rows x 1024 K (16 KB of packed codes).  The units,
//    in row-block-major order, are split evenly over a persistent grid of
//    CTAs (stream-K), so every SM streams the same number of bytes whatever
//    N and K are.
//  * Warp 8 is the producer: one lane issues, per unit, TMA loads of the packed
//    tile (4 boxes of 32 rows x 128 B, 128-byte swizzle) and of the X slice
//    (4 boxes of M rows x 256 elements) into a ring of shared-memory stages,
//    completing on the stage's "full" barrier.
//  * Warps 0..7 are consumers.  Warp w takes K chunk w (128 wide) of both
//    16-row tiles of the unit.  Lane (g, q) — g = lane/4, q = lane%4 — reads
//    16 bytes (32 codes) of rows g and g+8 of each tile, turns them into bf16
//    pairs in registers (LOP3 nibble isolation + exponent magic, one bf16x2
//    subtract of the zero point, one bf16x2 multiply by the scale) and uses
//    them directly as the A operand of m16n8k16 bf16 MMAs with fp32
//    accumulation; X supplies the B operand (M ≤ 8: one n8 MMA, M ≤ 16: two).
//    The MMA reduces over K in fragment order, so the nibble pairs are used in
//    the order the isolation yields them — (q0,q4)(q1,q5)(q2,q6)(q3,q7) — and
//    the X pairs are permuted to match with PRMT.
//  * The unit's scales and zero points land in the same stage and complete on
//    the same barrier, so consumers never wait on them: by TMA (boxes of 32
//    rows x 1024/g groups) when a scale row is 16-byte aligned; otherwise the
//    producer warp's 32 lanes copy them with 4-byte cp.async copies
//    (zero-filled outside the matrix), or with plain loads and stores when the
//    scale stride is not 4-byte aligned.  Per-channel (g = K, template G = 0):
//    the row block's 32 scales (and zeros) are contiguous, and 4 (8) lanes copy
//    them with 16-byte cp.async copies.
//  * At the end of a row block the 8 warps' partial tiles are summed in shared
//    memory in a fixed order and written to Y.  A row block that the stream-K
//    partition splits between CTAs is written instead as one fp32 partial per
//    CTA; a small second kernel, chained by programmatic dependent launch, adds
//    the parts in CTA (= K) order and writes Y.  No CTA ever waits on another,
//    so the split costs no synchronization latency inside the streaming kernel,
//    and the result is deterministic.
//  * Programmatic dependent launch lets the next kernel on the stream start
//    while this one drains: its CTAs are placed, set up their barriers and
//    prefetch their tensor maps, then wait (griddepcontrol.wait) before any
//    memory access.
#pragma once

#include "common.cuh"

namespace w4a16 {

constexpr int kDecRows = 32;                    // weight rows per unit
constexpr int kDecBlockK = 1024;                // K per unit
constexpr int kDecPBytes = kDecRows * kDecBlockK / 2;   // packed bytes per unit (16 KB)
constexpr int kDecConsumers = 8;
constexpr int kDecThreads = (kDecConsumers + 1) * 32;
constexpr int kDecMaxStages = 8;

// Unit u -> CTA that owns it under the even split u_c = floor(c·U/C).
__device__ __forceinline__ int64_t owner_of(int64_t u, int64_t U, int64_t C) {
    return ((u + 1) * C - 1) / U;
}

// Order in which a CTA visits its units [u0, u1): the partial row block at the
// start of the range, then the partial row block at its end, then the whole row
// blocks in between.  Row blocks shared with neighbouring CTAs are therefore
// finished first, and their cross-CTA reduction overlaps the streaming of the
// whole row blocks instead of sitting at the end of the CTA.
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
    float* ws_part;       // [(RB + C) slots][256·MB] fp32 partial row blocks
    int M;
    int N;
    int K;
    int RB;               // row blocks of 32 rows
    int KBn;              // K blocks of 1024
    int stages;
    int stage_bytes;      // packed + X + scale/zero bytes per stage (multiple of 1024)
    int sz_offset;        // offset of the scale/zero block inside a stage
    int sz_async;         // 1: scale rows are 4-byte aligned, copy with cp.async
    int sz_tma;           // 1: scale rows are 16-byte aligned, copy with TMA (tmS, tmZ)
    int64_t U;            // units = RB · KBn
};

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, uint32_t src_bytes) {
    // 4-byte async copy global -> shared; bytes beyond src_bytes (0 or 4) are zero-filled.
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
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

template <int MB, bool SYM, int G>
__global__ void __launch_bounds__(kDecThreads, MB == 1 ? 2 : 1)
    gemv_decode_kernel(const __grid_constant__ CUtensorMap tmP,
                       const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmS,
                       const __grid_constant__ CUtensorMap tmZ, const DecodeArgs a) {
    // G == 0: per-channel granularity, one scale (and zero) per row for all of K.
    constexpr int kG = G == 0 ? 1 : G;                 // divisor for the grouped forms
    constexpr int GB = G == 0 ? 1 : kDecBlockK / kG;   // groups per row per unit
    constexpr int RED = 2 * MB * 128;                  // partial elements per row block

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int S = a.stages;
    uint8_t* stages = smem;                                            // S x stage_bytes
    float* red = reinterpret_cast<float*>(stages + S * a.stage_bytes); // [8][RED]
    uint64_t* full = reinterpret_cast<uint64_t*>(red + kDecConsumers * RED);
    uint64_t* empty = full + kDecMaxStages;
    volatile int* abort_flag = reinterpret_cast<int*>(empty + kDecMaxStages);   // a wait was given up

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t C = gridDim.x;
    const int64_t cta = blockIdx.x;
    const int64_t u0 = cta * a.U / C;
    const int64_t u1 = (cta + 1) * a.U / C;
    const int nunits = (int)(u1 - u0);
    const int M = a.M;
    const uint32_t xbox_bytes = (uint32_t)M * 512u;
    const int Gtot = G == 0 ? 1 : a.K / kG;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            // TMA expect_tx arrive (+ 32 scale-copying lanes when scales are not copied by TMA)
            mbar_init(smem_u32(&full[s]), a.sz_tma ? 1 : 1 + 32);
            mbar_init(smem_u32(&empty[s]), kDecConsumers);
        }
        *abort_flag = 0;
        fence_mbar_init();
        grid_launch_dependents();            // the next kernel may start as this one drains
    }
    __syncthreads();

    if (warp == kDecConsumers) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&tmP);
            prefetch_tensormap(&tmX);
            if (a.sz_tma) {
                prefetch_tensormap(&tmS);
                if (!SYM) prefetch_tensormap(&tmZ);
            }
        }
        const uint32_t sz_tx = a.sz_tma ? (uint32_t)((SYM ? 1 : 2) * kDecRows * GB * 2) : 0u;
        const uint32_t tx = (uint32_t)kDecPBytes + 4u * xbox_bytes + sz_tx;
        // Nothing is requested before the preceding grid has completed.  Weights
        // do not depend on it, but requesting them early was measured to be
        // slower: CTAs that start while the previous grid drains would prefetch
        // their ring while the last-placed CTAs start cold, which staggers their
        // finish, and the early requests compete with the drain for HBM.
        grid_dependency_wait();
        UnitWalk wk;
        wk.init(u0, u1, a.KBn);
        int issued = 0;
        int s = 0;
        uint32_t ph = 0;
        for (int i = 0; i < nunits; ++i) {
            if (i > 0) {
                wk.advance();
                if (++s == S) { s = 0; ph ^= 1u; }
            }
            const int rb = wk.rb, kb = wk.kb;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(smem_u32(&empty[s]), ph ^ 1u);   // one lane waits
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            uint8_t* st = stages + s * a.stage_bytes;
            const uint32_t bar = smem_u32(&full[s]);
            if (lane == 0) {
                mbar_arrive_expect_tx(bar, tx);
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    tma_load_2d(smem_u32(st + b * 4096), &tmP, kb * 512 + b * 128, rb * kDecRows, bar);
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    tma_load_2d(smem_u32(st + kDecPBytes + b * xbox_bytes), &tmX,
                                kb * kDecBlockK + b * 256, 0, bar);
            }
            // scales (and zeros): 32 rows x GB groups
            uint16_t* sz = reinterpret_cast<uint16_t*>(st + a.sz_offset);
            const int g0 = G == 0 ? 0 : kb * GB;
            const int arrays = SYM ? 1 : 2;
            if constexpr (G == 0) {
                // per-channel: the row block's 32 scales (and zeros) are 64 contiguous,
                // 16-byte aligned bytes; lanes 0-3 copy the scales, 4-7 the zeros
                if (lane < 4 * arrays) {
                    const int arr = lane >> 2, j = lane & 3;
                    const int n = rb * kDecRows + 8 * j;
                    const int valid = min(max(a.N - n, 0), 8);
                    const uint16_t* src = (arr == 0 ? a.scales : a.zeros) + (valid > 0 ? n : 0);
                    cp_async_16(smem_u32(sz + arr * kDecRows + 8 * j), src, 2u * (uint32_t)valid);
                }
                cp_async_arrive_noinc(bar);
            } else if (a.sz_tma) {
                if (lane == 0) {
                    tma_load_2d(smem_u32(sz), &tmS, g0, rb * kDecRows, bar);
                    if (!SYM) tma_load_2d(smem_u32(sz + kDecRows * GB), &tmZ, g0, rb * kDecRows, bar);
                }
            } else if (a.sz_async) {
                // lane -> consecutive group pairs of a row
#pragma unroll 1
                for (int e = lane; e < kDecRows * (GB / 2); e += 32) {
                    const int r = e / (GB / 2);
                    const int j = 2 * (e % (GB / 2));
                    const int n = rb * kDecRows + r;
                    const bool in = n < a.N && g0 + j < Gtot;    // Gtot even: pairs never straddle
                    const int64_t off = in ? (int64_t)n * Gtot + g0 + j : 0;
                    for (int arr = 0; arr < arrays; ++arr) {
                        const uint16_t* src = (arr == 0 ? a.scales : a.zeros) + off;
                        cp_async_4(smem_u32(sz + arr * kDecRows * GB + r * GB + j), src, in ? 4u : 0u);
                    }
                }
                cp_async_arrive_noinc(bar);
            } else {
#pragma unroll 1
                for (int e = lane; e < kDecRows * GB; e += 32) {
                    const int r = e / GB;
                    const int j = e % GB;
                    const int n = rb * kDecRows + r;
                    const bool in = n < a.N && g0 + j < Gtot;
                    const int64_t off = (int64_t)n * Gtot + g0 + j;
                    for (int arr = 0; arr < arrays; ++arr) {
                        const uint16_t* src = arr == 0 ? a.scales : a.zeros;
                        sz[arr * kDecRows * GB + r * GB + j] = in ? ldg_u16(src + off) : (uint16_t)0;
                    }
                }
                mbar_arrive(bar);
            }
            ++issued;
        }
        // Do not leave while copies into this CTA's shared memory are in flight.
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i) {
            if (!mbar_wait(smem_u32(&full[i % S]), (uint32_t)(i / S) & 1u)) break;
        }
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int tid = threadIdx.x;            // 0..255
    const int g = lane >> 2;
    const int q = lane & 3;
    const int c = warp;                     // K chunk of the unit: k = 128·c .. 128·c+127
    const int grp_local = G == 0 ? 0 : (c * 128 + 32 * q) / kG;   // this lane's group in the unit

    float acc[2][MB][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[t][mb][j] = 0.0f;

    const bool m_ok0 = g < M;
    const bool m_ok1 = MB > 1 && (8 + g) < M;

    grid_dependency_wait();                 // Y and the workspace may be in use by the previous grid
    UnitWalk wk;
    wk.init(u0, u1, a.KBn);
    int s = 0;
    uint32_t ph = 0;
    for (int i = 0; i < nunits; ++i) {
        if (i > 0) {
            wk.advance();
            if (++s == S) { s = 0; ph ^= 1u; }
        }
        const int rb = wk.rb;

        // Once any wait has been given up, skip the remaining work but keep the
        // row-block barrier protocol below, so every consumer warp finishes.
        bool have = mbar_try_wait(smem_u32(&full[s]), ph);   // common case: data already here
        if (!have && lds_u32(const_cast<int*>(abort_flag)) == 0) {
            have = mbar_wait(smem_u32(&full[s]), ph);
            if (!have) *abort_flag = 1;
        }
        if (have) {
            const uint8_t* st = stages + s * a.stage_bytes;
            const uint16_t* ssm = reinterpret_cast<const uint16_t*>(st + a.sz_offset);
            const uint16_t* zsm = ssm + kDecRows * GB;

            // B fragments: X[m][k0 .. k0+31] with k0 = 128·c + 32·q, permuted to MMA pairs
            uint32_t bf[MB][4][2][2];
            {
                const uint8_t* xb = st + kDecPBytes + (c >> 1) * xbox_bytes + ((c & 1) * 256 + 64 * q);
#pragma unroll
                for (int mb = 0; mb < MB; ++mb) {
                    const bool ok = mb == 0 ? m_ok0 : m_ok1;
                    const uint8_t* xr = xb + (8 * mb + g) * 512;
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii) {
                        const uint4 v = ok ? lds128(xr + 16 * ii) : make_uint4(0, 0, 0, 0);
                        bf[mb][ii][0][0] = __byte_perm(v.x, v.z, 0x5410);   // (x0, x4)
                        bf[mb][ii][0][1] = __byte_perm(v.x, v.z, 0x7632);   // (x1, x5)
                        bf[mb][ii][1][0] = __byte_perm(v.y, v.w, 0x5410);   // (x2, x6)
                        bf[mb][ii][1][1] = __byte_perm(v.y, v.w, 0x7632);   // (x3, x7)
                    }
                }
            }
            // A fragments: rows 16t + g + 8h, 16 bytes at chunk c of the unit (128-byte swizzle).
            // Both 16-row tiles are loaded first and their MMA chains interleaved.
            const uint8_t* pb = st + (c >> 1) * 4096 + ((((c & 1) << 2) | q) ^ g) * 16 + g * 128;
            uint32_t w[2][2][4];
            uint32_t ss[2][2], zz[2][2];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const uint4 v = lds128(pb + (16 * t + 8 * hr) * 128);
                    w[t][hr][0] = v.x; w[t][hr][1] = v.y; w[t][hr][2] = v.z; w[t][hr][3] = v.w;
                    const int r = 16 * t + 8 * hr + g;
                    ss[t][hr] = __byte_perm(lds_u16(ssm + r * GB + grp_local), 0, 0x1010);
                    zz[t][hr] = SYM ? 0x43084308u
                                    : bf16x2_add(__byte_perm(lds_u16(zsm + r * GB + grp_local), 0, 0x1010),
                                                 0x43004300u);
                }
            }
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        // fragment registers produced in the order the MMA reads them:
                        // (row g, k-pair lo) (row g+8, lo) (row g, hi) (row g+8, hi)
                        uint32_t fa[4];
                        fa[0] = dq_pair<SYM>(w[t][0][ii] >> (8 * hh), zz[t][0], ss[t][0]);
                        fa[1] = dq_pair<SYM>(w[t][1][ii] >> (8 * hh), zz[t][1], ss[t][1]);
                        fa[2] = dq_pair<SYM>(w[t][0][ii] >> (8 * hh + 4), zz[t][0], ss[t][0]);
                        fa[3] = dq_pair<SYM>(w[t][1][ii] >> (8 * hh + 4), zz[t][1], ss[t][1]);
#pragma unroll
                        for (int mb = 0; mb < MB; ++mb)
                            mma_bf16_16816(acc[t][mb], fa[0], fa[1], fa[2], fa[3], bf[mb][ii][hh][0],
                                           bf[mb][ii][hh][1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
        }

        // ---------------------------------------------------------------- row block done?
        if (wk.segment_end()) {
            float* mine = red + warp * RED;
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int mb = 0; mb < MB; ++mb) {
                    *reinterpret_cast<float4*>(mine + ((t * MB + mb) * 32 + lane) * 4) =
                        make_float4(acc[t][mb][0], acc[t][mb][1], acc[t][mb][2], acc[t][mb][3]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[t][mb][j] = 0.0f;
                }
            named_bar_sync(1, kDecConsumers * 32);
            float v[MB];
#pragma unroll
            for (int k = 0; k < MB; ++k) {
                const int e = tid + 256 * k;
                float sum = 0.0f;
#pragma unroll
                for (int w = 0; w < kDecConsumers; ++w) sum += red[w * RED + e];
                v[k] = sum;
            }
            // The row block is whole here iff all its units lie in this CTA's range.
            const int64_t first_u = (int64_t)rb * a.KBn;
            const bool whole = first_u >= u0 && first_u + a.KBn <= u1;
            if (!whole) {
                // split row block: publish this CTA's part; the fixup kernel adds the parts
                float* part = a.ws_part + (int64_t)(rb + cta) * RED;
#pragma unroll
                for (int k = 0; k < MB; ++k) part[tid + 256 * k] = v[k];
            }
            named_bar_sync(1, kDecConsumers * 32);   // red[] is rewritten at the next row block
            if (whole) {
#pragma unroll
                for (int k = 0; k < MB; ++k) {
                    const int e = tid + 256 * k;
                    const int j = e & 3, ln = (e >> 2) & 31, tm = e >> 7;
                    const int mb = tm % MB, t = tm / MB;
                    const int n = rb * kDecRows + 16 * t + (ln >> 2) + 8 * (j >> 1);
                    const int m = 8 * mb + 2 * (ln & 3) + (j & 1);
                    if (n < a.N && m < M)
                        a.Y[(int64_t)m * a.N + n] = (uint16_t)f32_to_bf16_bits_rn(v[k]);
                }
            }
        }
    }
}

// Finishes the row blocks the stream-K partition split between CTAs: CTA b of
// this grid looks at the boundary between CTAs b and b+1 of the streaming grid;
// if the boundary falls inside a row block and is the first boundary in it, it
// adds the row block's fp32 parts in CTA order and writes Y.
template <int MB>
__global__ void __launch_bounds__(256) decode_fixup_kernel(const DecodeArgs a, int64_t C) {
    constexpr int RED = 2 * MB * 128;
    if (threadIdx.x == 0) grid_launch_dependents();
    const int64_t b = blockIdx.x;                       // boundary between CTAs b and b+1
    const int64_t u_next = (b + 1) * a.U / C;           // first unit of CTA b+1
    if (u_next % a.KBn == 0) return;                    // boundary on a row-block edge
    const int64_t rb = u_next / a.KBn;
    const int64_t c_first = owner_of(rb * a.KBn, a.U, C);
    if (c_first != b) return;                           // an earlier boundary handles it
    const int64_t c_last = owner_of(rb * a.KBn + a.KBn - 1, a.U, C);
    grid_dependency_wait();                             // the parts are the previous grid's output
    const int tid = threadIdx.x;
#pragma unroll
    for (int k = 0; k < MB; ++k) {
        const int e = tid + 256 * k;
        float sum = 0.0f;
        for (int64_t p = c_first; p <= c_last; ++p) sum += a.ws_part[(rb + p) * RED + e];
        const int j = e & 3, ln = (e >> 2) & 31, tm = e >> 7;
        const int mb = tm % MB, t = tm / MB;
        const int n = (int)rb * kDecRows + 16 * t + (ln >> 2) + 8 * (j >> 1);
        const int m = 8 * mb + 2 * (ln & 3) + (j & 1);
        if (n < a.N && m < a.M) a.Y[(int64_t)m * a.N + n] = (uint16_t)f32_to_bf16_bits_rn(sum);
    }
}

}  // namespace w4a16
