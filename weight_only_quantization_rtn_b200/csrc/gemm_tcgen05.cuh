// Prefill-path fused W4A16 GEMM (large M) on the 5th-generation tensor cores.
//
// Large-M work is compute bound, and there the per-use dequantization cost
// shows ("大模型推理中 Weight-only、W8A8 和 FP8 量化有什么区别？如何选型？", §二:
// "每次都要反量化的开销会凸显"; "推理优化中“用精度换性能“的核心技术：量化",
// §3.2).  So the dequantization runs in dedicated warps, overlapped with the
// tensor core through a multi-stage shared-memory pipeline, and each
// dequantized weight serves up to 256 activation rows:
//
//   D[128 x BM] (TMEM, fp32) += Ŵ[128 rows of N x K] · X[BM rows of M x K]ᵀ
//
// i.e. the CTA computes a 128 (n) x BM (m) tile of Yᵀ, with the dequantized
// weights as the UMMA A operand (M = 128) and the activations as B (N = BM).
//
// Warp roles (10 warps):
//   warp 0      producer: per 64-wide K block, one lane issues a TMA load of the
//               X tile (BM x 64 bf16, 128-byte swizzle) and one of the packed
//               tile (128 rows x 32 bytes, 32-byte swizzle).  Scales and zero
//               points arrive by TMA in slabs of 8 groups x 128 rows (one slab
//               serves g/8 K blocks, a two-slot ring with its own barriers; the
//               dequantizers copy a landed slab into registers and release it at
//               once) when their rows are 16-byte aligned; otherwise all 32 lanes copy the
//               block's aligned pair of groups per row into the stage with 4-byte
//               cp.async copies that complete on the stage's "full" barrier.
//   warp 1      TMEM allocator and, on one elected lane, the MMA issuer: waits
//               for the stage's X tile and dequantized A tile, issues four
//               tcgen05.mma (K = 16 each), and commits to the stage's "empty"
//               barrier so producer and dequantizers may reuse it.
//   warps 2..9  dequantizers, two per SM sub-partition: thread (w, l) takes
//               weight row 32·(w%4) + l and K half (w−2)/4 of the block: nibbles
//               from the packed tile -> bf16 pairs (q − z)·s -> 16-byte chunks
//               written into the A tile in the 128-byte swizzled K-major layout
//               the UMMA descriptor expects; fence.proxy.async makes the
//               generic-proxy writes visible to the tensor core before the
//               "a_full" arrive.  After the K loop the same warps drain TMEM
//               (tcgen05.ld), round to bf16 and store Y: warp w reads TMEM lanes
//               32·(w%4)..+31, the rows it dequantized, and every other 32-column
//               block of the accumulator.
//
// Tiles and split-K: CTA (x, z) of a launch computes output tile t = tile_base + x
// (m-tile t % tiles_m, n-tile t / tiles_m).  When a launch splits K, gridDim.z
// CTAs share each tile's K range (CTA z takes K blocks [z·kb_split,
// (z+1)·kb_split)), each writes its fp32 partial tile to the workspace, and
// tc_splitk_reduce_kernel, chained by programmatic dependent launch, adds the
// partials in z order and writes Y.  The host splits K when the tiles are fewer
// than the resident CTA slots (SMs x tc_ctas_per_sm), and splits only the last,
// partial wave of tiles (a second launch) when that wave would leave most slots
// idle.
//
// Every barrier wait is bounded (about one second); a timeout records an error
// in the device error word and the role stops issuing work, then the CTA
// drains and frees its TMEM before returning.
#pragma once

#include "common.cuh"

namespace w4a16 {

constexpr int kTcDequantWarps = 8;
constexpr int kTcThreads = (2 + kTcDequantWarps) * 32;
constexpr int kTcBlockK = 64;                 // K per pipeline stage (one 128-byte swizzle row)
constexpr int kTcTileN = 128;                 // UMMA M: weight rows per CTA

// Resident CTAs per SM.  With small activation tiles (BM ≤ 64) each K block
// carries little MMA work, and one CTA's chain of TMA wait -> dequantize ->
// MMA -> stage release leaves the SM mostly idle; two CTAs per SM overlap two
// such chains (measured 19% faster at M = 32, 11% at M = 64, K = N = 8192).
// Their stage rings are sized so that two fit in the SM's shared memory.
__host__ __device__ constexpr int tc_ctas_per_sm(int bm) { return bm <= 64 ? 2 : 1; }

// BITS: code width, 4 (two codes per byte) or 8 (W8A16, one code per byte).
template <int BM, int BITS = 4>
struct TcConfig {
    static constexpr int kRowBytes = kTcBlockK * BITS / 8;      // code bytes of a row per K block
    static constexpr int kXBytes = BM * kTcBlockK * 2;          // X tile
    static constexpr int kABytes = kTcTileN * kTcBlockK * 2;    // dequantized weight tile
    static constexpr int kPBytes = kTcTileN * kRowBytes;        // codes tile
    static constexpr int kSZBytes = 2 * kTcTileN * 4;              // scale and zero pairs per row
    static constexpr int kSlabBytes = 2 * 2 * kTcTileN * 8 * 2;  // two slots of scale + zero slabs
    // What TMA (and the scale copies) bring per K block: one slot of the load ring.
    static constexpr int kLoadBytes = kXBytes + kPBytes + kSZBytes;
    // 8-bit codes double the load per K block; their loads get a ring of their own,
    // deeper than the ring of dequantized A tiles (2 or 3), which needs only to
    // cover the MMA (M=2048, K=N=8192: 318 -> 275 us; M=32: 34.8 -> 31.7 us).  With
    // 4-bit codes, and 8-bit codes at BM = 128, each load slot carries its own A
    // tile (one ring): there the extra barrier traffic of two rings cost 2–9%.
    static constexpr bool kSplitRing = BITS == 8 && BM != 128;
    static constexpr int kSplitABufs = BM >= 128 ? 3 : 2;
    static constexpr int kBudget = 220 * 1024 / tc_ctas_per_sm(BM) - kSlabBytes -
                                   (kSplitRing ? kSplitABufs * kABytes : 0);
    static constexpr int kSlotBytes = kLoadBytes + (kSplitRing ? 0 : kABytes);
    static constexpr int kStagesRaw = kBudget / kSlotBytes;
    static constexpr int kStagesMax = kSplitRing ? 12 : 8;
    static constexpr int kStages = kStagesRaw > kStagesMax ? kStagesMax : kStagesRaw;
    static constexpr int kABufs = kSplitRing ? kSplitABufs : kStages;
    static constexpr int kBarrierBytes = 1024;
    static constexpr int kSmemBytes = kStages * kLoadBytes + kABufs * kABytes + kSlabBytes +
                                      kBarrierBytes + 1024;   // + align slack
    static constexpr int kTmemCols = BM < 32 ? 32 : BM;
};

// 8-bit codes (one word = 4 codes) -> two bf16x2 of bf16_rn((q − z)·s) in natural
// order.  2^23 + q is formed exactly by placing the byte in a binary32 mantissa;
// subtracting zoff = 2^23 + z (exact: < 2^24) leaves q − z, the product with the
// bf16 scale s is exact in binary32, and the conversion rounds once.
__device__ __forceinline__ void dequant4_bytes(uint32_t w, float s, float zoff, uint32_t out[2]) {
    float f[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        f[i] = (__uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u + (uint32_t)i)) - zoff) * s;
    uint32_t lo, hi;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(lo) : "f"(f[1]), "f"(f[0]));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(hi) : "f"(f[3]), "f"(f[2]));
    out[0] = lo;
    out[1] = hi;
}

template <int BM, bool SYM, int G, int BITS = 4>
__global__ void __launch_bounds__(kTcThreads, tc_ctas_per_sm(BM))
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                   const uint16_t* __restrict__ scales, const uint16_t* __restrict__ zeros,
                   uint16_t* __restrict__ Y, int M, int N, int K, int sz_async,
                   const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmZ,
                   int sz_tma, int kb_split, float* __restrict__ partials, int tile_base,
                   int tiles_n) {
    (void)tiles_n;                        // the order is m-tile fastest (below)
    static_assert(BITS == 4 || BITS == 8, "4- or 8-bit codes");
    using Cfg = TcConfig<BM, BITS>;
    constexpr int S = Cfg::kStages;                 // load ring (X, codes, scale pairs)
    constexpr int NA = Cfg::kABufs;                 // dequantized A ring
    constexpr bool kSplit = Cfg::kSplitRing;        // else A tile i lives in load slot i % S
    static_assert(S >= 2 && NA >= 2, "pipeline needs at least two slots per ring");
    static_assert((2 * S + 2 * NA + 5) * 8 + 8 <= Cfg::kBarrierBytes, "barrier area");
    static_assert(BM % 16 == 0 && BM >= 16 && BM <= 256, "UMMA N must be 16..256, step 16");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* xs = smem;                                   // S x kXBytes
    uint8_t* as = xs + S * Cfg::kXBytes;                  // NA x kABytes
    uint8_t* ps = as + NA * Cfg::kABytes;                 // S x kPBytes
    uint32_t* szs = reinterpret_cast<uint32_t*>(ps + S * Cfg::kPBytes);   // S x [2][128] u32 pairs
    uint16_t* slab = reinterpret_cast<uint16_t*>(szs + S * 2 * kTcTileN); // 2 x [2][128][8] u16
    uint64_t* bars = reinterpret_cast<uint64_t*>(slab + 2 * 2 * kTcTileN * 8);
    uint64_t* full = bars;             // [S] load slot landed
    uint64_t* empty = bars + S;        // [S] load slot free: its MMAs retired (and, with
                                       //     two rings, the dequantizers read its codes)
    uint64_t* afull = bars + 2 * S;    // [NA] dequantized A tile written
    uint64_t* aempty = afull + NA;     // [NA] MMAs reading the A tile retired
    uint64_t* accf = aempty + NA;      // all MMAs retired
    uint64_t* slab_full = accf + 1;    // [2] slab of scales/zeros landed
    uint64_t* slab_empty = accf + 3;   // [2] dequantizers done with the slab
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accf + 5);
    // G == 0: per-channel granularity, one scale (and zero) per row for all of K;
    // each dequantizing thread reads its row's pair once, nothing is staged.
    constexpr int kG = G == 0 ? 1 : G;                            // divisor for the grouped forms
    constexpr int kSlabKb = G == 0 ? 1 : 8 * G / kTcBlockK;       // K blocks served by one slab

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tile = tile_base + (int)blockIdx.x;
    // m-tiles vary fastest: a wave of CTAs covers few weight tiles and every
    // activation tile, so each weight tile is read from HBM about once per GEMM
    // while the activation tiles, which every wave reads again, stay in L2
    // (measured 1–2% faster at M=2048 than n-tiles fastest)
    const int tiles_m = (M + BM - 1) / BM;
    const int n0 = (tile / tiles_m) * kTcTileN;
    const int m0 = (tile % tiles_m) * BM;
    const int num_kb = (K + kTcBlockK - 1) / kTcBlockK;
    // this CTA's K blocks [kb0, kb0 + nkb); kb0 is a multiple of the slab length
    const int kb0 = (int)blockIdx.z * kb_split;
    const int nkb = min(num_kb - kb0, kb_split);
    const int Gn = G == 0 ? 1 : K / kG;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            // TMA arrive (+ 32 scale-copying lanes)
            mbar_init(smem_u32(&full[s]), (sz_tma || G == 0) ? 1 : 1 + 32);
            mbar_init(smem_u32(&empty[s]), kSplit ? 1 + kTcDequantWarps : 1);
        }
        for (int a = 0; a < NA; ++a) {
            mbar_init(smem_u32(&afull[a]), kTcDequantWarps);
            mbar_init(smem_u32(&aempty[a]), 1);
        }
        mbar_init(smem_u32(accf), 1);
        grid_launch_dependents();          // the split-K reduction may start as this grid drains
        for (int t = 0; t < 2; ++t) {
            mbar_init(smem_u32(&slab_full[t]), 1);
            mbar_init(smem_u32(&slab_empty[t]), kTcDequantWarps);
        }
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmP);
        if (sz_tma) {
            prefetch_tensormap(&tmS);
            if (!SYM) prefetch_tensormap(&tmZ);
        }
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int issued = 0;
        for (int i = 0; i < nkb; ++i) {
            const int kb = kb0 + i;
            const int s = i % S;
            const uint32_t ph = (uint32_t)(i / S) & 1u;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(smem_u32(&empty[s]), ph ^ 1u);   // one lane waits
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            const uint32_t bar = smem_u32(&full[s]);
            if (sz_tma && i % kSlabKb == 0) {
                // next slab of scales/zeros: its slot is free once the dequantizers
                // finished the slab two back
                const int t = i / kSlabKb, slot = t & 1;
                if (lane == 0) ok = mbar_wait(smem_u32(&slab_empty[slot]), ((uint32_t)(t >> 1) & 1u) ^ 1u);
                if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
                if (lane == 0) {
                    const uint32_t sb = smem_u32(&slab_full[slot]);
                    uint16_t* dsl = slab + slot * 2 * kTcTileN * 8;
                    mbar_arrive_expect_tx(sb, (SYM ? 1 : 2) * kTcTileN * 8 * 2);
                    tma_load_2d(smem_u32(dsl), &tmS, (kb / kSlabKb) * 8, n0, sb);
                    if (!SYM) tma_load_2d(smem_u32(dsl + kTcTileN * 8), &tmZ, (kb / kSlabKb) * 8, n0, sb);
                }
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(bar, Cfg::kXBytes + Cfg::kPBytes);
                tma_load_2d(smem_u32(xs + s * Cfg::kXBytes), &tmX, kb * kTcBlockK, m0, bar);
                tma_load_2d(smem_u32(ps + s * Cfg::kPBytes), &tmP, kb * Cfg::kRowBytes, n0, bar);
            }
            // the aligned pair of groups holding this block's group(s), per row and array
            const int jpair = ((kb * kTcBlockK) / kG) & ~1;
            uint32_t* dst = szs + s * 2 * kTcTileN;
            if (G == 0 || sz_tma) {
                // per-channel: nothing to stage; grouped: scales/zeros come with the slab
            } else if (sz_async) {
#pragma unroll
                for (int e = lane; e < 2 * kTcTileN; e += 32) {
                    const int arr = e / kTcTileN, r = e % kTcTileN;
                    const int n = n0 + r;
                    const bool in = n < N && !(SYM && arr == 1);
                    const uint16_t* src = (arr == 0 ? scales : zeros) +
                                          (in ? (int64_t)n * Gn + jpair : 0);
                    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst + e)),
                                 "l"(in ? src : scales), "r"(in ? 4u : 0u)
                                 : "memory");
                }
                asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
            } else {
                for (int e = lane; e < 2 * kTcTileN; e += 32) {
                    const int arr = e / kTcTileN, r = e % kTcTileN;
                    const int n = n0 + r;
                    uint32_t v = 0;
                    if (n < N && !(SYM && arr == 1)) {
                        const uint16_t* src = (arr == 0 ? scales : zeros) + (int64_t)n * Gn + jpair;
                        v = ldg_u16(src);
                        if (jpair + 1 < Gn) v |= (uint32_t)ldg_u16(src + 1) << 16;
                    }
                    dst[e] = v;
                }
                mbar_arrive(bar);
            }
            ++issued;
        }
        if (lane == 0) {
            // Do not leave while copies into this CTA's shared memory are in flight.
            for (int i = (issued > S ? issued - S : 0); i < issued; ++i) {
                if (!mbar_wait(smem_u32(&full[i % S]), (uint32_t)(i / S) & 1u)) break;
            }
            if (sz_tma && issued > 0) {
                const int slabs = (issued - 1) / kSlabKb + 1;   // slabs requested so far
                for (int t = (slabs > 2 ? slabs - 2 : 0); t < slabs; ++t)
                    if (!mbar_wait(smem_u32(&slab_full[t & 1]), (uint32_t)(t >> 1) & 1u)) break;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kTcTileN, BM);
            for (int i = 0; i < nkb; ++i) {
                const int s = i % S;
                const uint32_t ph = (uint32_t)(i / S) & 1u;
                const int ab = kSplit ? i % NA : s;
                if (!mbar_wait(smem_u32(&full[s]), ph)) break;
                if (!mbar_wait(smem_u32(&afull[ab]), (uint32_t)(i / NA) & 1u)) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(as + ab * Cfg::kABytes);
                const uint32_t x_base = smem_u32(xs + s * Cfg::kXBytes);
#pragma unroll
                for (int kk = 0; kk < kTcBlockK / 16; ++kk) {
                    tc_mma_bf16(tmem_d, sw128_kmajor_desc(a_base + kk * 32),
                                sw128_kmajor_desc(x_base + kk * 32), idesc,
                                (i | kk) != 0 ? 1u : 0u);
                }
                tc_commit(smem_u32(&empty[s]));       // X (and a one-ring A tile) read
                if (kSplit) tc_commit(smem_u32(&aempty[ab]));   // the A tile may be rewritten
            }
            // Signals the epilogue; also taken on the error path so that every
            // issued MMA has retired before TMEM is released.
            tc_commit(smem_u32(accf));
        }
    } else {
        // ------------------------------------------------------------ dequantize
        const int r = (warp & 3) * 32 + lane;   // weight row within the tile == TMEM lane
        const int h = (warp - 2) >> 2;          // K half of each 64-wide block
        const int n = n0 + r;
        const bool row_ok = n < N;
        // Zero pairs: 128 + z (the INT4 bf16 magic) for 4-bit codes, z itself for 8-bit.
        auto zero_of = [](uint32_t raw_dup) {
            return BITS == 4 ? bf16x2_add(raw_dup, 0x43004300u) : raw_dup;
        };
        uint32_t row_ss = 0u, row_zz = 0x43084308u;   // per-channel pair of this row
        if (G == 0 && row_ok) {
            row_ss = dup16(ldg_u16(scales + n));
            if (!SYM) row_zz = zero_of(dup16(ldg_u16(zeros + n)));
        }
        bool ok = true;
        // Scales by TMA slab: when a slab lands, each thread copies its row's 8 scales and
        // 8 zeros (two 16-byte reads, conflict-free) into registers, adds 128 to the zeros
        // once, and releases the slot; each K block then picks its pair with one PRMT.
        uint32_t sreg0 = 0u, sreg1 = 0u, sreg2 = 0u, sreg3 = 0u;   // this row's 8 slab scales
        uint32_t zreg0 = 0u, zreg1 = 0u, zreg2 = 0u, zreg3 = 0u;   // and its 8 zero pairs
        for (int i = 0; i < nkb; ++i) {
            const int kb = kb0 + i;
            const int s = i % S;
            const uint32_t ph = (uint32_t)(i / S) & 1u;
            const int t = i / kSlabKb, slot = t & 1;
            if (sz_tma && i % kSlabKb == 0) {
                if (!mbar_wait(smem_u32(&slab_full[slot]), (uint32_t)(t >> 1) & 1u)) {
                    ok = false;
                    break;
                }
                const uint16_t* srow = slab + slot * 2 * kTcTileN * 8 + r * 8;
                const uint4 sv = lds128(srow);
                sreg0 = sv.x; sreg1 = sv.y; sreg2 = sv.z; sreg3 = sv.w;
                if (!SYM) {
                    const uint4 zv = lds128(srow + kTcTileN * 8);
                    zreg0 = zero_of(zv.x);
                    zreg1 = zero_of(zv.y);
                    zreg2 = zero_of(zv.z);
                    zreg3 = zero_of(zv.w);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&slab_empty[slot]));   // slot no longer read
            }
            if (!mbar_wait(smem_u32(&full[s]), ph)) {
                ok = false;
                break;
            }
            uint32_t spair = 0u, zpair = 0u;
            if (G != 0 && !sz_tma) {
                spair = lds_u32(szs + s * 2 * kTcTileN + r);
                zpair = SYM ? 0u : lds_u32(szs + s * 2 * kTcTileN + kTcTileN + r);
            }
            const int ab = kSplit ? i % NA : s;
            const uint8_t* prow = ps + s * Cfg::kPBytes + r * Cfg::kRowBytes;
            const uint32_t arow = smem_u32(as + ab * Cfg::kABytes + r * 128);
            {
                uint4 v, v8 = make_uint4(0, 0, 0, 0);
                if constexpr (BITS == 4) {
                    // 32-byte swizzle: chunk h of row r sits at position h ^ bit 2 of r
                    v = lds128(prow + 16 * (h ^ ((r >> 2) & 1)));
                } else {
                    // 64-byte swizzle: 16-byte chunk c of row r sits at c ^ bits 2..1 of r;
                    // this thread's 32 codes are chunks 2h and 2h + 1
                    v = lds128(prow + 16 * ((2 * h) ^ ((r >> 1) & 3)));
                    v8 = lds128(prow + 16 * ((2 * h + 1) ^ ((r >> 1) & 3)));
                }
                uint32_t ss, zz;
                if (G == 0) {
                    ss = row_ss;
                    zz = row_zz;
                } else if (sz_tma) {
                    // group within the slab; its 2 bytes of the 8-byte register pair, twice
                    const int gi = (int)((uint32_t)(kb * kTcBlockK + 32 * h) / (uint32_t)kG) & 7;
                    const uint32_t sel = 0x1010u + (uint32_t)(gi & 3) * 0x2222u;
                    const bool up = (gi & 4) != 0;
                    ss = __byte_perm(up ? sreg2 : sreg0, up ? sreg3 : sreg1, sel);
                    zz = SYM ? 0x43084308u : __byte_perm(up ? zreg2 : zreg0, up ? zreg3 : zreg1, sel);
                } else {
                    const int half = ((kb * kTcBlockK + 32 * h) / kG) & 1;  // position in the pair
                    ss = dup16(spair >> (16 * half));
                    zz = SYM ? 0x43084308u : zero_of(dup16(zpair >> (16 * half)));
                }
                const uint32_t wv[8] = {v.x, v.y, v.z, v.w, v8.x, v8.y, v8.z, v8.w};
                // 8-bit: binary32 scale, and 2^23 + z (symmetric codes are flipped to
                // offset-128 form by XOR with 0x80 and take z = 128)
                const float s8 = __uint_as_float(ss << 16);
                const float zoff = SYM ? 8388736.0f : 8388608.0f + __uint_as_float(zz << 16);
                // two rings: the A tile is free once the MMAs of K block i − NA retired
                // (one ring: the load slot's "full" wait already implied it)
                if (kSplit && !mbar_wait(smem_u32(&aempty[ab]), ((uint32_t)(i / NA) & 1u) ^ 1u)) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t d[4];
                    if constexpr (BITS == 4) {
                        dequant8_natural<SYM>(wv[i], zz, ss, d);
                    } else {
                        const uint32_t flip = SYM ? 0x80808080u : 0u;
                        dequant4_bytes(wv[2 * i] ^ flip, s8, zoff, d);
                        dequant4_bytes(wv[2 * i + 1] ^ flip, s8, zoff, d + 2);
                    }
                    const int chunk = 4 * h + i;                 // 16-byte chunk: k = 8·chunk
                    const int phys = chunk ^ (r & 7);            // 128-byte swizzle
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(arow + phys * 16),
                                 "r"(d[0]), "r"(d[1]), "r"(d[2]), "r"(d[3])
                                 : "memory");
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(smem_u32(&afull[ab]));
                if (kSplit) mbar_arrive(smem_u32(&empty[s]));   // its codes and scale pairs were read
            }
        }
        // ------------------------------------------------------------ epilogue
        if (ok && mbar_wait(smem_u32(accf), 0)) {
            tc_fence_after();
            const uint32_t t_lane = (uint32_t)((warp & 3) * 32) << 16;
#pragma unroll 1
            for (int cb = h; cb < BM / 32; cb += 2) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_d + t_lane + cb * 32, v);
                tmem_wait_ld();
                if (row_ok && partials == nullptr) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int m = m0 + cb * 32 + j;
                        if (m < M)
                            Y[(int64_t)m * N + n] =
                                (uint16_t)f32_to_bf16_bits_rn(__uint_as_float(v[j]));
                    }
                } else if (partials != nullptr) {
                    // split-K: this CTA's fp32 part of its tile, [z][tile of the launch][BM][128]
                    float* part = partials +
                                  ((int64_t)blockIdx.z * gridDim.x + blockIdx.x) * (BM * kTcTileN);
#pragma unroll
                    for (int j = 0; j < 32; ++j) part[(cb * 32 + j) * kTcTileN + r] = __uint_as_float(v[j]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_d, Cfg::kTmemCols);
    }
    // A launch that started early behind another tile launch does not complete
    // before it: work queued after this launch may then rely on both.
    if (threadIdx.x == 0) grid_dependency_wait();
}

// Adds the split-K partial tiles in z order and rounds to bf16: for each tile of the
// preceding launch, Y[m0 + m][n0 + r] = Σ_z part[z][tile][m][r].  Four consecutive
// rows r per thread, grid-stride; the parts are the preceding grid's output.
__global__ void __launch_bounds__(256) tc_splitk_reduce_kernel(
    const float* __restrict__ partials, int splits, int tiles, int tile_base, int tiles_n, int bm,
    int M, int N, uint16_t* __restrict__ Y) {
    grid_dependency_wait();
    const int64_t per_tile = (int64_t)bm * kTcTileN;
    const int64_t stride = (int64_t)tiles * per_tile;          // one split's parts
    const int64_t items = stride / 4;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < items;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t idx = 4 * e;
        const int tl = (int)(idx / per_tile);
        const int within = (int)(idx - (int64_t)tl * per_tile);
        const int m_local = within / kTcTileN, r = within % kTcTileN;
        const int t = tile_base + tl;
        const int tiles_m = (M + bm - 1) / bm;
        const int m = (t % tiles_m) * bm + m_local;
        const int n = (t / tiles_m) * kTcTileN + r;
        if (m >= M || n >= N) continue;
        float4 acc = __ldcg(reinterpret_cast<const float4*>(partials + idx));
        for (int z = 1; z < splits; ++z) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(partials + z * stride + idx));
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
        uint16_t* y = Y + (int64_t)m * N + n;
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (n + q < N) y[q] = (uint16_t)f32_to_bf16_bits_rn(a4[q]);
    }
}

}  // namespace w4a16
