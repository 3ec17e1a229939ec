// Prefill-path fused W4A16 GEMM (large M) on the 5th-generation tensor cores.
//
// Large-M work is compute bound, and there the per-use dequantization cost
// shows (aigcbaba selection page §二: "每次都要反量化的开销会凸显"; qwbw.cn page
// §3.2).  So the dequantization runs in dedicated warps, overlapped with the
// tensor core through a multi-stage shared-memory pipeline, and each
// dequantized weight serves up to 256 activation rows:
//
//   D[128 x BM] (TMEM, fp32) += Ŵ[128 rows of N x K] · X[BM rows of M x K]ᵀ
//
// i.e. the CTA computes a 128 (n) x BM (m) tile of Yᵀ, with the dequantized
// weights as the UMMA A operand (M = 128) and the activations as B (N = BM).
//
// Warp roles (6 warps):
//   warp 0      producer: per 64-wide K block, one lane issues a TMA load of the
//               X tile (BM x 64 bf16, 128-byte swizzle) and one of the packed
//               tile (128 rows x 32 bytes); all 32 lanes copy the block's scales
//               and zero points (one aligned pair of groups per row) into the
//               stage with 4-byte cp.async copies.  Both complete on the stage's
//               "full" barrier, so the dequantizers never wait on global loads.
//   warp 1      TMEM allocator and, on one elected lane, the MMA issuer: waits
//               for the stage's X tile and dequantized A tile, issues four
//               tcgen05.mma (K = 16 each), and commits to the stage's "empty"
//               barrier so producer and dequantizers may reuse it.
//   warps 2..5  dequantizers, one weight row per thread: nibbles from the packed
//               tile -> bf16 pairs (q − z)·s -> 16-byte chunks written into the
//               A tile in the 128-byte swizzled K-major layout the UMMA
//               descriptor expects; fence.proxy.async makes the generic-proxy
//               writes visible to the tensor core before the "a_full" arrive.
//               After the K loop the same warps drain TMEM (tcgen05.ld), round
//               to bf16 and store Y.  Warp w reads TMEM lanes 32·(w%4)..+31,
//               which are the rows it dequantized.
//
// Every barrier wait is bounded (about one second); a timeout records an error
// in the device error word and the role stops issuing work, then the CTA
// drains and frees its TMEM before returning.
#pragma once

#include "common.cuh"

namespace w4a16 {

constexpr int kTcThreads = 192;
constexpr int kTcBlockK = 64;                 // K per pipeline stage (one 128-byte swizzle row)
constexpr int kTcTileN = 128;                 // UMMA M: weight rows per CTA

template <int BM>
struct TcConfig {
    static constexpr int kXBytes = BM * kTcBlockK * 2;          // X tile
    static constexpr int kABytes = kTcTileN * kTcBlockK * 2;    // dequantized weight tile
    static constexpr int kPBytes = kTcTileN * kTcBlockK / 2;    // packed codes tile
    static constexpr int kSZBytes = 2 * kTcTileN * 4;              // scale and zero pairs per row
    static constexpr int kStageBytes = kXBytes + kABytes + kPBytes + kSZBytes;
    static constexpr int kBudget = 220 * 1024;
    static constexpr int kStagesRaw = kBudget / kStageBytes;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kBarrierBytes = 1024;
    static constexpr int kSmemBytes = kStages * kStageBytes + kBarrierBytes + 1024;  // + align slack
    static constexpr int kTmemCols = BM < 32 ? 32 : BM;
};

template <int BM, bool SYM, int G>
__global__ void __launch_bounds__(kTcThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                   const uint16_t* __restrict__ scales, const uint16_t* __restrict__ zeros,
                   uint16_t* __restrict__ Y, int M, int N, int K, int sz_async) {
    using Cfg = TcConfig<BM>;
    constexpr int S = Cfg::kStages;
    static_assert(S >= 2, "pipeline needs at least two stages");
    static_assert(BM % 16 == 0 && BM >= 16 && BM <= 256, "UMMA N must be 16..256, step 16");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* xs = smem;                                   // S x kXBytes
    uint8_t* as = xs + S * Cfg::kXBytes;                  // S x kABytes
    uint8_t* ps = as + S * Cfg::kABytes;                  // S x kPBytes
    uint32_t* szs = reinterpret_cast<uint32_t*>(ps + S * Cfg::kPBytes);   // S x [2][128] u32 pairs
    uint64_t* bars = reinterpret_cast<uint64_t*>(szs + S * 2 * kTcTileN);
    uint64_t* full = bars;             // TMA bytes landed
    uint64_t* afull = bars + S;        // dequantized A tile written
    uint64_t* empty = bars + 2 * S;    // MMAs reading the stage retired
    uint64_t* accf = bars + 3 * S;     // all MMAs retired
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 3 * S + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kTcTileN;
    const int m0 = blockIdx.y * BM;
    const int num_kb = (K + kTcBlockK - 1) / kTcBlockK;
    const int Gn = K / G;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1 + 32);   // TMA expect_tx arrive + 32 scale lanes
            mbar_init(smem_u32(&afull[s]), 128);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        mbar_init(smem_u32(accf), 1);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmP);
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
        for (int kb = 0; kb < num_kb; ++kb) {
            const int s = kb % S;
            const uint32_t ph = (uint32_t)(kb / S) & 1u;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(smem_u32(&empty[s]), ph ^ 1u);   // one lane waits
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            const uint32_t bar = smem_u32(&full[s]);
            if (lane == 0) {
                mbar_arrive_expect_tx(bar, Cfg::kXBytes + Cfg::kPBytes);
                tma_load_2d(smem_u32(xs + s * Cfg::kXBytes), &tmX, kb * kTcBlockK, m0, bar);
                tma_load_2d(smem_u32(ps + s * Cfg::kPBytes), &tmP, kb * (kTcBlockK / 2), n0, bar);
            }
            // the aligned pair of groups holding this block's group(s), per row and array
            const int jpair = ((kb * kTcBlockK) / G) & ~1;
            uint32_t* dst = szs + s * 2 * kTcTileN;
            if (sz_async) {
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
            for (int kb = (issued > S ? issued - S : 0); kb < issued; ++kb) {
                if (!mbar_wait(smem_u32(&full[kb % S]), (uint32_t)(kb / S) & 1u)) break;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kTcTileN, BM);
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % S;
                const uint32_t ph = (uint32_t)(kb / S) & 1u;
                if (!mbar_wait(smem_u32(&full[s]), ph)) break;
                if (!mbar_wait(smem_u32(&afull[s]), ph)) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(as + s * Cfg::kABytes);
                const uint32_t x_base = smem_u32(xs + s * Cfg::kXBytes);
#pragma unroll
                for (int kk = 0; kk < kTcBlockK / 16; ++kk) {
                    tc_mma_bf16(tmem_d, sw128_kmajor_desc(a_base + kk * 32),
                                sw128_kmajor_desc(x_base + kk * 32), idesc,
                                (kb | kk) != 0 ? 1u : 0u);
                }
                tc_commit(smem_u32(&empty[s]));
            }
            // Signals the epilogue; also taken on the error path so that every
            // issued MMA has retired before TMEM is released.
            tc_commit(smem_u32(accf));
        }
    } else {
        // ------------------------------------------------------------ dequantize
        const int r = (warp & 3) * 32 + lane;   // weight row within the tile == TMEM lane
        const int n = n0 + r;
        const bool row_ok = n < N;
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
            const int s = kb % S;
            const uint32_t ph = (uint32_t)(kb / S) & 1u;
            if (!mbar_wait(smem_u32(&full[s]), ph)) {
                ok = false;
                break;
            }
            const uint32_t spair = lds_u32(szs + s * 2 * kTcTileN + r);
            const uint32_t zpair = SYM ? 0u : lds_u32(szs + s * 2 * kTcTileN + kTcTileN + r);
            const uint8_t* prow = ps + s * Cfg::kPBytes + r * 32;
            const uint32_t arow = smem_u32(as + s * Cfg::kABytes + r * 128);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 v = lds128(prow + 16 * h);
                const int half = ((kb * kTcBlockK + 32 * h) / G) & 1;   // position in the pair
                const uint32_t ss = dup16(spair >> (16 * half));
                const uint32_t zz = SYM ? 0x43084308u
                                        : bf16x2_add(dup16(zpair >> (16 * half)), 0x43004300u);
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t d[4];
                    dequant8_natural<SYM>(wv[i], zz, ss, d);
                    const int chunk = 4 * h + i;                 // 16-byte chunk: k = 8·chunk
                    const int phys = chunk ^ (r & 7);            // 128-byte swizzle
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(arow + phys * 16),
                                 "r"(d[0]), "r"(d[1]), "r"(d[2]), "r"(d[3])
                                 : "memory");
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(smem_u32(&afull[s]));
        }
        // ------------------------------------------------------------ epilogue
        if (ok && mbar_wait(smem_u32(accf), 0)) {
            tc_fence_after();
            const uint32_t t_lane = (uint32_t)((warp & 3) * 32) << 16;
#pragma unroll 1
            for (int cb = 0; cb < BM / 32; ++cb) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_d + t_lane + cb * 32, v);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int m = m0 + cb * 32 + j;
                        if (m < M)
                            Y[(int64_t)m * N + n] =
                                (uint16_t)f32_to_bf16_bits_rn(__uint_as_float(v[j]));
                    }
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
}

}  // namespace w4a16
