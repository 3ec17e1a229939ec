// W8A8: weights and activations both INT8, multiplied on the INT8 tensor cores
// ("Quantization & Acceleration: 解释 W8A8 与 W4A16 的差异与取舍", 数学机理 (1): both
// sides INT8, the INT8 tensor cores; activations are dynamic and quantized per
// token; "大模型推理中 Weight-only、W8A8 和 FP8 量化有什么区别？如何选型？", §三: an integer
// matrix multiply on both 8-bit sides, for compute-bound (large-batch) work).
//
//  * w8a8_quantize_act_kernel: one CTA per token (row of X): the row's absolute
//    maximum (exact in binary32, so the reduction order does not matter), s_x =
//    max|x| / 127 with an IEEE division, then q = rint(x / s_x) clamped to
//    [−128, 127] — the same binary32 operations as the oracle, so the codes and
//    scales are bit-identical.  Rows up to K = 32768 stay in registers between
//    the two steps (X is read once); longer rows are read a second time (L2).
//  * gemm_w8a8_kernel: Y[m, n] = s_x[m]·s_w[n]·Σ_k q_x[m, k]·q_w[n, k].  CTA tile
//    256 weight rows × BM tokens; per 128-K stage, TMA brings the weight codes
//    (256 rows × 128 B) and the token codes (BM rows × 128 B), both with the
//    128-byte swizzle, straight into the K-major layout the tensor core reads —
//    no dequantization on this path.  One thread issues, per 32-K step, two
//    tcgen05.mma.kind::i8 (M = 128 each, N = BM) that share the token tile, into
//    two int32 accumulators in tensor memory (exact: |Σ| < 127²·K).  The
//    256-row weight tile halves the shared-memory and L2 bytes per MAC of a
//    128-row one, whose kernel was bound by the L2 feed (51% of the INT8
//    roofline at M=2048, K=N=8192).  Eight epilogue warps read their 32 rows
//    (tcgen05.ld), convert to binary32, multiply by s_w[n] and s_x[m], round to
//    bf16 and store Y (consecutive lanes write consecutive n).  Tiles are
//    ordered m-tile fastest, as in the W4A16 tensor-core kernel.
#pragma once

#include "common.cuh"

namespace w4a16 {

constexpr int kW8a8Threads = 320;          // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int kW8a8TileN = 256;            // weight rows per CTA (two MMAs of M = 128)
constexpr int kW8a8BlockK = 128;           // K per stage: one 128-byte swizzle row of int8
constexpr int kW8a8ActThreads = 256;

// Instruction descriptor: kind::i8, signed 8-bit A and B, int32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_s8_s32(int mma_m, int mma_n) {
    return (2u << 4)                          // D = S32
           | (1u << 7)                        // A = signed 8-bit
           | (1u << 10)                       // B = signed 8-bit
           | ((uint32_t)(mma_n >> 3) << 17)   // N / 8
           | ((uint32_t)(mma_m >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void tc_mma_s8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <int BM>
struct W8a8Config {
    static constexpr int kABytes = kW8a8TileN * kW8a8BlockK;   // 32 KB
    static constexpr int kBBytes = BM * kW8a8BlockK;
    static constexpr int kStageBytes = kABytes + kBBytes;       // multiple of 1024
    static constexpr int kStages = (196608 / kStageBytes) > 8 ? 8 : (196608 / kStageBytes);
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256;
    static constexpr int kTmemCols = 2 * BM;                     // two int32 accumulators of BM columns
};

// Largest |x| of eight bf16 values.
__device__ __forceinline__ float chunk_absmax(uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        a = fmaxf(a, fabsf(__uint_as_float(w[i] << 16)));
        a = fmaxf(a, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
    }
    return a;
}

// Eight bf16 values -> eight int8 codes rint(x / sc) clamped to [-128, 127] (0 when sc == 0).
// Adding 1.5 * 2^23 to the clamped quotient rounds it to the nearest integer, ties
// to even (the binary32 addition's own rounding), and leaves that integer in the
// low mantissa bits: its low byte is the two's-complement code.
__device__ __forceinline__ uint2 chunk_codes(uint4 v, float sc) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float x = __uint_as_float(i & 1 ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16));
        float r = sc != 0.0f ? __fdiv_rn(x, sc) : 0.0f;
        r = fminf(fmaxf(r, -128.0f), 127.0f);
        t[i] = __float_as_uint(r + 12582912.0f);
    }
    const uint32_t lo = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
    return make_uint2(lo, hi);
}

// Per-token INT8 activations: X bf16 [M, K] -> q int8 [M, K], s fp32 [M].  Rows of up
// to kW8a8ActThreads * CACHE * 8 values stay in registers between the maximum and
// the rounding (one read of X); longer rows (CACHE = 0) are read twice.
template <int CACHE>
__global__ void __launch_bounds__(kW8a8ActThreads) w8a8_quantize_act_kernel(
    const uint16_t* __restrict__ X, int64_t M, int64_t K, int8_t* __restrict__ q, float* __restrict__ s) {
    __shared__ float red[kW8a8ActThreads / 32];
    const int64_t chunks = K / 8;                              // K is a multiple of 32
    constexpr bool cached = CACHE > 0;
    constexpr int kCache = CACHE > 0 ? CACHE : 1;
    for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
        const uint16_t* row = X + m * K;
        int8_t* qrow = q + m * K;
        uint4 v[kCache];
        float amax = 0.0f;
        if constexpr (cached) {
#pragma unroll
            for (int j = 0; j < kCache; ++j) {
                const int64_t c = threadIdx.x + (int64_t)j * kW8a8ActThreads;
                v[j] = c < chunks ? ldg_stream(row + 8 * c) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int j = 0; j < kCache; ++j) amax = fmaxf(amax, chunk_absmax(v[j]));
        } else {
            for (int64_t c = threadIdx.x; c < chunks; c += blockDim.x) amax = fmaxf(amax, chunk_absmax(ldg_cached(row + 8 * c)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
        __syncthreads();
        amax = red[0];
#pragma unroll
        for (int i = 1; i < kW8a8ActThreads / 32; ++i) amax = fmaxf(amax, red[i]);
        __syncthreads();                                       // red is reused by the next row
        const float sc = __fdiv_rn(amax, 127.0f);
        if (threadIdx.x == 0) s[m] = sc;
        if constexpr (cached) {
#pragma unroll
            for (int j = 0; j < kCache; ++j) {
                const int64_t c = threadIdx.x + (int64_t)j * kW8a8ActThreads;
                if (c < chunks) *reinterpret_cast<uint2*>(qrow + 8 * c) = chunk_codes(v[j], sc);
            }
        } else {
            for (int64_t c = threadIdx.x; c < chunks; c += blockDim.x)
                *reinterpret_cast<uint2*>(qrow + 8 * c) = chunk_codes(ldg_cached(row + 8 * c), sc);
        }
    }
}

template <int BM>
__global__ void __launch_bounds__(kW8a8Threads, 1)
    gemm_w8a8_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                     const uint16_t* __restrict__ sw, const float* __restrict__ sx,
                     uint16_t* __restrict__ Y, int M, int N, int K) {
    using Cfg = W8a8Config<BM>;
    constexpr int S = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * Cfg::kStageBytes);
    uint64_t* empty = full + S;
    uint64_t* dfull = empty + S;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(dfull + 1);
    volatile int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tiles_m = (M + BM - 1) / BM;
    const int m0 = ((int)blockIdx.x % tiles_m) * BM;
    const int n0 = ((int)blockIdx.x / tiles_m) * kW8a8TileN;
    const int nkb = (K + kW8a8BlockK - 1) / kW8a8BlockK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        mbar_init(smem_u32(dfull), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmW);
            prefetch_tensormap(&tmX);
            grid_dependency_wait();          // the codes may be the previous grid's output
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % S;
                const uint32_t ph = (uint32_t)(kb / S) & 1u;
                if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u)) {
                    *abort_flag = 1;
                    break;
                }
                const uint32_t st = smem_u32(smem + s * Cfg::kStageBytes);
                const uint32_t bar = smem_u32(&full[s]);
                mbar_arrive_expect_tx(bar, (uint32_t)Cfg::kStageBytes);
                tma_load_2d(st, &tmW, kb * kW8a8BlockK, n0, bar);
                tma_load_2d(st + Cfg::kABytes, &tmX, kb * kW8a8BlockK, m0, bar);
            }
            // do not leave while copies into this CTA's shared memory are in flight
            for (int kb = (nkb > S ? nkb - S : 0); kb < nkb; ++kb)
                if (!mbar_wait(smem_u32(&full[kb % S]), (uint32_t)(kb / S) & 1u)) break;
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_s8_s32(128, BM);
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % S;
                const bool ok = *abort_flag == 0 && mbar_wait(smem_u32(&full[s]), (uint32_t)(kb / S) & 1u);
                if (!ok) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t a = smem_u32(smem + s * Cfg::kStageBytes);
                const uint32_t b = a + Cfg::kABytes;
#pragma unroll
                for (int kk = 0; kk < kW8a8BlockK / 32; ++kk) {
                    const uint64_t bd = sw128_kmajor_desc(b + kk * 32);
                    const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
                    // weight rows 0..127 and 128..255 of the tile (16 KB apart)
                    tc_mma_s8(tbase, sw128_kmajor_desc(a + kk * 32), bd, idesc, acc);
                    tc_mma_s8(tbase + (uint32_t)BM, sw128_kmajor_desc(a + 16384 + kk * 32), bd, idesc, acc);
                }
                tc_commit(smem_u32(&empty[s]));       // the stage is free once these complete
            }
            tc_commit(smem_u32(dfull));               // the accumulators are final
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        const int quarter = warp & 3;                 // TMEM lanes 32·quarter .. +31
        const int half = (warp - 2) >> 2;             // accumulator 0 (rows 0..127) or 1 (128..255)
        const int n = n0 + 128 * half + 32 * quarter + lane;
        const bool got = mbar_wait(smem_u32(dfull), 0);
        tc_fence_after();
        grid_dependency_wait();                       // Y may be in use by the previous grid
        const float swn = n < N ? bf16_bits_to_f32(sw[n]) : 0.0f;
#pragma unroll 1
        for (int c0 = 0; c0 < BM; c0 += 32) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tbase + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(half * BM + c0), r);
            tmem_wait_ld();
            if (!got || *abort_flag != 0 || n >= N) continue;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int m = m0 + c0 + j;
                if (m < M) {
                    const float y = (float)(int32_t)r[j] * swn * __ldg(sx + m);
                    Y[(int64_t)m * N + n] = (uint16_t)f32_to_bf16_bits_rn(y);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, Cfg::kTmemCols);
    }
}

}  // namespace w4a16
