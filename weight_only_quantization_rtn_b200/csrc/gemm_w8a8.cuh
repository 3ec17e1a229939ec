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
//    scales are bit-identical.  The second pass reads the row again from L2.
//  * gemm_w8a8_kernel: Y[m, n] = s_x[m]·s_w[n]·Σ_k q_x[m, k]·q_w[n, k].  CTA tile
//    128 weight rows × BM tokens; per 128-K stage, TMA brings the weight codes
//    (128 rows × 128 B) and the token codes (BM rows × 128 B), both with the
//    128-byte swizzle, straight into the K-major layout the tensor core reads —
//    no dequantization on this path.  One thread issues four
//    tcgen05.mma.kind::i8 (M = 128, N = BM, K = 32) per stage with int32
//    accumulators in tensor memory (exact: |Σ| < 127²·K); four epilogue warps
//    read their 32 rows (tcgen05.ld), convert to binary32, multiply by s_w[n]
//    and s_x[m], round to bf16 and store Y (consecutive lanes write consecutive
//    n).  Tiles are ordered m-tile fastest, as in the W4A16 tensor-core kernel.
#pragma once

#include "common.cuh"

namespace w4a16 {

constexpr int kW8a8Threads = 192;          // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kW8a8TileN = 128;            // weight rows per CTA (MMA M)
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
    static constexpr int kABytes = kW8a8TileN * kW8a8BlockK;   // 16 KB
    static constexpr int kBBytes = BM * kW8a8BlockK;
    static constexpr int kStageBytes = kABytes + kBBytes;       // multiple of 1024
    static constexpr int kStages = (196608 / kStageBytes) > 8 ? 8 : (196608 / kStageBytes);
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256;
    static constexpr int kTmemCols = BM < 32 ? 32 : BM;          // int32 accumulators, BM columns
};

// Per-token INT8 activations: X bf16 [M, K] -> q int8 [M, K], s fp32 [M].
__global__ void __launch_bounds__(kW8a8ActThreads) w8a8_quantize_act_kernel(
    const uint16_t* __restrict__ X, int64_t M, int64_t K, int8_t* __restrict__ q, float* __restrict__ s) {
    __shared__ float red[kW8a8ActThreads / 32];
    const int64_t chunks = K / 8;                              // K is a multiple of 32
    for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
        const uint16_t* row = X + m * K;
        float amax = 0.0f;
        for (int64_t c = threadIdx.x; c < chunks; c += blockDim.x) {
            const uint4 v = ldg_cached(row + 8 * c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                amax = fmaxf(amax, fabsf(__uint_as_float(w[i] << 16)));
                amax = fmaxf(amax, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
            }
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
        for (int64_t c = threadIdx.x; c < chunks; c += blockDim.x) {
            const uint4 v = ldg_cached(row + 8 * c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t packed[2] = {0u, 0u};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float x = __uint_as_float(i & 1 ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16));
                int c8 = 0;
                if (sc != 0.0f) {
                    float r = rintf(__fdiv_rn(x, sc));
                    r = fminf(fmaxf(r, -128.0f), 127.0f);
                    c8 = (int)r;
                }
                packed[i >> 2] |= ((uint32_t)c8 & 0xFFu) << (8 * (i & 3));
            }
            *reinterpret_cast<uint2*>(q + m * K + 8 * c) = make_uint2(packed[0], packed[1]);
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
            constexpr uint32_t idesc = idesc_s8_s32(kW8a8TileN, BM);
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
                for (int kk = 0; kk < kW8a8BlockK / 32; ++kk)
                    tc_mma_s8(tbase, sw128_kmajor_desc(a + kk * 32), sw128_kmajor_desc(b + kk * 32), idesc,
                              (kb > 0 || kk > 0) ? 1u : 0u);
                tc_commit(smem_u32(&empty[s]));       // the stage is free once these complete
            }
            tc_commit(smem_u32(dfull));               // the accumulators are final
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        const int quarter = warp & 3;                 // TMEM lanes 32·quarter .. +31
        const int n = n0 + 32 * quarter + lane;
        const bool got = mbar_wait(smem_u32(dfull), 0);
        tc_fence_after();
        grid_dependency_wait();                       // Y may be in use by the previous grid
        const float swn = n < N ? bf16_bits_to_f32(sw[n]) : 0.0f;
#pragma unroll 1
        for (int c0 = 0; c0 < BM; c0 += 32) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tbase + ((uint32_t)(32 * quarter) << 16) + (uint32_t)c0, r);
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
