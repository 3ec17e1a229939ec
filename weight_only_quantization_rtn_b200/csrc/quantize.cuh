// Quantize/pack and dequantize kernels (HBM-bound, one pass each).
//
// Quantization follows "推理优化中“用精度换性能“的核心技术：量化",
// §2.3 (x_int = round(x/s) + z) and §3.3 (asymmetric s = (max − min)/(2^b − 1),
// z = round(−min/s); symmetric s = max|x|/max_int, z = 0), with b = 4 and
// groups of g elements along K (§3.4).  Arithmetic is binary32 with IEEE
// round-to-nearest division (__fdiv_rn) and round-half-to-even (rintf); the
// scale is rounded to bf16 before z and q are formed, the asymmetric range is
// widened to contain 0, and codes are clamped to the INT4 range.
#pragma once

#include "common.cuh"

namespace w4a16 {

// Clamp in binary32 before converting to an integer.
__device__ __forceinline__ float clampf(float r, float lo, float hi) {
    return r < lo ? lo : (r > hi ? hi : r);
}

// Eight bf16 elements (one 16-byte load) widened to binary32.
__device__ __forceinline__ void unpack8(const uint4 v, float x[8]) {
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(wv[i] << 16);
        x[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
    }
}

// Asymmetric scale and zero point of a group from its range [mn, mx] (already
// widened to contain 0): s = bf16_rn((mx − mn)/15), z = clamp(rint(−mn/s), 0, 15).
// Returns the bf16 bits of s; z = 0 when s rounds to 0.
__device__ __forceinline__ uint32_t asym_params(float mn, float mx, float* s, int32_t* z) {
    const uint32_t s_bits = f32_to_bf16_bits_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
    *s = bf16_bits_to_f32(s_bits);
    *z = *s != 0.0f ? (int32_t)clampf(rintf(__fdiv_rn(-mn, *s)), 0.0f, 15.0f) : 0;
    return s_bits;
}

// Symmetric scale s = bf16_rn(max|x| / 7).
__device__ __forceinline__ uint32_t sym_params(float amax, float* s) {
    const uint32_t s_bits = f32_to_bf16_bits_rn(__fdiv_rn(amax, 7.0f));
    *s = bf16_bits_to_f32(s_bits);
    return s_bits;
}

// Codes of eight elements, element i in nibble i: q = clamp(rint(x/s) + z, 0, 15)
// (asymmetric) or clamp(rint(x/s), −8, 7) as 4-bit two's complement (symmetric).
// All codes are 0 when s is 0.  rint is the binary32 addition of 1.5·2^23 to the
// quotient (clamped to ±32 first, which changes no code): the sum rounds to the
// nearest integer, ties to even, and its bit pattern minus that of 1.5·2^23 is
// the integer itself, so no float-to-integer conversion is needed.
template <bool SYM>
__device__ __forceinline__ uint32_t codes8(const float x[8], float s, int32_t z) {
    uint32_t word = 0;
    if (s == 0.0f) return word;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float r = clampf(__fdiv_rn(x[i], s), -32.0f, 32.0f);
        int32_t q = __float_as_int(r + 12582912.0f) - 0x4B400000;
        if (SYM) {
            q = q < -8 ? -8 : (q > 7 ? 7 : q);
            word |= ((uint32_t)q & 0xFu) << (4 * i);
        } else {
            q += z;
            q = q < 0 ? 0 : (q > 15 ? 15 : q);
            word |= (uint32_t)q << (4 * i);
        }
    }
    return word;
}

// Range of eight elements: asymmetric min/max (folded into mn, mx) or max|x| (into mx).
template <bool SYM>
__device__ __forceinline__ void range8(const float x[8], float& mn, float& mx) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (SYM) {
            const float a = fabsf(x[i]);
            mx = a > mx ? a : mx;
        } else {
            mn = x[i] < mn ? x[i] : mn;
            mx = x[i] > mx ? x[i] : mx;
        }
    }
}

// One thread owns 8 consecutive elements (one 16-byte load, one 32-bit packed
// store); TPG = G/8 consecutive lanes own one group and combine their range
// with butterfly shuffles.  Loops are warp-uniform so every shuffle has all 32
// lanes present.
template <int G, bool SYM>
__global__ void __launch_bounds__(256) quantize_pack_kernel(const uint16_t* __restrict__ W,
                                                            int64_t total_chunks,
                                                            uint32_t* __restrict__ packed32,
                                                            uint16_t* __restrict__ scales,
                                                            uint16_t* __restrict__ zeros) {
    constexpr int TPG = G / 8;
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t base = warp0 * 32; base < total_chunks; base += nwarps * 32) {
        const int64_t c = base + lane;
        const bool valid = c < total_chunks;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (valid) v = ldg_stream(W + c * 8);
        float x[8];
        unpack8(v, x);
        float mn = 0.0f, mx = 0.0f;                     // asymmetric range widened to contain 0
        range8<SYM>(x, mn, mx);
#pragma unroll
        for (int o = 1; o < TPG; o <<= 1) {
            const float omx = __shfl_xor_sync(0xffffffffu, mx, o);
            mx = omx > mx ? omx : mx;
            if (!SYM) {
                const float omn = __shfl_xor_sync(0xffffffffu, mn, o);
                mn = omn < mn ? omn : mn;
            }
        }
        float s;
        int32_t z = 0;
        const uint32_t s_bits = SYM ? sym_params(mx, &s) : asym_params(mn, mx, &s, &z);
        const uint32_t word = codes8<SYM>(x, s, z);
        if (valid) {
            packed32[c] = word;
            if ((lane & (TPG - 1)) == 0) {
                const int64_t grp = c / TPG;
                scales[grp] = (uint16_t)s_bits;
                if (zeros != nullptr) zeros[grp] = (uint16_t)f32_to_bf16_bits_rn((float)z);
            }
        }
    }
}

// Per-channel granularity (g = K: one scale, and one zero point, per output row;
// "量化实战深入（GPTQ / AWQ / SmoothQuant / KV 量化）", 量化粒度 table;
// "推理优化中“用精度换性能“的核心技术：量化", §3.4).  One CTA of 256 threads per row
// and step: a first pass over the row finds its range (min/max are exact, so the
// order of the reduction does not matter), a second pass forms the codes.  The
// row (at most 64 KB at K = 32768) is still in L2 for the second read.
constexpr int kQuantRowThreads = 256;

template <bool SYM>
__global__ void __launch_bounds__(kQuantRowThreads) quantize_rows_kernel(
    const uint16_t* __restrict__ W, int64_t N, int64_t K, uint32_t* __restrict__ packed32,
    uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros) {
    __shared__ float part_mn[kQuantRowThreads / 32], part_mx[kQuantRowThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t cpr = K / 8;                            // 8-element chunks per row
    for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
        const uint16_t* row = W + n * K;
        float mn = 0.0f, mx = 0.0f;
        for (int64_t c = threadIdx.x; c < cpr; c += kQuantRowThreads) {
            float x[8];
            unpack8(ldg_stream(row + c * 8), x);
            range8<SYM>(x, mn, mx);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float omx = __shfl_xor_sync(0xffffffffu, mx, o);
            const float omn = __shfl_xor_sync(0xffffffffu, mn, o);
            mx = omx > mx ? omx : mx;
            mn = omn < mn ? omn : mn;
        }
        if (lane == 0) {
            part_mn[warp] = mn;
            part_mx[warp] = mx;
        }
        __syncthreads();
#pragma unroll
        for (int w = 0; w < kQuantRowThreads / 32; ++w) {
            mn = part_mn[w] < mn ? part_mn[w] : mn;
            mx = part_mx[w] > mx ? part_mx[w] : mx;
        }
        __syncthreads();                                  // part_* are rewritten for the next row
        float s;
        int32_t z = 0;
        const uint32_t s_bits = SYM ? sym_params(mx, &s) : asym_params(mn, mx, &s, &z);
        for (int64_t c = threadIdx.x; c < cpr; c += kQuantRowThreads) {
            float x[8];
            unpack8(ldg_stream(row + c * 8), x);
            packed32[n * cpr + c] = codes8<SYM>(x, s, z);
        }
        if (threadIdx.x == 0) {
            scales[n] = (uint16_t)s_bits;
            if (zeros != nullptr) zeros[n] = (uint16_t)f32_to_bf16_bits_rn((float)z);
        }
    }
}

// Ŵ = bf16_rn((q − z)·s): one thread expands 32 codes (one 16-byte load) into
// 64 bytes of bf16; the 32 codes always lie in one group since g ≥ 32.
template <int G, bool SYM>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint4* __restrict__ packed16,
                                                         const uint16_t* __restrict__ scales,
                                                         const uint16_t* __restrict__ zeros,
                                                         int64_t total_chunks,
                                                         uint4* __restrict__ W_hat) {
    // One 4-byte word (8 codes) per thread and step, so that a warp's loads are
    // 128 contiguous bytes and its stores (8 bf16 = 16 bytes each) 512.
    constexpr int WPG = G / 8;   // words per group
    const uint32_t* packed = reinterpret_cast<const uint32_t*>(packed16);
    const int64_t total_words = total_chunks * 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < total_words; w += stride) {
        uint32_t v;
        asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(packed + w));
        const int64_t grp = w / WPG;
        const uint32_t ss = dup16(ldg_u16(scales + grp));
        const uint32_t zz = zero_pair<SYM>(SYM ? 0u : (uint32_t)ldg_u16(zeros + grp));
        uint32_t d[4];
        dequant8_natural<SYM>(v, zz, ss, d);
        W_hat[w] = make_uint4(d[0], d[1], d[2], d[3]);
    }
}

// Per-channel Ŵ (g = K): one CTA per row and step, the row's scale and zero
// point read once; one 4-byte word (8 codes) per thread as above.
template <bool SYM>
__global__ void __launch_bounds__(256) dequantize_rows_kernel(const uint32_t* __restrict__ packed,
                                                              const uint16_t* __restrict__ scales,
                                                              const uint16_t* __restrict__ zeros,
                                                              int64_t N, int64_t K,
                                                              uint4* __restrict__ W_hat) {
    const int64_t wpr = K / 8;                            // words per row
    for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
        const uint32_t ss = dup16(ldg_u16(scales + n));
        const uint32_t zz = zero_pair<SYM>(SYM ? 0u : (uint32_t)ldg_u16(zeros + n));
        for (int64_t c = threadIdx.x; c < wpr; c += blockDim.x) {
            uint32_t v;
            asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(packed + n * wpr + c));
            uint32_t d[4];
            dequant8_natural<SYM>(v, zz, ss, d);
            W_hat[n * wpr + c] = make_uint4(d[0], d[1], d[2], d[3]);
        }
    }
}

// X'[m, k] = bf16_rn(X[m, k]·a[k]): the per-input-channel activation scale for
// the tensor-core GEMM, formed once per call ("推理优化中“用精度换性能“的核心技术：
// 量化", §5.2 and §6.2, the activation half of the equivalent scaling).  The
// product of two bf16 values is exact in binary32 and mul.rn.bf16x2 rounds it
// once.  One 16-byte chunk (8 elements) per thread and step; K is a multiple of
// 8, so a chunk never crosses a row.
__global__ void __launch_bounds__(256) scale_activations_kernel(const uint4* __restrict__ X,
                                                                const uint4* __restrict__ a,
                                                                int64_t chunks, int64_t row_chunks,
                                                                uint4* __restrict__ Xs) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 v = X[i];
        const uint4 s = a[i % row_chunks];
        Xs[i] = make_uint4(bf16x2_mul(v.x, s.x), bf16x2_mul(v.y, s.y), bf16x2_mul(v.z, s.z),
                           bf16x2_mul(v.w, s.w));
    }
}

}  // namespace w4a16
