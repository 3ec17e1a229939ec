// W8A16: the 8-bit form of weight-only RTN quantization, one code per byte.
//
// The page "推理优化中“用精度换性能“的核心技术：量化"
// states the INT8 form directly in §3.3: asymmetric s = (max − min)/255,
// z = round(−min/s); symmetric s = max|x|/max_int with max_int = 127 ("量化实战深入（GPTQ / AWQ / SmoothQuant / KV 量化）"
// §二, absmax with b = 8).  "大模型推理中 Weight-only、W8A8 和 FP8 量化有什么区别？如何选型？" (详细版) lists W8A16 beside
// W4A16.  Readings as for INT4: round half to even in binary32, s rounded to
// bf16 before z and q, the asymmetric range widened to contain 0, codes clamped
// to [0, 255] or [−128, 127] (symmetric codes stored as int8), x̂ =
// bf16_rn((q − z)·s) — |q − z| ≤ 255 times an 8-bit significand is exact in
// binary32, so one rounding.
//
// Kernels (this translation unit shares no device code with the INT4 one):
//  * w8_quantize_kernel / w8_quantize_rows_kernel: one pass over W, grouped
//    (G/8 lanes per group, butterfly shuffles) or per-channel (g = K, one CTA
//    per row, block-wide range reduction and a second pass from L2);
//  * w8_dequantize_kernel: 8 codes (one 8-byte load) per thread and step.
// The fused GEMMs for 8-bit codes are instances of the INT4 translation unit's
// kernels: gemv_decode_kernel for M ≤ 16 and gemm_tc_kernel for larger M.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/w4a16.h"

namespace w8 {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;
constexpr int kThreads = 256;

__device__ __forceinline__ float bf16_to_f32(uint32_t bits) { return __uint_as_float(bits << 16); }

__device__ __forceinline__ uint32_t f32_to_bf16_rn(float f) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ float clampf(float r, float lo, float hi) {
    return r < lo ? lo : (r > hi ? hi : r);
}

__device__ __forceinline__ uint4 ldg16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Eight bf16 elements widened to binary32.
__device__ __forceinline__ void unpack8(const uint4 v, float x[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Range of eight elements: min/max widened to contain 0 (asym) or max|x| (sym, into mx).
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

// Scale (bf16 bits) and zero point of a group from its range.
template <bool SYM>
__device__ __forceinline__ uint32_t params(float mn, float mx, float* s, int32_t* z) {
    const float s32 = SYM ? __fdiv_rn(mx, 127.0f) : __fdiv_rn(__fsub_rn(mx, mn), 255.0f);
    const uint32_t s_bits = f32_to_bf16_rn(s32);
    *s = bf16_to_f32(s_bits);
    *z = (!SYM && *s != 0.0f) ? (int32_t)clampf(rintf(__fdiv_rn(-mn, *s)), 0.0f, 255.0f) : 0;
    return s_bits;
}

// Codes of eight elements as eight bytes (element i in byte i).  rint is the
// binary32 addition of 1.5·2^23 to the quotient (clamped to ±512 first, which
// changes no code): the sum rounds to the nearest integer, ties to even, and its
// bit pattern minus that of 1.5·2^23 is the integer.
template <bool SYM>
__device__ __forceinline__ uint2 codes8(const float x[8], float s, int32_t z) {
    uint32_t b[2] = {0u, 0u};
    if (s != 0.0f) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float r = clampf(__fdiv_rn(x[i], s), -512.0f, 512.0f);
            int32_t q = __float_as_int(r + 12582912.0f) - 0x4B400000;
            if (SYM) {
                q = q < -128 ? -128 : (q > 127 ? 127 : q);
            } else {
                q += z;
                q = q < 0 ? 0 : (q > 255 ? 255 : q);
            }
            b[i >> 2] |= ((uint32_t)q & 0xFFu) << (8 * (i & 3));
        }
    }
    return make_uint2(b[0], b[1]);
}

// Grouped quantization: one thread per 8 consecutive elements, TPG = G/8 lanes per group.
template <int G, bool SYM>
__global__ void __launch_bounds__(kThreads) w8_quantize_kernel(const uint16_t* __restrict__ W,
                                                              int64_t chunks,
                                                              uint2* __restrict__ codes,
                                                              uint16_t* __restrict__ scales,
                                                              uint16_t* __restrict__ zeros) {
    constexpr int TPG = G / 8;
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t base = warp0 * 32; base < chunks; base += nwarps * 32) {
        const int64_t c = base + lane;
        const bool valid = c < chunks;
        float x[8];
        unpack8(valid ? ldg16(W + c * 8) : make_uint4(0, 0, 0, 0), x);
        float mn = 0.0f, mx = 0.0f;
        range8<SYM>(x, mn, mx);
#pragma unroll
        for (int o = 1; o < TPG; o <<= 1) {
            const float omx = __shfl_xor_sync(0xffffffffu, mx, o);
            const float omn = __shfl_xor_sync(0xffffffffu, mn, o);
            mx = omx > mx ? omx : mx;
            mn = omn < mn ? omn : mn;
        }
        float s;
        int32_t z;
        const uint32_t s_bits = params<SYM>(mn, mx, &s, &z);
        const uint2 q = codes8<SYM>(x, s, z);
        if (valid) {
            codes[c] = q;
            if ((lane & (TPG - 1)) == 0) {
                scales[c / TPG] = (uint16_t)s_bits;
                if (zeros != nullptr) zeros[c / TPG] = (uint16_t)f32_to_bf16_rn((float)z);
            }
        }
    }
}

// Per-channel quantization (g = K): one CTA per row and step, a block-wide range
// reduction (min/max are exact, order-free), then the codes from a second pass.
template <bool SYM>
__global__ void __launch_bounds__(kThreads) w8_quantize_rows_kernel(
    const uint16_t* __restrict__ W, int64_t N, int64_t K, uint2* __restrict__ codes,
    uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros) {
    __shared__ float part_mn[kThreads / 32], part_mx[kThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t cpr = K / 8;
    for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
        const uint16_t* row = W + n * K;
        float mn = 0.0f, mx = 0.0f;
        for (int64_t c = threadIdx.x; c < cpr; c += kThreads) {
            float x[8];
            unpack8(ldg16(row + c * 8), x);
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
        for (int w = 0; w < kThreads / 32; ++w) {
            mn = part_mn[w] < mn ? part_mn[w] : mn;
            mx = part_mx[w] > mx ? part_mx[w] : mx;
        }
        __syncthreads();                                  // part_* are rewritten for the next row
        float s;
        int32_t z;
        const uint32_t s_bits = params<SYM>(mn, mx, &s, &z);
        for (int64_t c = threadIdx.x; c < cpr; c += kThreads) {
            float x[8];
            unpack8(ldg16(row + c * 8), x);
            codes[n * cpr + c] = codes8<SYM>(x, s, z);
        }
        if (threadIdx.x == 0) {
            scales[n] = (uint16_t)s_bits;
            if (zeros != nullptr) zeros[n] = (uint16_t)f32_to_bf16_rn((float)z);
        }
    }
}

// Code byte i of a 32-bit word as a signed (SYM) or unsigned integer.
template <bool SYM>
__device__ __forceinline__ int32_t code_of(uint32_t word, int i) {
    const uint32_t b = (word >> (8 * i)) & 0xFFu;
    return SYM ? (int32_t)(int8_t)b : (int32_t)b;
}

// x̂ = bf16_rn((q − z)·s): the product is exact in binary32, rounded once.
__device__ __forceinline__ uint32_t dequant1(int32_t q, int32_t z, float s) {
    return f32_to_bf16_rn((float)(q - z) * s);
}

// Ŵ from the codes: 8 codes (one 8-byte load) per thread and step; `gpw` = 8-code
// words per group (g/8; K/8 for per-channel).
template <bool SYM>
__global__ void __launch_bounds__(kThreads) w8_dequantize_kernel(const uint2* __restrict__ codes,
                                                                const uint16_t* __restrict__ scales,
                                                                const uint16_t* __restrict__ zeros,
                                                                int64_t words, int64_t gpw,
                                                                uint4* __restrict__ W_hat) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words; w += stride) {
        uint2 v;
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                     : "=r"(v.x), "=r"(v.y)
                     : "l"(codes + w));
        const int64_t grp = w / gpw;
        const float s = bf16_to_f32(__ldg(scales + grp));
        const int32_t z = SYM ? 0 : (int32_t)bf16_to_f32(__ldg(zeros + grp));
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t word = j < 2 ? v.x : v.y;
            const uint32_t lo = dequant1(code_of<SYM>(word, 2 * (j & 1)), z, s);
            const uint32_t hi = dequant1(code_of<SYM>(word, 2 * (j & 1) + 1), z, s);
            o[j] = lo | (hi << 16);
        }
        W_hat[w] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// ---------------------------------------------------------------- host side
struct DeviceInfo {
    bool ready = false;
    int sm_count = 0;
    int cc_major = 0;
    int cc_minor = 0;
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];

w4a16_status device_info(DeviceInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return W4A16_ECUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo& d = g_devices[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return W4A16_ECUDA;
        d.ready = true;
    }
    *out = d;
    if (d.cc_major != 10 || d.cc_minor != 0) return W4A16_EUNSUPPORTED;   // built for sm_100a only
    return W4A16_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool grouped(int32_t g) { return g == 32 || g == 64 || g == 128; }
bool per_channel(int32_t g, int64_t K) { return !grouped(g) && (int64_t)g == K; }

// The same shape rules as the INT4 entry points: g ∈ {32, 64, 128} dividing K,
// or g = K (per-channel) with K a multiple of 32.
w4a16_status check_shape(int64_t N, int64_t K, int32_t g, int32_t sym) {
    if (sym != 0 && sym != 1) return W4A16_EINVAL;
    if (N < 0 || K <= 0 || N > kMaxDim || K > kMaxDim) return W4A16_EINVAL;
    if (grouped(g)) return K % g == 0 ? W4A16_OK : W4A16_EINVAL;
    return (per_channel(g, K) && K % 32 == 0) ? W4A16_OK : W4A16_EINVAL;
}

int grid_for(int64_t items, int sm_count) {
    const int64_t blocks = (items + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)sm_count * 8;
    return (int)(blocks < 1 ? 1 : (blocks < cap ? blocks : cap));
}

w4a16_status launch_status() { return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ECUDA; }


}  // namespace w8

using namespace w8;

extern "C" {

w4a16_status w8a16_quantize(const void* W, int64_t N, int64_t K, int32_t g, int32_t sym,
                            void* codes, void* scales, void* zeros, void* stream) {
    w4a16_status st = check_shape(N, K, g, sym);
    if (st != W4A16_OK) return st;
    if (N == 0) return W4A16_OK;
    if (!W || !codes || !scales || (!sym && !zeros)) return W4A16_EINVAL;
    if (!aligned16(W) || !aligned16(codes) || !aligned16(scales) || (zeros && !aligned16(zeros)))
        return W4A16_EINVAL;
    DeviceInfo di;
    if ((st = device_info(&di)) != W4A16_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto* Wp = static_cast<const uint16_t*>(W);
    auto* Cp = static_cast<uint2*>(codes);
    auto* Sp = static_cast<uint16_t*>(scales);
    auto* Zp = static_cast<uint16_t*>(zeros);
    if (per_channel(g, K)) {
        const int grid = (int)(N < (int64_t)di.sm_count * 8 ? N : (int64_t)di.sm_count * 8);
        if (sym) w8_quantize_rows_kernel<true><<<grid, kThreads, 0, s>>>(Wp, N, K, Cp, Sp, Zp);
        else w8_quantize_rows_kernel<false><<<grid, kThreads, 0, s>>>(Wp, N, K, Cp, Sp, Zp);
        return launch_status();
    }
    const int64_t chunks = N * K / 8;
    const int grid = grid_for(chunks, di.sm_count);
#define W8_Q_CASE(GG)                                                                          \
    case GG:                                                                                   \
        if (sym) w8_quantize_kernel<GG, true><<<grid, kThreads, 0, s>>>(Wp, chunks, Cp, Sp, Zp); \
        else w8_quantize_kernel<GG, false><<<grid, kThreads, 0, s>>>(Wp, chunks, Cp, Sp, Zp);  \
        break;
    switch (g) {
        W8_Q_CASE(32)
        W8_Q_CASE(64)
        W8_Q_CASE(128)
        default: return W4A16_EINVAL;
    }
#undef W8_Q_CASE
    return launch_status();
}

w4a16_status w8a16_dequantize(const void* codes, const void* scales, const void* zeros,
                              int64_t N, int64_t K, int32_t g, int32_t sym, void* W_hat,
                              void* stream) {
    w4a16_status st = check_shape(N, K, g, sym);
    if (st != W4A16_OK) return st;
    if (N == 0) return W4A16_OK;
    if (!codes || !scales || !W_hat || (!sym && !zeros)) return W4A16_EINVAL;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(W_hat) || (!sym && !aligned16(zeros)))
        return W4A16_EINVAL;
    DeviceInfo di;
    if ((st = device_info(&di)) != W4A16_OK) return st;
    const int64_t words = N * K / 8;
    const int64_t gpw = (per_channel(g, K) ? K : (int64_t)g) / 8;
    const int grid = grid_for(words, di.sm_count);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto* Cp = static_cast<const uint2*>(codes);
    auto* Sp = static_cast<const uint16_t*>(scales);
    auto* Zp = static_cast<const uint16_t*>(zeros);
    auto* Wp = static_cast<uint4*>(W_hat);
    if (sym) w8_dequantize_kernel<true><<<grid, kThreads, 0, s>>>(Cp, Sp, Zp, words, gpw, Wp);
    else w8_dequantize_kernel<false><<<grid, kThreads, 0, s>>>(Cp, Sp, Zp, words, gpw, Wp);
    return launch_status();
}

}  // extern "C"
