// C ABI of the W4A16 library: argument checks, M-dispatch, launches.
// The public contract is documented in include/w4a16.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/w4a16.h"
#include "common.cuh"
#include "gemm_tcgen05.cuh"
#include "gemv_decode.cuh"
#include "quantize.cuh"

using namespace w4a16;

namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

struct DeviceInfo {
    bool ready = false;
    int sm_count = 0;
    int cc_major = 0;
    int cc_minor = 0;
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_group(int32_t g) { return g == 32 || g == 64 || g == 128; }

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

w4a16_status encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_encode_tiled == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || p == nullptr)
            return W4A16_ECUDA;
        g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    *fn = g_encode_tiled;
    return W4A16_OK;
}

w4a16_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? W4A16_OK : W4A16_ECUDA;
}

// ---------------------------------------------------------------- plans
// Decode kernel tiling: 16-row warp tiles, two per CTA; S CTAs of a cluster
// split K when the row tiles alone would leave SMs idle.
constexpr int kDecodeTPW = 2;
constexpr int kDecodeRows = 16 * kDecodeTPW;

int decode_split(int64_t N, int64_t K, int sm_count) {
    const int64_t row_blocks = (N + kDecodeRows - 1) / kDecodeRows;
    const int64_t chunks = (K + 127) / 128;
    // Aim for about 4 CTAs per SM; keep at least 2 K chunks per warp per CTA.
    const int64_t want = (int64_t)sm_count * 4;
    int s = 1;
    while (s < 8 && row_blocks * s < want && chunks / (s + 1) >= 2 * kDecodeWarps) ++s;
    return s;
}

int tc_tile_m(int64_t M) {
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;
}

int tc_smem_bytes(int bm) {
    switch (bm) {
        case 32: return TcConfig<32>::kSmemBytes;
        case 64: return TcConfig<64>::kSmemBytes;
        case 128: return TcConfig<128>::kSmemBytes;
        default: return TcConfig<256>::kSmemBytes;
    }
}

w4a16_status check_shape(int64_t M, int64_t N, int64_t K, int32_t g, int32_t sym) {
    if (!valid_group(g)) return W4A16_EINVAL;
    if (sym != 0 && sym != 1) return W4A16_EINVAL;
    if (M < 0 || N < 0 || K <= 0) return W4A16_EINVAL;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return W4A16_EINVAL;
    if (K % g != 0) return W4A16_EINVAL;
    return W4A16_OK;
}

w4a16_status make_plan(int64_t M, int64_t N, int64_t K, int32_t g, int32_t sym, int32_t path,
                       int32_t split_k, int sm_count, w4a16_plan* p) {
    w4a16_status st = check_shape(M, N, K, g, sym);
    if (st != W4A16_OK) return st;
    if (path < W4A16_PATH_AUTO || path > W4A16_PATH_TENSORCORE) return W4A16_EINVAL;
    if (split_k < 0 || split_k > 8) return W4A16_EINVAL;
    int chosen = path;
    if (chosen == W4A16_PATH_AUTO) chosen = M <= 16 ? W4A16_PATH_DECODE : W4A16_PATH_TENSORCORE;
    if (chosen == W4A16_PATH_DECODE && M > 16) return W4A16_EINVAL;
    if (chosen == W4A16_PATH_TENSORCORE && split_k > 1) return W4A16_EINVAL;
    *p = w4a16_plan{};
    p->path = chosen;
    if (chosen == W4A16_PATH_DECODE) {
        const int64_t row_blocks = (N + kDecodeRows - 1) / kDecodeRows;
        p->split_k = split_k > 0 ? split_k : decode_split(N, K, sm_count);
        p->tile_m = M <= 8 ? 8 : 16;
        p->tile_n = kDecodeRows;
        p->grid = row_blocks * p->split_k;
        p->threads = kDecodeThreads;
        p->smem_bytes = 0;
    } else {
        const int bm = tc_tile_m(M);
        p->split_k = 1;
        p->tile_m = bm;
        p->tile_n = kTcTileN;
        p->grid = ((N + kTcTileN - 1) / kTcTileN) * ((M + bm - 1) / bm);
        p->threads = kTcThreads;
        p->smem_bytes = tc_smem_bytes(bm);
    }
    return W4A16_OK;
}

// ---------------------------------------------------------------- launches
template <int MB, bool SYM, int G>
w4a16_status launch_decode_t(const w4a16_plan& p, const void* X, int M, int64_t K,
                             const void* packed, const void* scales, const void* zeros, int64_t N,
                             void* Y, cudaStream_t stream) {
    const int total_chunks = (int)((K + 127) / 128);
    const int cps = (total_chunks + p.split_k - 1) / p.split_k;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.grid, 1, 1);
    cfg.blockDim = dim3(kDecodeThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)p.split_k;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(
        &cfg, gemv_decode_kernel<MB, kDecodeTPW, SYM, G>, static_cast<const uint16_t*>(X), M, K,
        static_cast<const uint8_t*>(packed), static_cast<const uint16_t*>(scales),
        static_cast<const uint16_t*>(zeros), N, static_cast<uint16_t*>(Y), (int)p.split_k, cps);
    return e == cudaSuccess ? W4A16_OK : W4A16_ECUDA;
}

template <bool SYM, int G>
w4a16_status launch_decode_g(const w4a16_plan& p, const void* X, int M, int64_t K,
                             const void* packed, const void* scales, const void* zeros, int64_t N,
                             void* Y, cudaStream_t stream) {
    if (p.tile_m == 8) return launch_decode_t<1, SYM, G>(p, X, M, K, packed, scales, zeros, N, Y, stream);
    return launch_decode_t<2, SYM, G>(p, X, M, K, packed, scales, zeros, N, Y, stream);
}

w4a16_status launch_decode(const w4a16_plan& p, const void* X, int M, int64_t K,
                           const void* packed, const void* scales, const void* zeros, int64_t N,
                           int32_t g, int32_t sym, void* Y, cudaStream_t stream) {
#define W4A16_DECODE_CASE(GG)                                                                 \
    case GG:                                                                                  \
        return sym ? launch_decode_g<true, GG>(p, X, M, K, packed, scales, zeros, N, Y, stream) \
                   : launch_decode_g<false, GG>(p, X, M, K, packed, scales, zeros, N, Y, stream);
    switch (g) {
        W4A16_DECODE_CASE(32)
        W4A16_DECODE_CASE(64)
        W4A16_DECODE_CASE(128)
        default: return W4A16_EINVAL;
    }
#undef W4A16_DECODE_CASE
}

w4a16_status encode_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                       uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                       uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    PFN_cuTensorMapEncodeTiled_v12000 fn;
    w4a16_status st = encoder(&fn);
    if (st != W4A16_OK) return st;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? W4A16_OK : W4A16_ECUDA;
}

template <int BM, bool SYM, int G>
w4a16_status launch_tc_t(const w4a16_plan& p, const CUtensorMap& tmX, const CUtensorMap& tmP,
                         const void* scales, const void* zeros, void* Y, int M, int N, int K,
                         cudaStream_t stream) {
    auto kern = gemm_tc_kernel<BM, SYM, G>;
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 TcConfig<BM>::kSmemBytes) != cudaSuccess)
            return W4A16_ECUDA;
        attr_set[dev] = true;
    }
    dim3 grid((unsigned)((N + kTcTileN - 1) / kTcTileN), (unsigned)((M + BM - 1) / BM), 1);
    kern<<<grid, kTcThreads, TcConfig<BM>::kSmemBytes, stream>>>(
        tmX, tmP, static_cast<const uint16_t*>(scales), static_cast<const uint16_t*>(zeros),
        static_cast<uint16_t*>(Y), M, N, K);
    return launch_status();
}

template <bool SYM, int G>
w4a16_status launch_tc_g(const w4a16_plan& p, const CUtensorMap& tmX, const CUtensorMap& tmP,
                         const void* scales, const void* zeros, void* Y, int M, int N, int K,
                         cudaStream_t stream) {
    switch (p.tile_m) {
        case 32: return launch_tc_t<32, SYM, G>(p, tmX, tmP, scales, zeros, Y, M, N, K, stream);
        case 64: return launch_tc_t<64, SYM, G>(p, tmX, tmP, scales, zeros, Y, M, N, K, stream);
        case 128: return launch_tc_t<128, SYM, G>(p, tmX, tmP, scales, zeros, Y, M, N, K, stream);
        default: return launch_tc_t<256, SYM, G>(p, tmX, tmP, scales, zeros, Y, M, N, K, stream);
    }
}

w4a16_status launch_tc(const w4a16_plan& p, const void* X, int64_t M, int64_t K,
                       const void* packed, const void* scales, const void* zeros, int64_t N,
                       int32_t g, int32_t sym, void* Y, cudaStream_t stream) {
    CUtensorMap tmX, tmP;
    w4a16_status st = encode_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K,
                                (uint64_t)M, (uint64_t)K * 2, kTcBlockK, (uint32_t)p.tile_m,
                                CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != W4A16_OK) return st;
    st = encode_2d(&tmP, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)(K / 2), (uint64_t)N,
                   (uint64_t)(K / 2), kTcBlockK / 2, kTcTileN, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != W4A16_OK) return st;
    const int m = (int)M, n = (int)N, k = (int)K;
#define W4A16_TC_CASE(GG)                                                                     \
    case GG:                                                                                  \
        return sym ? launch_tc_g<true, GG>(p, tmX, tmP, scales, zeros, Y, m, n, k, stream)      \
                   : launch_tc_g<false, GG>(p, tmX, tmP, scales, zeros, Y, m, n, k, stream);
    switch (g) {
        W4A16_TC_CASE(32)
        W4A16_TC_CASE(64)
        W4A16_TC_CASE(128)
        default: return W4A16_EINVAL;
    }
#undef W4A16_TC_CASE
}

int grid_for(int64_t work_items, int threads, int sm_count) {
    const int64_t blocks = (work_items + threads - 1) / threads;
    const int64_t cap = (int64_t)sm_count * 8;   // grid-stride loops beyond 8 CTAs per SM
    return (int)(blocks < cap ? (blocks < 1 ? 1 : blocks) : cap);
}

}  // namespace

// ==================================================================== ABI
extern "C" {

int32_t w4a16_abi_version(void) { return W4A16_ABI_VERSION; }

const char* w4a16_status_string(w4a16_status s) {
    switch (s) {
        case W4A16_OK: return "W4A16_OK";
        case W4A16_EINVAL: return "W4A16_EINVAL: invalid argument";
        case W4A16_EUNSUPPORTED: return "W4A16_EUNSUPPORTED: device is not sm_100";
        case W4A16_ECUDA: return "W4A16_ECUDA: CUDA runtime error";
        case W4A16_EWORKSPACE: return "W4A16_EWORKSPACE: workspace too small";
        case W4A16_EDEVICE: return "W4A16_EDEVICE: a kernel gave up a bounded wait";
        default: return "W4A16: unknown status";
    }
}

w4a16_status w4a16_quantize(const void* W, int64_t N, int64_t K, int32_t g, int32_t sym,
                            void* packed, void* scales, void* zeros, void* stream) {
    w4a16_status st = check_shape(0, N, K, g, sym);
    if (st != W4A16_OK) return st;
    if (N == 0) return W4A16_OK;
    if (!W || !packed || !scales || (!sym && !zeros)) return W4A16_EINVAL;
    if (!aligned16(W) || !aligned16(packed) || !aligned16(scales) || (zeros && !aligned16(zeros)))
        return W4A16_EINVAL;
    DeviceInfo di;
    if ((st = device_info(&di)) != W4A16_OK) return st;
    const int64_t chunks = N * K / 8;
    const int grid = grid_for(chunks, 256, di.sm_count);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto* Wp = static_cast<const uint16_t*>(W);
    auto* Pp = static_cast<uint32_t*>(packed);
    auto* Sp = static_cast<uint16_t*>(scales);
    auto* Zp = static_cast<uint16_t*>(zeros);
#define W4A16_Q_CASE(GG)                                                                      \
    case GG:                                                                                  \
        if (sym) quantize_pack_kernel<GG, true><<<grid, 256, 0, s>>>(Wp, chunks, Pp, Sp, Zp); \
        else quantize_pack_kernel<GG, false><<<grid, 256, 0, s>>>(Wp, chunks, Pp, Sp, Zp);    \
        break;
    switch (g) {
        W4A16_Q_CASE(32)
        W4A16_Q_CASE(64)
        W4A16_Q_CASE(128)
        default: return W4A16_EINVAL;
    }
#undef W4A16_Q_CASE
    return launch_status();
}

w4a16_status w4a16_dequantize(const void* packed, const void* scales, const void* zeros,
                              int64_t N, int64_t K, int32_t g, int32_t sym, void* W_hat,
                              void* stream) {
    w4a16_status st = check_shape(0, N, K, g, sym);
    if (st != W4A16_OK) return st;
    if (N == 0) return W4A16_OK;
    if (!packed || !scales || !W_hat || (!sym && !zeros)) return W4A16_EINVAL;
    if (!aligned16(packed) || !aligned16(scales) || !aligned16(W_hat) || (!sym && !aligned16(zeros)))
        return W4A16_EINVAL;
    DeviceInfo di;
    if ((st = device_info(&di)) != W4A16_OK) return st;
    const int64_t chunks = N * K / 32;
    const int grid = grid_for(chunks, 256, di.sm_count);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto* Pp = static_cast<const uint4*>(packed);
    auto* Sp = static_cast<const uint16_t*>(scales);
    auto* Zp = static_cast<const uint16_t*>(zeros);
    auto* Wp = static_cast<uint4*>(W_hat);
#define W4A16_D_CASE(GG)                                                                       \
    case GG:                                                                                   \
        if (sym) dequantize_kernel<GG, true><<<grid, 256, 0, s>>>(Pp, Sp, Zp, chunks, Wp);     \
        else dequantize_kernel<GG, false><<<grid, 256, 0, s>>>(Pp, Sp, Zp, chunks, Wp);        \
        break;
    switch (g) {
        W4A16_D_CASE(32)
        W4A16_D_CASE(64)
        W4A16_D_CASE(128)
        default: return W4A16_EINVAL;
    }
#undef W4A16_D_CASE
    return launch_status();
}

size_t w4a16_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int32_t g) {
    (void)M;
    (void)N;
    (void)K;
    (void)g;
    return 0;
}

w4a16_status w4a16_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t g, int32_t sym,
                             int32_t path, int32_t split_k, w4a16_plan* plan) {
    if (!plan) return W4A16_EINVAL;
    return make_plan(M, N, K, g, sym, path, split_k, 148, plan);
}

w4a16_status w4a16_gemm_ex(const void* X, int64_t M, int64_t K, const void* packed,
                           const void* scales, const void* zeros, int64_t N, int32_t g,
                           int32_t sym, void* Y, void* workspace, size_t workspace_bytes,
                           int32_t path, int32_t split_k, void* stream) {
    (void)workspace;
    w4a16_plan p;
    w4a16_status st = make_plan(M, N, K, g, sym, path, split_k, 148, &p);
    if (st != W4A16_OK) return st;
    if (workspace_bytes < w4a16_gemm_workspace_size(M, N, K, g)) return W4A16_EWORKSPACE;
    if (M == 0 || N == 0) return W4A16_OK;
    if (!X || !packed || !scales || !Y || (!sym && !zeros)) return W4A16_EINVAL;
    if (!aligned16(X) || !aligned16(packed) || !aligned16(scales) || !aligned16(Y) ||
        (!sym && !aligned16(zeros)))
        return W4A16_EINVAL;
    DeviceInfo di;
    if ((st = device_info(&di)) != W4A16_OK) return st;
    if (di.sm_count != 148) {
        st = make_plan(M, N, K, g, sym, path, split_k, di.sm_count, &p);
        if (st != W4A16_OK) return st;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (p.path == W4A16_PATH_DECODE)
        return launch_decode(p, X, (int)M, K, packed, scales, zeros, N, g, sym, Y, s);
    return launch_tc(p, X, M, K, packed, scales, zeros, N, g, sym, Y, s);
}

w4a16_status w4a16_gemm(const void* X, int64_t M, int64_t K, const void* packed,
                        const void* scales, const void* zeros, int64_t N, int32_t g,
                        int32_t sym, void* Y, void* workspace, size_t workspace_bytes,
                        void* stream) {
    return w4a16_gemm_ex(X, M, K, packed, scales, zeros, N, g, sym, Y, workspace,
                         workspace_bytes, W4A16_PATH_AUTO, 0, stream);
}

w4a16_status w4a16_device_error(int32_t* code) {
    if (!code) return W4A16_EINVAL;
    if (cudaDeviceSynchronize() != cudaSuccess) return W4A16_ECUDA;
    int value = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&value, g_device_error, sizeof(int)) != cudaSuccess) return W4A16_ECUDA;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return W4A16_ECUDA;
    *code = value;
    return W4A16_OK;
}

}  // extern "C"
