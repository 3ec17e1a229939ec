// C ABI of the W4A16 library: argument checks, M-dispatch, launches.
// The public contract is documented in include/w4a16.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "../../include/w4a16.h"
#include "common.cuh"
#include "gemm_tcgen05.cuh"
#include "gemm_w8a8.cuh"
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

// Group sizes along K with kernels of their own.
bool grouped(int32_t g) { return g == 32 || g == 64 || g == 128; }

// Per-channel granularity: one group spanning the whole row (g == K), one scale
// and zero point per output feature ("量化实战深入（GPTQ / AWQ / SmoothQuant / KV 量化）", 量化粒度 table;
// "推理优化中“用精度换性能“的核心技术：量化", §3.4).
// Kernels take it as group size 0.
bool per_channel(int32_t g, int64_t K) { return !grouped(g) && (int64_t)g == K; }

// g is one of the grouped sizes with K a multiple of it, or g == K with K a
// multiple of 32 (packed rows of whole 16-byte chunks, as TMA needs).
bool valid_group(int32_t g, int64_t K) {
    if (grouped(g)) return K % g == 0;
    return per_channel(g, K) && K % 32 == 0;
}

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
constexpr int kSmemPerBlockMax = 232448;  // opt-in maximum per CTA (227 KB)
constexpr int kMaxCtas = 65535;

// Decode kernel geometry for (M, N, K, g): 256-row x 256-K units, one CTA per
// SM with a ring of shared-memory stages and scale slabs filling its shared
// memory.
struct DecodeGeometry {
    int bits;          // code width, 4 or 8
    int mb;            // n8 MMA column blocks (1: M ≤ 8, 2: M ≤ 16)
    int rb;            // row blocks of 256 rows
    int kbn;           // K blocks of 256
    int64_t units;     // rb · kbn
    int gu;            // scale groups per row per unit (1 for per-channel)
    int sw;            // groups per staged scale row without TMA slabs (0 with them)
    int sz_tma;        // scales staged by TMA in 8-group slabs (rows 16-byte aligned)
    int slabs;         // slab ring slots (0 without TMA slabs)
    int slab_off;      // slab ring inside the dynamic shared memory
    int xf_off;        // fragment-ordered X inside a stage
    int sz_off;        // scales and zeros inside a stage
    int stage_bytes;   // multiple of 1024
    int stages;
    int ctas_per_sm;
    int smem_bytes;    // dynamic shared memory per CTA
};

// Outside the stages: zero fragments, barriers and flags (< 1024 bytes), plus
// slack to align the dynamic shared memory base to 1024 bytes.
constexpr int kDecFixedSmem = 1024 + 1024;

// Scale (and zero) groups of one row inside a 256-wide K block.
int decode_block_k(int bits) { return bits == 8 ? dec_block_k<8>() : dec_block_k<4>(); }
int decode_unit_groups(int32_t g, int64_t K, int bits) {
    return per_channel(g, K) ? 1 : decode_block_k(bits) / g;
}

// Stage: codes tile (16 KB, TMA, 128-byte swizzle) | X slice, natural order
// (M x 512 B, TMA) | X in fragment order (rows 576 B apart, the last one 512 B;
// 128-byte aligned) | without TMA slabs, scales and zeros (2 x 256 rows x gu bf16).
DecodeGeometry decode_geometry(int64_t M, int64_t N, int64_t K, int g, int bits = 4) {
    DecodeGeometry d{};
    d.bits = bits;
    d.mb = M <= 8 ? 1 : 2;
    d.rb = (int)((N + kDecRows - 1) / kDecRows);
    const int bk = decode_block_k(bits);
    const int xrb = bk * 2, xfrb = bk * 2 + 64;   // X rows: natural, fragment order (padded)
    d.kbn = (int)((K + bk - 1) / bk);
    d.units = (int64_t)d.rb * d.kbn;
    d.gu = decode_unit_groups(g, K, bits);
    d.sz_tma = (!per_channel(g, K) && (K / g) % 8 == 0) ? 1 : 0;
    const int m = M < 1 ? 1 : (int)M;
    const int xnat_end = kDecPBytes + m * xrb;
    d.xf_off = (xnat_end + 127) / 128 * 128;
    const int xf_end = d.xf_off + (m - 1) * xfrb + xrb;
    d.sz_off = (xf_end + 127) / 128 * 128;      // TMA destinations are 128-byte aligned
    // Scales in the stage only without TMA slabs; with them, a ring of slab slots.
    // A unit with a single group whose rows hold an even number of groups stages
    // the 4-byte aligned pair around it (the copy mode decode_scale_copy picks).
    const bool pairs = !d.sz_tma && !per_channel(g, K) && d.gu == 1 && (K / g) % 2 == 0;
    d.sw = d.sz_tma ? 0 : (pairs ? 2 : d.gu);
    const int stage_raw = d.sz_off + 2 * kDecRows * d.sw * 2;
    d.stage_bytes = (stage_raw + 1023) / 1024 * 1024;
    // Slab slots: one the consumers read, plus enough for the units the producer
    // may run ahead (the ring depth) at 8/gu units per slab, plus one for a slab
    // boundary in between; at least 2, at most one per stage plus one.
    const int ups = d.sz_tma ? 8 / d.gu : 1;
    auto slabs_for = [&](int stages) {
        if (!d.sz_tma) return 0;
        int sl = (stages + 1 + ups - 1) / ups + 1;
        if (sl > stages + 1) sl = stages + 1;
        if (sl < 2) sl = 2;
        if (sl > kDecMaxSlabs) sl = kDecMaxSlabs;
        return sl;
    };
    auto fits = [&](int stages, int budget) {
        return stages * d.stage_bytes + slabs_for(stages) * kDecSlabBytes <= budget;
    };
    // One CTA per SM (16 consumer warps; two such CTAs would not fit the registers).
    int one = 0;
    while (one < kDecMaxStages && fits(one + 1, kSmemPerBlockMax - kDecFixedSmem)) ++one;
    d.ctas_per_sm = 1;
    d.stages = one;
    d.slabs = slabs_for(d.stages);
    d.slab_off = d.stages * d.stage_bytes;
    d.smem_bytes = d.slab_off + d.slabs * kDecSlabBytes + kDecFixedSmem;
    return d;
}

// The stage layout's invariants: every TMA destination (codes, X, scale and zero
// slabs) 128-byte aligned, the codes tile 1024-byte aligned (128-byte swizzle),
// the fragment-ordered X 128-byte aligned (bank spread of the consumers' loads),
// and the ring within the shared memory of one CTA.
bool decode_geometry_ok(const DecodeGeometry& d, int64_t M) {
    const int m = M < 1 ? 1 : (int)M;
    const int sw = d.sw;                       // scales in the stage only without slabs
    const int xrb = decode_block_k(d.bits) * 2, xfrb = xrb + 64;
    return (d.bits == 4 || d.bits == 8) && d.stage_bytes % 1024 == 0 && kDecPBytes % 128 == 0 &&
           d.xf_off % 128 == 0 && d.xf_off >= kDecPBytes + m * xrb && d.sz_off % 128 == 0 &&
           d.sz_off >= d.xf_off + (m - 1) * xfrb + xrb &&
           (kDecRows * sw * 2) % 128 == 0 && d.sz_off + 2 * kDecRows * sw * 2 <= d.stage_bytes &&
           d.stages >= 2 && d.stages <= kDecMaxStages && d.slab_off % 1024 == 0 &&
           (d.sz_tma ? d.slabs >= 2 && d.slabs <= kDecMaxSlabs : d.slabs == 0) &&
           kDecSlabBytes % 1024 == 0 && d.smem_bytes <= kSmemPerBlockMax;
}

// Workspace of a decode launch with `ctas` CTAs: (rb + ctas) slots, slot rb + c
// holding CTA c's part of a row block that the stream-K partition splits —
// per slot 16 ready flags, then 16 warps x 32 lanes x 4·mb fp32 partial sums.
// Scratch: no initialization is needed (a flag counts only when it holds the
// ready pattern, which the consuming CTA clears again).
int64_t decode_flag_bytes(const DecodeGeometry& d, int64_t ctas) {
    return ((int64_t)(d.rb + ctas) * kDecConsumers * 4 + 255) / 256 * 256;
}

int64_t decode_workspace_bytes(const DecodeGeometry& d, int64_t ctas) {
    return decode_flag_bytes(d, ctas) + (int64_t)(d.rb + ctas) * kDecConsumers * 32 * 16 * d.mb;
}

// Row blocks the even unit split cuts between CTAs.
int64_t decode_split_blocks(const DecodeGeometry& d, int64_t ctas) {
    int64_t n = 0, last = -1;
    for (int64_t b = 1; b < ctas; ++b) {
        const int64_t u = b * d.units / ctas;
        if (u % d.kbn != 0 && u / d.kbn != last) {
            ++n;
            last = u / d.kbn;
        }
    }
    return n;
}

int tc_tile_m(int64_t M) {
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;
}

// Split-K for the tensor-core path: when the (n, m) tiles are fewer than the
// resident CTA slots, split each tile's K blocks over up to slots / tiles CTAs (at most 8, at
// least 4 K blocks each); split boundaries are multiples of the scale slab
// (g/8 blocks) when scales come by TMA.  Returns K blocks per split.
int tc_kb_split(int num_kb, int splits, int g, bool sz_tma) {
    int kbs = (num_kb + splits - 1) / splits;
    const int slab = sz_tma ? g / 8 : 1;
    return (kbs + slab - 1) / slab * slab;
}

// Tensor-core launch schedule.  Output tiles (128 weight rows x bm activation
// rows) run unsplit in a "head" launch; K is split over `splits` CTAs per tile for
// the "tail" tiles, whose partials a reduce kernel adds.  A wave is one CTA per
// resident slot (SMs x tc_ctas_per_sm(bm)).  All tiles are tail when they are
// fewer than the slots; otherwise only a last partial wave that would leave more
// than half of the slots idle becomes the tail.  Splits: up to slots / tail tiles,
// at most 8, at least 4 K blocks each.
struct TcSchedule {
    int tiles_n;      // n-tiles (128 weight rows each)
    int64_t head;     // unsplit tiles [0, head)
    int64_t tail;     // split tiles [head, head + tail)
    int splits;       // K splits of each tail tile (1 when there is no tail)
    int kb_split;     // K blocks per split
};

TcSchedule tc_schedule(int64_t M, int64_t N, int64_t K, int g, int bm, int sm_count) {
    TcSchedule t{};
    sm_count *= tc_ctas_per_sm(bm);           // resident CTA slots
    t.tiles_n = (int)((N + kTcTileN - 1) / kTcTileN);
    const int64_t tiles = (int64_t)t.tiles_n * ((M + bm - 1) / bm);
    const int num_kb = (int)((K + kTcBlockK - 1) / kTcBlockK);
    const bool sz_tma = !per_channel(g, K) && (K / g) % 8 == 0;
    int64_t tail = 0;
    if (tiles < sm_count) {
        tail = tiles;
    } else {
        const int64_t rem = tiles % sm_count;
        if (rem > 0 && rem <= sm_count / 2) tail = rem;
    }
    int s = 1;
    if (tail > 0) {
        s = (int)(sm_count / tail);
        if (s > 8) s = 8;
        if (s > num_kb / 4) s = num_kb / 4;
        if (s < 1) s = 1;
    }
    t.kb_split = tc_kb_split(num_kb, s, g, sz_tma);
    t.splits = (num_kb + t.kb_split - 1) / t.kb_split;
    if (t.splits < 2) {                       // nothing to split: one unsplit launch
        t.splits = 1;
        t.kb_split = num_kb;
        tail = 0;
    }
    t.head = tiles - tail;
    t.tail = tail;
    return t;
}

template <int BITS>
void tc_smem_and_stages(int bm, int* smem, int* stages) {
    switch (bm) {
        case 32: *smem = TcConfig<32, BITS>::kSmemBytes; *stages = TcConfig<32, BITS>::kStages; break;
        case 64: *smem = TcConfig<64, BITS>::kSmemBytes; *stages = TcConfig<64, BITS>::kStages; break;
        case 128: *smem = TcConfig<128, BITS>::kSmemBytes; *stages = TcConfig<128, BITS>::kStages; break;
        default: *smem = TcConfig<256, BITS>::kSmemBytes; *stages = TcConfig<256, BITS>::kStages; break;
    }
}

w4a16_status check_shape(int64_t M, int64_t N, int64_t K, int32_t g, int32_t sym) {
    if (sym != 0 && sym != 1) return W4A16_EINVAL;
    if (M < 0 || N < 0 || K <= 0) return W4A16_EINVAL;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return W4A16_EINVAL;
    if (!valid_group(g, K)) return W4A16_EINVAL;
    return W4A16_OK;
}

// M-dispatch: small M streams the weights (HBM-bound) with the decode kernel;
// larger M is tensor-core bound and goes to the tcgen05 kernel.
int choose_path(int64_t M) { return M <= 16 ? W4A16_PATH_DECODE : W4A16_PATH_TENSORCORE; }

// bits: code width, 4 or 8 (8-bit codes run only on the tensor-core kernel here;
// their small-M GEMV has its own launcher).
w4a16_status make_plan(int64_t M, int64_t N, int64_t K, int32_t g, int32_t sym, int32_t path,
                       int32_t ctas, int sm_count, w4a16_plan* p, int bits = 4) {
    w4a16_status st = check_shape(M, N, K, g, sym);
    if (st != W4A16_OK) return st;
    if (path < W4A16_PATH_AUTO || path > W4A16_PATH_TENSORCORE) return W4A16_EINVAL;
    if (ctas < 0 || ctas > kMaxCtas) return W4A16_EINVAL;
    const int chosen = path == W4A16_PATH_AUTO ? choose_path(M) : path;
    if (chosen == W4A16_PATH_DECODE && M > 16) return W4A16_EINVAL;
    if (chosen == W4A16_PATH_TENSORCORE && ctas != 0) return W4A16_EINVAL;
    *p = w4a16_plan{};
    p->path = chosen;
    if (chosen == W4A16_PATH_DECODE) {
        const DecodeGeometry d = decode_geometry(M, N, K, g, bits);
        if (!decode_geometry_ok(d, M)) return W4A16_EUNSUPPORTED;
        // At most one resident wave: the CTA that finishes a split row block waits
        // for parts from its neighbours, which must be running too.
        const int64_t resident = (int64_t)sm_count * d.ctas_per_sm;
        int64_t grid = ctas > 0 ? ctas : resident;
        if (grid > resident) grid = resident;
        if (grid > d.units) grid = d.units;
        if (grid < 1) grid = 1;
        p->tile_m = 8 * d.mb;
        p->tile_n = kDecRows;
        p->grid = grid;
        p->threads = kDecThreads;
        p->smem_bytes = d.smem_bytes;
        p->stages = d.stages;
        p->kernels = 1;
        p->split_tiles = decode_split_blocks(d, grid);
        p->workspace_bytes = decode_workspace_bytes(d, grid);
    } else {
        const int bm = tc_tile_m(M);
        const TcSchedule ts = tc_schedule(M, N, K, g, bm, sm_count);
        p->tile_m = bm;
        p->tile_n = kTcTileN;
        p->grid = ts.head + ts.tail * ts.splits;
        p->threads = kTcThreads;
        if (bits == 8) tc_smem_and_stages<8>(bm, &p->smem_bytes, &p->stages);
        else tc_smem_and_stages<4>(bm, &p->smem_bytes, &p->stages);
        p->kernels = (ts.head > 0 ? 1 : 0) + (ts.tail > 0 ? 2 : 0);
        p->split_tiles = ts.tail;
        p->workspace_bytes = ts.tail > 0 ? (int64_t)ts.splits * ts.tail * bm * kTcTileN * 4 : 0;
    }
    return W4A16_OK;
}

// SM count of the current device, queried once per device (148 when no device
// can be queried, e.g. for host-only planning on a machine without a GPU).
int current_sm_count() {
    static std::atomic<int> cached[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return 148;
    }
    int sms = cached[dev].load(std::memory_order_relaxed);
    if (sms > 0) return sms;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
        cudaGetLastError();
        return 148;
    }
    cached[dev].store(sms, std::memory_order_relaxed);
    return sms;
}

// Tensor maps are encoded on the host for every launch; a call repeated with
// the same buffers (the common case: fixed weights, reused activation and output
// buffers) finds its maps in this per-thread cache instead of re-encoding them.
struct TmKey {
    const void* base;
    uint64_t inner, outer, row_bytes;
    uint32_t box_inner, box_outer;
    int dtype, swizzle;
    bool operator==(const TmKey& o) const {
        return base == o.base && inner == o.inner && outer == o.outer && row_bytes == o.row_bytes &&
               box_inner == o.box_inner && box_outer == o.box_outer && dtype == o.dtype &&
               swizzle == o.swizzle;
    }
};

struct TmEntry {
    bool valid;
    TmKey key;
    CUtensorMap map;
};

constexpr int kTmCacheSize = 256;

size_t tm_hash(const TmKey& k) {
    uint64_t h = reinterpret_cast<uintptr_t>(k.base) * 0x9E3779B97F4A7C15ull;
    for (uint64_t v : {k.inner, k.outer, k.row_bytes, (uint64_t)k.box_inner, (uint64_t)k.box_outer,
                       (uint64_t)k.dtype, (uint64_t)k.swizzle})
        h = (h ^ v) * 0x100000001B3ull;
    return (size_t)(h >> 17) % kTmCacheSize;
}

w4a16_status encode_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                       uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                       uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    thread_local TmEntry cache[kTmCacheSize];
    const TmKey key{base, inner, outer, row_bytes, box_inner, box_outer, (int)dtype, (int)swizzle};
    TmEntry& e = cache[tm_hash(key)];
    if (e.valid && e.key == key) {
        *map = e.map;
        return W4A16_OK;
    }
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
    if (r != CUDA_SUCCESS) return W4A16_ECUDA;
    e.valid = true;
    e.key = key;
    e.map = *map;
    return W4A16_OK;
}

// ---------------------------------------------------------------- decode launch
template <int MB, bool SYM, int G, int BITS>
w4a16_status launch_decode_t(const w4a16_plan& p, const CUtensorMap& tmP, const CUtensorMap& tmX,
                             const CUtensorMap& tmS, const CUtensorMap& tmZ,
                             const DecodeArgs& args, cudaStream_t stream) {
    auto kern = gemv_decode_kernel<MB, SYM, G, BITS>;
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemPerBlockMax) != cudaSuccess)
            return W4A16_ECUDA;
        attr_set[dev] = true;
    }
    // Programmatic dependent launch: the kernel's CTAs are placed and set up while
    // the previous grid on the stream drains; they read nothing before their
    // dependency wait.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.grid, 1, 1);
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)p.smem_bytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tmP, tmX, tmS, tmZ, args) != cudaSuccess) return W4A16_ECUDA;
    return W4A16_OK;
}

// Bytes per scale copy for grouped scales: the largest of 16, 8, 4 that divides
// both a unit's scale bytes per row (gu·2) and the scale row stride (K/g·2), so
// that copies are aligned and never cross the end of a row; 2 = plain loads.
int decode_scale_copy(int gu, int64_t groups) {
    for (int cs = 16; cs >= 4; cs /= 2)
        if (cs <= gu * 2 && (gu * 2) % cs == 0 && (groups * 2) % cs == 0) return cs;
    // one group per unit (8-bit codes at g = 128): the aligned pair holding it
    if (gu == 1 && groups % 2 == 0) return 3;
    return 2;
}

w4a16_status launch_decode(const w4a16_plan& p, const void* X, int64_t M, int64_t K,
                           const void* packed, const void* scales, const void* zeros, int64_t N,
                           int32_t g, int32_t sym, void* Y, void* workspace, cudaStream_t stream,
                           const void* act_scale = nullptr, bool static_weights = false, int bits = 4) {
    const DecodeGeometry d = decode_geometry(M, N, K, g, bits);
    const int bk = decode_block_k(bits);
    const uint64_t row_bytes = (uint64_t)K * (uint64_t)bits / 8;   // code bytes per weight row
    CUtensorMap tmP, tmX;
    w4a16_status st = encode_2d(&tmP, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, row_bytes, (uint64_t)N,
                                row_bytes, kDecUnitRowBytes, kDecRows, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != W4A16_OK) return st;
    st = encode_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K, (uint64_t)M,
                   (uint64_t)K * 2, (uint32_t)bk, (uint32_t)M, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != W4A16_OK) return st;
    const bool pc = per_channel(g, K);
    DecodeArgs args{};
    args.scales = static_cast<const uint16_t*>(scales);
    args.zeros = static_cast<const uint16_t*>(zeros);
    args.Y = static_cast<uint16_t*>(Y);
    args.act_scale = static_cast<const uint16_t*>(act_scale);
    args.ws_flag = static_cast<uint32_t*>(workspace);
    args.ws_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                            decode_flag_bytes(d, p.grid));
    args.M = (int)M;
    args.N = (int)N;
    args.K = (int)K;
    args.RB = d.rb;
    args.KBn = d.kbn;
    args.Gtot = pc ? 1 : (int)(K / g);
    args.stages = d.stages;
    args.stage_bytes = d.stage_bytes;
    args.xf_off = d.xf_off;
    args.sz_off = d.sz_off;
    args.sz_tma = d.sz_tma;
    args.slab_off = d.slab_off;
    args.slabs = d.slabs;
    args.sz_copy = pc ? 16 : decode_scale_copy(d.gu, K / g);
    // Scales and zeros [N][K/g] in slabs of 8 groups x 256 rows, when their rows are
    // 16-byte aligned; otherwise the kernel copies them with cp.async and these are unused.
    CUtensorMap tmS = tmP, tmZ = tmP;
    if (d.sz_tma) {
        st = encode_2d(&tmS, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, scales, (uint64_t)(K / g), (uint64_t)N,
                       (uint64_t)(K / g) * 2, 8, kDecRows, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (st != W4A16_OK) return st;
        if (!sym) {
            st = encode_2d(&tmZ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, zeros, (uint64_t)(K / g), (uint64_t)N,
                           (uint64_t)(K / g) * 2, 8, kDecRows, CU_TENSOR_MAP_SWIZZLE_NONE);
            if (st != W4A16_OK) return st;
        }
    }
    args.early = static_weights ? 1 : 0;
    args.U = d.units;
    const int gsel = pc ? 0 : g;                   // kernel group size, 0 = per-channel
#define W4A16_DEC_G(MBV, SYMV, BV)                                                              \
    switch (gsel) {                                                                             \
        case 32: return launch_decode_t<MBV, SYMV, 32, BV>(p, tmP, tmX, tmS, tmZ, args, stream);   \
        case 64: return launch_decode_t<MBV, SYMV, 64, BV>(p, tmP, tmX, tmS, tmZ, args, stream);   \
        case 128: return launch_decode_t<MBV, SYMV, 128, BV>(p, tmP, tmX, tmS, tmZ, args, stream); \
        case 0: return launch_decode_t<MBV, SYMV, 0, BV>(p, tmP, tmX, tmS, tmZ, args, stream);     \
        default: return W4A16_EINVAL;                                                           \
    }
#define W4A16_DEC_MS(BV)                      \
    if (d.mb == 1) {                          \
        if (sym) W4A16_DEC_G(1, true, BV)     \
        W4A16_DEC_G(1, false, BV)             \
    }                                         \
    if (sym) W4A16_DEC_G(2, true, BV)         \
    W4A16_DEC_G(2, false, BV)
    if (bits == 8) {
        W4A16_DEC_MS(8)
    }
    W4A16_DEC_MS(4)
#undef W4A16_DEC_MS
#undef W4A16_DEC_G
}

template <int BM, bool SYM, int G, int BITS>
w4a16_status launch_tc_t(const w4a16_plan& p, const CUtensorMap& tmX, const CUtensorMap& tmP,
                         const CUtensorMap& tmS, const CUtensorMap& tmZ, int sz_tma,
                         const void* scales, const void* zeros, void* Y, int M, int N, int K,
                         int g, void* workspace, cudaStream_t stream) {
    auto kern = gemm_tc_kernel<BM, SYM, G, BITS>;
    using Cfg = TcConfig<BM, BITS>;
    const int sz_async = (G != 0 && (K / g) % 2 == 0) ? 1 : 0;   // 4-byte aligned scale rows
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg::kSmemBytes) != cudaSuccess)
            return W4A16_ECUDA;
        // all of the SM's unified L1 / shared storage as shared memory, so that
        // tc_ctas_per_sm(BM) CTAs are resident at once
        if (cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
            return W4A16_ECUDA;
        attr_set[dev] = true;
    }
    // the same schedule make_plan reported (it used this device's SM count)
    const TcSchedule ts = tc_schedule(M, N, K, g, BM, current_sm_count());
    const auto* sc = static_cast<const uint16_t*>(scales);
    const auto* ze = static_cast<const uint16_t*>(zeros);
    auto* y = static_cast<uint16_t*>(Y);
    const int num_kb = (K + kTcBlockK - 1) / kTcBlockK;
    if (ts.head > 0) {
        kern<<<dim3((unsigned)ts.head, 1, 1), kTcThreads, Cfg::kSmemBytes, stream>>>(
            tmX, tmP, sc, ze, y, M, N, K, sz_async, tmS, tmZ, sz_tma, num_kb, nullptr, 0, ts.tiles_n);
        w4a16_status st = launch_status();
        if (st != W4A16_OK) return st;
    }
    if (ts.tail == 0) return W4A16_OK;
    float* partials = static_cast<float*>(workspace);
    // The tail may start while the head drains (programmatic dependent launch);
    // the reduce waits for the tail, and the tail waits for the head before it ends.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ts.tail, 1, (unsigned)ts.splits);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = ts.head > 0 ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kern, tmX, tmP, sc, ze, y, M, N, K, sz_async, tmS, tmZ, sz_tma,
                           ts.kb_split, partials, (int)ts.head, ts.tiles_n) != cudaSuccess)
        return W4A16_ECUDA;
    // Sum of the partial tiles, chained by programmatic dependent launch.
    const int64_t items = ts.tail * BM * kTcTileN / 4;
    int64_t blocks = (items + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    cudaLaunchConfig_t rcfg = {};
    rcfg.gridDim = dim3((unsigned)blocks, 1, 1);
    rcfg.blockDim = dim3(256, 1, 1);
    rcfg.stream = stream;
    rcfg.attrs = attr;
    rcfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&rcfg, tc_splitk_reduce_kernel, static_cast<const float*>(partials),
                           ts.splits, (int)ts.tail, (int)ts.head, ts.tiles_n, BM, M, N, y) != cudaSuccess)
        return W4A16_ECUDA;
    return W4A16_OK;
}

template <bool SYM, int G, int BITS>
w4a16_status launch_tc_g(const w4a16_plan& p, const CUtensorMap& tmX, const CUtensorMap& tmP,
                         const CUtensorMap& tmS, const CUtensorMap& tmZ, int sz_tma,
                         const void* scales, const void* zeros, void* Y, int M, int N, int K,
                         int g, void* workspace, cudaStream_t stream) {
#define W4A16_TC_TILE(BMV) \
    launch_tc_t<BMV, SYM, G, BITS>(p, tmX, tmP, tmS, tmZ, sz_tma, scales, zeros, Y, M, N, K, g, \
                             workspace, stream)
    switch (p.tile_m) {
        case 32: return W4A16_TC_TILE(32);
        case 64: return W4A16_TC_TILE(64);
        case 128: return W4A16_TC_TILE(128);
        default: return W4A16_TC_TILE(256);
    }
#undef W4A16_TC_TILE
}

w4a16_status launch_tc(const w4a16_plan& p, const void* X, int64_t M, int64_t K,
                       const void* packed, const void* scales, const void* zeros, int64_t N,
                       int32_t g, int32_t sym, void* Y, void* workspace, cudaStream_t stream,
                       int bits = 4) {
    CUtensorMap tmX, tmP;
    w4a16_status st = encode_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K,
                                (uint64_t)M, (uint64_t)K * 2, kTcBlockK, (uint32_t)p.tile_m,
                                CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != W4A16_OK) return st;
    // codes [N][K·bits/8]: boxes of 128 rows x one K block (32 bytes with the 32-byte
    // swizzle for 4-bit codes, 64 bytes with the 64-byte swizzle for 8-bit codes)
    const uint64_t row_bytes = (uint64_t)K * (uint64_t)bits / 8;
    st = encode_2d(&tmP, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, row_bytes, (uint64_t)N, row_bytes,
                   (uint32_t)(kTcBlockK * bits / 8), kTcTileN,
                   bits == 8 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    if (st != W4A16_OK) return st;
    // Scales and zeros [N][K/g] in slabs of 8 groups x 128 rows, when their rows are
    // 16-byte aligned; otherwise the kernel copies them with cp.async.
    const bool pc = per_channel(g, K);             // per-channel: each row's pair read once
    const int sz_tma = (!pc && (K / g) % 8 == 0) ? 1 : 0;
    CUtensorMap tmS = tmP, tmZ = tmP;
    if (sz_tma) {
        st = encode_2d(&tmS, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, scales, (uint64_t)(K / g), (uint64_t)N,
                       (uint64_t)(K / g) * 2, 8, kTcTileN, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (st != W4A16_OK) return st;
        if (!sym) {
            st = encode_2d(&tmZ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, zeros, (uint64_t)(K / g),
                           (uint64_t)N, (uint64_t)(K / g) * 2, 8, kTcTileN, CU_TENSOR_MAP_SWIZZLE_NONE);
            if (st != W4A16_OK) return st;
        }
    }
    const int m = (int)M, n = (int)N, k = (int)K;
#define W4A16_TC_CASE(GG)                                                                      \
    case GG:                                                                                   \
        if (bits == 8)                                                                         \
            return sym ? launch_tc_g<true, GG, 8>(p, tmX, tmP, tmS, tmZ, sz_tma, scales, zeros, Y, \
                                                  m, n, k, g, workspace, stream)               \
                       : launch_tc_g<false, GG, 8>(p, tmX, tmP, tmS, tmZ, sz_tma, scales, zeros, \
                                                   Y, m, n, k, g, workspace, stream);         \
        return sym ? launch_tc_g<true, GG, 4>(p, tmX, tmP, tmS, tmZ, sz_tma, scales, zeros, Y, m, n, \
                                              k, g, workspace, stream)                         \
                   : launch_tc_g<false, GG, 4>(p, tmX, tmP, tmS, tmZ, sz_tma, scales, zeros, Y, m, \
                                               n, k, g, workspace, stream);
    switch (pc ? 0 : g) {
        W4A16_TC_CASE(32)
        W4A16_TC_CASE(64)
        W4A16_TC_CASE(128)
        W4A16_TC_CASE(0)
        default: return W4A16_EINVAL;
    }
#undef W4A16_TC_CASE
}

int grid_for(int64_t work_items, int threads, int sm_count) {
    const int64_t blocks = (work_items + threads - 1) / threads;
    const int64_t cap = (int64_t)sm_count * 8;   // grid-stride loops beyond 8 CTAs per SM
    return (int)(blocks < cap ? (blocks < 1 ? 1 : blocks) : cap);
}

// Built-in scratch for w4a16_gemm_decode_noalloc (callers that cannot
// allocate).  In host code this name is only a host-side stand-in; the device
// address comes from cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[W4A16_NOALLOC_SCRATCH_BYTES];
void* g_noalloc_ptr[kMaxDevices] = {};

w4a16_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return W4A16_ECUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return W4A16_ECUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return W4A16_OK;
}

// Workspace of an activation-scaled GEMM: the tensor-core path forms X' once into
// the workspace, after the GEMM's own scratch (rounded to 256 bytes); the decode
// path scales X inside the kernel and needs nothing extra.
int64_t act_scaled_workspace_bytes(const w4a16_plan& p, int64_t M, int64_t K) {
    if (p.path == W4A16_PATH_DECODE) return p.workspace_bytes;
    return (p.workspace_bytes + 255) / 256 * 256 + M * K * 2;
}

// The fused GEMM behind every W4A16 GEMM entry point; act_scale (bf16 [K]) or null.
w4a16_status gemm_impl(const void* X, int64_t M, int64_t K, const void* packed, const void* scales,
                       const void* zeros, int64_t N, int32_t g, int32_t sym, const void* act_scale,
                       void* Y, void* workspace, size_t workspace_bytes, int32_t path, int32_t ctas,
                       void* stream) {
    const bool static_weights = (path & W4A16_STATIC_WEIGHTS) != 0;
    path &= ~W4A16_STATIC_WEIGHTS;
    w4a16_plan p;
    w4a16_status st = make_plan(M, N, K, g, sym, path, ctas, current_sm_count(), &p);
    if (st != W4A16_OK) return st;
    if (M == 0 || N == 0) return W4A16_OK;
    if (!X || !packed || !scales || !Y || (!sym && !zeros)) return W4A16_EINVAL;
    if (!aligned16(X) || !aligned16(packed) || !aligned16(scales) || !aligned16(Y) ||
        (!sym && !aligned16(zeros)) || (act_scale && !aligned16(act_scale)))
        return W4A16_EINVAL;
    const int64_t need = act_scale ? act_scaled_workspace_bytes(p, M, K) : p.workspace_bytes;
    if (workspace_bytes < (size_t)need) return W4A16_EWORKSPACE;
    if (need > 0 && (workspace == nullptr || !aligned16(workspace))) return W4A16_EINVAL;
    DeviceInfo di;
    if ((st = device_info(&di)) != W4A16_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (p.path == W4A16_PATH_DECODE)
        return launch_decode(p, X, M, K, packed, scales, zeros, N, g, sym, Y, workspace, s, act_scale,
                             static_weights);
    if (act_scale) {
        // Large M: every X tile is read by all N/128 CTAs of its row of tiles, so X' is
        // formed once, by an elementwise pass into the workspace, rather than per tile.
        void* xs = static_cast<uint8_t*>(workspace) + (p.workspace_bytes + 255) / 256 * 256;
        const int64_t chunks = M * K / 8;
        scale_activations_kernel<<<grid_for(chunks, 256, di.sm_count), 256, 0, s>>>(
            static_cast<const uint4*>(X), static_cast<const uint4*>(act_scale), chunks, K / 8,
            static_cast<uint4*>(xs));
        if ((st = launch_status()) != W4A16_OK) return st;
        X = xs;
    }
    return launch_tc(p, X, M, K, packed, scales, zeros, N, g, sym, Y, workspace, s, 4);
}

}  // namespace

// ==================================================================== ABI
// ---------------------------------------------------------------- W8A8 launch
bool w8a8_shape_ok(int64_t M, int64_t N, int64_t K) {
    return M >= 0 && N >= 0 && K > 0 && K % 32 == 0 && M <= kMaxDim && N <= kMaxDim && K <= kMaxDim;
}

template <int BM>
w4a16_status launch_w8a8_t(const void* qx, const void* sx, int64_t M, int64_t K, const void* qw,
                           const void* sw, int64_t N, void* Y, cudaStream_t stream) {
    using Cfg = W8a8Config<BM>;
    CUtensorMap tmW, tmX;
    w4a16_status st = encode_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, (uint64_t)K, (uint64_t)N,
                                (uint64_t)K, kW8a8BlockK, kW8a8TileN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != W4A16_OK) return st;
    st = encode_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, (uint64_t)K, (uint64_t)M, (uint64_t)K,
                   kW8a8BlockK, (uint32_t)BM, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != W4A16_OK) return st;
    auto kern = gemm_w8a8_kernel<BM>;
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes) !=
            cudaSuccess)
            return W4A16_ECUDA;
        attr_set[dev] = true;
    }
    const int64_t tiles = ((N + kW8a8TileN - 1) / kW8a8TileN) * ((M + BM - 1) / BM);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)tiles, 1, 1);
    cfg.blockDim = dim3(kW8a8Threads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)Cfg::kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tmW, tmX, static_cast<const uint16_t*>(sw),
                           static_cast<const float*>(sx), static_cast<uint16_t*>(Y), (int)M, (int)N,
                           (int)K) != cudaSuccess)
        return W4A16_ECUDA;
    return W4A16_OK;
}

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
    if (per_channel(g, K)) {
        const int rgrid = (int)(N < (int64_t)di.sm_count * 8 ? N : (int64_t)di.sm_count * 8);
        if (sym) quantize_rows_kernel<true><<<rgrid, kQuantRowThreads, 0, s>>>(Wp, N, K, Pp, Sp, Zp);
        else quantize_rows_kernel<false><<<rgrid, kQuantRowThreads, 0, s>>>(Wp, N, K, Pp, Sp, Zp);
        return launch_status();
    }
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
    if (per_channel(g, K)) {
        const int rgrid = (int)(N < (int64_t)di.sm_count * 8 ? N : (int64_t)di.sm_count * 8);
        const auto* P32 = static_cast<const uint32_t*>(packed);
        if (sym) dequantize_rows_kernel<true><<<rgrid, 256, 0, s>>>(P32, Sp, Zp, N, K, Wp);
        else dequantize_rows_kernel<false><<<rgrid, 256, 0, s>>>(P32, Sp, Zp, N, K, Wp);
        return launch_status();
    }
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
    w4a16_plan p;
    if (make_plan(M, N, K, g, 0, W4A16_PATH_AUTO, 0, current_sm_count(), &p) != W4A16_OK) return 0;
    return (size_t)p.workspace_bytes;
}

w4a16_status w4a16_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t g, int32_t sym,
                             int32_t path, int32_t ctas, w4a16_plan* plan) {
    if (!plan) return W4A16_EINVAL;
    return make_plan(M, N, K, g, sym, path & ~W4A16_STATIC_WEIGHTS, ctas, current_sm_count(), plan);
}

w4a16_status w8a16_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t g, int32_t sym,
                             int32_t path, w4a16_plan* plan) {
    if (!plan) return W4A16_EINVAL;
    return make_plan(M, N, K, g, sym, path & ~W4A16_STATIC_WEIGHTS, 0, current_sm_count(), plan, 8);
}

w4a16_status w4a16_gemm_ex(const void* X, int64_t M, int64_t K, const void* packed,
                           const void* scales, const void* zeros, int64_t N, int32_t g,
                           int32_t sym, void* Y, void* workspace, size_t workspace_bytes,
                           int32_t path, int32_t ctas, void* stream) {
    return gemm_impl(X, M, K, packed, scales, zeros, N, g, sym, nullptr, Y, workspace,
                     workspace_bytes, path, ctas, stream);
}

w4a16_status w4a16_gemm_host(const void* X_host, int64_t M, int64_t K, const void* packed,
                             const void* scales, const void* zeros, int64_t N, int32_t g,
                             int32_t sym, void* Y_host, void* X_dev, void* Y_dev,
                             void* workspace, size_t workspace_bytes, int32_t flags,
                             void* stream) {
    // every argument check of the GEMM first, on its plan, so that an invalid call
    // queues no copy
    w4a16_plan p;
    w4a16_status st = make_plan(M, N, K, g, sym, flags & ~W4A16_STATIC_WEIGHTS, 0, current_sm_count(), &p);
    if (st != W4A16_OK) return st;
    if (M == 0 || N == 0) return W4A16_OK;
    if (!X_host || !Y_host || !X_dev || !Y_dev || !aligned16(X_dev) || !aligned16(Y_dev))
        return W4A16_EINVAL;
    if (!packed || !scales || (!sym && !zeros) || !aligned16(packed) || !aligned16(scales) ||
        (!sym && !aligned16(zeros)))
        return W4A16_EINVAL;
    if (workspace_bytes < (size_t)p.workspace_bytes) return W4A16_EWORKSPACE;
    if (p.workspace_bytes > 0 && (workspace == nullptr || !aligned16(workspace))) return W4A16_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(X_dev, X_host, (size_t)(M * K * 2), cudaMemcpyHostToDevice, s) != cudaSuccess)
        return W4A16_ECUDA;
    st = w4a16_gemm_ex(X_dev, M, K, packed, scales, zeros, N, g, sym, Y_dev, workspace,
                       workspace_bytes, flags, 0, stream);
    if (st != W4A16_OK) return st;
    if (cudaMemcpyAsync(Y_host, Y_dev, (size_t)(M * N * 2), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return W4A16_ECUDA;
    return W4A16_OK;
}

w4a16_status w4a16_gemm(const void* X, int64_t M, int64_t K, const void* packed,
                        const void* scales, const void* zeros, int64_t N, int32_t g,
                        int32_t sym, void* Y, void* workspace, size_t workspace_bytes,
                        void* stream) {
    return w4a16_gemm_ex(X, M, K, packed, scales, zeros, N, g, sym, Y, workspace,
                         workspace_bytes, W4A16_PATH_AUTO, 0, stream);
}

size_t w4a16_gemm_act_scaled_workspace_size(int64_t M, int64_t N, int64_t K, int32_t g) {
    w4a16_plan p;
    if (make_plan(M, N, K, g, 0, W4A16_PATH_AUTO, 0, current_sm_count(), &p) != W4A16_OK) return 0;
    return (size_t)act_scaled_workspace_bytes(p, M, K);
}

w4a16_status w4a16_gemm_act_scaled(const void* X, int64_t M, int64_t K, const void* act_scale,
                                   const void* packed, const void* scales, const void* zeros,
                                   int64_t N, int32_t g, int32_t sym, void* Y, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    if (!act_scale && M > 0 && N > 0) return W4A16_EINVAL;
    return gemm_impl(X, M, K, packed, scales, zeros, N, g, sym, act_scale, Y, workspace,
                     workspace_bytes, W4A16_PATH_AUTO, 0, stream);
}

w4a16_status w4a16_gemm_decode_noalloc(const void* X, int64_t M, int64_t K, const void* packed,
                                       const void* scales, const void* zeros, int64_t N,
                                       int32_t g, int32_t sym, void* Y, void* stream) {
    w4a16_plan p;
    w4a16_status st = make_plan(M, N, K, g, sym, W4A16_PATH_DECODE, 0, current_sm_count(), &p);
    if (st != W4A16_OK) return st;
    if (M == 0 || N == 0) return W4A16_OK;
    if (!X || !packed || !scales || !Y || (!sym && !zeros)) return W4A16_EINVAL;
    if (!aligned16(X) || !aligned16(packed) || !aligned16(scales) || !aligned16(Y) ||
        (!sym && !aligned16(zeros)))
        return W4A16_EINVAL;
    if ((size_t)p.workspace_bytes > W4A16_NOALLOC_SCRATCH_BYTES) return W4A16_EWORKSPACE;
    DeviceInfo di;
    if ((st = device_info(&di)) != W4A16_OK) return st;
    void* scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != W4A16_OK) return st;
    return launch_decode(p, X, M, K, packed, scales, zeros, N, g, sym, Y, scratch,
                         static_cast<cudaStream_t>(stream));
}

size_t w8a16_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int32_t g) {
    w4a16_plan p;
    if (make_plan(M, N, K, g, 0, W4A16_PATH_AUTO, 0, current_sm_count(), &p, 8) != W4A16_OK) return 0;
    return (size_t)p.workspace_bytes;
}

w4a16_status w8a16_gemm_ex(const void* X, int64_t M, int64_t K, const void* codes,
                           const void* scales, const void* zeros, int64_t N, int32_t g,
                           int32_t sym, void* Y, void* workspace, size_t workspace_bytes,
                           int32_t path, void* stream) {
    const bool static_weights = (path & W4A16_STATIC_WEIGHTS) != 0;
    path &= ~W4A16_STATIC_WEIGHTS;
    w4a16_status st = check_shape(M, N, K, g, sym);
    if (st != W4A16_OK) return st;
    if (M == 0 || N == 0) return W4A16_OK;
    if (!X || !codes || !scales || !Y || (!sym && !zeros)) return W4A16_EINVAL;
    if (!aligned16(X) || !aligned16(codes) || !aligned16(scales) || !aligned16(Y) ||
        (!sym && !aligned16(zeros)))
        return W4A16_EINVAL;
    DeviceInfo di;
    if ((st = device_info(&di)) != W4A16_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    w4a16_plan p;
    st = make_plan(M, N, K, g, sym, path, 0, current_sm_count(), &p, 8);
    if (st != W4A16_OK) return st;
    if (workspace_bytes < (size_t)p.workspace_bytes) return W4A16_EWORKSPACE;
    if (p.workspace_bytes > 0 && (workspace == nullptr || !aligned16(workspace))) return W4A16_EINVAL;
    if (p.path == W4A16_PATH_DECODE)
        return launch_decode(p, X, M, K, codes, scales, zeros, N, g, sym, Y, workspace, s, nullptr,
                             static_weights, 8);
    return launch_tc(p, X, M, K, codes, scales, zeros, N, g, sym, Y, workspace, s, 8);
}

w4a16_status w8a16_gemm(const void* X, int64_t M, int64_t K, const void* codes, const void* scales,
                        const void* zeros, int64_t N, int32_t g, int32_t sym, void* Y,
                        void* workspace, size_t workspace_bytes, void* stream) {
    return w8a16_gemm_ex(X, M, K, codes, scales, zeros, N, g, sym, Y, workspace, workspace_bytes,
                         W4A16_PATH_AUTO, stream);
}

w4a16_status w8a8_quantize_activations(const void* X, int64_t M, int64_t K, void* q, void* s,
                                        void* stream) {
    if (!w8a8_shape_ok(M, 0, K)) return W4A16_EINVAL;
    if (M == 0) return W4A16_OK;
    if (!X || !q || !s || !aligned16(X) || !aligned16(q) || !aligned16(s)) return W4A16_EINVAL;
    const int grid = (int)(M < (int64_t(1) << 30) ? M : (int64_t(1) << 30));   // one CTA per token
    const int64_t chunks = K / 8;
    const uint16_t* x = static_cast<const uint16_t*>(X);
    int8_t* qq = static_cast<int8_t*>(q);
    float* ss = static_cast<float*>(s);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (chunks <= 4 * kW8a8ActThreads)
        w8a8_quantize_act_kernel<4><<<grid, kW8a8ActThreads, 0, st>>>(x, M, K, qq, ss);
    else if (chunks <= 16 * kW8a8ActThreads)
        w8a8_quantize_act_kernel<16><<<grid, kW8a8ActThreads, 0, st>>>(x, M, K, qq, ss);
    else
        w8a8_quantize_act_kernel<0><<<grid, kW8a8ActThreads, 0, st>>>(x, M, K, qq, ss);
    return launch_status();
}

w4a16_status w8a8_gemm(const void* qx, const void* sx, int64_t M, int64_t K, const void* qw,
                       const void* sw, int64_t N, void* Y, void* stream) {
    if (!w8a8_shape_ok(M, N, K)) return W4A16_EINVAL;
    if (M == 0 || N == 0) return W4A16_OK;
    if (!qx || !sx || !qw || !sw || !Y) return W4A16_EINVAL;
    if (!aligned16(qx) || !aligned16(sx) || !aligned16(qw) || !aligned16(sw) || !aligned16(Y))
        return W4A16_EINVAL;
    DeviceInfo di;
    w4a16_status st = device_info(&di);
    if (st != W4A16_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M <= 64) return launch_w8a8_t<64>(qx, sx, M, K, qw, sw, N, Y, s);
    if (M <= 128) return launch_w8a8_t<128>(qx, sx, M, K, qw, sw, N, Y, s);
    return launch_w8a8_t<256>(qx, sx, M, K, qw, sw, N, Y, s);
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
