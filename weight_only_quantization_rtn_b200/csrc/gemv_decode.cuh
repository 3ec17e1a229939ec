// Decode-path fused W4A16 GEMM for small M (M ≤ 16).
//
// Decode is bound by reading the weights once from HBM (qwbw.cn,
// "推理优化中“用精度换性能“的核心技术：量化", §1 and §3.2; aigcbaba selection page
// §二: "反复读大权重只算一个 token").  The kernel therefore streams the packed
// INT4 codes with 128-bit loads that each lane issues several of before using
// any, dequantizes them in registers, and spends as few instructions per
// weight as possible:
//
//  * A warp owns a tile of 16 weight rows.  Lane (g, t) — g = lane/4, t = lane%4 —
//    loads 16 bytes (32 codes) of rows g and g+8 at K offset 32·t of a 128-wide
//    K chunk.  The codes become bf16 pairs in registers (LOP3 nibble isolation +
//    exponent magic, one bf16x2 subtract of the zero point, one bf16x2 multiply
//    by the scale) and are used directly as the A operand of m16n8k16 bf16 MMAs
//    with fp32 accumulation; the activations X form the B operand (M ≤ 8 → one
//    n8 MMA, M ≤ 16 → two).  The tensor core replaces the per-weight FMAs and
//    the warp-shuffle reductions a CUDA-core GEMV would need, which matters
//    because at HBM speed the ALU budget is about 2.7 instructions per weight.
//    The MMA reduces over K in whatever order the fragments assign, so the
//    nibble pairs are used in the order the LOP3 isolation yields them —
//    (q0,q4) (q1,q5) (q2,q6) (q3,q7) — and X is permuted to match (PRMT).
//  * The 8 warps of a CTA take interleaved 128-wide K chunks of the CTA's K
//    range; their partial tiles are summed in shared memory in a fixed order.
//  * When the row tiles alone cannot fill the GPU, S CTAs of one thread-block
//    cluster split K and their partial sums are added through distributed
//    shared memory in cluster-rank order: deterministic, no workspace, no
//    atomics, no second launch.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace w4a16 {

namespace cg = cooperative_groups;

constexpr int kDecodeWarps = 8;
constexpr int kDecodeThreads = kDecodeWarps * 32;
constexpr int kDecodeUnroll = 2;   // K chunks whose loads are issued together per warp

template <int MB, int TPW>
struct DecodeSmem {
    // Per warp partial fragments: [warp][tile][mb][lane][4]
    float part[kDecodeWarps][TPW][MB][32][4];
    // CTA partial (sum over warps), read by peer CTAs of the cluster
    float cta[TPW][MB][32][4];
};

// MB: n8 MMA columns blocks (1: M ≤ 8, 2: M ≤ 16); TPW: 16-row tiles per CTA.
template <int MB, int TPW, bool SYM, int G>
__global__ void __launch_bounds__(kDecodeThreads) gemv_decode_kernel(
    const uint16_t* __restrict__ X, int M, int64_t K, const uint8_t* __restrict__ packed,
    const uint16_t* __restrict__ scales, const uint16_t* __restrict__ zeros, int64_t N,
    uint16_t* __restrict__ Y, int split_k, int chunks_per_split) {
    __shared__ __align__(16) DecodeSmem<MB, TPW> sm;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int gq = lane >> 2;   // fragment row group
    const int tq = lane & 3;    // fragment thread-in-group
    cg::cluster_group cluster = cg::this_cluster();
    const int ks = (int)cluster.block_rank();     // cluster rank = K split index
    const int64_t rb = blockIdx.x / split_k;      // row block
    const int64_t row0 = rb * (16 * TPW);
    const int64_t KB = K / 2;                     // bytes per packed row
    const int64_t Gn = K / G;                     // groups per row
    const int total_chunks = (int)((K + 127) / 128);
    const int cbeg = ks * chunks_per_split;
    const int cend = min(total_chunks, cbeg + chunks_per_split);

    float acc[TPW][MB][4];
#pragma unroll
    for (int t = 0; t < TPW; ++t)
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[t][mb][j] = 0.0f;

    // Row pointers of this lane: rows gq and gq+8 of each tile.
    int64_t rows[TPW][2];
    bool row_ok[TPW][2];
#pragma unroll
    for (int t = 0; t < TPW; ++t)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            rows[t][h] = row0 + 16 * t + gq + 8 * h;
            row_ok[t][h] = rows[t][h] < N;
        }
    // Activation rows this lane supplies to the B fragments.
    bool m_ok[MB];
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) m_ok[mb] = (8 * mb + gq) < M;

    for (int c0 = cbeg + warp; c0 < cend; c0 += kDecodeWarps * kDecodeUnroll) {
        // ---- issue every load of this step before consuming any
        uint4 wq[kDecodeUnroll][TPW][2];
        uint32_t sraw[kDecodeUnroll][TPW][2], zraw[kDecodeUnroll][TPW][2];
        uint4 xv[kDecodeUnroll][MB][4];
        bool k_ok[kDecodeUnroll];
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            const int c = c0 + u * kDecodeWarps;
            const int64_t kbase = (int64_t)c * 128 + 32 * tq;
            k_ok[u] = (c < cend) && (kbase < K);
            const int64_t grp = kbase / G;
#pragma unroll
            for (int t = 0; t < TPW; ++t)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const bool ok = k_ok[u] && row_ok[t][h];
                    wq[u][t][h] = ok ? ldg_stream(packed + rows[t][h] * KB + kbase / 2)
                                     : make_uint4(0, 0, 0, 0);
                    sraw[u][t][h] = ok ? ldg_u16(scales + rows[t][h] * Gn + grp) : 0u;
                    zraw[u][t][h] = (ok && !SYM) ? ldg_u16(zeros + rows[t][h] * Gn + grp) : 0u;
                }
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) {
                const bool ok = k_ok[u] && m_ok[mb];
                const uint16_t* xp = X + (int64_t)(8 * mb + gq) * K + kbase;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    xv[u][mb][i] = ok ? ldg_cached(xp + 8 * i) : make_uint4(0, 0, 0, 0);
            }
        }
        // ---- dequantize + MMA
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            // B fragments: X pairs permuted to (x0,x4)(x1,x5) / (x2,x6)(x3,x7) per 8 codes
            uint32_t bf[MB][4][2][2];
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 v = xv[u][mb][i];   // X[k..k+7]: (x0x1)(x2x3)(x4x5)(x6x7)
                    bf[mb][i][0][0] = __byte_perm(v.x, v.z, 0x5410);   // (x0, x4)
                    bf[mb][i][0][1] = __byte_perm(v.x, v.z, 0x7632);   // (x1, x5)
                    bf[mb][i][1][0] = __byte_perm(v.y, v.w, 0x5410);   // (x2, x6)
                    bf[mb][i][1][1] = __byte_perm(v.y, v.w, 0x7632);   // (x3, x7)
                }
#pragma unroll
            for (int t = 0; t < TPW; ++t) {
                const uint32_t ss0 = dup16(sraw[u][t][0]), ss1 = dup16(sraw[u][t][1]);
                const uint32_t zz0 = zero_pair<SYM>(zraw[u][t][0]);
                const uint32_t zz1 = zero_pair<SYM>(zraw[u][t][1]);
                const uint32_t w0[4] = {wq[u][t][0].x, wq[u][t][0].y, wq[u][t][0].z,
                                        wq[u][t][0].w};
                const uint32_t w1[4] = {wq[u][t][1].x, wq[u][t][1].y, wq[u][t][1].z,
                                        wq[u][t][1].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t a0[4], a1[4];   // rows gq and gq+8: (q0,q4)(q1,q5)(q2,q6)(q3,q7)
                    dequant8_interleaved<SYM>(w0[i], zz0, ss0, a0);
                    dequant8_interleaved<SYM>(w1[i], zz1, ss1, a1);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int mb = 0; mb < MB; ++mb)
                            mma_bf16_16816(acc[t][mb], a0[2 * hh], a1[2 * hh], a0[2 * hh + 1],
                                           a1[2 * hh + 1], bf[mb][i][hh][0], bf[mb][i][hh][1]);
                }
            }
        }
    }

    // ---- reduce the 8 warps (fixed order), then the cluster's CTAs (rank order)
#pragma unroll
    for (int t = 0; t < TPW; ++t)
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
            *reinterpret_cast<float4*>(sm.part[warp][t][mb][lane]) =
                make_float4(acc[t][mb][0], acc[t][mb][1], acc[t][mb][2], acc[t][mb][3]);
    __syncthreads();
    constexpr int kElems = TPW * MB * 32 * 4;
    float* cta_flat = &sm.cta[0][0][0][0];
    for (int e = threadIdx.x; e < kElems; e += kDecodeThreads) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) s += (&sm.part[w][0][0][0][0])[e];
        cta_flat[e] = s;
    }
    cluster.sync();
    for (int e = threadIdx.x; e < kElems; e += kDecodeThreads) {
        if (e % split_k != ks) continue;            // outputs are shared out among the ranks
        float s = 0.0f;
        for (int r = 0; r < split_k; ++r) s += cluster.map_shared_rank(cta_flat, r)[e];
        // decode fragment position e = ((t*MB + mb)*32 + lane)*4 + j
        const int j = e & 3;
        const int ln = (e >> 2) & 31;
        const int tm = e >> 7;
        const int mb = tm % MB;
        const int t = tm / MB;
        const int64_t n = row0 + 16 * t + (ln >> 2) + 8 * (j >> 1);
        const int m = 8 * mb + 2 * (ln & 3) + (j & 1);
        if (n < N && m < M) Y[(int64_t)m * N + n] = (uint16_t)f32_to_bf16_bits_rn(s);
    }
    cluster.sync();   // keep this CTA's shared memory alive until every peer has read it
}

}  // namespace w4a16
