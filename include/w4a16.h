/*
 * w4a16.h — C ABI of the B200 (sm_100a) W4A16 weight-only RTN library.
 *
 * W4A16: weights stored as 4-bit integer codes, activations kept in 16-bit
 * floating point (bf16 here).  The method, as the pages describe it:
 *
 *  - "推理优化中“用精度换性能“的核心技术：量化":
 *      §2.2  INT4 holds [−8, 7] or [0, 15];
 *      §2.3  x_int = round(x_float / s) + z,  x̂_float = (x_int − z) × s;
 *      §3.3  symmetric:  s = max|x| / max_int, z = 0;
 *            asymmetric: s = (max(x) − min(x)) / (2^b − 1), z = round(−min(x)/s);
 *      §3.4  group-wise granularity: each group of 128 weights shares one
 *            16-bit scale and an optional 16-bit zero point (4.25 bits/weight);
 *      §3.2  weight-only inference: load INT4 from memory, dequantize to
 *            16-bit, multiply with 16-bit activations.
 *  - "量化实战深入（GPTQ / AWQ / SmoothQuant / KV 量化）",
 *      §二  q = round(x/s) + z, x ≈ s·(q − z); absmax s = max|x| / (2^(b−1) − 1);
 *           per-group = one scale per 128 elements.
 *  - "大模型推理中 Weight-only、W8A8 和 FP8 量化有什么区别？如何选型？",
 *      §二  a fused kernel reads INT4, unpacks and scales in registers or shared
 *           memory, and multiplies with the high-precision activations.
 *  - "LLM 量化中 W4A16 表示什么…｜蚂蚁集团 C/C++面经解析", 显存收益主要来自权重 / 性能取决于 kernel:
 *           0.5 byte per INT4 weight; dequantize inside the GEMM while reading
 *           INT4, rather than expanding the whole matrix first.
 *
 * Readings fixed by this library where the pages leave a step open:
 *  round() is round-half-to-even in binary32; s is computed in binary32 and
 *  rounded to bf16, and z and q use that bf16 s; codes are clamped to the INT4
 *  range; the asymmetric range is widened to contain 0 (so z is an integer in
 *  [0, 15] and 0 is on the grid); a group whose s rounds to 0 gets z = q = 0;
 *  symmetric codes are 4-bit two's complement and s = max|x| / 7; groups run
 *  along K (input channels); the dequantized weight is bf16_rn((q − z)·s).
 *
 * Layouts (all row-major, contiguous, every pointer 16-byte aligned):
 *  W       bf16  [N, K]      weights, N = output features, K = input features
 *  X       bf16  [M, K]      activations
 *  Y       bf16  [M, N]      Y = X · Ŵᵀ, fp32 accumulation, rounded once to bf16
 *  packed  uint8 [N, K/2]    byte i of a row holds element 2i in its low nibble
 *                            and element 2i+1 in its high nibble
 *  scales  bf16  [N, K/g]    one scale per group of g consecutive elements of a row
 *  zeros   bf16  [N, K/g]    zero point per group (an integer 0..15 stored in bf16);
 *                            all 0 in symmetric mode
 *
 * Supported: g ∈ {32, 64, 128} with K a positive multiple of g, or g = K with K
 * a positive multiple of 32 — per-channel granularity, one scale (and zero) per
 * output feature, scales/zeros [N, 1] ("量化实战深入（GPTQ / AWQ / SmoothQuant / KV 量化）",
 * 量化粒度 table; "推理优化中“用精度换性能“的核心技术：量化", §3.4); N ≥ 0, M ≥ 0 (M = 0 or N = 0 is a no-op), N, K, M < 2^31.  Every pointer is a DEVICE
 * pointer owned by the caller; the library allocates no device memory and keeps
 * no state beyond per-device constants (device properties, tensor-map encoder)
 * and the fixed scratch array of w4a16_gemm_decode_noalloc.  Device scratch,
 * where a kernel needs it, is otherwise the caller's `workspace`.
 * Each call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 * stream).  Arguments are checked on the host before any launch; a rejected
 * call launches nothing and returns W4A16_EINVAL.  No call aborts, throws or
 * falls back to the CPU.
 */
#ifndef W4A16_H_
#define W4A16_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define W4A16_ABI_VERSION 5   /* 3: w4a16_plan.split_tiles; the decode path is one kernel;
                                 4: W4A16_STATIC_WEIGHTS, w8a16_gemm_ex/_plan, W8A8;
                                 5: w4a16_gemm_host */

typedef enum w4a16_status {
    W4A16_OK = 0,
    W4A16_EINVAL = 1,        /* bad size, group, mode, alignment or null pointer; nothing launched */
    W4A16_EUNSUPPORTED = 2,  /* valid request the current device cannot run (needs sm_100) */
    W4A16_ECUDA = 3,         /* the CUDA runtime reported an error while launching */
    W4A16_EWORKSPACE = 4,    /* workspace smaller than w4a16_gemm_workspace_size() */
    W4A16_EDEVICE = 5        /* a kernel gave up a bounded wait (see w4a16_device_error) */
} w4a16_status;

/* GEMM kernel choice (roofline-driven: decode is weight-bandwidth bound, prefill
 * is tensor-core bound — "Quantization & Acceleration: 解释 W8A8 与 W4A16 的差异与取舍",
 * 关键判据; "大模型推理中 Weight-only、W8A8 和 FP8 量化有什么区别？如何选型？", §二 and §五). */
typedef enum w4a16_path {
    W4A16_PATH_AUTO = 0,       /* choose from M (roofline: M ≤ 16 is weight-bandwidth bound) */
    W4A16_PATH_DECODE = 1,     /* small-M kernel, M ≤ 16: persistent stream-K grid; TMA streams
                                  packed codes and X into a shared-memory ring; in-register
                                  dequantization feeds bf16 MMAs with fp32 accumulation; a
                                  row block split across CTAs is finished by its first
                                  owner, which adds the other owners' parts in a fixed order */
    W4A16_PATH_TENSORCORE = 2  /* large-M kernel: TMA-fed INT4 tile dequantized into shared
                                  memory and fed to tcgen05 bf16 MMA with TMEM accumulators;
                                  when the output tiles are fewer than the resident CTA
                                  slots (two per SM for tiles of at most 64 activation rows,
                                  else one), or the last wave of tiles would leave most
                                  slots idle, those tiles split
                                  K and a reduce kernel adds the parts in a fixed order */
} w4a16_path;

/* Flag OR'ed into the `path` argument of w4a16_gemm_ex (w4a16_gemm_plan accepts
 * and ignores it): the caller states that the kernel before this call on its
 * stream does not write packed, scales or zeros.  The decode kernel (M ≤ 16) then
 * streams the weights as soon as its CTAs are resident, while that kernel drains
 * (programmatic dependent launch), and waits for it only before reading X and
 * writing Y.  Inference with fixed weights meets the condition; a call right
 * after quantizing the same weights on the same stream does not, and its result
 * is then undefined.  The tensor-core path reads nothing before the previous
 * kernel completes either way.  Why it helps: on the layers of a 7B-shaped decode
 * step the first stage lands a few microseconds after the weights are requested,
 * a sizeable part of a 3–4 µs layer. */
#define W4A16_STATIC_WEIGHTS 0x100

/* The launch a GEMM call would make (filled by w4a16_gemm_plan). */
typedef struct w4a16_plan {
    int32_t path;            /* w4a16_path actually used (never AUTO) */
    int32_t tile_m;          /* activation rows per tile (decode: 8 or 16 MMA columns;
                                tensor core: 32/64/128/256) */
    int32_t tile_n;          /* output features per tile */
    int32_t threads;         /* threads per CTA */
    int64_t grid;            /* CTAs launched */
    int32_t smem_bytes;      /* dynamic shared memory per CTA */
    int32_t stages;          /* shared-memory pipeline depth */
    int32_t kernels;         /* kernels the call launches: decode 1; tensor core 1 unsplit,
                                2 when every tile splits K (+ the reduce), 3 with an unsplit
                                head, a split tail and the reduce */
    int64_t workspace_bytes; /* device workspace this launch needs */
    int64_t split_tiles;     /* output tiles whose K range is split between CTAs, so that
                                partial sums pass through the workspace: decode, the 256-row
                                blocks its stream-K partition cuts; tensor core, the tail tiles */
} w4a16_plan;

/* Quantize W[N, K] group-wise by RTN (asymmetric when sym == 0, symmetric when
 * sym == 1) and pack two codes per byte.  g = K quantizes per channel: each
 * row's range is reduced over the whole row.
 *   W       in   bf16 [N, K]
 *   packed  out  uint8 [N, K/2]
 *   scales  out  bf16 [N, K/g]
 *   zeros   out  bf16 [N, K/g]; may be NULL when sym == 1 (else written as 0)
 * Inputs must be finite.  Bit-exact with the host oracle. */
w4a16_status w4a16_quantize(const void* W, int64_t N, int64_t K, int32_t g, int32_t sym,
                            void* packed, void* scales, void* zeros, void* stream);

/* Expand packed codes to Ŵ[n, k] = bf16_rn((q − z)·s) ("推理优化中“用精度换性能“的核心技术：量化", §2.3).
 * This is the unfused form the fused GEMM avoids; it is provided for checking
 * and for callers that need Ŵ.
 *   packed, scales in; zeros in (ignored, may be NULL, when sym == 1)
 *   W_hat   out  bf16 [N, K] */
w4a16_status w4a16_dequantize(const void* packed, const void* scales, const void* zeros,
                              int64_t N, int64_t K, int32_t g, int32_t sym, void* W_hat,
                              void* stream);

/* Bytes of device workspace w4a16_gemm needs for this shape.  The decode path
 * stores there the fp32 partial sums of the 256-row blocks that its stream-K
 * partition splits between CTAs, with a ready flag per part.  The tensor-core path, for the output tiles
 * whose K it splits into S parts (all tiles when they are fewer than the
 * resident CTA slots, else only a mostly-empty last wave), stores S fp32 partial tiles of
 * 128 weight rows x tile_m activation rows per split tile, and needs 0 bytes
 * when it splits nothing.  In both cases a second, small kernel adds the parts
 * in a fixed order.  The contents are scratch: no
 * initialization is needed and nothing is kept between calls, but two calls
 * that may run at the same time (for instance on two streams) need two
 * workspaces.  Uses the current device's SM count. */
size_t w4a16_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int32_t g);

/* Fused W4A16 GEMM: Y[M, N] = X[M, K] · Ŵ[N, K]ᵀ with Ŵ = bf16_rn((q − z)·s)
 * formed in registers/shared memory from the packed codes, fp32 accumulation,
 * one rounding of each output to bf16.  Never materialises Ŵ in global memory.
 *   X in bf16 [M, K]; packed/scales/zeros as produced by w4a16_quantize
 *   (zeros ignored, may be NULL, when sym == 1); Y out bf16 [M, N].
 *   workspace/workspace_bytes: device scratch of at least
 *   w4a16_gemm_workspace_size() bytes, 16-byte aligned (see there).
 * Results are deterministic: the same inputs give bitwise-equal Y. */
w4a16_status w4a16_gemm(const void* X, int64_t M, int64_t K, const void* packed,
                        const void* scales, const void* zeros, int64_t N, int32_t g,
                        int32_t sym, void* Y, void* workspace, size_t workspace_bytes,
                        void* stream);

/* w4a16_gemm with the dispatch decision overridden: `path` forces a kernel
 * (AUTO = same as w4a16_gemm) and `ctas` (decode only; 0 = automatic) sets the
 * size of the persistent grid, hence where the stream-K partition splits row
 * blocks; it is capped at one resident wave (one or two CTAs per SM, as the
 * plan reports), because the CTA finishing a split row block waits for parts
 * from CTAs that run beside it.  Used by tests, benchmarks and
 * profiling to exercise both kernels and many partitions at the same shape.
 * Returns W4A16_EINVAL if the forced kernel cannot run the shape (DECODE with
 * M > 16, or `ctas` given for the tensor-core path), W4A16_EWORKSPACE if the
 * workspace is smaller than the plan's workspace_bytes. */
w4a16_status w4a16_gemm_ex(const void* X, int64_t M, int64_t K, const void* packed,
                           const void* scales, const void* zeros, int64_t N, int32_t g,
                           int32_t sym, void* Y, void* workspace, size_t workspace_bytes,
                           int32_t path, int32_t ctas, void* stream);

/* w4a16_gemm_ex with the activations and the result in HOST memory: copies
 * X_host (bf16 [M, K]) into X_dev, runs the GEMM into Y_dev, and copies Y_dev into
 * Y_host (bf16 [M, N]), all three in order on `stream`; one call per layer of a
 * host-driven step.  X_dev (M·K·2 bytes) and Y_dev (M·N·2 bytes) are device
 * scratch owned by the caller, 16-byte aligned; nothing is allocated.  With
 * page-locked host buffers the call returns before the copies complete: the
 * caller synchronizes the stream before reading Y_host or reusing X_host.
 * `flags` is w4a16_gemm_ex's `path` (kernel choice, W4A16_STATIC_WEIGHTS).
 * Errors as w4a16_gemm_ex (checked before the first copy), plus W4A16_EINVAL for
 * a null host or scratch pointer and W4A16_ECUDA when a copy cannot be queued. */
w4a16_status w4a16_gemm_host(const void* X_host, int64_t M, int64_t K, const void* packed,
                             const void* scales, const void* zeros, int64_t N, int32_t g,
                             int32_t sym, void* Y_host, void* X_dev, void* Y_dev,
                             void* workspace, size_t workspace_bytes, int32_t flags,
                             void* stream);

/* Bytes of device workspace w4a16_gemm_act_scaled needs for this shape: the
 * plan's workspace for M ≤ 16; for the tensor-core path that, rounded up to 256
 * bytes, plus M·K bf16 for the scaled activations.  0 for rejected shapes. */
size_t w4a16_gemm_act_scaled_workspace_size(int64_t M, int64_t N, int64_t K, int32_t g);

/* W4A16 GEMM with a per-input-channel activation scale:
 *   Y[M, N] = X'[M, K] · Ŵ[N, K]ᵀ,  X'[m, k] = bf16_rn(X[m, k] · a[k]).
 * This is the activation half of the equivalent scaling W·X = (W·diag(a)⁻¹)·
 * (diag(a)·X) that activation-aware weight quantization and SmoothQuant use to
 * move outlier magnitude between activations and weights ("推理优化中“用精度换
 * 性能“的核心技术：量化", §5.2 and §6.2; "大模型推理中 Weight-only、W8A8 和 FP8
 * 量化有什么区别？如何选型？", §三): the weights are quantized after being
 * divided by a, and the GEMM multiplies each activation by a[k].  The product
 * of two bf16 values is exact in binary32 and is rounded once, so the result
 * equals a w4a16_gemm on activations the caller scaled in bf16 beforehand.
 * M ≤ 16 (decode kernel): the scale is fused into the kernel's X path (one warp
 * scales each staged X slice as it reorders it; no extra bytes, measured cost
 * a few percent).  Larger M (tensor-core kernel): every X tile is read by the
 * N/128 CTAs of its row of output tiles, so X' is formed once by an elementwise
 * pass into the workspace before the GEMM, rather than once per tile.
 *   act_scale  in  bf16 [K], 16-byte aligned (computing it needs calibration
 *              data, so it is the caller's); other arguments as w4a16_gemm, same
 *              dispatch; workspace at least w4a16_gemm_act_scaled_workspace_size().
 * Returns W4A16_EINVAL for a null act_scale (when M, N > 0). */
w4a16_status w4a16_gemm_act_scaled(const void* X, int64_t M, int64_t K, const void* act_scale,
                                   const void* packed, const void* scales, const void* zeros,
                                   int64_t N, int32_t g, int32_t sym, void* Y, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Host-only: report the launch w4a16_gemm_ex would make, including the
 * workspace it needs.  Returns W4A16_EINVAL for shapes or overrides it would
 * reject. */
w4a16_status w4a16_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t g, int32_t sym,
                             int32_t path, int32_t ctas, w4a16_plan* plan);

/* Size of the built-in device scratch used by w4a16_gemm_decode_noalloc. */
#define W4A16_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

/* Decode-path GEMM (M ≤ 16) that allocates nothing and takes no workspace.
 * The pages have no counterpart: this exists for callers that cannot allocate
 * device memory — plug-ins whose host framework owns every device allocation
 * through its own pool, and hosts that forbid allocation after start-up so
 * that memory use stays fixed.
 * Same arguments, result and determinism as w4a16_gemm_ex with
 * path = W4A16_PATH_DECODE and ctas = 0, minus the workspace: the split-K
 * partial sums live in a file-scope device array of
 * W4A16_NOALLOC_SCRATCH_BYTES that every GPU which loads the library keeps
 * until the process exits.  Returns W4A16_EWORKSPACE, launching nothing, when
 * the problem needs more scratch than that (its plan's workspace_bytes: about
 * 1000 row blocks plus CTAs at M ≤ 8, 500 at M 9–16, i.e. N up to roughly
 * 218 000 and 90 000 rows on 148 SMs), and W4A16_EINVAL for M > 16 or any
 * argument w4a16_gemm_ex would reject.
 * The first call on a device looks up the array's device address for that
 * device (cudaGetSymbolAddress, with the device current).  All calls share the
 * one array and it keeps the last call's contents; nothing in it needs to
 * start at zero.  Calls that overlap on the GPU (other streams, other threads)
 * race on it: serialize them. */
w4a16_status w4a16_gemm_decode_noalloc(const void* X, int64_t M, int64_t K, const void* packed,
                                       const void* scales, const void* zeros, int64_t N,
                                       int32_t g, int32_t sym, void* Y, void* stream);

/* ---------------------------------------------------------------------------
 * W8A16: the same method with 8-bit codes (the INT8 form
 * "推理优化中“用精度换性能“的核心技术：量化" states in §3.3: asymmetric s = (max − min)/255, z = round(−min/s); symmetric
 * s = max|x|/127, "量化实战深入（GPTQ / AWQ / SmoothQuant / KV 量化）" §二 absmax with b = 8;
 * W8A16 is listed beside W4A16 in "大模型推理中 Weight-only、W8A8 和 FP8 量化有什么区别？如何选型？", 详细版).  Readings as above with the 8-bit
 * ranges: codes clamped to [0, 255] (asym) or [−128, 127] (sym, stored as
 * int8 two's complement); zeros are integers 0..255 stored in bf16.
 * Layouts: codes uint8 [N, K] (element k of a row in byte k); scales and
 * zeros bf16 [N, K/g] as for INT4.  Same g and K rules, alignment, stream and
 * error conventions as the INT4 entry points.
 * ------------------------------------------------------------------------- */

/* Quantize W[N, K] (bf16) to 8-bit codes: codes uint8 [N, K], scales and zeros
 * bf16 [N, K/g] (zeros may be NULL when sym == 1, else written as 0).
 * Bit-exact with the host oracle. */
w4a16_status w8a16_quantize(const void* W, int64_t N, int64_t K, int32_t g, int32_t sym,
                            void* codes, void* scales, void* zeros, void* stream);

/* Ŵ[n, k] = bf16_rn((q − z)·s) from 8-bit codes (W_hat bf16 [N, K]). */
w4a16_status w8a16_dequantize(const void* codes, const void* scales, const void* zeros,
                              int64_t N, int64_t K, int32_t g, int32_t sym, void* W_hat,
                              void* stream);

/* Bytes of device workspace w8a16_gemm needs: for M ≤ 16 the decode kernel's
 * split row blocks (the same layout and size rule as w4a16_gemm_workspace_size:
 * it depends on the row blocks and the grid), for larger M the tensor-core
 * kernel's split-K partial tiles.  Uses the current device's SM count; 0 for
 * rejected shapes.  (Before ABI version 4 the M ≤ 16 path needed none.) */
size_t w8a16_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int32_t g);

/* Host-only: the launch w8a16_gemm_ex would make with this `path` (AUTO: the
 * decode kernel for M ≤ 16, else the tensor-core kernel, both with 8-bit codes),
 * including its workspace.  Returns W4A16_EINVAL for shapes or paths
 * w8a16_gemm_ex would reject. */
w4a16_status w8a16_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t g, int32_t sym,
                             int32_t path, w4a16_plan* plan);

/* Fused W8A16 GEMM: Y[M, N] = X[M, K] · Ŵ[N, K]ᵀ with Ŵ = bf16_rn((q − z)·s)
 * formed on chip, binary32 accumulation, one rounding of each output to bf16;
 * deterministic.  M ≤ 16: the decode kernel with 8-bit codes (units of 256
 * rows x 128 K, i.e. the same 32 KB TMA tiles; each word of 4 codes becomes two
 * bf16 pairs — the byte in a binary32 mantissa, 2^23 + z subtracted, the exact
 * product with s rounded once — and feeds one mma.sync; split row blocks are
 * finished in the kernel, as for INT4).  M > 16: the tensor-core kernel with 8-bit
 * codes (64-byte code rows per K block, binary32-exact dequantization into the
 * shared-memory A tile, tcgen05 MMA), split-K as for INT4.  workspace: at least
 * w8a16_gemm_workspace_size() bytes, 16-byte aligned, when that is nonzero;
 * W4A16_EWORKSPACE if it is smaller. */
w4a16_status w8a16_gemm(const void* X, int64_t M, int64_t K, const void* codes,
                        const void* scales, const void* zeros, int64_t N, int32_t g,
                        int32_t sym, void* Y, void* workspace, size_t workspace_bytes,
                        void* stream);

/* w8a16_gemm with the kernel choice overridden, as w4a16_gemm_ex does for 4-bit
 * codes (`path` AUTO, DECODE (M ≤ 16) or TENSORCORE, optionally OR'ed with
 * W4A16_STATIC_WEIGHTS); the workspace is that of w8a16_gemm_plan for the same
 * path.  Used by tests and benchmarks to measure both kernels at one shape. */
w4a16_status w8a16_gemm_ex(const void* X, int64_t M, int64_t K, const void* codes,
                           const void* scales, const void* zeros, int64_t N, int32_t g,
                           int32_t sym, void* Y, void* workspace, size_t workspace_bytes,
                           int32_t path, void* stream);

/* ---------------------------------------------------------------------------
 * W8A8: weights and activations both INT8 on the INT8 tensor cores
 * ("Quantization & Acceleration: 解释 W8A8 与 W4A16 的差异与取舍", 数学机理 (1): both
 * sides quantized to INT8; activations are dynamic and quantized per token;
 * "大模型推理中 Weight-only、W8A8 和 FP8 量化有什么区别？如何选型？", §三: integer
 * matrix multiply on both 8-bit sides, for compute-bound work).  Weights are
 * quantized once with w8a16_quantize(sym = 1, g = K): int8 codes [N, K] and one
 * bf16 scale per output channel [N].  Activations are quantized per call.
 * K must be a multiple of 32; every pointer 16-byte aligned. */

/* Per-token INT8 activations: for each row m of X (bf16 [M, K]),
 * s[m] = max_k |X[m, k]| / 127 (binary32, IEEE division) and
 * q[m, k] = round_half_even(X[m, k] / s[m]) clamped to [−128, 127] (0 for a
 * row of zeros, whose s is 0).  q: int8 [M, K]; s: fp32 [M].  The codes and
 * scales are bit-identical to the host reference's.  X must be finite. */
w4a16_status w8a8_quantize_activations(const void* X, int64_t M, int64_t K, void* q, void* s,
                                        void* stream);

/* W8A8 GEMM: Y[m, n] = bf16_rn(s_x[m] · s_w[n] · Σ_k q_x[m, k]·q_w[n, k]) with the
 * integer sum accumulated exactly in int32 on the tensor cores (tcgen05.mma
 * kind::i8), converted to binary32 and multiplied by the two scales.
 *   qx int8 [M, K], sx fp32 [M] (from w8a8_quantize_activations);
 *   qw int8 [N, K], sw bf16 [N] (w8a16_quantize, sym = 1, g = K); Y bf16 [M, N].
 * CTA tile 128 weight rows x 64/128/256 tokens, one CTA per tile; no workspace. */
w4a16_status w8a8_gemm(const void* qx, const void* sx, int64_t M, int64_t K, const void* qw,
                       const void* sw, int64_t N, void* Y, void* stream);

/* Read and clear the current device's error word, written by a kernel that gave
 * up a bounded wait (a pipeline barrier that did not complete within about one
 * second).  *code = 0 when no kernel reported one.  Synchronizes the device. */
w4a16_status w4a16_device_error(int32_t* code);

/* Human-readable name of a status code (static string, never NULL). */
const char* w4a16_status_string(w4a16_status status);

/* W4A16_ABI_VERSION of the loaded library. */
int32_t w4a16_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H_ */
