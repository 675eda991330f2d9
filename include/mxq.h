/*
 * mxq.h -- block-scaled post-training weight quantization with a searched E4M3 block
 * scale, on NVIDIA B200 (sm_100a).
 *
 * For every block of B contiguous input-dimension weights of W [n, k] (or every 64 x 64
 * tile, for E4M3 elements) the library picks one scale and emits the quantized codes:
 *
 *   naive    the amax snap s0 = RNE_E4M3(amax / qmax)
 *            ("Is Finer Better? The Limits of Microscaling Formats in LLMs", sec. 2.1:
 *            s = Q_scale(xmax / C), q = Q_elem(x / s), x^ = s * q);
 *   sse      the candidate scale minimising sum_j (w_j - s q_j)^2;
 *   hopt     the candidate scale minimising sum_j h_j (w_j - s q_j)^2 with
 *            h_j = E[x_j^2] over calibration activations ("quantization_algorithms.txt",
 *            sec. 1, the diagonal approximation of the output-error objective);
 *
 * over candidates on the E4M3 scale grid (all 126 positive finite values, or a window of
 * codes around the naive snap; qwantize "Results", sections "INT8 (FP8 E4M3 scales)" and
 * "NVFP4 (FP8 E4M3 scales)"), on another 8-bit scale grid (UE8M0 powers of two -- MXFP4 --,
 * UE4M4 or UE5M3; qwantize "Results", sections "MXFP4 (UE8M0 power-of-2 scales)" and
 * "Exotic Scales"), or, for E4M3 elements, on a logarithmic grid of float32 tile scales
 * ("quantization_algorithms.txt", sec. 1).
 *
 * Element grids: E2M1 {0, 0.5, 1, 1.5, 2, 3, 4, 6} (qmax 6); symmetric INT4 [-7, 7]
 * (qmax 7; the NVINT4 rows of qwantize "Results", "GPTQ Quantization"); symmetric INT8
 * [-127, 127] with effective scale fl32(amax_e4m3 / 127) (qwantize "Results", INT8
 * section); E4M3 elements (max 448). Every rounding onto a grid is round-to-nearest with
 * ties to the even code and saturation; the quotient w / s is the IEEE float32 quotient.
 * Candidate ties go to the smallest scale.
 *
 * Conventions for every call below:
 *  - Pointers named as device pointers are device memory (any allocator) owned by the
 *    caller; the library allocates no device memory for data. Workspace sizes come from the
 *    *_workspace queries.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 *    stream) unless stated otherwise. Results are valid after the stream synchronises.
 *  - Arguments are validated on the host before any launch; a rejected call launches
 *    nothing and returns a status. A CUDA launch failure returns MXQ_ERR_CUDA and
 *    mxq_last_error() (per host thread) describes it. No exception crosses the boundary.
 *  - Calls are reentrant. Mutable state, all of it set up on first use and guarded by
 *    locks: the per-thread error text; per device, the raised shared-memory limit of each
 *    tensor-core kernel; per device, the three library streams and the ring of events
 *    that mxq_gptq_factor and mxq_gptq create on first use (their calls on one device are
 *    ordered on the host); and per device the address of the static scratch of
 *    mxq_act_sqmean_noalloc.
 *  - Empty problems (n, k or rows == 0) return MXQ_OK without launching.
 *  - Weights and activations may not contain NaN or infinities (the result is then
 *    unspecified, but no launch faults).
 */
#ifndef MXQ_H
#define MXQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MXQ_API __attribute__((visibility("default")))
#else
#define MXQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MXQ_OK = 0,
    MXQ_ERR_INVALID_ARG = 1,   /* null pointer, bad enum or parameter value */
    MXQ_ERR_SHAPE = 2,         /* negative size, k % block != 0, ld < cols, ... */
    MXQ_ERR_DTYPE = 3,         /* unsupported input element type */
    MXQ_ERR_ALIGN = 4,         /* pointer or leading dimension not 16-byte aligned */
    MXQ_ERR_UNSUPPORTED = 5,   /* valid but not implemented combination */
    MXQ_ERR_CUDA = 6,          /* a CUDA call failed; see mxq_last_error() */
    MXQ_ERR_WORKSPACE = 7      /* workspace missing or smaller than the query's answer */
} mxq_status;

typedef enum { MXQ_F32 = 0, MXQ_BF16 = 1 } mxq_dtype;
typedef enum { MXQ_FMT_NVFP4 = 0, MXQ_FMT_INT8 = 1, MXQ_FMT_E4M3 = 2, MXQ_FMT_INT4 = 3 } mxq_fmt;
typedef enum { MXQ_NAIVE = 0, MXQ_SSE = 1, MXQ_HOPT = 2 } mxq_mode;
/* 8-bit block-scale grids (code -> value; every listed code finite):
 *  MXQ_SCALE_E4M3   codes 0..126: 0, m/8 2^-6 (e = 0), (1 + m/8) 2^(e-7); candidates 1..126
 *  MXQ_SCALE_UE4M4  codes 0..255: 0, m/16 2^-6 (e = 0), (1 + m/16) 2^(e-7) (max 496);
 *                   candidates 1..255
 *  MXQ_SCALE_UE5M3  codes 0..255: 0, m/8 2^-14 (e = 0), (1 + m/8) 2^(e-15) (max 122880);
 *                   candidates 1..255
 *  MXQ_SCALE_UE8M0  codes 0..254: 2^(code - 127) (OCP E8M0; 255 is NaN); candidates 0..254 */
typedef enum { MXQ_SCALE_E4M3 = 0, MXQ_SCALE_UE4M4 = 1, MXQ_SCALE_UE5M3 = 2,
               MXQ_SCALE_UE8M0 = 3 } mxq_scale_fmt;

/* Quantizer settings.
 *  fmt        MXQ_FMT_NVFP4: E2M1 elements, one scale byte (grid `scale_fmt`) per block of
 *             `block` (16 or 32) contiguous weights along k. With MXQ_SCALE_UE8M0 this is
 *             MXFP4.
 *             MXQ_FMT_INT4: int4 elements in [-7, 7], one scale byte (grid `scale_fmt`:
 *             E4M3 -- NVINT4 --, UE4M4 or UE5M3) per block of `block` (16 or 32) weights.
 *             MXQ_FMT_INT8: int8 elements in [-127, 127], one E4M3 byte (the stored amax)
 *             per block of `block` (32, 64, 128 or 256) weights; effective scale
 *             fl32(E4M3 / 127).
 *             MXQ_FMT_E4M3: E4M3 elements, one float32 scale per `block` x `block` tile
 *             (block = tile_rows = 64).
 *  mode       MXQ_NAIVE, MXQ_SSE or MXQ_HOPT.
 *  block      see fmt.
 *  tile_rows  1 for NVFP4 and INT8; 64 (= block) for E4M3 tiles.
 *  window     NVFP4 / INT4 / INT8 search: -1 = every candidate code of the scale grid
 *             (E4M3: the 126 positive finite values 0x01..0x7E); w >= 0 = codes
 *             [c0 - w, c0 + w] clipped to the candidate codes around the naive code c0
 *             ([1, max(w, 1)] when c0 is a zero scale). Ignored for E4M3 tiles.
 *  log_points E4M3 tiles: P grid points g_p = fl32(2^(lo + (hi - lo) p / (P - 1))),
 *             candidate s_p = fl32(fl32(amax_tile / 448) * g_p); 2 <= P <= 256.
 *  log_lo_exp2, log_hi_exp2  lo and hi (finite, lo < hi); the pages' grid is -2, 2.
 *  scale_fmt  the block-scale grid (mxq_scale_fmt) of NVFP4 and INT4 elements; INT8 and
 *             E4M3 tiles need MXQ_SCALE_E4M3 (0); UE8M0 only with NVFP4 elements.
 *             Naive scale: UE8M0 2^(floor(log2 amax) - 2) (the OCP rule, 2 = the largest
 *             E2M1 exponent), clamped to codes 0..254 (0 for amax = 0); every other grid
 *             its nearest value (RNE, saturating) to fl32(amax / qmax).
 *  ctas_per_sm  how many CTAs per SM the NVFP4 (E4M3-scale) search may occupy: 0 = as many
 *             as fit (fastest alone); 1 leaves room beside it for a streaming kernel on
 *             another stream, e.g. the next batch's h pass, which then overlaps the search.
 *             Results are the same for every value (the fused error sums of
 *             mxq_quantize_err group blocks by CTA, so they can differ in the last bits).
 *             Other quantizers ignore it.
 */
typedef struct mxq_params {
    int32_t fmt;
    int32_t mode;
    int32_t block;
    int32_t tile_rows;
    int32_t window;
    int32_t log_points;
    float log_lo_exp2;
    float log_hi_exp2;
    int32_t scale_fmt;
    int32_t ctas_per_sm;
} mxq_params;

/* Weight error metrics from the four sums that mxq_error produces. */
typedef struct mxq_metrics {
    double sse;         /* sum (w - w^)^2 */
    double w_sq;        /* sum w^2 */
    double hsse;        /* sum h_j (w - w^)^2   (0 without h) */
    double hw_sq;       /* sum h_j w^2          (0 without h) */
    double weight_rel;  /* sqrt(sse / w_sq): ||Q(W) - W||_F / ||W||_F (qwantize "Results") */
    double h_rel;       /* sqrt(hsse / hw_sq)   (0 without h) */
} mxq_metrics;

/* ------------------------------------------------------------------------------------
 * h pass: h_j = E_r[x_rj^2] = (1/R) sum_r x_rj^2 over the rows of the calibration
 * activations X ("quantization_algorithms.txt", sec. 1: h_j = E[x_j^2]).
 *
 *  X          device, [rows, cols] row-major with leading dimension ld (elements);
 *             16-byte aligned; dtype MXQ_BF16 or MXQ_F32.
 *  cols       multiple of 8 (bf16) or 4 (f32); ld >= cols with ld * elsize % 16 == 0.
 *  h          device float [cols], written as fl32(sum / rows) (the sum is exact to within
 *             ~2e-6 relative: float32 over at most 32 rows, then double).
 *  workspace  device, at least mxq_act_sqmean_workspace(rows, cols) bytes, 8-byte aligned.
 * ------------------------------------------------------------------------------------ */
MXQ_API size_t mxq_act_sqmean_workspace(int64_t rows, int64_t cols);
MXQ_API mxq_status mxq_act_sqmean(const void* X, int32_t dtype, int64_t rows, int64_t cols, int64_t ld,
                          float* h, void* workspace, size_t workspace_bytes, void* stream);

/* mxq_act_sqmean without a workspace argument, for callers that cannot allocate device
 * memory (their device memory belongs to another allocator or a fixed arena, or they must
 * not call cudaMalloc after start-up because it can synchronise the device). The pages
 * have no counterpart: this is an interface variant, not part of the method.
 * The scratch is a 1 MiB static device array inside the library, present on every GPU that
 * loads it until the process exits; it covers every width up to 131072 columns (wider X is
 * rejected with MXQ_ERR_SHAPE, launching nothing). No cudaMalloc, cudaFree or other
 * allocation happens. All calls share the array: calls that overlap on the GPU race, so
 * order them (e.g. one stream). The first call on each device, with that device current,
 * looks up the array's device address and caches it for the life of the process; make it
 * before any stream capture begins. The cached address does not survive a cudaDeviceReset:
 * after resetting a device, do not call this entry point on it again.
 * Arguments and result as for mxq_act_sqmean. */
MXQ_API mxq_status mxq_act_sqmean_noalloc(const void* X, int32_t dtype, int64_t rows,
                                          int64_t cols, int64_t ld, float* h, void* stream);

/* The two halves of mxq_act_sqmean, for row-sharded activations (one shard per GPU):
 *  mxq_act_sqsum writes colsum[j] = sum over this shard's rows of x_rj^2 (device double
 *  [cols]); workspace as for mxq_act_sqmean. After the shards' colsum vectors are gathered
 *  into device memory partials [parts, cols] (row-major), mxq_act_sqmean_finalize writes
 *  h[j] = fl32((sum_p partials[p][j]) / total_rows), summing p in ascending order. */
MXQ_API mxq_status mxq_act_sqsum(const void* X, int32_t dtype, int64_t rows, int64_t cols, int64_t ld,
                         double* colsum, void* workspace, size_t workspace_bytes, void* stream);
MXQ_API mxq_status mxq_act_sqmean_finalize(const double* partials, int64_t parts, int64_t cols,
                                   int64_t total_rows, float* h, void* stream);

/* ------------------------------------------------------------------------------------
 * Gram blocks of the activations, for the block-Hessian objective: the page's exact
 * output-error objective of a block, || X_b (W_b - s Q(W_b / s))^T ||_F^2 =
 * R d^T G_b d per row, with G_b = X_b^T X_b / R ("quantization_algorithms.txt", sec. 1;
 * h is its diagonal). Computed on the tensor cores from one read of X.
 *
 *  X          device bf16 [rows, cols] row-major, leading dimension ld (elements); 16-byte
 *             aligned, ld * 2 % 16 == 0. (float32 X: MXQ_ERR_DTYPE.)
 *  block      B = 16, 32 or 64 (64: the E4M3 tile width, for the tile GPTQ); cols % B == 0.
 *  G          device float [cols/B][B][B], 16-byte aligned: G[b][i][j] =
 *             fl32(sum_r x_r,bB+i x_r,bB+j / rows) (the sum: float32 over at most 512 rows
 *             inside the tensor cores, then double); symmetric to within that rounding.
 *  h          device float [cols] or NULL: h[c] = G[c/B][c%B][c%B].
 *  workspace  device, at least mxq_act_block_gram_workspace(rows, cols, block) bytes,
 *             16-byte aligned.
 * A launch whose internal waits time out (none does on a working GPU) writes NaN to G and h.
 * ------------------------------------------------------------------------------------ */
MXQ_API size_t mxq_act_block_gram_workspace(int64_t rows, int64_t cols, int32_t block);
MXQ_API mxq_status mxq_act_block_gram(const void* X, int32_t dtype, int64_t rows, int64_t cols,
                                      int64_t ld, int32_t block, float* G, float* h,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * Scale search and quantization (naive / sse / hopt), fused in one kernel per format.
 *
 *  W       device, [n, k] row-major, leading dimension ld (elements), 16-byte aligned,
 *          ld * elsize % 16 == 0; dtype MXQ_BF16 or MXQ_F32.
 *  h       device float [k], 16-byte aligned; required for MXQ_HOPT, ignored otherwise.
 *  p       host pointer to the settings.
 *  codes   device, dense row-major:
 *            NVFP4 uint8 [n, k/2]: element 2i in the low nibble, nibble = sign << 3 | e2m1
 *            INT4  uint8 [n, k/2]: element 2i in the low nibble, nibble = the signed code
 *                  in two's complement (-7 .. 7)
 *            INT8  int8  [n, k]:   two's complement in [-127, 127]
 *            E4M3  uint8 [n, k]:   sign << 7 | e4m3 code
 *          The sign bit of a zero magnitude is the weight's sign bit (INT8 has no -0).
 *  scales  device, dense row-major:
 *            NVFP4, INT4, INT8: uint8 scale codes [n, k/block] of the scale grid; a zero
 *            scale (code 0 of E4M3 / UE4M4 / UE5M3) only from a naive snap that rounds
 *            to zero (then every magnitude is 0);
 *            E4M3: float [n/64, k/64] tile scales (0 for an all-zero tile).
 *  Shapes: k % block == 0; for E4M3 tiles n % 64 == 0 and k % 64 == 0.
 *  Result: identical to the plain definition evaluated with IEEE float32 quotients and
 *  float32 dequantised values, candidate errors accumulated in double in element order,
 *  ties to the smallest scale (NVFP4, INT4 and INT8: exactly, including ties; E4M3 tiles:
 *  exactly wherever the two best tile errors differ by more than 1e-6 relative).
 * ------------------------------------------------------------------------------------ */
MXQ_API mxq_status mxq_quantize(const void* W, int32_t dtype, int64_t n, int64_t k, int64_t ld,
                        const float* h, const mxq_params* p, void* codes, void* scales,
                        void* stream);

/* ------------------------------------------------------------------------------------
 * Block-Hessian H-optimal search: the scale minimising d^T G_b d per block (d = w - w^,
 * G_b the block's Gram matrix from mxq_act_block_gram, or any symmetric B x B matrices),
 * i.e. the page's output-error objective || X_b d ||^2 / R instead of its diagonal
 * approximation ("quantization_algorithms.txt", sec. 1).
 *
 *  W, codes, scales  as for mxq_quantize; p->fmt MXQ_FMT_NVFP4 or MXQ_FMT_INT4, any
 *                    p->scale_fmt they accept, p->block 16 or 32, p->mode MXQ_HOPT,
 *                    p->window as for mxq_quantize.
 *  G                 device float [k/B][B][B], 16-byte aligned.
 *  Result: identical to the definition e = sum_i sum_j G_ij (d_i d_j) (double, i then j,
 *  d_i = (double)w_i - (double)fl32(s q_i) signed), lowest code on ties -- exactly,
 *  including ties.
 * ------------------------------------------------------------------------------------ */
MXQ_API mxq_status mxq_quantize_gram(const void* W, int32_t dtype, int64_t n, int64_t k,
                                     int64_t ld, const float* G, const mxq_params* p,
                                     void* codes, void* scales, void* stream);

/* ------------------------------------------------------------------------------------
 * Element projection at one fixed scale -- the per-element step of the search above,
 * exposed so that it can be verified exhaustively.
 *
 *  w          device float [count], 4-byte aligned (only |w| is used).
 *  fmt        MXQ_FMT_NVFP4: q = RNE_E2M1(fl32(|w| / scale)) code 0..7;
 *             MXQ_FMT_INT4:  q = min(7, RNE_int(fl32(|w| / scale)));
 *             MXQ_FMT_INT8:  q = min(127, RNE_int(fl32(|w| / fl32(scale / 127)))), scale
 *                            the stored E4M3 amax;
 *             MXQ_FMT_E4M3:  q = RNE_E4M3(fl32(|w| / scale)) code 0..126, any float
 *                            scale > 0.
 *  scale_fmt  NVFP4 / INT4: the grid that `scale` must be a positive value of
 *             (mxq_scale_fmt); INT8: MXQ_SCALE_E4M3; ignored for E4M3 elements.
 *  q          device uint8 [count]: the magnitude codes.
 * ------------------------------------------------------------------------------------ */
MXQ_API mxq_status mxq_project(const float* w, int64_t count, int32_t fmt, int32_t scale_fmt,
                               float scale, uint8_t* q, void* stream);

/* ------------------------------------------------------------------------------------
 * Dequantisation: out [n, k] float (device, dense) = s * q with the layouts above
 * (NVFP4: grid(scale) * E2M1(code); INT4: grid(scale) * code; INT8: code *
 * fl32(E4M3(scale) / 127), the product rounded to float; E4M3: tile scale * E4M3(code),
 * rounded to float). A UE8M0 scale byte 255 (NaN) decodes to NaN.
 * ------------------------------------------------------------------------------------ */
MXQ_API mxq_status mxq_dequant(const void* codes, const void* scales, const mxq_params* p, int64_t n,
                       int64_t k, float* out, void* stream);

/* ------------------------------------------------------------------------------------
 * Scale bytes for sm_100 block-scaled tensor-core GEMMs. The quantizer writes scales
 * row-major [n, kb] (kb = k / block); block-scaled MMA instructions (and the libraries
 * built on them) read them in 128 x 4 tiles of 512 bytes: tiles ordered by row tile, then
 * column tile; inside a tile, row m and column c at byte (m % 32) * 16 + (m / 32) * 4 + c;
 * rows padded to a multiple of 128 and columns to a multiple of 4 with zeros. This layout
 * is the hardware's, not the pages'.
 *  scales  device uint8 [n, kb]; out  device uint8, mxq_swizzled_scales_bytes(n, kb) bytes.
 * ------------------------------------------------------------------------------------ */
MXQ_API size_t mxq_swizzled_scales_bytes(int64_t n, int64_t kb);
MXQ_API mxq_status mxq_swizzle_scales(const uint8_t* scales, int64_t n, int64_t kb,
                                      uint8_t* out, void* stream);

/* ------------------------------------------------------------------------------------
 * The product of two NVFP4 operands in this library's output format, on the block-scaled
 * tensor cores: D = A^ B^T with A^ = dequant(A) [m, k] and B^ = dequant(B) [n, k], each an
 * NVFP4 matrix of 16-element blocks along k -- E2M1 codes and one E4M3 scale per block
 * ("Is Finer Better? The Limits of Microscaling Formats in LLMs", sec. 2.1: x^ = s q). The
 * hardware (tcgen05.mma kind::mxf4nvf4, scale_vec::4X) reads the codes as mxq_quantize packs
 * them and the scales in the layout mxq_swizzle_scales writes, so quantized weights feed a
 * block-scaled GEMM as they are; e.g. Y = X_q W_q^T with X quantized along its rows.
 *
 *  a_codes    device uint8 [m, k/2] (NVFP4 codes, element 2i in the low nibble), 16-byte
 *             aligned; b_codes likewise [n, k/2].
 *  a_scales   device, the E4M3 block scales of A [m, k/16] rewritten by mxq_swizzle_scales
 *             (mxq_swizzled_scales_bytes(m, k/16) bytes), 16-byte aligned; b_scales likewise.
 *  k          a multiple of 64; m, n, k below 2^31.
 *  D          device float [m, n] row-major, 16-byte aligned: D[i][j] = sum_c A^[i][c] B^[j][c],
 *             float32 accumulation in the tensor cores (each product of two scaled E2M1
 *             values is exact), within (k + 2) 2^-24 (|A^| |B^|^T)_ij of the exact sum.
 *  workspace  device, mxq_nvfp4_gemm_workspace() bytes, 16-byte aligned. A launch whose
 *             internal waits time out (none does on a working GPU) writes NaN over D.
 * ------------------------------------------------------------------------------------ */
MXQ_API size_t mxq_nvfp4_gemm_workspace(void);
MXQ_API mxq_status mxq_nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales,
                                  const uint8_t* b_codes, const uint8_t* b_scales, int64_t m,
                                  int64_t n, int64_t k, float* D, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * Weight error (qwantize "Results": ||Q(W) - W||_F / ||W||_F) and the h-weighted error
 * (the diagonal objective, "quantization_algorithms.txt", sec. 1), without materialising
 * the dequantised matrix.
 *
 *  sums       device double [4]: sum (w - w^)^2, sum w^2, sum h_j (w - w^)^2,
 *             sum h_j w^2 (the last two 0 when h is NULL). Deterministic (fixed-order
 *             combine).
 *  workspace  device, at least mxq_error_workspace(n, k) bytes, 8-byte aligned.
 * mxq_metrics_from_sums (host, synchronous) turns four host doubles into mxq_metrics.
 * ------------------------------------------------------------------------------------ */
MXQ_API size_t mxq_error_workspace(int64_t n, int64_t k);
MXQ_API mxq_status mxq_error(const void* W, int32_t dtype, int64_t n, int64_t k, int64_t ld,
                     const void* codes, const void* scales, const float* h,
                     const mxq_params* p, double* sums, void* workspace,
                     size_t workspace_bytes, void* stream);
MXQ_API mxq_status mxq_metrics_from_sums(const double* host_sums, mxq_metrics* out);

/* mxq_quantize followed by mxq_error on its result, in one call: codes and scales as
 * mxq_quantize writes them (identical bytes), sums as mxq_error defines them, h-weighted
 * with h when h is not NULL (H-optimal uses the same h for the search). The NVFP4 search
 * with E4M3 scales (mode SSE or H-optimal) adds each block's sums at its winning scale as
 * it emits the block, so the weights are read once; every other quantizer runs the error
 * pass after the search. The sums group the blocks differently from mxq_error's, so the two
 * can differ in the last bits (each is deterministic). workspace:
 * mxq_quantize_err_workspace(n, k, p) bytes, 8-byte aligned. */
MXQ_API size_t mxq_quantize_err_workspace(int64_t n, int64_t k, const mxq_params* p);
MXQ_API mxq_status mxq_quantize_err(const void* W, int32_t dtype, int64_t n, int64_t k,
                                    int64_t ld, const float* h, const mxq_params* p,
                                    void* codes, void* scales, double* sums, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * Output error of a quantized weight (qwantize "Results": ||X_s Wq^T - X_s W^T||_F /
 * ||X_s W^T||_F on sampled calibration rows X_s), on the tensor cores: both products with
 * float32 accumulation (bf16 operands; the 4-bit codes are expanded to bf16 exactly), the
 * squared Frobenius norms summed in double in a fixed order.
 *  X       device bf16 [m, k], leading dimension ldx; W device bf16 [n, k], ldw; both
 *          16-byte aligned with ld * 2 % 16 == 0.
 *  codes, scales, p  the quantized W (p->fmt MXQ_FMT_NVFP4 or MXQ_FMT_INT4, any scale grid
 *          and block they accept; row-major scales).
 *  sums    device double [2]: sum (X Wq^T - X W^T)^2, sum (X W^T)^2 (NaN after an internal
 *          wait timed out, which no working GPU does).
 *  workspace  mxq_output_error_workspace(m, n) bytes, 16-byte aligned.
 * ------------------------------------------------------------------------------------ */
MXQ_API size_t mxq_output_error_workspace(int64_t m, int64_t n);
MXQ_API mxq_status mxq_output_error(const void* X, int64_t m, int64_t k, int64_t ldx,
                                    const void* W, int64_t n, int64_t ldw, const void* codes,
                                    const void* scales, const mxq_params* p, double* sums,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * FP8-GPTQ on 64 x 64 tiles ("quantization_algorithms.txt", section 1, the 64x64 tile
 * scheme): E4M3 elements at fixed tile scales, the columns of every tile quantised one
 * after another with each residual propagated through the inverse of the damped Gram
 * matrix of the tile's 64 input dimensions (GPTQ's update in its Cholesky form).
 *
 * mxq_gptq_prepare: per column block b, H = (G_b + G_b^T) / 2 + lambda I with
 * lambda = damp * mean(diag G_b) (1 when that mean is 0), and U the upper Cholesky factor
 * of H^-1 (H^-1 = U^T U), computed in float64 and rounded to float32 once.
 *  G        device float [nblocks][64][64], 16-byte aligned: the Gram blocks of
 *           mxq_act_block_gram with block 64 (any scaling of them gives the same codes).
 *  damp     relative damping, finite and >= 0 (GPTQ's customary value is 0.01).
 *  U        device float [nblocks][64][64], 16-byte aligned; the strict lower triangle is
 *           written as 0. A block whose damped H is not positive definite (impossible for
 *           a Gram matrix) yields NaN entries.
 *
 * mxq_gptq_tiles: for every row r of every 64 x 64 tile (rows independent), columns
 * c = 0 .. 63 in order: q = RNE_E4M3(fl32(|w_c| / s)) (code 0..126, 0 when s == 0),
 * wq = +-fl32(s E4M3(q)) with the sign of w_c, err = fl32(fl32(w_c - wq) / U_cc),
 * w_j = fl32(w_j - fl32(err U_cj)) for j > c; w starts as the tile's weights.
 *  W        as for mxq_quantize (bf16 or float32), n % 64 == 0, k % 64 == 0.
 *  U        device float [k/64][64][64], 16-byte aligned (mxq_gptq_prepare's output).
 *  scales   device float [n/64][k/64], 4-byte aligned: the tile scales (e.g. those of
 *           mxq_quantize with MXQ_FMT_E4M3), finite and >= 0.
 *  codes    device uint8 [n, k], 16-byte aligned: sign << 7 | e4m3 code (the layout of
 *           mxq_quantize's E4M3 codes; mxq_dequant and mxq_error read them with the same
 *           scales).
 *  Result: identical to the definition above evaluated in that order (every step a
 *  separately rounded IEEE float32 operation), given the same U.
 * ------------------------------------------------------------------------------------ */
MXQ_API mxq_status mxq_gptq_prepare(const float* G, int64_t nblocks, double damp, float* U,
                                    void* stream);
MXQ_API mxq_status mxq_gptq_tiles(const void* W, int32_t dtype, int64_t n, int64_t k,
                                  int64_t ld, const float* U, const float* scales,
                                  uint8_t* codes, void* stream);

/* ------------------------------------------------------------------------------------
 * GPTQ with the block quantizer as its inner step (qwantize "Results", "GPTQ
 * Quantization": the GPTQ block is the quantization block; after a block is quantised its
 * error is compensated in all remaining columns through the inverse Hessian; sequential
 * order, or "ordered" -- blocks sorted by descending Hessian-weighted quantization loss).
 * The algorithm is Frantar et al. 2022, Algorithm 1, in its Cholesky form.
 *
 * mxq_act_gram: H = X^T X / R, the full cols x cols Gram matrix (the GPTQ Hessian up to a
 *  factor) of bf16 X [rows, cols] (ld as for mxq_act_sqmean), float32, row-major, 16-byte
 *  aligned. Computed on the tensor cores (tcgen05, pairs of SMs, 256 x 512 tiles of H) over
 *  the tiles that reach the upper triangle: bf16 products (exact), float32 accumulation
 *  over the rows in order (the last wave's tiles in row chunks added in double in a fixed
 *  order), then the upper triangle copied onto the lower one: H is exactly symmetric,
 *  deterministic, and each entry is within rows * 2^-24 * (|X|^T |X|)_ij / rows of the
 *  exact value. workspace: mxq_act_gram_workspace(rows, cols) bytes, 16-byte aligned (at
 *  most one 256 x 512 float32 partial tile per pair of SMs). A launch whose internal waits
 *  time out (none does on a working GPU) writes NaN over all of H.
 *
 * mxq_gptq_factor: U [k][k] float32 (upper, the strict lower triangle written as 0), the
 *  upper Cholesky factor of (H~ + lambda I)^-1, H~ = (H + H^T) / 2 with rows and columns in
 *  sweep order (position t*block + j is column perm[t]*block + j; natural order when perm
 *  is NULL), lambda = damp * mean(diag H) (1 when that mean is 0); computed in float64,
 *  rounded to float32 once.
 *   H       device float [k][k], 16-byte aligned.
 *   block   the quantization block (16 or 32); k % block == 0; perm device int32 [k/block]
 *           (a permutation of 0 .. k/block - 1; other values are clamped into range and
 *           give a meaningless result) or NULL.
 *   damp    finite, >= 0 (GPTQ's customary 0.01).
 *   workspace  mxq_gptq_factor_workspace(k) bytes (two float64 k x k matrices, k rounded
 *           up to a multiple of 64), 16-byte aligned.
 *   The call is asynchronous like the others: its kernels run on two streams of the library
 *   (one per device, created on first use) that wait for `stream` and that `stream` waits
 *   for before its next work; concurrent calls on one device are ordered on the host.
 *
 * mxq_gptq_order: the ordered variant's block sequence. loss_b = sum over rows and the
 *  block's columns of h_j (w_ij - w^_ij)^2 (float64) for the plain quantizer's result
 *  (mxq_quantize with p and h); perm = the blocks by descending loss, the lower block first
 *  on equal loss. k / block <= 2048.
 *   W, p    as for mxq_quantize (p->fmt MXQ_FMT_NVFP4 or MXQ_FMT_INT4, block 16 or 32).
 *   h       device float [k] (required: the loss weights; also the H-optimal search's).
 *   perm    device int32 [k / block].
 *   workspace  mxq_gptq_order_workspace(n, k, p) bytes, 16-byte aligned.
 *
 * mxq_gptq: the sweep. Rows are independent; for each row and each block position
 *  t = 0 .. k/block - 1 (block b = perm[t], or t): the block's scale is the quantizer's pick
 *  (p->mode, p->window, p->scale_fmt as for mxq_quantize) for the block's CURRENT weights;
 *  then for its columns j in order, at position q = t*block + j:
 *    code = the element projection at that scale, wq = +-fl32(s g(code)),
 *    err_j = fl32(fl32(w - wq) / U[q][q]), w at the block's later positions q' -=
 *    fl32(err_j U[q][q']);
 *  then at every later position q': acc = 0, acc = fma(err_j, U[t*block + j][q'], acc) for
 *  j = 0 .. block-1, w -= acc. Every step one IEEE float32 operation.
 *   W       as for mxq_quantize; h as for mxq_quantize (H-optimal); U mxq_gptq_factor's
 *           output for the same perm; codes / scales: mxq_quantize's layouts (original
 *           column order).
 *   workspace  mxq_gptq_workspace(n, k) bytes (the working weights, n x k float32),
 *           16-byte aligned. n <= 65535 x 64.
 *  Result: identical to the definition above, including ties (each scale search scores
 *  every candidate exactly in float64, element order; lowest code on equal errors).
 * ------------------------------------------------------------------------------------ */
MXQ_API size_t mxq_act_gram_workspace(int64_t rows, int64_t cols);
MXQ_API mxq_status mxq_act_gram(const void* X, int32_t dtype, int64_t rows, int64_t cols,
                                int64_t ld, float* H, void* workspace, size_t workspace_bytes,
                                void* stream);
MXQ_API size_t mxq_gptq_factor_workspace(int64_t k);
MXQ_API mxq_status mxq_gptq_factor(const float* H, int64_t k, int32_t block,
                                   const int32_t* perm, double damp, float* U, void* workspace,
                                   size_t workspace_bytes, void* stream);
MXQ_API size_t mxq_gptq_order_workspace(int64_t n, int64_t k, const mxq_params* p);
MXQ_API mxq_status mxq_gptq_order(const void* W, int32_t dtype, int64_t n, int64_t k,
                                  int64_t ld, const float* h, const mxq_params* p,
                                  int32_t* perm, void* workspace, size_t workspace_bytes,
                                  void* stream);
MXQ_API size_t mxq_gptq_workspace(int64_t n, int64_t k);
MXQ_API mxq_status mxq_gptq(const void* W, int32_t dtype, int64_t n, int64_t k, int64_t ld,
                            const float* h, const float* U, const int32_t* perm,
                            const mxq_params* p, void* codes, void* scales, void* workspace,
                            size_t workspace_bytes, void* stream);

/* The tensor-core kernels (mxq_act_block_gram, mxq_act_gram, mxq_output_error,
 * mxq_nvfp4_gemm) bound every wait of their pipelines (a poll of an mbarrier); a wait that
 * runs out sets an error word, the kernel lets its copies and MMAs finish and frees its
 * tensor memory, and the call's outputs become NaN. mxq_set_wait_polls sets that bound for
 * the launches that follow, process-wide (0 restores the default, 2^26 polls: seconds). A
 * small bound makes the waits run out on purpose, to test that path; the library stays
 * usable afterwards. No page counterpart: this is the library's own failure handling. */
MXQ_API void mxq_set_wait_polls(uint32_t polls);

/* Human-readable text for a status; the last failure's detail on this host thread. */
MXQ_API const char* mxq_status_string(mxq_status s);
MXQ_API const char* mxq_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* MXQ_H */
