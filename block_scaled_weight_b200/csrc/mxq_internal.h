// mxq_internal.h -- launch plumbing shared between the C-ABI layer and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mxq {

// ---- h pass -------------------------------------------------------------------------
// The activation matrix is cut into column strips of kStripCols and into `chunks` row
// chunks; one CTA per (strip, chunk) writes double column sums of squares into
// partial[chunk][cols]. The chunk count depends only on (rows, cols), so the reduction
// order (and the result) is the same on every run and every device.
constexpr int kHpassThreads = 256;
// Resident 256-thread CTAs per SM and the one-wave target grid on a 148-SM B200; strips x
// chunks never exceeds kHpassTargetCtas, so the workspace is at most
// max(kHpassTargetCtas x 256, cols) doubles. Two of the three register-bound slots of an SM:
// the third stays free for a search CTA of the previous batch running beside the h pass
// (3 per SM streamed 3 % faster alone, but left no room).
constexpr int kHpassCtasPerSm = 2;
constexpr int kHpassTargetCtas = 148 * kHpassCtasPerSm;
int hpass_chunks(int64_t rows, int64_t cols, int dtype);
cudaError_t launch_hpass_partial(const void* X, int dtype, int64_t rows, int64_t cols,
                                 int64_t ld, int chunks, double* partial, cudaStream_t st);
// out[j] = sum_{p < parts} partial[p][j] (ascending p); if h != nullptr also
// h[j] = fl32(out[j] / total_rows). Either output may be null.
cudaError_t launch_hpass_finalize(const double* partial, int64_t parts, int64_t cols,
                                  int64_t total_rows, double* colsum, float* h, cudaStream_t st);

// ---- Gram blocks (tensor cores) ---------------------------------------------------------
// G [cols/B][B][B] = fl32(X_b^T X_b / rows) and optionally h = diag(G), for bf16 X.
int gram_chunks(int64_t rows, int64_t cols, int B);
size_t gram_workspace(int64_t rows, int64_t cols, int B);
cudaError_t launch_gram(const void* X, int64_t rows, int64_t cols, int64_t ld, int B, float* G,
                        float* h, void* workspace, cudaStream_t st);

// ---- quantization ---------------------------------------------------------------------
struct QuantArgs {
  const void* W;
  int dtype;
  int64_t n, k, ld;
  const float* h;      // null unless mode == HOPT
  const float* G;      // Gram blocks [k/B][B][B] for the block-Hessian search
  int fmt, mode, block, window;
  int scale_fmt;       // block-scale grid of NVFP4 / INT4 elements (mxq_grids.h)
  void* codes;
  void* scales;
  int log_points;
  float log_grid[256];  // E4M3 tiles: g_p
  // fused error sums (NVFP4 searches with E4M3 scales): per-CTA partials, the four sums, and
  // h for the h-weighted sums of an SSE search (HOPT uses h)
  double* err_partial = nullptr;
  double* err_sums = nullptr;
  const float* h_err = nullptr;
  int ctas_per_sm = 0;  // NVFP4 search: CTAs per SM of its persistent grid (0: all that fit)
};
cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t st);
// Partial slots the fused error sums of an NVFP4 search need (search CTAs + exact-pass CTAs).
int fp4_error_parts(int64_t n, int64_t k, int B, int ctas_per_sm);
// E2M1 on a scale grid other than E4M3, and INT4 on any grid (mxq_quant_grid.cu).
cudaError_t launch_quantize_grid(const QuantArgs& a, cudaStream_t st);
// Block-Hessian search (d^T G_b d) for E2M1 / INT4 elements on any scale grid.
cudaError_t launch_quantize_gram(const QuantArgs& a, cudaStream_t st);
cudaError_t launch_project(const float* w, int64_t count, int fmt, float scale, uint8_t* q,
                           cudaStream_t st);

// ---- dequant / error ------------------------------------------------------------------
struct DecodeArgs {
  const void* codes;
  const void* scales;
  int fmt, block;
  int scale_fmt;  // NVFP4 / INT4: the block-scale grid
  int64_t n, k;
};
cudaError_t launch_dequant(const DecodeArgs& d, float* out, cudaStream_t st);
size_t swizzled_scales_bytes(int64_t n, int64_t kb);
cudaError_t launch_swizzle_scales(const uint8_t* in, int64_t n, int64_t kb, uint8_t* out,
                                  cudaStream_t st);
int error_partials(int64_t n, int64_t k);
// sums[i] = sum over p < parts of partial[p][i], in a fixed order.
cudaError_t launch_error_final(const double* partial, int parts, double* sums, cudaStream_t st);
cudaError_t launch_error(const DecodeArgs& d, const void* W, int dtype, int64_t ld,
                         const float* h, double* partial, int parts, double* sums,
                         cudaStream_t st);

// ---- output error on the tensor cores (mxq_outerr.cu) ------------------------------------
size_t outerr_workspace(int64_t m, int64_t n);
cudaError_t launch_outerr(const void* X, int64_t m, int64_t k, int64_t ldx, const void* W,
                          int64_t n, int64_t ldw, const uint8_t* codes, const uint8_t* scales,
                          int fmt, int scale_fmt, int block, double* sums, void* workspace,
                          cudaStream_t st);

// ---- NVFP4 x NVFP4 product on the block-scaled tensor cores (mxq_nvfp4_mm.cu) -----------
size_t nvfp4_mm_workspace();
cudaError_t launch_nvfp4_mm(const uint8_t* a_codes, const uint8_t* a_sf, const uint8_t* b_codes,
                            const uint8_t* b_sf, int64_t m, int64_t n, int64_t k, float* D,
                            void* workspace, cudaStream_t st);

// ---- FP8-GPTQ on 64 x 64 tiles (mxq_gptq.cu) ---------------------------------------------
cudaError_t launch_gptq_prepare(const float* G, int64_t nblocks, double damp, float* U,
                                cudaStream_t st);
cudaError_t launch_gptq_tiles(const void* W, int dtype, int64_t n, int64_t k, int64_t ld,
                              const float* U, const float* scales, uint8_t* codes,
                              cudaStream_t st);

// ---- GPTQ with the block quantizer (mxq_gptq_full.cu) ----------------------------------
struct GptqArgs {
  const void* W;
  int dtype;
  int64_t n, k, ld;
  const float* h;          // HOPT search weights (and the ordered variant's loss weights)
  const float* U;          // [k][k] factor in sweep order
  const int32_t* perm;     // [k / block] block order, or null
  int fmt, mode, block, window, scale_fmt;
  void* codes;
  void* scales;
  void* workspace;         // gptq_sweep_workspace(n, k) bytes
};
size_t gptq_factor_workspace(int64_t k);
cudaError_t launch_gptq_factor(const float* H, int64_t k, int B, const int32_t* perm,
                               double damp, float* U, void* ws, cudaStream_t st);
size_t gptq_sweep_workspace(int64_t n, int64_t k);
cudaError_t launch_gptq_sweep(const GptqArgs& g, cudaStream_t st);
int gptq_sort_max();
cudaError_t launch_gptq_order(const GptqArgs& g, const uint8_t* codes, const uint8_t* scales,
                              double* loss, int32_t* perm, cudaStream_t st);
// ---- the full Gram matrix on the tensor cores (mxq_gram_full.cu) ---------------------------
size_t gram_full_workspace(int64_t rows, int64_t cols);
cudaError_t launch_gram_full(const void* X, int64_t rows, int64_t cols, int64_t ld, float* H,
                             void* workspace, cudaStream_t st, const char** why);

int sm_count();
// Bound (in polls) of every pipeline wait of the tensor-core kernels: 2^26 unless a caller
// lowered it with mxq_set_wait_polls (to exercise the timeout path).
uint32_t wait_polls();
// Raises func's dynamic shared-memory limit to `bytes` on the current device, once per
// (device, kernel): the attribute is per device, so each GPU a process uses needs its own.
cudaError_t ensure_dynamic_smem(const void* func, int bytes);
// Sets the per-thread text that mxq_last_error() returns.
void set_error_text(const char* fmt, ...) __attribute__((format(printf, 1, 2)));

}  // namespace mxq
