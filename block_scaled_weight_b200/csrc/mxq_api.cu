// mxq_api.cu -- the extern "C" boundary of libmxq.so: host-side validation, workspace
// queries and kernel launches. See include/mxq.h for the contract of every call.
#include "../../include/mxq.h"
#include "mxq_grids.h"
#include "mxq_internal.h"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

namespace mxq {

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

namespace {
std::atomic<uint32_t> g_wait_polls{0};
}

uint32_t wait_polls() {
  const uint32_t p = g_wait_polls.load(std::memory_order_relaxed);
  return p ? p : (1u << 26);
}

cudaError_t ensure_dynamic_smem(const void* func, int bytes) {
  // The attribute belongs to the (device, kernel) pair: remember each pair raised so far.
  struct Done { int dev; const void* func; int bytes; };
  static std::mutex mu;
  static std::vector<Done> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const Done& d : done)
    if (d.dev == dev && d.func == func && d.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  done.push_back(Done{dev, func, bytes});
  return cudaSuccess;
}

}  // namespace mxq

namespace {

thread_local char g_err[512] = "";

mxq_status fail(mxq_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
mxq_status fail(mxq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return s;
}

mxq_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return MXQ_OK;
  return fail(MXQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }
int elsize(int32_t dt) { return dt == MXQ_BF16 ? 2 : 4; }

mxq_status check_matrix(const void* X, int32_t dt, int64_t rows, int64_t cols, int64_t ld,
                        const char* name) {
  if (dt != MXQ_BF16 && dt != MXQ_F32) return fail(MXQ_ERR_DTYPE, "%s: dtype %d", name, dt);
  if (rows < 0 || cols < 0) return fail(MXQ_ERR_SHAPE, "%s: negative shape", name);
  if (ld < cols) return fail(MXQ_ERR_SHAPE, "%s: ld %lld < cols %lld", name, (long long)ld,
                             (long long)cols);
  if (rows == 0 || cols == 0) return MXQ_OK;
  if (!X) return fail(MXQ_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(X, 16)) return fail(MXQ_ERR_ALIGN, "%s not 16-byte aligned", name);
  if ((ld * elsize(dt)) % 16 != 0)
    return fail(MXQ_ERR_ALIGN, "%s: ld * element size not a multiple of 16 bytes", name);
  return MXQ_OK;
}

mxq_status check_params(const mxq_params* p, int64_t n, int64_t k) {
  if (!p) return fail(MXQ_ERR_INVALID_ARG, "params is NULL");
  if (p->mode < MXQ_NAIVE || p->mode > MXQ_HOPT) return fail(MXQ_ERR_INVALID_ARG, "mode %d", p->mode);
  if (p->ctas_per_sm < 0) return fail(MXQ_ERR_INVALID_ARG, "ctas_per_sm %d", p->ctas_per_sm);
  switch (p->fmt) {
    case MXQ_FMT_NVFP4:
    case MXQ_FMT_INT4:
      if (p->block != 16 && p->block != 32)
        return fail(MXQ_ERR_UNSUPPORTED, "%s block %d (16 or 32)",
                    p->fmt == MXQ_FMT_NVFP4 ? "NVFP4" : "INT4", p->block);
      if (p->tile_rows != 1) return fail(MXQ_ERR_UNSUPPORTED, "NVFP4 / INT4 tile_rows must be 1");
      if (!mxq::grid_known(p->scale_fmt))
        return fail(MXQ_ERR_INVALID_ARG, "scale_fmt %d", p->scale_fmt);
      if (p->fmt == MXQ_FMT_INT4 && p->scale_fmt == MXQ_SCALE_UE8M0)
        return fail(MXQ_ERR_UNSUPPORTED, "UE8M0 scales are for E2M1 elements (MXFP4)");
      break;
    case MXQ_FMT_INT8:
      if (p->block != 32 && p->block != 64 && p->block != 128 && p->block != 256)
        return fail(MXQ_ERR_UNSUPPORTED, "INT8 block %d (32, 64, 128 or 256)", p->block);
      if (p->tile_rows != 1) return fail(MXQ_ERR_UNSUPPORTED, "INT8 tile_rows must be 1");
      if (p->scale_fmt != MXQ_SCALE_E4M3)
        return fail(MXQ_ERR_UNSUPPORTED, "INT8 stores its amax as E4M3 (scale_fmt 0)");
      break;
    case MXQ_FMT_E4M3:
      if (p->block != 64 || p->tile_rows != 64)
        return fail(MXQ_ERR_UNSUPPORTED, "E4M3 tiles are 64 x 64");
      if (p->mode != MXQ_NAIVE) {
        if (p->log_points < 2 || p->log_points > 256)
          return fail(MXQ_ERR_INVALID_ARG, "log_points %d (2..256)", p->log_points);
        if (!std::isfinite(p->log_lo_exp2) || !std::isfinite(p->log_hi_exp2) ||
            !(p->log_lo_exp2 < p->log_hi_exp2) || std::fabs(p->log_lo_exp2) > 64 ||
            std::fabs(p->log_hi_exp2) > 64)
          return fail(MXQ_ERR_INVALID_ARG, "log grid exponents");
      }
      if (n % 64 != 0) return fail(MXQ_ERR_SHAPE, "n %% 64 != 0 for E4M3 tiles");
      if (p->scale_fmt != MXQ_SCALE_E4M3)
        return fail(MXQ_ERR_UNSUPPORTED, "E4M3 tiles have float scales (scale_fmt 0)");
      break;
    default:
      return fail(MXQ_ERR_INVALID_ARG, "fmt %d", p->fmt);
  }
  if (p->window < -1) return fail(MXQ_ERR_INVALID_ARG, "window %d", p->window);
  if (k % p->block != 0) return fail(MXQ_ERR_SHAPE, "k %% block != 0");
  return MXQ_OK;
}

}  // namespace

void mxq::set_error_text(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
}

extern "C" {

const char* mxq_status_string(mxq_status s) {
  switch (s) {
    case MXQ_OK: return "ok";
    case MXQ_ERR_INVALID_ARG: return "invalid argument";
    case MXQ_ERR_SHAPE: return "bad shape";
    case MXQ_ERR_DTYPE: return "unsupported dtype";
    case MXQ_ERR_ALIGN: return "misaligned pointer or leading dimension";
    case MXQ_ERR_UNSUPPORTED: return "unsupported combination";
    case MXQ_ERR_CUDA: return "CUDA error";
    case MXQ_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

const char* mxq_last_error(void) { return g_err; }

void mxq_set_wait_polls(uint32_t polls) { mxq::g_wait_polls.store(polls, std::memory_order_relaxed); }

size_t mxq_act_sqmean_workspace(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0) return 0;
  // the strip width only shapes the grid; the chunk count for bf16 is never smaller
  const int ch = std::max(mxq::hpass_chunks(rows, cols, MXQ_BF16), mxq::hpass_chunks(rows, cols, MXQ_F32));
  return (size_t)ch * (size_t)cols * sizeof(double);
}

static mxq_status act_common(const void* X, int32_t dtype, int64_t rows, int64_t cols,
                             int64_t ld, void* workspace, size_t ws, double** partial,
                             int* chunks) {
  mxq_status s = check_matrix(X, dtype, rows, cols, ld, "X");
  if (s != MXQ_OK) return s;
  const int vec = dtype == MXQ_BF16 ? 8 : 4;
  if (cols % vec != 0) return fail(MXQ_ERR_SHAPE, "cols %% %d != 0", vec);
  if (rows == 0 || cols == 0) return MXQ_OK;
  const size_t need = mxq_act_sqmean_workspace(rows, cols);
  if (!workspace || ws < need)
    return fail(MXQ_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws, need);
  if (!aligned(workspace, 8)) return fail(MXQ_ERR_ALIGN, "workspace not 8-byte aligned");
  *partial = (double*)workspace;
  *chunks = mxq::hpass_chunks(rows, cols, dtype);
  return MXQ_OK;
}

mxq_status mxq_act_sqmean(const void* X, int32_t dtype, int64_t rows, int64_t cols, int64_t ld,
                          float* h, void* workspace, size_t workspace_bytes, void* stream) {
  double* partial = nullptr;
  int chunks = 0;
  mxq_status s = act_common(X, dtype, rows, cols, ld, workspace, workspace_bytes, &partial,
                            &chunks);
  if (s != MXQ_OK) return s;
  if (cols == 0) return MXQ_OK;
  if (!h) return fail(MXQ_ERR_INVALID_ARG, "h is NULL");
  cudaStream_t st = (cudaStream_t)stream;
  if (rows == 0) return cuda_status(cudaMemsetAsync(h, 0, cols * sizeof(float), st), "memset h");
  s = cuda_status(mxq::launch_hpass_partial(X, dtype, rows, cols, ld, chunks, partial, st),
                  "h pass");
  if (s != MXQ_OK) return s;
  return cuda_status(mxq::launch_hpass_finalize(partial, chunks, cols, rows, nullptr, h, st),
                     "h finalize");
}

mxq_status mxq_act_sqsum(const void* X, int32_t dtype, int64_t rows, int64_t cols, int64_t ld,
                         double* colsum, void* workspace, size_t workspace_bytes, void* stream) {
  double* partial = nullptr;
  int chunks = 0;
  mxq_status s = act_common(X, dtype, rows, cols, ld, workspace, workspace_bytes, &partial,
                            &chunks);
  if (s != MXQ_OK) return s;
  if (cols == 0) return MXQ_OK;
  if (!colsum) return fail(MXQ_ERR_INVALID_ARG, "colsum is NULL");
  cudaStream_t st = (cudaStream_t)stream;
  if (rows == 0)
    return cuda_status(cudaMemsetAsync(colsum, 0, cols * sizeof(double), st), "memset colsum");
  s = cuda_status(mxq::launch_hpass_partial(X, dtype, rows, cols, ld, chunks, partial, st),
                  "h pass");
  if (s != MXQ_OK) return s;
  return cuda_status(mxq::launch_hpass_finalize(partial, chunks, cols, 0, colsum, nullptr, st),
                     "h partial combine");
}

mxq_status mxq_act_sqmean_finalize(const double* partials, int64_t parts, int64_t cols,
                                   int64_t total_rows, float* h, void* stream) {
  if (parts < 0 || cols < 0 || total_rows < 0) return fail(MXQ_ERR_SHAPE, "negative size");
  if (cols == 0) return MXQ_OK;
  if (!h || (parts > 0 && !partials)) return fail(MXQ_ERR_INVALID_ARG, "NULL pointer");
  if (partials && !aligned(partials, 8)) return fail(MXQ_ERR_ALIGN, "partials not 8-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  if (parts == 0 || total_rows == 0)
    return cuda_status(cudaMemsetAsync(h, 0, cols * sizeof(float), st), "memset h");
  return cuda_status(mxq::launch_hpass_finalize(partials, parts, cols, total_rows, nullptr, h, st),
                     "h finalize");
}

size_t mxq_act_block_gram_workspace(int64_t rows, int64_t cols, int32_t block) {
  if (rows <= 0 || cols <= 0 || (block != 16 && block != 32 && block != 64)) return 0;
  return mxq::gram_workspace(rows, cols, block);
}

mxq_status mxq_act_block_gram(const void* X, int32_t dtype, int64_t rows, int64_t cols,
                              int64_t ld, int32_t block, float* G, float* h, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (dtype != MXQ_BF16) return fail(MXQ_ERR_DTYPE, "block Gram needs bf16 X (dtype %d)", dtype);
  mxq_status s = check_matrix(X, dtype, rows, cols, ld, "X");
  if (s != MXQ_OK) return s;
  if (block != 16 && block != 32 && block != 64)
    return fail(MXQ_ERR_UNSUPPORTED, "block %d (16, 32 or 64)", block);
  if (cols % block != 0) return fail(MXQ_ERR_SHAPE, "cols %% block != 0");
  if (cols == 0) return MXQ_OK;
  if (!G) return fail(MXQ_ERR_INVALID_ARG, "G is NULL");
  if (!aligned(G, 16) || (h && !aligned(h, 4)))
    return fail(MXQ_ERR_ALIGN, "G not 16-byte or h not 4-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  if (rows == 0) {
    mxq_status z = cuda_status(cudaMemsetAsync(G, 0, (size_t)cols * block * sizeof(float), st),
                               "memset G");
    if (z != MXQ_OK || !h) return z;
    return cuda_status(cudaMemsetAsync(h, 0, (size_t)cols * sizeof(float), st), "memset h");
  }
  if (rows > 0x7fffffff - 64) return fail(MXQ_ERR_SHAPE, "rows beyond 2^31 - 64");
  const size_t need = mxq::gram_workspace(rows, cols, block);
  if (!workspace || workspace_bytes < need)
    return fail(MXQ_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
  if (!aligned(workspace, 16)) return fail(MXQ_ERR_ALIGN, "workspace not 16-byte aligned");
  return cuda_status(mxq::launch_gram(X, rows, cols, ld, block, G, h, workspace, st),
                     "block Gram");
}

// Validation shared by mxq_quantize and mxq_quantize_err; fills `a` for a non-empty
// problem (a->n == 0 when there is nothing to launch).
static mxq_status prepare_quantize(const void* W, int32_t dtype, int64_t n, int64_t k,
                                   int64_t ld, const float* h, const mxq_params* p, void* codes,
                                   void* scales, mxq::QuantArgs* a) {
  mxq_status s = check_matrix(W, dtype, n, k, ld, "W");
  if (s != MXQ_OK) return s;
  s = check_params(p, n, k);
  if (s != MXQ_OK) return s;
  a->n = 0;
  if (n == 0 || k == 0) return MXQ_OK;
  if (!codes || !scales) return fail(MXQ_ERR_INVALID_ARG, "codes or scales is NULL");
  if (!aligned(codes, 16)) return fail(MXQ_ERR_ALIGN, "codes not 16-byte aligned");
  if (p->fmt == MXQ_FMT_E4M3 && !aligned(scales, 4))
    return fail(MXQ_ERR_ALIGN, "scales not 4-byte aligned");
  if (p->mode == MXQ_HOPT) {
    if (!h) return fail(MXQ_ERR_INVALID_ARG, "H-optimal needs h");
    if (!aligned(h, 16)) return fail(MXQ_ERR_ALIGN, "h not 16-byte aligned");
  }
  a->W = W;
  a->dtype = dtype;
  a->n = n;
  a->k = k;
  a->ld = ld;
  a->h = p->mode == MXQ_HOPT ? h : nullptr;
  a->fmt = p->fmt;
  a->mode = p->mode;
  a->block = p->block;
  a->window = p->window;
  a->scale_fmt = p->scale_fmt;
  a->ctas_per_sm = p->ctas_per_sm;
  a->codes = codes;
  a->scales = scales;
  a->log_points = p->fmt == MXQ_FMT_E4M3 && p->mode != MXQ_NAIVE ? p->log_points : 0;
  for (int i = 0; i < a->log_points; ++i) {
    const double lo = p->log_lo_exp2, hi = p->log_hi_exp2;
    a->log_grid[i] = (float)std::exp2(lo + (hi - lo) * (double)i / (double)(a->log_points - 1));
  }
  return MXQ_OK;
}

mxq_status mxq_quantize(const void* W, int32_t dtype, int64_t n, int64_t k, int64_t ld,
                        const float* h, const mxq_params* p, void* codes, void* scales,
                        void* stream) {
  mxq::QuantArgs a{};
  mxq_status s = prepare_quantize(W, dtype, n, k, ld, h, p, codes, scales, &a);
  if (s != MXQ_OK || a.n == 0) return s;
  return cuda_status(mxq::launch_quantize(a, (cudaStream_t)stream), "quantize");
}

// The NVFP4 search with E4M3 scales adds the error sums itself; every other quantizer is
// followed by the error pass.
static bool fused_error(const mxq_params* p) {
  return p->fmt == MXQ_FMT_NVFP4 && p->scale_fmt == 0 && p->mode != MXQ_NAIVE;
}

size_t mxq_quantize_err_workspace(int64_t n, int64_t k, const mxq_params* p) {
  if (n <= 0 || k <= 0 || !p) return 0;
  const int64_t parts = fused_error(p) && (p->block == 16 || p->block == 32)
                            ? mxq::fp4_error_parts(n, k, p->block, p->ctas_per_sm)
                            : mxq::error_partials(n, k);
  return (size_t)parts * 4 * sizeof(double);
}

mxq_status mxq_quantize_err(const void* W, int32_t dtype, int64_t n, int64_t k, int64_t ld,
                            const float* h, const mxq_params* p, void* codes, void* scales,
                            double* sums, void* workspace, size_t workspace_bytes,
                            void* stream) {
  mxq::QuantArgs a{};
  mxq_status s = prepare_quantize(W, dtype, n, k, ld, h, p, codes, scales, &a);
  if (s != MXQ_OK) return s;
  if (!sums) return fail(MXQ_ERR_INVALID_ARG, "sums is NULL");
  if (!aligned(sums, 8)) return fail(MXQ_ERR_ALIGN, "sums not 8-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  if (a.n == 0) return cuda_status(cudaMemsetAsync(sums, 0, 4 * sizeof(double), st), "memset");
  if (h && !aligned(h, 16)) return fail(MXQ_ERR_ALIGN, "h not 16-byte aligned");
  const size_t need = mxq_quantize_err_workspace(n, k, p);
  if (!workspace || workspace_bytes < need)
    return fail(MXQ_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
  if (!aligned(workspace, 8)) return fail(MXQ_ERR_ALIGN, "workspace not 8-byte aligned");
  if (fused_error(p)) {
    a.err_partial = (double*)workspace;
    a.err_sums = sums;
    a.h_err = p->mode == MXQ_HOPT ? nullptr : h;
    return cuda_status(mxq::launch_quantize(a, st), "quantize with error sums");
  }
  cudaError_t e = mxq::launch_quantize(a, st);
  if (e != cudaSuccess) return cuda_status(e, "quantize");
  mxq::DecodeArgs d{codes, scales, p->fmt, p->block, p->scale_fmt, n, k};
  return cuda_status(mxq::launch_error(d, W, dtype, ld, h, (double*)workspace,
                                       mxq::error_partials(n, k), sums, st),
                     "error");
}

mxq_status mxq_quantize_gram(const void* W, int32_t dtype, int64_t n, int64_t k, int64_t ld,
                             const float* G, const mxq_params* p, void* codes, void* scales,
                             void* stream) {
  mxq_status s = check_matrix(W, dtype, n, k, ld, "W");
  if (s != MXQ_OK) return s;
  s = check_params(p, n, k);
  if (s != MXQ_OK) return s;
  if (p->fmt != MXQ_FMT_NVFP4 && p->fmt != MXQ_FMT_INT4)
    return fail(MXQ_ERR_UNSUPPORTED, "block-Hessian search: NVFP4 or INT4 elements");
  if (p->mode != MXQ_HOPT) return fail(MXQ_ERR_INVALID_ARG, "block-Hessian search: mode MXQ_HOPT");
  if (n == 0 || k == 0) return MXQ_OK;
  if (!codes || !scales || !G) return fail(MXQ_ERR_INVALID_ARG, "codes, scales or G is NULL");
  if (!aligned(codes, 16) || !aligned(G, 16))
    return fail(MXQ_ERR_ALIGN, "codes or G not 16-byte aligned");
  mxq::QuantArgs a{};
  a.W = W;
  a.dtype = dtype;
  a.n = n;
  a.k = k;
  a.ld = ld;
  a.G = G;
  a.fmt = p->fmt;
  a.mode = p->mode;
  a.block = p->block;
  a.window = p->window;
  a.scale_fmt = p->scale_fmt;
  a.codes = codes;
  a.scales = scales;
  return cuda_status(mxq::launch_quantize_gram(a, (cudaStream_t)stream), "quantize (block Hessian)");
}

mxq_status mxq_project(const float* w, int64_t count, int32_t fmt, int32_t scale_fmt,
                       float scale, uint8_t* q, void* stream) {
  if (count < 0) return fail(MXQ_ERR_SHAPE, "negative count");
  if (fmt < MXQ_FMT_NVFP4 || fmt > MXQ_FMT_INT4) return fail(MXQ_ERR_INVALID_ARG, "fmt %d", fmt);
  if (fmt != MXQ_FMT_E4M3 && !mxq::grid_known(scale_fmt))
    return fail(MXQ_ERR_INVALID_ARG, "scale_fmt %d", scale_fmt);
  if (fmt == MXQ_FMT_INT8 && scale_fmt != MXQ_SCALE_E4M3)
    return fail(MXQ_ERR_UNSUPPORTED, "INT8 stores its amax as E4M3 (scale_fmt 0)");
  if (count == 0) return MXQ_OK;
  if (!w || !q) return fail(MXQ_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(w, 4)) return fail(MXQ_ERR_ALIGN, "w not 4-byte aligned");
  if (!(scale > 0.0f) || !std::isfinite(scale))
    return fail(MXQ_ERR_INVALID_ARG, "scale must be positive and finite");
  if (fmt != MXQ_FMT_E4M3 && !mxq::grid_has_value(scale_fmt, scale))
    return fail(MXQ_ERR_INVALID_ARG, "scale is not a positive value of scale grid %d", scale_fmt);
  return cuda_status(mxq::launch_project(w, count, fmt, scale, q, (cudaStream_t)stream),
                     "project");
}

mxq_status mxq_dequant(const void* codes, const void* scales, const mxq_params* p, int64_t n,
                       int64_t k, float* out, void* stream) {
  if (n < 0 || k < 0) return fail(MXQ_ERR_SHAPE, "negative shape");
  mxq_status s = check_params(p, n, k);
  if (s != MXQ_OK) return s;
  if (n == 0 || k == 0) return MXQ_OK;
  if (!codes || !scales || !out) return fail(MXQ_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(codes, 16) || !aligned(out, 16) || !aligned(scales, 4))
    return fail(MXQ_ERR_ALIGN, "codes/out not 16-byte or scales not 4-byte aligned");
  mxq::DecodeArgs d{codes, scales, p->fmt, p->block, p->scale_fmt, n, k};
  return cuda_status(mxq::launch_dequant(d, out, (cudaStream_t)stream), "dequant");
}

size_t mxq_swizzled_scales_bytes(int64_t n, int64_t kb) {
  if (n <= 0 || kb <= 0) return 0;
  return mxq::swizzled_scales_bytes(n, kb);
}

mxq_status mxq_swizzle_scales(const uint8_t* scales, int64_t n, int64_t kb, uint8_t* out,
                              void* stream) {
  if (n < 0 || kb < 0) return fail(MXQ_ERR_SHAPE, "negative shape");
  if (n == 0 || kb == 0) return MXQ_OK;
  if (!scales || !out) return fail(MXQ_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(mxq::launch_swizzle_scales(scales, n, kb, out, (cudaStream_t)stream),
                     "swizzle scales");
}

size_t mxq_nvfp4_gemm_workspace(void) { return mxq::nvfp4_mm_workspace(); }

mxq_status mxq_nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales,
                          const uint8_t* b_codes, const uint8_t* b_scales, int64_t m, int64_t n,
                          int64_t k, float* D, void* workspace, size_t workspace_bytes,
                          void* stream) {
  if (m < 0 || n < 0 || k < 0) return fail(MXQ_ERR_SHAPE, "negative shape");
  if (m > 0x7fffffff || n > 0x7fffffff || k > 0x7fffffff)
    return fail(MXQ_ERR_SHAPE, "m, n and k must be below 2^31");
  if (k % 64 != 0) return fail(MXQ_ERR_SHAPE, "k %% 64 != 0");
  if (m == 0 || n == 0) return MXQ_OK;
  if (!D) return fail(MXQ_ERR_INVALID_ARG, "D is NULL");
  if (!aligned(D, 16)) return fail(MXQ_ERR_ALIGN, "D not 16-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  if (k == 0) return cuda_status(cudaMemsetAsync(D, 0, (size_t)m * n * sizeof(float), st), "memset D");
  if (!a_codes || !a_scales || !b_codes || !b_scales)
    return fail(MXQ_ERR_INVALID_ARG, "NULL operand");
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_scales, 16) ||
      !aligned(b_scales, 16))
    return fail(MXQ_ERR_ALIGN, "operands must be 16-byte aligned");
  if (!workspace || workspace_bytes < mxq::nvfp4_mm_workspace())
    return fail(MXQ_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes,
                mxq::nvfp4_mm_workspace());
  if (!aligned(workspace, 16)) return fail(MXQ_ERR_ALIGN, "workspace not 16-byte aligned");
  return cuda_status(mxq::launch_nvfp4_mm(a_codes, a_scales, b_codes, b_scales, m, n, k, D,
                                          workspace, st),
                     "NVFP4 product");
}

size_t mxq_error_workspace(int64_t n, int64_t k) {
  if (n <= 0 || k <= 0) return 0;
  return (size_t)mxq::error_partials(n, k) * 4 * sizeof(double);
}

mxq_status mxq_error(const void* W, int32_t dtype, int64_t n, int64_t k, int64_t ld,
                     const void* codes, const void* scales, const float* h,
                     const mxq_params* p, double* sums, void* workspace,
                     size_t workspace_bytes, void* stream) {
  mxq_status s = check_matrix(W, dtype, n, k, ld, "W");
  if (s != MXQ_OK) return s;
  s = check_params(p, n, k);
  if (s != MXQ_OK) return s;
  if (!sums) return fail(MXQ_ERR_INVALID_ARG, "sums is NULL");
  if (!aligned(sums, 8)) return fail(MXQ_ERR_ALIGN, "sums not 8-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  if (n == 0 || k == 0) return cuda_status(cudaMemsetAsync(sums, 0, 4 * sizeof(double), st), "memset");
  if (!codes || !scales) return fail(MXQ_ERR_INVALID_ARG, "codes or scales is NULL");
  if (!aligned(codes, 16) || !aligned(scales, 4))
    return fail(MXQ_ERR_ALIGN, "codes not 16-byte or scales not 4-byte aligned");
  if (h && !aligned(h, 16)) return fail(MXQ_ERR_ALIGN, "h not 16-byte aligned");
  const size_t need = mxq_error_workspace(n, k);
  if (!workspace || workspace_bytes < need)
    return fail(MXQ_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
  if (!aligned(workspace, 8)) return fail(MXQ_ERR_ALIGN, "workspace not 8-byte aligned");
  mxq::DecodeArgs d{codes, scales, p->fmt, p->block, p->scale_fmt, n, k};
  return cuda_status(mxq::launch_error(d, W, dtype, ld, h, (double*)workspace,
                                       mxq::error_partials(n, k), sums, st),
                     "error");
}

mxq_status mxq_gptq_prepare(const float* G, int64_t nblocks, double damp, float* U,
                            void* stream) {
  if (nblocks < 0) return fail(MXQ_ERR_SHAPE, "nblocks %lld", (long long)nblocks);
  if (!std::isfinite(damp) || damp < 0) return fail(MXQ_ERR_INVALID_ARG, "damp %g", damp);
  if (nblocks == 0) return MXQ_OK;
  if (nblocks > 0x7fffffff) return fail(MXQ_ERR_SHAPE, "nblocks beyond 2^31 - 1");
  if (!G || !U) return fail(MXQ_ERR_INVALID_ARG, "G or U is NULL");
  if (!aligned(G, 16) || !aligned(U, 16)) return fail(MXQ_ERR_ALIGN, "G or U not 16-byte aligned");
  return cuda_status(mxq::launch_gptq_prepare(G, nblocks, damp, U, (cudaStream_t)stream),
                     "GPTQ prepare");
}

mxq_status mxq_gptq_tiles(const void* W, int32_t dtype, int64_t n, int64_t k, int64_t ld,
                          const float* U, const float* scales, uint8_t* codes, void* stream) {
  mxq_status s = check_matrix(W, dtype, n, k, ld, "W");
  if (s != MXQ_OK) return s;
  if (n % 64 != 0 || k % 64 != 0) return fail(MXQ_ERR_SHAPE, "n and k must be multiples of 64");
  if (n == 0 || k == 0) return MXQ_OK;
  if (k / 64 > 65535) return fail(MXQ_ERR_SHAPE, "k beyond 64 * 65535");
  if (!U || !scales || !codes) return fail(MXQ_ERR_INVALID_ARG, "U, scales or codes is NULL");
  if (!aligned(U, 16) || !aligned(codes, 16) || !aligned(scales, 4))
    return fail(MXQ_ERR_ALIGN, "U or codes not 16-byte, or scales not 4-byte aligned");
  return cuda_status(mxq::launch_gptq_tiles(W, dtype, n, k, ld, U, scales, codes,
                                            (cudaStream_t)stream),
                     "GPTQ tiles");
}

size_t mxq_act_gram_workspace(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0) return 0;
  return mxq::gram_full_workspace(rows, cols);
}

mxq_status mxq_act_gram(const void* X, int32_t dtype, int64_t rows, int64_t cols, int64_t ld,
                        float* H, void* workspace, size_t workspace_bytes, void* stream) {
  if (dtype != MXQ_BF16) return fail(MXQ_ERR_DTYPE, "Gram matrix needs bf16 X (dtype %d)", dtype);
  mxq_status s = check_matrix(X, dtype, rows, cols, ld, "X");
  if (s != MXQ_OK) return s;
  if (cols == 0) return MXQ_OK;
  if (!H) return fail(MXQ_ERR_INVALID_ARG, "H is NULL");
  if (!aligned(H, 16)) return fail(MXQ_ERR_ALIGN, "H not 16-byte aligned");
  if (rows > 0x7fffffff || cols > 0x7fffffff || ld > 0x7fffffff)
    return fail(MXQ_ERR_SHAPE, "rows, cols and ld must be below 2^31");
  cudaStream_t st = (cudaStream_t)stream;
  if (rows == 0)
    return cuda_status(cudaMemsetAsync(H, 0, (size_t)cols * cols * sizeof(float), st), "memset H");
  const size_t need = mxq_act_gram_workspace(rows, cols);
  if (!workspace || workspace_bytes < need)
    return fail(MXQ_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
  if (!aligned(workspace, 16)) return fail(MXQ_ERR_ALIGN, "workspace not 16-byte aligned");
  const char* why = "";
  cudaError_t e = mxq::launch_gram_full(X, rows, cols, ld, H, workspace, st, &why);
  if (e == cudaErrorUnknown && why[0]) return fail(MXQ_ERR_CUDA, "Gram matrix: %s", why);
  return cuda_status(e, "Gram matrix");
}

size_t mxq_gptq_factor_workspace(int64_t k) {
  return k > 0 ? mxq::gptq_factor_workspace(k) : 0;
}

mxq_status mxq_gptq_factor(const float* H, int64_t k, int32_t block, const int32_t* perm,
                           double damp, float* U, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (k < 0) return fail(MXQ_ERR_SHAPE, "k %lld", (long long)k);
  if (block != 16 && block != 32) return fail(MXQ_ERR_UNSUPPORTED, "block %d (16 or 32)", block);
  if (k % block != 0) return fail(MXQ_ERR_SHAPE, "k %% block != 0");
  if (!std::isfinite(damp) || damp < 0) return fail(MXQ_ERR_INVALID_ARG, "damp %g", damp);
  if (k == 0) return MXQ_OK;
  if (k > 65536) return fail(MXQ_ERR_SHAPE, "k beyond 65536");
  if (!H || !U) return fail(MXQ_ERR_INVALID_ARG, "H or U is NULL");
  if (!aligned(H, 16) || !aligned(U, 16) || (perm && !aligned(perm, 4)))
    return fail(MXQ_ERR_ALIGN, "H or U not 16-byte, or perm not 4-byte aligned");
  const size_t need = mxq::gptq_factor_workspace(k);
  if (!workspace || workspace_bytes < need)
    return fail(MXQ_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
  if (!aligned(workspace, 16)) return fail(MXQ_ERR_ALIGN, "workspace not 16-byte aligned");
  return cuda_status(mxq::launch_gptq_factor(H, k, block, perm, damp, U, workspace,
                                             (cudaStream_t)stream),
                     "GPTQ factor");
}

namespace {
size_t round256(size_t x) { return (x + 255) / 256 * 256; }

mxq_status check_gptq_params(const mxq_params* p, int64_t n, int64_t k) {
  mxq_status s = check_params(p, n, k);
  if (s != MXQ_OK) return s;
  if (p->fmt != MXQ_FMT_NVFP4 && p->fmt != MXQ_FMT_INT4)
    return fail(MXQ_ERR_UNSUPPORTED, "GPTQ: NVFP4 or INT4 elements (E4M3 tiles: mxq_gptq_tiles)");
  return MXQ_OK;
}
}  // namespace

size_t mxq_gptq_order_workspace(int64_t n, int64_t k, const mxq_params* p) {
  if (n <= 0 || k <= 0 || !p || p->block <= 0) return 0;
  return round256((size_t)n * (size_t)(k / 2)) + round256((size_t)n * (size_t)(k / p->block)) +
         round256((size_t)(k / p->block) * sizeof(double));
}

mxq_status mxq_gptq_order(const void* W, int32_t dtype, int64_t n, int64_t k, int64_t ld,
                          const float* h, const mxq_params* p, int32_t* perm, void* workspace,
                          size_t workspace_bytes, void* stream) {
  mxq_status s = check_matrix(W, dtype, n, k, ld, "W");
  if (s != MXQ_OK) return s;
  s = check_gptq_params(p, n, k);
  if (s != MXQ_OK) return s;
  if (k == 0) return MXQ_OK;
  if (k / p->block > mxq::gptq_sort_max())
    return fail(MXQ_ERR_SHAPE, "more than %d blocks per row", mxq::gptq_sort_max());
  if (!h || !perm) return fail(MXQ_ERR_INVALID_ARG, "h or perm is NULL");
  if (!aligned(h, 16) || !aligned(perm, 4))
    return fail(MXQ_ERR_ALIGN, "h not 16-byte or perm not 4-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  if (n == 0) {
    std::vector<int32_t> id((size_t)(k / p->block));
    for (size_t i = 0; i < id.size(); ++i) id[i] = (int32_t)i;
    return cuda_status(cudaMemcpyAsync(perm, id.data(), id.size() * sizeof(int32_t),
                                       cudaMemcpyHostToDevice, st),
                       "perm copy");
  }
  const size_t need = mxq_gptq_order_workspace(n, k, p);
  if (!workspace || workspace_bytes < need)
    return fail(MXQ_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
  if (!aligned(workspace, 16)) return fail(MXQ_ERR_ALIGN, "workspace not 16-byte aligned");
  char* ws = (char*)workspace;
  uint8_t* codes = (uint8_t*)ws;
  uint8_t* scales = codes + round256((size_t)n * (size_t)(k / 2));
  double* loss = (double*)(scales + round256((size_t)n * (size_t)(k / p->block)));
  s = mxq_quantize(W, dtype, n, k, ld, h, p, codes, scales, stream);
  if (s != MXQ_OK) return s;
  mxq::GptqArgs g{};
  g.W = W;
  g.dtype = dtype;
  g.n = n;
  g.k = k;
  g.ld = ld;
  g.h = h;
  g.fmt = p->fmt;
  g.block = p->block;
  g.scale_fmt = p->scale_fmt;
  return cuda_status(mxq::launch_gptq_order(g, codes, scales, loss, perm, st), "GPTQ order");
}

size_t mxq_gptq_workspace(int64_t n, int64_t k) {
  return n > 0 && k > 0 ? mxq::gptq_sweep_workspace(n, k) : 0;
}

mxq_status mxq_gptq(const void* W, int32_t dtype, int64_t n, int64_t k, int64_t ld,
                    const float* h, const float* U, const int32_t* perm, const mxq_params* p,
                    void* codes, void* scales, void* workspace, size_t workspace_bytes,
                    void* stream) {
  mxq_status s = check_matrix(W, dtype, n, k, ld, "W");
  if (s != MXQ_OK) return s;
  s = check_gptq_params(p, n, k);
  if (s != MXQ_OK) return s;
  if (n == 0 || k == 0) return MXQ_OK;
  if (n > (int64_t)65535 * 64) return fail(MXQ_ERR_SHAPE, "n beyond 65535 x 64 rows");
  if (!U || !codes || !scales) return fail(MXQ_ERR_INVALID_ARG, "U, codes or scales is NULL");
  if (!aligned(U, 16) || !aligned(codes, 16) || (perm && !aligned(perm, 4)))
    return fail(MXQ_ERR_ALIGN, "U or codes not 16-byte, or perm not 4-byte aligned");
  if (p->mode == MXQ_HOPT) {
    if (!h) return fail(MXQ_ERR_INVALID_ARG, "H-optimal needs h");
    if (!aligned(h, 16)) return fail(MXQ_ERR_ALIGN, "h not 16-byte aligned");
  }
  const size_t need = mxq::gptq_sweep_workspace(n, k);
  if (!workspace || workspace_bytes < need)
    return fail(MXQ_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
  if (!aligned(workspace, 16)) return fail(MXQ_ERR_ALIGN, "workspace not 16-byte aligned");
  mxq::GptqArgs g{};
  g.W = W;
  g.dtype = dtype;
  g.n = n;
  g.k = k;
  g.ld = ld;
  g.h = p->mode == MXQ_HOPT ? h : nullptr;
  g.U = U;
  g.perm = perm;
  g.fmt = p->fmt;
  g.mode = p->mode;
  g.block = p->block;
  g.window = p->window;
  g.scale_fmt = p->scale_fmt;
  g.codes = codes;
  g.scales = scales;
  g.workspace = workspace;
  return cuda_status(mxq::launch_gptq_sweep(g, (cudaStream_t)stream), "GPTQ sweep");
}

size_t mxq_output_error_workspace(int64_t m, int64_t n) {
  if (m <= 0 || n <= 0) return 0;
  return mxq::outerr_workspace(m, n);
}

mxq_status mxq_output_error(const void* X, int64_t m, int64_t k, int64_t ldx, const void* W,
                            int64_t n, int64_t ldw, const void* codes, const void* scales,
                            const mxq_params* p, double* sums, void* workspace,
                            size_t workspace_bytes, void* stream) {
  mxq_status s = check_matrix(X, MXQ_BF16, m, k, ldx, "X");
  if (s != MXQ_OK) return s;
  s = check_matrix(W, MXQ_BF16, n, k, ldw, "W");
  if (s != MXQ_OK) return s;
  s = check_params(p, n, k);
  if (s != MXQ_OK) return s;
  if (p->fmt != MXQ_FMT_NVFP4 && p->fmt != MXQ_FMT_INT4)
    return fail(MXQ_ERR_UNSUPPORTED, "output error: NVFP4 or INT4 codes");
  if (!sums) return fail(MXQ_ERR_INVALID_ARG, "sums is NULL");
  if (!aligned(sums, 8)) return fail(MXQ_ERR_ALIGN, "sums not 8-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  if (m == 0 || n == 0 || k == 0)
    return cuda_status(cudaMemsetAsync(sums, 0, 2 * sizeof(double), st), "memset");
  if (!codes || !scales) return fail(MXQ_ERR_INVALID_ARG, "codes or scales is NULL");
  if (!aligned(codes, 8)) return fail(MXQ_ERR_ALIGN, "codes not 8-byte aligned");
  if (m > 0x7fffff00 || n > 0x7fffff00) return fail(MXQ_ERR_SHAPE, "rows beyond 2^31");
  const size_t need = mxq::outerr_workspace(m, n);
  if (!workspace || workspace_bytes < need)
    return fail(MXQ_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
  if (!aligned(workspace, 16)) return fail(MXQ_ERR_ALIGN, "workspace not 16-byte aligned");
  return cuda_status(mxq::launch_outerr(X, m, k, ldx, W, n, ldw, (const uint8_t*)codes,
                                        (const uint8_t*)scales, p->fmt, p->scale_fmt, p->block,
                                        sums, workspace, st),
                     "output error");
}

mxq_status mxq_metrics_from_sums(const double* s, mxq_metrics* out) {
  if (!s || !out) return fail(MXQ_ERR_INVALID_ARG, "NULL pointer");
  out->sse = s[0];
  out->w_sq = s[1];
  out->hsse = s[2];
  out->hw_sq = s[3];
  out->weight_rel = s[1] > 0 ? std::sqrt(s[0] / s[1]) : 0.0;
  out->h_rel = s[3] > 0 ? std::sqrt(s[2] / s[3]) : 0.0;
  return MXQ_OK;
}

}  // extern "C"
