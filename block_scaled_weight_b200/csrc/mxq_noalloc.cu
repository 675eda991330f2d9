// mxq_noalloc.cu -- mxq_act_sqmean_noalloc: the h pass without any caller-provided or
// library-allocated workspace.
//
// Why it exists: mxq_act_sqmean needs a device workspace for its per-chunk column sums,
// which the caller must allocate. Some callers cannot: code that runs inside a host
// application whose device memory is entirely owned by another allocator or a fixed
// arena (so a cudaMalloc would bypass its accounting or fail), and latency-critical
// services that must not allocate after start-up because cudaMalloc can synchronise the
// device. This variant keeps the scratch in a file-scope static device array instead.
//
// The array is 1 MiB and lives in every GPU's memory from the moment the library is
// loaded on that GPU until the process exits. 1 MiB covers every activation width up to
// 131072 columns, for any number of rows; wider inputs are rejected (MXQ_ERR_SHAPE).
//
// Sharing: every call on a device uses the same array. Calls whose work overlaps on the
// GPU (two streams, or two host threads without ordering between them) race on it; order
// them, for example by issuing them on one stream. Nothing in the array needs clearing:
// each call writes every scratch entry it later reads.
//
// Set-up: the first call on each device, with that device current, looks the array's
// device address up (cudaGetSymbolAddress) and caches it; make that first call before any
// stream capture begins. The cache lives as long as the process and does not survive a
// cudaDeviceReset (which unloads the module and may move the array): a caller that resets
// a device must not call this entry point on it afterwards.
#include "../../include/mxq.h"
#include "mxq_internal.h"

#include <cmath>
#include <cstdio>
#include <mutex>

namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;
// The h pass needs at most max(kHpassTargetCtas x 256, cols) doubles of scratch (strips x
// row chunks never exceeds one wave of kHpassTargetCtas CTAs; a strip is at most 256
// columns wide): within 1 MiB for every width up to 131072 columns, whatever the rows.
static_assert(size_t(mxq::kHpassTargetCtas) * 256 * sizeof(double) <= kScratchBytes,
              "a one-wave h pass grid must fit the static scratch");
static_assert(size_t(131072) * sizeof(double) <= kScratchBytes,
              "the documented width limit must fit the static scratch");
__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device (host code cannot use the symbol
// itself: on the host it is only a stand-in, not a device address).
mxq_status scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    mxq::set_error_text("cudaGetDevice: %s", cudaGetErrorString(e));
    return MXQ_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    mxq::set_error_text("device ordinal %d beyond %d", dev, kMaxDevices);
    return MXQ_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) {
      mxq::set_error_text("cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      return MXQ_ERR_CUDA;
    }
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return MXQ_OK;
}

}  // namespace

extern "C" mxq_status mxq_act_sqmean_noalloc(const void* X, int32_t dtype, int64_t rows,
                                             int64_t cols, int64_t ld, float* h,
                                             void* stream) {
  if (dtype != MXQ_BF16 && dtype != MXQ_F32) {
    mxq::set_error_text("X: dtype %d", dtype);
    return MXQ_ERR_DTYPE;
  }
  if (rows < 0 || cols < 0 || ld < cols) {
    mxq::set_error_text("X: bad shape (rows %lld, cols %lld, ld %lld)", (long long)rows,
                        (long long)cols, (long long)ld);
    return MXQ_ERR_SHAPE;
  }
  const int vec = dtype == MXQ_BF16 ? 8 : 4;
  const int esz = dtype == MXQ_BF16 ? 2 : 4;
  if (cols % vec != 0) {
    mxq::set_error_text("cols %% %d != 0", vec);
    return MXQ_ERR_SHAPE;
  }
  if (cols == 0) return MXQ_OK;
  if (!h) {
    mxq::set_error_text("h is NULL");
    return MXQ_ERR_INVALID_ARG;
  }
  cudaStream_t st = (cudaStream_t)stream;
  if (rows == 0) {
    cudaError_t e = cudaMemsetAsync(h, 0, cols * sizeof(float), st);
    if (e != cudaSuccess) {
      mxq::set_error_text("memset h: %s", cudaGetErrorString(e));
      return MXQ_ERR_CUDA;
    }
    return MXQ_OK;
  }
  if (!X) {
    mxq::set_error_text("X is NULL");
    return MXQ_ERR_INVALID_ARG;
  }
  if ((uintptr_t)X % 16 != 0 || (ld * esz) % 16 != 0) {
    mxq::set_error_text("X not 16-byte aligned or ld * element size not a multiple of 16");
    return MXQ_ERR_ALIGN;
  }
  const size_t need = mxq_act_sqmean_workspace(rows, cols);
  if (need > kScratchBytes) {
    mxq::set_error_text("cols %lld needs %zu bytes of scratch; the static scratch holds %zu "
                        "(up to 131072 columns)", (long long)cols, need, kScratchBytes);
    return MXQ_ERR_SHAPE;
  }
  void* scratch = nullptr;
  mxq_status s = scratch_on_current_device(&scratch);
  if (s != MXQ_OK) return s;
  const int chunks = mxq::hpass_chunks(rows, cols, dtype);
  cudaError_t e = mxq::launch_hpass_partial(X, dtype, rows, cols, ld, chunks, (double*)scratch,
                                            st);
  if (e == cudaSuccess)
    e = mxq::launch_hpass_finalize((const double*)scratch, chunks, cols, rows, nullptr, h, st);
  if (e != cudaSuccess) {
    mxq::set_error_text("h pass: %s", cudaGetErrorString(e));
    return MXQ_ERR_CUDA;
  }
  return MXQ_OK;
}
