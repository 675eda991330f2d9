// mxq_nvfp4_mm.cu -- D = A^ B^T for two operands in the library's own NVFP4 output format, on
// the block-scaled tensor cores. An NVFP4 block is 16 E2M1 values and one E4M3 scale, and
// x^ = s q ("Is Finer Better? The Limits of Microscaling Formats in LLMs", sec. 2.1); here the
// hardware applies the scales: tcgen05.mma kind::mxf4nvf4 with scale_vec::4X multiplies
// packed E2M1 operands (element 2i in the low nibble, as mxq_quantize packs them) and
// scales each 16-element slice of a row by its UE4M3 scale byte, read from tensor memory.
//
// The scale bytes come in the 128 x 4 tile layout that mxq_swizzle_scales writes: for a tile
// of 128 rows and 4 consecutive scales (64 elements of K), row m and scale c at byte
// (m % 32) * 16 + (m / 32) * 4 + c of a 512-byte tile, tiles ordered by row tile, then K.
// One tile is exactly what one MMA of K = 64 consumes for 128 rows; tcgen05.cp copies it from
// shared memory into four tensor-memory columns (32x128b, replicated over the four lane
// quarters), where the MMA reads it.
//
// One CTA per 128 x 128 tile of D. Per stage (256 elements of K): a TMA warp loads 128 rows
// x 128 bytes of each operand's codes (128-byte swizzle) and the four scale tiles of each
// (two 2 KB bulk copies); one thread copies the scale tiles into tensor memory and issues
// four MMAs (K = 64 each, M = N = 128) into a float32 accumulator; the epilogue warps read
// the accumulator (tcgen05.ld) and store D. Every wait is bounded; a timeout sets the error
// word and the call's D is overwritten with NaN.
#include "mxq_common.cuh"
#include "mxq_internal.h"
#include "mxq_tc.cuh"

namespace mxq {
namespace {

constexpr int kMmM = 128, kMmN = 128;
constexpr int kMmKStage = 256;                    // elements of K per stage (128 bytes a row)
constexpr int kMmStages = 4;
constexpr int kMmCodes = 128 * 128;               // 16 KB: 128 rows x 128 bytes
constexpr int kMmSf = 4 * 512;                    // four 512-byte scale tiles
constexpr int kMmStage = 2 * kMmCodes + 2 * kMmSf;  // 36 KB
constexpr int kMmBarOff = kMmStages * kMmStage;
constexpr int kMmSmem = kMmBarOff + 256 + 1024;
constexpr int kMmThreads = 192;
constexpr uint32_t kMmIdesc = tc::idesc_nvf4(kMmM, kMmN);
// tensor memory: the accumulator (128 columns), then per stage 16 columns of A scales and
// 16 of B scales
constexpr uint32_t kMmTmemCols = 256;
constexpr uint32_t kMmSfCol = 128;

static_assert(kMmSmem <= 227 * 1024, "shared memory per CTA");

struct MmParams {
  int64_t m, n, k;
  const uint8_t* sfa;       // swizzled scales of A
  const uint8_t* sfb;
  int64_t sf_tiles_k;       // scale tiles per row tile: ceil(k / 64)
  float* D;
  int* err;
  uint32_t polls;
};

__global__ void __launch_bounds__(kMmThreads, 1)
k_nvfp4_mm(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
           MmParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + kMmBarOff);
  uint64_t* empty = full + kMmStages;
  uint64_t* accfull = empty + kMmStages;
  uint32_t* tmem_slot = (uint32_t*)(accfull + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t mt = blockIdx.y, nt = blockIdx.x;
  const int nchunks = (int)((P.k + kMmKStage - 1) / kMmKStage);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMmStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(accfull, 1);
    *abort_flag = 0;
    tc::mbar_init_fence();
  }
  if (warp == 5) {
    tc::tmem_alloc(tmem_slot, kMmTmemCols);
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(P.err, 1);
  };

  if (warp == 4) {
    // ---- TMA producer ----------------------------------------------------------------
    if (lane == 0) {
      int issued[kMmStages];
#pragma unroll
      for (int s = 0; s < kMmStages; ++s) issued[s] = 0;
      for (int c = 0; c < nchunks; ++c) {
        const int s = c % kMmStages;
        if (!tc::mbar_wait(&empty[s], ((uint32_t)(c / kMmStages) & 1u) ^ 1u, abort_flag,
                           P.polls)) {
          fail();
          break;
        }
        // scale tiles of this chunk that exist (a tile = 64 elements of K)
        const int64_t t0 = (int64_t)c * 4;
        const int ntile = (int)(P.sf_tiles_k - t0 < 4 ? P.sf_tiles_k - t0 : 4);
        const uint32_t sf_bytes = (uint32_t)ntile * 512u;
        tc::mbar_expect_tx(&full[s], 2u * kMmCodes + 2u * sf_bytes);
        uint8_t* st = smem + s * kMmStage;
        tc::tma_load_2d(st, &amap, c * 128, (int)(mt * kMmM), &full[s]);
        tc::tma_load_2d(st + kMmCodes, &bmap, c * 128, (int)(nt * kMmN), &full[s]);
        tc::bulk_load(st + 2 * kMmCodes, P.sfa + (mt * P.sf_tiles_k + t0) * 512, sf_bytes,
                      &full[s]);
        tc::bulk_load(st + 2 * kMmCodes + kMmSf, P.sfb + (nt * P.sf_tiles_k + t0) * 512,
                      sf_bytes, &full[s]);
        ++issued[s];
      }
      // every copy this thread started has landed before the CTA can exit
#pragma unroll
      for (int s = 0; s < kMmStages; ++s)
        if (issued[s] > 0)
          for (uint32_t i = 0; i < tc::kDefaultPolls &&
                               !tc::mbar_try_wait(&full[s], (uint32_t)(issued[s] - 1) & 1u);
               ++i) {
          }
    }
  } else if (warp == 5) {
    // ---- scale copies and MMAs ---------------------------------------------------------
    if (lane == 0) {
      bool ok = true;
      for (int c = 0; c < nchunks && ok; ++c) {
        const int s = c % kMmStages;
        if (!tc::mbar_wait(&full[s], (uint32_t)(c / kMmStages) & 1u, abort_flag, P.polls)) {
          fail();
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t base = tc::smem_u32(smem + s * kMmStage);
        const int64_t t0 = (int64_t)c * 4;
        const int nsteps = (int)(P.sf_tiles_k - t0 < 4 ? P.sf_tiles_k - t0 : 4);
        const uint32_t sfa_col = tmem + kMmSfCol + (uint32_t)s * 32u;
        const uint32_t sfb_col = sfa_col + 16u;
        for (int j = 0; j < nsteps; ++j) {
          tc::tmem_cp_32x128b_x4(sfa_col + 4u * j, tc::desc_rows16(base + 2 * kMmCodes + 512 * j));
          tc::tmem_cp_32x128b_x4(sfb_col + 4u * j,
                                 tc::desc_rows16(base + 2 * kMmCodes + kMmSf + 512 * j));
        }
        for (int j = 0; j < nsteps; ++j) {
          const uint64_t a = tc::desc_k_sw128(base + 32u * j);          // 64 E2M1 = 32 bytes
          const uint64_t b = tc::desc_k_sw128(base + kMmCodes + 32u * j);
          tc::mma_nvf4(tmem, a, b, kMmIdesc, sfa_col + 4u * j, sfb_col + 4u * j,
                       (c | j) != 0 ? 1u : 0u);
        }
        tc::commit_local(&empty[s]);
      }
      tc::commit_local(accfull);
      // the accumulator hand-off doubles as the drain: every MMA and copy has completed
      for (uint32_t i = 0; i < tc::kDefaultPolls && !tc::mbar_try_wait(accfull, 0); ++i) {
      }
    }
  } else {
    // ---- epilogue ------------------------------------------------------------------------
    const bool ok = tc::mbar_wait(accfull, 0, abort_flag, P.polls);
    if (!__all_sync(kFull, ok)) {
      if (lane == 0) fail();
    } else {
      tc::fence_after_sync();
      const int64_t row = mt * kMmM + warp * 32 + lane;
      const uint32_t lanes = (uint32_t)(warp * 32) << 16;
#pragma unroll 1
      for (int c = 0; c < kMmN / 32; ++c) {
        float v[32];
        tc::tmem_ld32(tmem + lanes + (uint32_t)(c * 32), v);
        const int64_t col = nt * kMmN + c * 32;
        if (row < P.m)
          for (int q = 0; q < 32 && col + q < P.n; ++q) P.D[row * P.n + col + q] = v[q];
      }
    }
  }
  __syncthreads();
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kMmTmemCols);
  }
}

// After a timed-out launch (*err set) every entry of D becomes NaN.
__global__ void k_nvfp4_mm_check(const int* err, float* D, int64_t total) {
  if (!*err) return;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x)
    D[i] = __int_as_float(0x7fc00000);
}

}  // namespace

size_t nvfp4_mm_workspace() { return 256; }

cudaError_t launch_nvfp4_mm(const uint8_t* a_codes, const uint8_t* a_sf, const uint8_t* b_codes,
                            const uint8_t* b_sf, int64_t m, int64_t n, int64_t k, float* D,
                            void* workspace, cudaStream_t st) {
  CUtensorMap amap, bmap;
  if (!encode_2d(&amap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a_codes, m, k / 2, k / 2, 128, 128) ||
      !encode_2d(&bmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, b_codes, n, k / 2, k / 2, 128, 128))
    return cudaErrorInvalidValue;
  int* err = (int*)workspace;
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  e = ensure_dynamic_smem((const void*)k_nvfp4_mm, kMmSmem);
  if (e != cudaSuccess) return e;
  MmParams P{m, n, k, a_sf, b_sf, (k + 63) / 64, D, err, wait_polls()};
  const dim3 grid((unsigned)((n + kMmN - 1) / kMmN), (unsigned)((m + kMmM - 1) / kMmM));
  k_nvfp4_mm<<<grid, kMmThreads, kMmSmem, st>>>(amap, bmap, P);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_nvfp4_mm_check<<<64, 256, 0, st>>>(err, D, m * n);
  return cudaGetLastError();
}

}  // namespace mxq
