// mxq_outerr.cu -- the output error of a quantized weight on the tensor cores:
// ||X Wq^T - X W^T||_F^2 and ||X W^T||_F^2 (qwantize "Results": output error
// ||X_s Wq^T - X_s W^T||_F / ||X_s W^T||_F on sampled calibration rows X_s).
//
// A CTA computes a 128 x 64 tile of both products, Y = X W^T and Yq = X Wq^T, over the
// whole K: per 64-column stage a TMA producer warp loads the X tile (128 x 64 bf16) and the
// W tile (64 x 64 bf16), four dequant warps expand the same 64 x 64 slice of the packed
// 4-bit codes and their scales to bf16 (exact: an element value times a scale has at most
// 8 significant bits) straight into the 128-byte-swizzled K-major layout the MMA reads, and
// one thread of the MMA warp issues tcgen05.mma kind::f16 (M = 128, N = 64, K = 16) into two
// tensor-memory accumulators. The epilogue warps read both accumulators (tcgen05.ld),
// square and sum in double; a one-CTA pass adds the per-CTA partials in a fixed order.
// Every wait is bounded (on timeout the CTA sets the error word and the sums become NaN).
#include "mxq_common.cuh"
#include "mxq_grids.h"
#include "mxq_internal.h"

#include <cuda.h>
#include <cuda_fp16.h>

#include <cstring>

namespace mxq {
namespace {

constexpr int kOeM = 128, kOeN = 64, kOeK = 64;      // CTA tile and K per stage
constexpr int kOeStages = 3;
constexpr int kOeXBytes = kOeM * kOeK * 2;           // 16 KB
constexpr int kOeWBytes = kOeN * kOeK * 2;           // 8 KB
constexpr int kOeStageBytes = kOeXBytes + 2 * kOeWBytes;
constexpr int kOeThreads = 192;
constexpr uint32_t kOeSpin = 1u << 26;

__device__ __forceinline__ uint32_t s_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void bar_init(uint64_t* b, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(s_u32(b)), "r"(n));
}
__device__ __forceinline__ void bar_expect(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(s_u32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(s_u32(b)) : "memory");
}
__device__ __forceinline__ bool bar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(s_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool bar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag,
                                         uint32_t polls) {
  for (uint32_t it = 0; it < polls; ++it) {
    if (bar_try(b, parity)) return true;
    if ((it & 1023u) == 1023u && *abort_flag) return false;
  }
  return false;
}

// K-major operand, 128-byte swizzle: rows of 64 bf16 (128 B), 8-row groups 1 KB apart
// (stride byte offset); the leading byte offset is unused for swizzled K-major layouts.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)((1024u >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// kind::f16, D float32, A and B bf16, both K-major, N = 64, M = 128.
constexpr uint32_t kOeIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kOeN >> 3) << 17) |
                              ((uint32_t)(kOeM >> 4) << 24);

__device__ __forceinline__ void umma(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(kOeIdesc), "r"(acc));
}
__device__ __forceinline__ void umma_commit(uint64_t* b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   s_u32(b))
               : "memory");
}
__device__ __forceinline__ void tma2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* b) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(s_u32(dst)),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(s_u32(b))
      : "memory");
}
__device__ __forceinline__ void tld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

struct OeParams {
  int64_t m, n, k;
  const uint8_t* codes;    // [n][k/2] nibbles
  const uint8_t* scales;   // [n][k/B]
  int block;
  int int4;                // 0: E2M1 nibbles, 1: two's-complement INT4 nibbles
  double* partial;         // [ctas][2]
  int* err;
  uint32_t polls;          // bound of every pipeline wait (the drains keep kOeSpin)
};

struct OeScaleTab {
  float v[256];
};

}  // namespace
}  // namespace mxq

namespace mxq {
namespace {

constexpr int kOeBar = kOeStages * kOeStageBytes;
// barriers (256 B), scale table (1 KB), reduction scratch (256 B), 1 KB alignment slack
constexpr int kOeUsed = kOeBar + 256 + 1024 + 256;
constexpr int kOeSmem = kOeUsed + 1024;

// Two bf16 values (element values times the block scale; exact) packed into a word.
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const uint32_t ua = __float_as_uint(a) >> 16, ub = __float_as_uint(b) >> 16;
  return ua | (ub << 16);
}

__global__ void __launch_bounds__(kOeThreads, 1)
k_outerr_tc(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap,
            OeParams P, OeScaleTab ST) {
  extern __shared__ uint8_t oe_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)oe_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + kOeBar);
  uint64_t* qfull = full + kOeStages;
  uint64_t* empty = qfull + kOeStages;
  uint64_t* accfull = empty + kOeStages;
  uint64_t* done = accfull + 1;
  uint32_t* tmem_slot = (uint32_t*)(done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  float* stab = (float*)(smem + kOeBar + 256);
  double* red = (double*)(smem + kOeBar + 256 + 1024);   // [4 warps][2]

  if ((size_t)(smem - oe_raw) + kOeUsed > (size_t)kOeSmem) {   // never: slack covers alignment
    if (threadIdx.x == 0) atomicExch(P.err, 1);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.x * kOeM, n0 = (int64_t)blockIdx.y * kOeN;
  const int nk = (int)((P.k + kOeK - 1) / kOeK);
  for (int i = threadIdx.x; i < 256; i += kOeThreads) stab[i] = ST.v[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < kOeStages; ++s) {
      bar_init(&full[s], 1);
      bar_init(&qfull[s], 128);
      bar_init(&empty[s], 1);
    }
    bar_init(accfull, 1);
    bar_init(done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;" ::"r"(
        s_u32(tmem_slot)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  }
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(P.err, 1);
  };

  if (warp == 0) {
    // ---- TMA producer: X tile (128 x 64) and W tile (64 x 64) per stage ---------------
    if (lane == 0) {
      int issued[kOeStages];
#pragma unroll
      for (int s = 0; s < kOeStages; ++s) issued[s] = 0;
      for (int it = 0; it < nk; ++it) {
        const int s = it % kOeStages;
        if (!bar_wait(&empty[s], ((uint32_t)(it / kOeStages) & 1u) ^ 1u, abort_flag, P.polls)) { fail(); break; }
        bar_expect(&full[s], kOeXBytes + kOeWBytes);
        uint8_t* st = smem + s * kOeStageBytes;
        tma2d(st, &xmap, it * kOeK, (int)m0, &full[s]);
        tma2d(st + kOeXBytes, &wmap, it * kOeK, (int)n0, &full[s]);
        ++issued[s];
      }
#pragma unroll
      for (int s = 0; s < kOeStages; ++s)
        if (issued[s] > 0)
          for (uint32_t i = 0; i < kOeSpin && !bar_try(&full[s], (uint32_t)(issued[s] - 1) & 1u); ++i) {
          }
    }
  } else if (warp == 5) {
    // ---- MMA issuer ----------------------------------------------------------------------
    if (lane == 0) {
      const uint32_t d_ref = tmem, d_q = tmem + kOeN;
      bool ok = true;
      for (int it = 0; it < nk && ok; ++it) {
        const int s = it % kOeStages;
        const uint32_t ph = (uint32_t)(it / kOeStages) & 1u;
        ok = bar_wait(&full[s], ph, abort_flag, P.polls) && bar_wait(&qfull[s], ph, abort_flag, P.polls);
        if (!ok) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t xs = s_u32(smem + s * kOeStageBytes);
        const uint32_t ws = xs + kOeXBytes, qs = ws + kOeWBytes;
#pragma unroll
        for (int kk = 0; kk < kOeK / 16; ++kk) {
          const uint64_t a = kmajor_desc(xs + 32u * kk);
          const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
          umma(d_ref, a, kmajor_desc(ws + 32u * kk), acc);
          umma(d_q, a, kmajor_desc(qs + 32u * kk), acc);
        }
        umma_commit(&empty[s]);
      }
      if (!ok) fail();
      umma_commit(accfull);
      umma_commit(done);
      for (uint32_t i = 0; i < kOeSpin && !bar_try(done, 0); ++i) {
      }
    }
  } else {
    // ---- warps 1-4: expand the codes to bf16, then the epilogue ----------------------------
    const int t = threadIdx.x - 32;          // 0 .. 127
    const int r = t >> 1, hf = t & 1;        // W-tile row, half of its 64 columns
    const int64_t row = n0 + r;
    const int64_t kb = P.k / P.block;
    bool ok = true;
    // codes and scales of a stage: fetched one stage ahead, so that the global-load latency
    // overlaps the expansion of the previous stage
    auto fetch = [&](int it, uint32_t (&cw)[4], float (&sc)[4]) {
      const int64_t kk0 = (int64_t)it * kOeK + 32 * hf;
#pragma unroll
      for (int q = 0; q < 4; ++q) { cw[q] = 0u; sc[q] = 0.0f; }
      if (it < nk && row < P.n && kk0 < P.k) {
        const uint2* cp = reinterpret_cast<const uint2*>(P.codes + row * (P.k / 2) + kk0 / 2);
        const uint2 c0 = __ldg(cp), c1 = (kk0 + 16 < P.k) ? __ldg(cp + 1) : make_uint2(0u, 0u);
        cw[0] = c0.x; cw[1] = c0.y; cw[2] = c1.x; cw[3] = c1.y;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int64_t e0 = kk0 + 8 * q;
          sc[q] = e0 < P.k ? stab[__ldg(P.scales + row * kb + e0 / P.block)] : 0.0f;
        }
      }
    };
    uint32_t cw[4], cwn[4];
    float sc[4], scn[4];
    fetch(0, cw, sc);
    for (int it = 0; it < nk; ++it) {
      const int s = it % kOeStages;
      fetch(it + 1, cwn, scn);
      ok = bar_wait(&empty[s], ((uint32_t)(it / kOeStages) & 1u) ^ 1u, abort_flag, P.polls);
      if (!__all_sync(kFull, ok)) { ok = false; break; }
      uint32_t wd[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {           // 8 elements per word
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t byte = (cw[q] >> (8 * u)) & 0xffu;
          float v0, v1;
          if (P.int4) {
            v0 = (float)((int)(byte << 28) >> 28);
            v1 = (float)((int)(byte << 24) >> 28);
          } else {
            const uint32_t h2 = e2m1x2_to_f16x2(byte);
            v0 = __half2float(__ushort_as_half(lo16(h2)));
            v1 = __half2float(__ushort_as_half(hi16(h2)));
          }
          wd[4 * q + u] = pack_bf16(__fmul_rn(v0, sc[q]), __fmul_rn(v1, sc[q]));
        }
      }
      uint8_t* qt = smem + s * kOeStageBytes + kOeXBytes + kOeWBytes + r * 128;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 4 * hf + j;
        *reinterpret_cast<uint4*>(qt + ((c ^ (r & 7)) << 4)) =
            make_uint4(wd[4 * j], wd[4 * j + 1], wd[4 * j + 2], wd[4 * j + 3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      bar_arrive(&qfull[s]);
#pragma unroll
      for (int q = 0; q < 4; ++q) { cw[q] = cwn[q]; sc[q] = scn[q]; }
    }
    if (!ok && lane == 0) fail();
    // epilogue: this warp's tensor-memory lanes 32 (warp % 4) ..
    double sdd = 0.0, syy = 0.0;
    const bool got = __all_sync(kFull, ok && bar_wait(accfull, 0, abort_flag, P.polls));
    if (got) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t lanebase = (uint32_t)((warp & 3) * 32) << 16;
#pragma unroll
      for (int h = 0; h < kOeN / 32; ++h) {
        float yr[32], yq[32];
        tld32(tmem + lanebase + (uint32_t)(32 * h), yr);
        tld32(tmem + lanebase + (uint32_t)(kOeN + 32 * h), yq);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const double d = (double)yq[j] - (double)yr[j];
          sdd += d * d;
          syy += (double)yr[j] * (double)yr[j];
        }
      }
    } else if (lane == 0) {
      fail();
    }
    sdd = warp_sum(sdd);
    syy = warp_sum(syy);
    if (lane == 0) {
      red[(warp - 1) * 2] = sdd;
      red[(warp - 1) * 2 + 1] = syy;
    }
  }
  __syncthreads();
  if (threadIdx.x == 32) {
    const int64_t cta = (int64_t)blockIdx.y * gridDim.x + blockIdx.x;
    P.partial[cta * 2] = ((red[0] + red[2]) + red[4]) + red[6];
    P.partial[cta * 2 + 1] = ((red[1] + red[3]) + red[5]) + red[7];
  }
  if (warp == 5) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(tmem));
  }
}

__global__ void k_outerr_final(const double* __restrict__ partial, int parts, const int* err,
                               double* sums) {
  __shared__ double red[2][256];
  double a = 0.0, b = 0.0;
  for (int p = threadIdx.x; p < parts; p += 256) {
    a += partial[2 * p];
    b += partial[2 * p + 1];
  }
  red[0][threadIdx.x] = a;
  red[1][threadIdx.x] = b;
  __syncthreads();
  for (int half = 128; half > 0; half >>= 1) {
    if ((int)threadIdx.x < half) {
      red[0][threadIdx.x] += red[0][threadIdx.x + half];
      red[1][threadIdx.x] += red[1][threadIdx.x + half];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const bool bad = *err != 0;
    sums[0] = bad ? __longlong_as_double(0x7ff8000000000000ll) : red[0][0];
    sums[1] = bad ? __longlong_as_double(0x7ff8000000000000ll) : red[1][0];
  }
}

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                             const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                             const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                             CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn oe_encode() {
  static EncodeFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return (EncodeFn)p;
  }();
  return fn;
}

bool make_map(EncodeFn enc, CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
              int64_t ld, uint32_t box_rows) {
  std::memset(map, 0, sizeof *map);
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t outerr_workspace(int64_t m, int64_t n) {
  const int64_t ctas = ((m + kOeM - 1) / kOeM) * ((n + kOeN - 1) / kOeN);
  return 256 + (size_t)ctas * 2 * sizeof(double);
}

cudaError_t launch_outerr(const void* X, int64_t m, int64_t k, int64_t ldx, const void* W,
                          int64_t n, int64_t ldw, const uint8_t* codes, const uint8_t* scales,
                          int fmt, int scale_fmt, int block, double* sums, void* workspace,
                          cudaStream_t st) {
  EncodeFn enc = oe_encode();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap xmap, wmap;
  if (!make_map(enc, &xmap, X, m, k, ldx, kOeM) || !make_map(enc, &wmap, W, n, k, ldw, kOeN))
    return cudaErrorInvalidValue;
  OeScaleTab T;
  const GridInfo g = grid_info(scale_fmt);
  for (int c = 0; c < 256; ++c) T.v[c] = c < g.ncodes ? (float)grid_value(scale_fmt, c) : __builtin_nanf("");
  int* err = (int*)workspace;
  double* partial = (double*)((char*)workspace + 256);
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((m + kOeM - 1) / kOeM), (unsigned)((n + kOeN - 1) / kOeN));
  OeParams P{m, n, k, codes, scales, block, fmt == 3 ? 1 : 0, partial, err, wait_polls()};
  e = ensure_dynamic_smem((const void*)k_outerr_tc, (int)kOeSmem);
  if (e != cudaSuccess) return e;
  k_outerr_tc<<<grid, kOeThreads, kOeSmem, st>>>(xmap, wmap, P, T);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_outerr_final<<<1, 256, 0, st>>>(partial, (int)(grid.x * grid.y), err, sums);
  return cudaGetLastError();
}

}  // namespace mxq
