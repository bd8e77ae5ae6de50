// out = act(x W + bias) on the sm_100a tensor cores, bias and activation in
// the GEMM's own epilogue (the layer's f1 with SiLU, f2 without).
//
// x [T, K] bf16 (row stride x_stride), W [K, N] bf16 row-major, out [T, N] bf16.
// Output tile 128 x 256, K in blocks of 64:
//   A = x tile  (128 rows x 64 K, K-major, 128B swizzle: one TMA box)
//   B = W block (64 K rows x 256 N, N-major: four TMA boxes of 64 N columns)
//   D = fp32 accumulator in tensor memory, two 256-column buffers so that the
//       epilogue of one tile overlaps the MMAs of the next
// Persistent CTAs walk the tiles (row-block major, so CTAs running at the
// same time share x rows in L2).  Warp roles (320 threads): warp 0 TMA
// producer, warp 1 MMA issuer and tensor-memory owner, warps 2-9 epilogue
// (thread = output row = TMEM lane, two warps per lane quarter splitting the
// columns): tcgen05.ld 32 columns at a time, add the
// fp32 bias, SiLU as h + h tanh(h) with h = x/2 (one MUFU op per element),
// round to bf16, 16-byte stores of the thread's own row.  Rows past T are
// zero-filled by TMA on the way in and not stored on the way out.  Every wait
// is bounded and reports HSTU_ERR_TIMEOUT through the workspace status word.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "device_common.cuh"
#include "hstu_internal.h"

namespace hstu {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kXStage = kBM * kBK * 2;         // 16 KB
constexpr int kWChunk = kBK * 64 * 2;          // 64 K rows x 64 N columns = 8 KB
constexpr int kWStage = kWChunk * (kBN / 64);  // 32 KB
constexpr int kEpiWarps = 8;                  // two per TMEM lane quarter: each takes half the columns
constexpr int kGemmThreads = 32 * (2 + kEpiWarps);
constexpr uint32_t kAccCols = kBN;             // one fp32 accumulator: 256 columns

struct __align__(1024) GemmSmem {
  uint8_t x[kStages][kXStage];
  uint8_t w[kStages][kWStage];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kGemmSmem = sizeof(GemmSmem) + 1024;
static_assert(kGemmSmem <= 227 * 1024, "shared memory budget");

struct GemmArgs {
  int T, K, N;
  long long out_stride;  // elements
  int silu;
  const float* bias;
  __nv_bfloat16* out;
  WsHeader* hdr;
};

__device__ __forceinline__ float act(float x, int silu) {
  if (!silu) return x;
  const float h = 0.5f * x;  // SiLU(x) = x sigmoid(x) = h (1 + tanh h)
  return fmaf(h, tanh_approx(h), h);
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bias_act_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tm_x,
                         const __grid_constant__ CUtensorMap tm_w) {
  extern __shared__ uint8_t smem_raw[];
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (a.T + kBM - 1) / kBM, tiles_n = a.N / kBN, n_tiles = tiles_m * tiles_n;
  const int nk = a.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], kEpiWarps);
    }
    mbar_init(&sm.done, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 2 * kAccCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_w);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x) {
        const int m0 = (tile / tiles_n) * kBM, n0 = (tile % tiles_n) * kBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          ok = mbar_wait(&sm.empty[s], ((it / kStages) & 1) ^ 1, abort_flag, a.hdr, 21);
          if (!ok) break;
          mbar_arrive_expect_tx(&sm.full[s], kXStage + kWStage);
          tma_load_2d(sm.x[s], &tm_x, &sm.full[s], kb * kBK, m0);
#pragma unroll
          for (int c = 0; c < kBN / 64; ++c)
            tma_load_2d(sm.w[s] + c * kWChunk, &tm_w, &sm.full[s], n0 + 64 * c, kb * kBK);
        }
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (int j = max(0, it - kStages); j < it; ++j)
        mbar_wait(&sm.full[j % kStages], (j / kStages) & 1, nullptr, a.hdr, 29);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kBM, kBN, 0, 1);
      int it = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++tc) {
        const int b = tc & 1;
        // accumulator b held tile tc - 2 until the epilogue read it
        ok = mbar_wait(&sm.acc_empty[b], ((tc >> 1) & 1) ^ 1, abort_flag, a.hdr, 22);
        if (!ok) break;
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          ok = mbar_wait(&sm.full[s], (it / kStages) & 1, abort_flag, a.hdr, 23);
          if (!ok) break;
          tc_fence_after();
          const uint32_t xb = smem_u32(sm.x[s]), wb = smem_u32(sm.w[s]);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ss(tmem + b * kAccCols, sw128_desc(xb + kk * 32, 16, 1024),
                   sw128_desc(wb + kk * 16 * 128, kWChunk, 1024), idesc, (kb | kk) != 0);
          mma_commit(&sm.empty[s]);
        }
        if (ok) mma_commit(&sm.acc_full[b]);
      }
      // tensor memory is freed below only after every issued MMA completed
      mma_commit(&sm.done);
      mbar_wait(&sm.done, 0, nullptr, a.hdr, 28);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // the TMEM lanes this warp may read
    const int half = (warp - 2) >> 2;  // columns half*128 .. +127 of the tile
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    int tc = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tc) {
      const int b = tc & 1;
      const int m0 = (tile / tiles_n) * kBM, n0 = (tile % tiles_n) * kBN;
      const bool ok = __all_sync(~0u, mbar_wait(&sm.acc_full[b], (tc >> 1) & 1, abort_flag, a.hdr, 24));
      if (!ok) break;
      tc_fence_after();
      const int row = m0 + r;
      __nv_bfloat16* orow = a.out + (size_t)row * a.out_stride + n0;
#pragma unroll 1
      for (int c = half * (kBN / 64); c < (half + 1) * (kBN / 64); ++c) {
        uint32_t acc[32];
        tmem_ld32(tmem + lane_base + b * kAccCols + c * 32, acc);
        float bias[32];
        if (a.bias) {
          const float4* bp = reinterpret_cast<const float4*>(a.bias + n0 + c * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 v = __ldg(bp + e);
            bias[4 * e] = v.x;
            bias[4 * e + 1] = v.y;
            bias[4 * e + 2] = v.z;
            bias[4 * e + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) bias[e] = 0.f;
        }
        tmem_wait_ld(acc);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(act(__uint_as_float(acc[2 * e]) + bias[2 * e], a.silu),
                              act(__uint_as_float(acc[2 * e + 1]) + bias[2 * e + 1], a.silu));
        if (row < a.T) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      // this accumulator may take the tile after next
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 2 * kAccCols);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [rows, cols] bf16 row-major with a row stride: box = box_rows x 64 columns, 128B swizzle
bool encode_2d(CUtensorMap* m, const void* base, long long rows, long long cols, long long stride,
               int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)stride * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool gemm_sm100_supported(int K, int N) { return K > 0 && N > 0 && K % kBK == 0 && N % kBN == 0; }

cudaError_t launch_gemm_sm100(const void* x, long long T, int K, long long x_stride, const void* w, int N,
                              const float* bias, void* out, long long out_stride, bool silu, void* hdr,
                              cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static int sms[64];
  static unsigned long long attr_set = 0;
  if (!(attr_set & (1ull << dev))) {
    cudaError_t e =
        cudaFuncSetAttribute(gemm_bias_act_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  if (T == 0) return cudaSuccess;
  CUtensorMap tx, tw;
  if (!encode_2d(&tx, x, T, K, x_stride, kBM) || !encode_2d(&tw, w, K, N, N, kBK)) return cudaErrorInvalidValue;
  GemmArgs a;
  a.T = (int)T;
  a.K = K;
  a.N = N;
  a.out_stride = out_stride;
  a.silu = silu ? 1 : 0;
  a.bias = bias;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.hdr = static_cast<WsHeader*>(hdr);
  const long long tiles = ((T + kBM - 1) / kBM) * (N / kBN);
  const int grid = (int)std::min<long long>(tiles, sms[dev]);
  gemm_bias_act_kernel<<<grid, kGemmThreads, kGemmSmem, s>>>(a, tx, tw);
  return cudaGetLastError();
}

}  // namespace hstu
