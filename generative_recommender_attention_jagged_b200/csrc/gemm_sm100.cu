// out = act(x W + bias) on a pair of SMs (tcgen05 cta_group::2), bias and
// activation in the epilogue: the layer's f1 (SiLU) and f2 projections.
//
// Why a pair: a single-SM 128 x 256 tile reads its A and B operands from
// shared memory at 96 B/clk while TMA writes the next stages at about the
// same rate, more than the SM's shared memory delivers, so the tensor core
// waits.  Two CTAs of a cluster share one 256 x 256 output tile: each holds
// its own 128 rows of x and half (128 columns) of the W block, the MMA
// (M = 256, N = 256, K = 16, issued by the even CTA) reads both CTAs' shared
// memory, and each SM then reads 64 B/clk of operands and takes 64 B/clk of
// TMA writes.  Each CTA's accumulator is its 128 rows x 256 columns in its
// own tensor memory (two buffers: the epilogue of one tile overlaps the MMAs
// of the next).
//
// Roles (320 threads per CTA): warp 0 TMA producer (both CTAs load their own
// x rows and W half into a 6-stage ring; the bytes complete on the even CTA's
// barrier), warp 1 MMA issuer (even CTA only) and tensor-memory owner (both
// CTAs allocate collectively), warps 2-9 epilogue (thread = output row, two
// warps per lane quarter splitting each 64-column box): tcgen05.ld, fp32
// bias, SiLU as h + h tanh h with h = x / 2, bf16 into one of two
// 128B-swizzled staging boxes that one thread stores with TMA (whole
// 128-byte row segments) while the other box fills.  The odd CTA's epilogue
// frees an accumulator by a remote arrive on the even CTA's barrier.  Every
// wait is bounded; whatever happens, both CTAs meet at a cluster barrier
// before tensor memory is freed and the CTAs exit, so neither leaves while
// the other's MMAs may still read its shared memory or copies into it are in
// flight.
//
// Measured (T = 53,095 rows, K = 512): the wide SiLU projection (N = 2048)
// at about two thirds of the measured bf16 peak, twice as fast as cuBLASLt + a
// SiLU pass.  A narrow output (N = 512: 5.6 tiles per pair, the last round 62%
// full) is dominated by the launch's fill and tail, where cuBLASLt is faster.
//
// The remote arrive and every wait use CTA scope (a cluster-scope release or
// acquire costs a memory barrier per use: 10% of this kernel's time).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "hstu_internal.h"
#include "pair_common.cuh"

namespace hstu {
namespace {

constexpr int kBM = 128;                          // rows per CTA (256 per pair)
constexpr int kBN = 256;                          // columns per pair tile (128 of W per CTA)
constexpr int kBK = 64;
constexpr int kStages = 6;
constexpr int kXStage = kBM * kBK * 2;            // 16 KB
constexpr int kWChunk = kBK * 64 * 2;             // 64 K rows x 64 N columns = 8 KB
constexpr int kWStage = kWChunk * (kBN / 2 / 64); // this CTA's 128 columns: 16 KB
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr uint32_t kAccCols = kBN;                // one fp32 accumulator: 256 columns

constexpr int kOutBox = kBM * 128;               // 128 rows x 64 bf16 columns of output: 16 KB

struct __align__(1024) Smem2 {
  uint8_t x[kStages][kXStage];
  uint8_t w[kStages][kWStage];
  uint8_t out[2][kOutBox];      // two 128B-swizzled TMA boxes (128 rows x 64 columns), used in turn
  uint64_t full[kStages];       // even CTA: both CTAs' bytes of the stage landed
  uint64_t empty[kStages];      // both CTAs: the MMAs that read the stage completed
  uint64_t acc_full[2];         // both CTAs: accumulator b holds a finished tile
  uint64_t acc_empty[2];        // even CTA: both CTAs' epilogues read accumulator b
  uint64_t done;                // both CTAs: every MMA completed
  uint32_t tmem_base;
  int abort;
  int issued;                   // stages whose copies this CTA issued
};
constexpr size_t kSmem2 = sizeof(Smem2) + 1024;
static_assert(kSmem2 <= 227 * 1024, "shared memory budget");

struct Gemm2Args {
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

// the 256 epilogue threads agree on a flag (barrier 2), so that they leave
// the tile loop together and never split across named barrier 1
__device__ __forceinline__ bool epi_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 2, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}

// TMA store of a 2-D box from shared memory (bulk group of this thread)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, const void* src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const Gemm2Args a, const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_out) {
  extern __shared__ uint8_t smem_raw[];
  Smem2& sm = aligned_smem<Smem2>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int tiles_m = (a.T + 2 * kBM - 1) / (2 * kBM), tiles_n = a.N / kBN;
  const int n_units = tiles_m * tiles_n;
  const int nk = a.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], 2 * kEpiWarps);
    }
    mbar_init(&sm.done, 1);
    sm.abort = 0;
    sm.issued = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    // both CTAs allocate together (same warp, same destination offset)
    tmem_alloc_pair(&sm.tmem_base, 2 * kAccCols);
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_out);
  }
  tc_fence_before();
  // barriers of both CTAs are initialised before any CTA touches the other's
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int u = pair; ok && u < n_units; u += n_pairs) {
        const int m0 = (u / tiles_n) * 2 * kBM + rank * kBM;
        const int n0 = (u % tiles_n) * kBN + rank * (kBN / 2);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          ok = mbar_wait(&sm.empty[s], ((it / kStages) & 1) ^ 1, abort_flag, a.hdr, 31);
          if (!ok) break;
          if (leader) mbar_arrive_expect_tx(&sm.full[s], 2 * (kXStage + kWStage));
          tma_load_2d_pair(sm.x[s], &tm_x, &sm.full[s], kb * kBK, m0);
#pragma unroll
          for (int c = 0; c < kBN / 2 / 64; ++c)
            tma_load_2d_pair(sm.w[s] + c * kWChunk, &tm_w, &sm.full[s], n0 + 64 * c, kb * kBK);
          sm.issued = it + 1;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (even CTA)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = idesc_bf16(2 * kBM, kBN, 0, 1);
      int it = 0, tc = 0;
      bool ok = true;
      for (int u = pair; ok && u < n_units; u += n_pairs, ++tc) {
        const int b = tc & 1;
        // accumulator b held tile tc - 2 until both epilogues read it
        ok = mbar_wait(&sm.acc_empty[b], ((tc >> 1) & 1) ^ 1, abort_flag, a.hdr, 32);
        if (!ok) break;
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          ok = mbar_wait(&sm.full[s], (it / kStages) & 1, abort_flag, a.hdr, 33);
          if (!ok) break;
          tc_fence_after();
          const uint32_t xb = smem_u32(sm.x[s]), wb = smem_u32(sm.w[s]);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ss_pair(tmem + b * kAccCols, sw128_desc(xb + kk * 32, 16, 1024),
                        sw128_desc(wb + kk * 16 * 128, kWChunk, 1024), idesc, (kb | kk) != 0);
          mma_commit_pair(&sm.empty[s]);
        }
        if (ok) mma_commit_pair(&sm.acc_full[b]);
      }
      // both CTAs learn when every issued MMA completed
      mma_commit_pair(&sm.done);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int quarter = warp & 3;      // the TMEM lanes this warp may read
    const int half = (warp - 2) >> 2;  // columns half*128 .. +127 of the tile
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    // the even CTA's acc_empty barriers, as seen from this CTA
    const uint32_t empty_addr0 = map_shared(smem_u32(&sm.acc_empty[0]), 0);
    const uint32_t empty_addr1 = map_shared(smem_u32(&sm.acc_empty[1]), 0);
    int tc = 0;
    for (int u = pair; u < n_units; u += n_pairs, ++tc) {
      const int b = tc & 1;
      const bool ok = epi_all(mbar_wait(&sm.acc_full[b], (tc >> 1) & 1, abort_flag, a.hdr, 34));
      if (!ok) break;
      tc_fence_after();
      const int row0 = (u / tiles_n) * 2 * kBM + rank * kBM;
      const int n0 = (u % tiles_n) * kBN;
      // box bx (columns 64 bx .. 64 bx + 63) is staged in buffer (4 tc + bx) & 1;
      // the warps of column half h convert its 32 columns 64 bx + 32 h ..
#pragma unroll 1
      for (int bx = 0; bx < kBN / 64; ++bx) {
        const int c = 2 * bx + half;  // 32-column chunk of this warp
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
        // the store issued two boxes ago has read the buffer this box reuses
        if (tc > 0 || bx >= 2) {
          if (warp == 2 && lane == 0) bulk_wait_read1();
          named_bar_sync(1, 32 * kEpiWarps);
        }
        tmem_wait_ld(acc);
        if (bx == kBN / 64 - 1) {
          // this CTA's part of accumulator b is read: tell the even CTA's issuer
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(b ? empty_addr1 : empty_addr0);
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(act(__uint_as_float(acc[2 * e]) + bias[2 * e], a.silu),
                              act(__uint_as_float(acc[2 * e + 1]) + bias[2 * e + 1], a.silu));
        // the row's 64 bytes into the box: 16-byte chunk j of the box row at
        // j ^ (r & 7) (the TMA store's 128-byte swizzle)
        const uint32_t box = smem_u32(sm.out[bx & 1]) + r * 128;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = half * 4 + e;
          asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(box + ((j ^ (r & 7)) << 4)), "r"(pk[4 * e]),
                       "r"(pk[4 * e + 1]), "r"(pk[4 * e + 2]), "r"(pk[4 * e + 3])
                       : "memory");
        }
        // the box goes out as one TMA store (rows past T are dropped)
        fence_proxy_async_smem();
        named_bar_sync(1, 32 * kEpiWarps);
        if (warp == 2 && lane == 0) {
          tma_store_2d(&tm_out, sm.out[bx & 1], n0 + 64 * bx, row0);
          bulk_commit();
        }
      }
    }
    // the last stores have completed before the CTA's shared memory is released
    if (warp == 2 && lane == 0) bulk_wait_all();
  }

  // Every MMA completed (both CTAs see the commit) and both CTAs meet, the
  // issued counts published; the even CTA then accounts for every copy into
  // either CTA (a stage expected but not issued by the odd CTA, or issued but
  // not expected, which only a timed-out wait leaves behind), and both meet
  // again before tensor memory is freed and either exits, so no copy lands
  // in a CTA that has left.
  if (warp == 1 && lane == 0) mbar_wait(&sm.done, 0, nullptr, a.hdr, 38);
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (leader && warp == 0 && lane == 0) {
    const int mine = sm.issued;
    const int peer = (int)ld_shared_cluster_u32(map_shared(smem_u32(&sm.issued), 1));
    const int last = max(mine, peer);
    for (int t = max(0, last - kStages); t < last; ++t) {
      uint64_t* bar = &sm.full[t % kStages];
      if (t < mine && t >= peer) mbar_complete_tx(bar, kXStage + kWStage);       // odd half never issued
      if (t >= mine && t < peer) mbar_arrive_expect_tx(bar, kXStage + kWStage);  // odd half never expected
      mbar_wait(bar, (t / kStages) & 1, nullptr, a.hdr, 39);
    }
  }
  __syncwarp();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 1)
    tmem_dealloc_pair(tmem, 2 * kAccCols);
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
bool encode_2d(CUtensorMap* m, const void* base, long long rows, long long cols, long long stride, int box_rows) {
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
    cudaError_t e = cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem2);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  if (T == 0) return cudaSuccess;
  CUtensorMap tx, tw;
  CUtensorMap to;
  if (!encode_2d(&tx, x, T, K, x_stride, kBM) || !encode_2d(&tw, w, K, N, N, kBK) ||
      !encode_2d(&to, out, T, N, out_stride, kBM))
    return cudaErrorInvalidValue;
  Gemm2Args a;
  a.T = (int)T;
  a.K = K;
  a.N = N;
  a.out_stride = out_stride;
  a.silu = silu ? 1 : 0;
  a.bias = bias;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.hdr = static_cast<WsHeader*>(hdr);
  const long long units = ((T + 2 * kBM - 1) / (2 * kBM)) * (N / kBN);
  const int pairs = (int)std::max<long long>(1, std::min<long long>(units, sms[dev] / 2));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem2;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_pair_kernel, a, tx, tw, to);
}

}  // namespace hstu
