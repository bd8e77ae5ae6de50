// Backward of the attention core o = A V over jagged users (CUDA cores, fp32).
//
// ("Generative Recommenders at Scale", Inside NVIDIA's GPU-native stack: SiLU
// weighting with relative attention bias; "How Generative Recommenders Are
// Redefining RecSys at Scale", Summary: the models are trained.)  With g = dL/do,
// on the allowed set:
//   ds_ij = (g_i . v_j) SiLU'(s_ij) / N_max,  SiLU'(x) = sig(x) (1 + x (1 - sig(x)))
//   dq_i  = alpha sum_j ds_ij k_j          (query-side kernel, one warp per (row, head);
//   d rab_pos, d rab_ts += ds_ij            it also adds the bias gradients)
//   dv_j  = sum_i a_ij g_i,  a_ij = SiLU(s_ij) / N_max
//   dk_j  = alpha sum_i ds_ij q_i          (key-side kernel, one warp per (key, head))
// Scores are recomputed in fp32 exactly as the CUDA-core forward does them
// (exact integer time buckets, expf).
//
// Head dims 32, 64 and 128 take the tiled kernel: one CTA per (user, head,
// block of 64 keys) keeps K, V and the block's d_k, d_v accumulators on chip
// and walks the 64-row query blocks that see the keys.  Per query block it
// stages Q and g in shared memory, forms S = Q K^T and dP = g V^T (4x4
// register tiles, fp32 FMA), turns them into a and ds, then accumulates
// d_v += a^T g and d_k += ds^T Q, and adds ds K into d_q with vector atomics
// (d_q is zeroed first).  Bias gradients come from the block pair's ds tile in
// shared memory: one thread per position difference (127 per pair) sums its
// pairs and adds the result to d rab_pos with one atomic, and a row walk folds
// each run of equal time buckets into a per-CTA histogram (warp-aggregated
// when a warp's lanes share the bucket) that goes to d rab_ts at the end.
// Other head dims take the warp-per-row kernels below, whose warps fold runs
// of equal bias indices of their own row before the atomics.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <type_traits>

#include "device_common.cuh"
#include "hstu_internal.h"

namespace hstu {
namespace {

constexpr int kMaxPerLane = 8;  // d <= 256

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(~0u, x, o);
  return x;
}

__device__ __forceinline__ int find_user(const int32_t* off, int B, int row) {
  int lo = 0, hi = B - 1;  // largest u with off[u] <= row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= row) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

struct BwdOut {
  const float* d_o;  // [T, H, d]
  float *dq, *dk, *dv, *d_rp, *d_rt;
};

template <typename T>
__global__ void __launch_bounds__(256) attn_bwd_q_kernel(const AttnArgs a, const BucketTable tab, const BwdOut b) {
  __shared__ long long thr[kMaxBuckets];
  for (int x = threadIdx.x; x < kMaxBuckets; x += blockDim.x) thr[x] = tab.thr[x];
  __syncthreads();
  if (a.hdr->status != 0) return;
  const int lane = threadIdx.x & 31;
  const int d = a.d, per_lane = (d + 31) >> 5;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  const long long total = (long long)a.T_q * a.H;
  for (long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total;
       w += (long long)gridDim.x * (blockDim.x >> 5)) {
    const int row = (int)(w / a.H), head = (int)(w % a.H);
    const int u = find_user(a.q_offsets, a.B, row);
    const int q0 = a.q_offsets[u];
    const int n = a.q_offsets[u + 1] - q0;
    const int hist = n - (a.num_cand ? a.num_cand[u] : 0);
    const int i = row - q0;
    const long long t_i = a.ts[q0 + i];
    const int p_i = min(i, hist);
    float qv[kMaxPerLane], gv[kMaxPerLane], acc[kMaxPerLane];
#pragma unroll
    for (int x = 0; x < kMaxPerLane; ++x) {
      const int e = lane + 32 * x;
      const bool in = x < per_lane && e < d;
      qv[x] = in ? ld_f(q + (size_t)row * a.qkv_stride + head * d + e) : 0.f;
      gv[x] = in ? b.d_o[((size_t)row * a.H + head) * d + e] : 0.f;
      acc[x] = 0.f;
    }
    // allowed keys: [0, i] for history rows; [0, hist) and i for candidates
    const int j_end = i < hist ? i + 1 : hist;
    int run_idx = -1, run_b = -1;
    float run_pos = 0.f, run_ts = 0.f;  // lane 0: a run of equal bias indices not yet added
    for (int jj = 0; jj <= j_end; ++jj) {
      int j = jj;
      if (jj == j_end) {
        if (i < hist) break;
        j = i;
      }
      const size_t base = (size_t)(q0 + j) * a.qkv_stride + head * d;
      float qk = 0.f, gvj = 0.f;
#pragma unroll
      for (int x = 0; x < kMaxPerLane; ++x) {
        const int e = lane + 32 * x;
        if (x < per_lane && e < d) {
          qk = fmaf(qv[x], ld_f(k + base + e), qk);
          gvj = fmaf(gv[x], ld_f(v + base + e), gvj);
        }
      }
      qk = warp_sum(qk);
      gvj = warp_sum(gvj);
      const int p_j = min(j, hist);
      const int bkt = bucket_of_dt(thr, t_i - a.ts[q0 + j]);
      const int pidx = p_i - p_j + a.n_max - 1;
      const float s = a.alpha * qk + a.rab_pos[pidx] + a.rab_ts[bkt];
      const float sig = 1.f / (1.f + expf(-s));
      const float ds = gvj * sig * (1.f + s * (1.f - sig)) / (float)a.n_max;
#pragma unroll
      for (int x = 0; x < kMaxPerLane; ++x) {
        const int e = lane + 32 * x;
        if (x < per_lane && e < d) acc[x] = fmaf(a.alpha * ds, ld_f(k + base + e), acc[x]);
      }
      if (lane == 0) {
        if (pidx != run_idx) {
          if (run_idx >= 0) atomicAdd(b.d_rp + run_idx, run_pos);
          run_idx = pidx;
          run_pos = 0.f;
        }
        run_pos += ds;
        if (bkt != run_b) {
          if (run_b >= 0) atomicAdd(b.d_rt + run_b, run_ts);
          run_b = bkt;
          run_ts = 0.f;
        }
        run_ts += ds;
      }
    }
    if (lane == 0) {
      if (run_idx >= 0) atomicAdd(b.d_rp + run_idx, run_pos);
      if (run_b >= 0) atomicAdd(b.d_rt + run_b, run_ts);
    }
#pragma unroll
    for (int x = 0; x < kMaxPerLane; ++x) {
      const int e = lane + 32 * x;
      if (x < per_lane && e < d) b.dq[((size_t)row * a.H + head) * d + e] = acc[x];
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256) attn_bwd_kv_kernel(const AttnArgs a, const BucketTable tab,
                                                          const BwdOut b) {
  __shared__ long long thr[kMaxBuckets];
  for (int x = threadIdx.x; x < kMaxBuckets; x += blockDim.x) thr[x] = tab.thr[x];
  __syncthreads();
  if (a.hdr->status != 0) return;
  const int lane = threadIdx.x & 31;
  const int d = a.d, per_lane = (d + 31) >> 5;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  const long long total = (long long)a.T_q * a.H;
  for (long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total;
       w += (long long)gridDim.x * (blockDim.x >> 5)) {
    const int row = (int)(w / a.H), head = (int)(w % a.H);
    const int u = find_user(a.q_offsets, a.B, row);
    const int q0 = a.q_offsets[u];
    const int n = a.q_offsets[u + 1] - q0;
    const int hist = n - (a.num_cand ? a.num_cand[u] : 0);
    const int j = row - q0;
    const long long t_j = a.ts[q0 + j];
    const int p_j = min(j, hist);
    float kv[kMaxPerLane], vv[kMaxPerLane], dk[kMaxPerLane], dv[kMaxPerLane];
#pragma unroll
    for (int x = 0; x < kMaxPerLane; ++x) {
      const int e = lane + 32 * x;
      const bool in = x < per_lane && e < d;
      const size_t base = (size_t)row * a.qkv_stride + head * d + e;
      kv[x] = in ? ld_f(k + base) : 0.f;
      vv[x] = in ? ld_f(v + base) : 0.f;
      dk[x] = dv[x] = 0.f;
    }
    // queries that see key j: every i >= j when j is history (history rows
    // causally, candidates because j < h), only i = j when j is a candidate
    const int i_end = j < hist ? n : j + 1;
    for (int i = j; i < i_end; ++i) {
      const size_t qb = (size_t)(q0 + i) * a.qkv_stride + head * d;
      const size_t gb = ((size_t)(q0 + i) * a.H + head) * d;
      float qk = 0.f, gvj = 0.f;
#pragma unroll
      for (int x = 0; x < kMaxPerLane; ++x) {
        const int e = lane + 32 * x;
        if (x < per_lane && e < d) {
          qk = fmaf(ld_f(q + qb + e), kv[x], qk);
          gvj = fmaf(b.d_o[gb + e], vv[x], gvj);
        }
      }
      qk = warp_sum(qk);
      gvj = warp_sum(gvj);
      const int p_i = min(i, hist);
      const int bkt = bucket_of_dt(thr, a.ts[q0 + i] - t_j);
      const float s = a.alpha * qk + a.rab_pos[p_i - p_j + a.n_max - 1] + a.rab_ts[bkt];
      const float sig = 1.f / (1.f + expf(-s));
      const float wgt = s * sig / (float)a.n_max;
      const float ds = gvj * sig * (1.f + s * (1.f - sig)) / (float)a.n_max;
#pragma unroll
      for (int x = 0; x < kMaxPerLane; ++x) {
        const int e = lane + 32 * x;
        if (x < per_lane && e < d) {
          dv[x] = fmaf(wgt, b.d_o[gb + e], dv[x]);
          dk[x] = fmaf(a.alpha * ds, ld_f(q + qb + e), dk[x]);
        }
      }
    }
#pragma unroll
    for (int x = 0; x < kMaxPerLane; ++x) {
      const int e = lane + 32 * x;
      if (x < per_lane && e < d) {
        b.dk[((size_t)row * a.H + head) * d + e] = dk[x];
        b.dv[((size_t)row * a.H + head) * d + e] = dv[x];
      }
    }
  }
}


// ---------------------------------------------------------------- tiled path
constexpr int kBT = 64;           // query rows / keys per block
constexpr int kBwdThreads = 256;  // 16 x 16 threads

template <int D>
struct BwdSmem {
  static constexpr int kDP = D + 4;         // row stride (floats): 16-byte rows, two-way conflicts at most
  static constexpr int kSP = kBT + 4;
  float k[kBT][kDP], v[kBT][kDP], q[kBT][kDP], g[kBT][kDP];
  float a[kBT][kSP];    // a_ij / N_max     [query][key]
  float ds[kBT][kSP];   // ds_ij            [query][key]
  float dst[kBT][kSP];  // ds_ij            [key][query]
  int bk[kBT][kSP];     // time bucket of each pair [query][key]
  uint4 oct[32];        // octave table of the bucket edges (|dt| + 1 < 2^32)
  float rts[kMaxBuckets];  // rab_ts
  float rpw[128];       // rab_pos over the block pair's position differences wbase .. wbase + 126
  float drt[kMaxBuckets];
  long long thr[kMaxBuckets];
  long long tq[kBT], tk[kBT];
};

__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// rows [r0, r0 + 64) of a [rows, H, D] tensor (row stride `stride` elements)
// into shared memory as fp32; rows at or past `rows` are zero
template <int D, typename T>
__device__ __forceinline__ void stage_rows(float (*dst)[D + 4], const T* src, int r0, int rows, int stride,
                                           int head) {
  constexpr int kVec = D / 4;
  for (int x = threadIdx.x; x < kBT * kVec; x += kBwdThreads) {
    const int r = x / kVec, c = (x % kVec) * 4;
    float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < rows) {
      const T* p = src + (size_t)(r0 + r) * stride + (size_t)head * D + c;
      if constexpr (sizeof(T) == 4) {
        val = *reinterpret_cast<const float4*>(p);
      } else {
        const uint2 raw = *reinterpret_cast<const uint2*>(p);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        val = make_float4(lo.x, lo.y, hi.x, hi.y);
      }
    }
    *reinterpret_cast<float4*>(&dst[r][c]) = val;
  }
}

// A query block's rows in registers: a thread holds chunks tid + 256 x of
// 4 elements (fp32 as float4, bf16 as 4 packed halves), so the next block's
// loads are in flight while the current block's d_q product runs.
template <int D, typename T>
struct RowRegs {
  static constexpr int kN = kBT * (D / 4) / kBwdThreads;
  using V = typename std::conditional<sizeof(T) == 4, float4, uint2>::type;
  V v[kN];
  __device__ __forceinline__ void load(const T* src, int r0, int rows, int stride, int head) {
#pragma unroll
    for (int x = 0; x < kN; ++x) {
      const int id = threadIdx.x + kBwdThreads * x;
      const int r = id / (D / 4), c = (id % (D / 4)) * 4;
      if (r0 + r < rows) {
        v[x] = *reinterpret_cast<const V*>(src + (size_t)(r0 + r) * stride + (size_t)head * D + c);
      } else {
        if constexpr (sizeof(T) == 4) v[x] = make_float4(0.f, 0.f, 0.f, 0.f);
        else v[x] = make_uint2(0u, 0u);
      }
    }
  }
  __device__ __forceinline__ void store(float (*dst)[D + 4]) const {
#pragma unroll
    for (int x = 0; x < kN; ++x) {
      const int id = threadIdx.x + kBwdThreads * x;
      const int r = id / (D / 4), c = (id % (D / 4)) * 4;
      float4 val;
      if constexpr (sizeof(T) == 4) {
        val = v[x];
      } else {
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v[x].x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v[x].y));
        val = make_float4(lo.x, lo.y, hi.x, hi.y);
      }
      *reinterpret_cast<float4*>(&dst[r][c]) = val;
    }
  }
};

// The DE dims of thread dg in the d_k / d_v / d_q products come in chunks of
// kC = min(DE, 4): chunk c holds dims kC dg + 16 kC c ..  so the 16 threads of
// a row read one contiguous span of shared memory.
template <int DE>
__device__ __forceinline__ int dim_of(int dg, int e) {
  constexpr int kC = DE < 4 ? DE : 4;
  return kC * dg + 16 * kC * (e / kC) + e % kC;
}

template <int DE>
__device__ __forceinline__ void lds_dims(const float* row, int dg, float (&x)[DE]) {
  if constexpr (DE >= 4) {
#pragma unroll
    for (int c = 0; c < DE / 4; ++c) {
      const float4 t = lds4(row + 4 * dg + 64 * c);
      x[4 * c] = t.x;
      x[4 * c + 1] = t.y;
      x[4 * c + 2] = t.z;
      x[4 * c + 3] = t.w;
    }
  } else {
    const float2 t = *reinterpret_cast<const float2*>(row + 2 * dg);
    x[0] = t.x;
    x[1] = t.y;
  }
}

// global atomics of one row's DE dims (16- or 8-byte vector adds)
template <int DE>
__device__ __forceinline__ void red_add_dims(float* row, int dg, const float (&x)[DE]) {
  if constexpr (DE >= 4) {
#pragma unroll
    for (int c = 0; c < DE / 4; ++c)
      atomicAdd(reinterpret_cast<float4*>(row + 4 * dg + 64 * c),
                make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]));
  } else {
    atomicAdd(reinterpret_cast<float2*>(row + 2 * dg), make_float2(x[0], x[1]));
  }
}

template <int D, typename T>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_tiled_kernel(const AttnArgs a, const BucketTable tab, const BwdOut b) {
  constexpr int DE = D / 16;  // dims per thread in the d_k / d_v / d_q products
  extern __shared__ __align__(16) uint8_t smem_raw[];
  BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>(smem_raw);
  if (a.hdr->status != 0) return;
  const int tid = threadIdx.x;
  const int u = blockIdx.x / a.H, head = blockIdx.x % a.H;
  const int kb = blockIdx.y;
  const int q0 = a.q_offsets[u];
  const int n = a.q_offsets[u + 1] - q0;
  const int j0 = kb * kBT;
  if (j0 >= n) return;
  const int hist = n - (a.num_cand ? a.num_cand[u] : 0);
  const T* q = static_cast<const T*>(a.q) + (size_t)q0 * a.qkv_stride;
  const T* k = static_cast<const T*>(a.k) + (size_t)q0 * a.qkv_stride;
  const T* v = static_cast<const T*>(a.v) + (size_t)q0 * a.qkv_stride;
  const float* g = b.d_o + (size_t)q0 * a.H * D;
  for (int x = tid; x < kMaxBuckets; x += kBwdThreads) {
    sm.thr[x] = tab.thr[x];
    sm.drt[x] = 0.f;
    sm.rts[x] = x < a.nb ? a.rab_ts[x] : 0.f;
  }
  if (tid < 32) sm.oct[tid] = make_uint4(tab.oct[tid][0], tab.oct[tid][1], tab.oct[tid][2], tab.oct[tid][3]);
  stage_rows<D>(sm.k, k, j0, n, a.qkv_stride, head);
  stage_rows<D>(sm.v, v, j0, n, a.qkv_stride, head);
  if (tid < kBT) sm.tk[tid] = a.ts[q0 + min(j0 + tid, n - 1)];

  const int ty = tid >> 4, tx = tid & 15;  // S tile: rows ty + 16 r, keys tx + 16 c
  const int rg = tid >> 4, dg = tid & 15;  // products: keys / queries 4 rg .. 4 rg + 3, dims dim_of(dg, .)
  float dk[4][DE], dv[4][DE];
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int e = 0; e < DE; ++e) dk[x][e] = dv[x][e] = 0.f;
  const float inv_n = 1.f / (float)a.n_max;
  const int nqb = (n + kBT - 1) / kBT;
  // history keys are seen by every later row (candidates included); a block
  // of candidate keys only by the candidates themselves
  const int qb_end = j0 < hist ? nqb : kb + 1;
  RowRegs<D, T> nq;
  RowRegs<D, float> ng;
  long long nts = 0;
  auto fetch = [&](int qb) {
    nq.load(q, qb * kBT, n, a.qkv_stride, head);
    ng.load(g, qb * kBT, n, a.H * D, head);
    if (tid < kBT) nts = a.ts[q0 + min(qb * kBT + tid, n - 1)];
  };
  fetch(kb);
  for (int qb = kb; qb < qb_end; ++qb) {
    const int i0 = qb * kBT;
    __syncthreads();  // the previous block pair is done with q, g, a, ds, dst and bk
    nq.store(sm.q);
    ng.store(sm.g);
    if (tid < kBT) sm.tq[tid] = nts;
    // rab_pos over the pair's position differences: p_i - p_j - wbase lies in [0, 126]
    const int wbase = min(i0, hist) - min(j0 + kBT - 1, hist);
    if (tid < 127) {
      const int idx = wbase + tid + a.n_max - 1;
      sm.rpw[tid] = (idx >= 0 && idx < 2 * a.n_max - 1) ? a.rab_pos[idx] : 0.f;
    }
    __syncthreads();

    // S = Q K^T and dP = g V^T on 4 x 4 register tiles
    float s[4][4], dp[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[r][c] = dp[r][c] = 0.f;
#pragma unroll 2
    for (int e = 0; e < D; e += 4) {
      float4 qv[4], gv[4], kv[4], vv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        qv[r] = lds4(&sm.q[ty + 16 * r][e]);
        gv[r] = lds4(&sm.g[ty + 16 * r][e]);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        kv[c] = lds4(&sm.k[tx + 16 * c][e]);
        vv[c] = lds4(&sm.v[tx + 16 * c][e]);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          s[r][c] = fmaf(qv[r].x, kv[c].x, fmaf(qv[r].y, kv[c].y, fmaf(qv[r].z, kv[c].z, fmaf(qv[r].w, kv[c].w, s[r][c]))));
          dp[r][c] = fmaf(gv[r].x, vv[c].x, fmaf(gv[r].y, vv[c].y, fmaf(gv[r].z, vv[c].z, fmaf(gv[r].w, vv[c].w, dp[r][c]))));
        }
    }

    // a and ds of the block pair, and each pair's time bucket
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int li = ty + 16 * r, lj = tx + 16 * c;
        const int i = i0 + li, j = j0 + lj;
        const bool allowed = i < n && j < n && (i < hist ? j <= i : (j < hist || j == i));
        float av = 0.f, dsv = 0.f;
        int bkt = 0;
        if (allowed) {
          const int p_i = min(i, hist), p_j = min(j, hist);
          // the octave table below 2^32 (one lookup), the edge search above
          const long long dt = sm.tq[li] - sm.tk[lj];
          const unsigned long long xdt = abs_dt_plus1(dt);
          bkt = xdt < (1ull << 32) ? bucket_oct(sm.oct, (unsigned int)xdt) : bucket_of_dt(sm.thr, dt);
          const float sv = a.alpha * s[r][c] + sm.rpw[p_i - p_j - wbase] + sm.rts[bkt];
          const float sig = 1.f / (1.f + expf(-sv));
          av = sv * sig * inv_n;
          dsv = dp[r][c] * sig * (1.f + sv * (1.f - sig)) * inv_n;
        }
        sm.a[li][lj] = av;
        sm.ds[li][lj] = dsv;
        sm.dst[lj][li] = dsv;
        sm.bk[li][lj] = bkt;
      }
    __syncthreads();
    // Bias gradients from the ds tile (ds is 0 outside the allowed set).
    // d rab_pos: thread w < 127 sums the pairs with p_i - p_j = wbase + w; in
    // row i that is key position p_i - wbase - w, or the row's own key when
    // that position is the history length (candidates sit at position h).
    // d rab_ts: the other 128 threads fold 32 columns of one row each (the
    // bucket only changes near the diagonal), warp-aggregated when all lanes
    // share the bucket.
    if (tid < 127) {
      const int w = tid;
      float acc = 0.f;
#pragma unroll 8
      for (int li = 0; li < kBT; ++li) {
        const int i = i0 + li;
        const int pj = min(i, hist) - wbase - w;
        // a history key at position pj, or (pj == h) a candidate row's own key
        const bool key = pj >= 0 && (pj < hist || (pj == hist && i >= hist));
        const int lj = (pj < hist ? pj : i) - j0;
        if (key && lj >= 0 && lj < kBT) acc += sm.ds[li][lj];
      }
      if (acc != 0.f) atomicAdd(b.d_rp + wbase + w + a.n_max - 1, acc);
    } else if (tid >= 128) {
      const int t = tid - 128;
      const int li = t >> 1, c0 = (t & 1) * 32;
      // lane l starts at column l of its half: the lanes' reads fall in 32 distinct banks
      const int rot = tid & 31;
      int run_b = sm.bk[li][c0 + rot];
      float run_v = 0.f;
      for (int x = 0; x < 32; ++x) {
        const int c = c0 + ((x + rot) & 31);
        const int bb = sm.bk[li][c];
        if (bb != run_b) {
          if (run_v != 0.f) atomicAdd(&sm.drt[run_b], run_v);
          run_b = bb;
          run_v = 0.f;
        }
        run_v += sm.ds[li][c];
      }
      // the last run goes through the warp aggregate when every lane shares its bucket
      const unsigned same = __match_any_sync(~0u, run_b);
      if (same == ~0u) {
        float x = run_v;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(~0u, x, o);
        if ((tid & 31) == 0 && x != 0.f) atomicAdd(&sm.drt[run_b], x);
      } else if (run_v != 0.f) {
        atomicAdd(&sm.drt[run_b], run_v);
      }
    }

    // d_v += a^T g, d_k += ds^T Q (keys 4 rg .. 4 rg + 3)
#pragma unroll 4
    for (int i = 0; i < kBT; ++i) {
      const float4 av = lds4(&sm.a[i][4 * rg]);
      const float4 dsv = lds4(&sm.ds[i][4 * rg]);
      float gr[DE], qr[DE];
      lds_dims(sm.g[i], dg, gr);
      lds_dims(sm.q[i], dg, qr);
      const float aw[4] = {av.x, av.y, av.z, av.w};
      const float dw[4] = {dsv.x, dsv.y, dsv.z, dsv.w};
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int e = 0; e < DE; ++e) {
          dv[x][e] = fmaf(aw[x], gr[e], dv[x][e]);
          dk[x][e] = fmaf(dw[x], qr[e], dk[x][e]);
        }
    }
    // the next query block's rows load while d_q is formed
    if (qb + 1 < qb_end) fetch(qb + 1);
    // d_q of this query block += alpha ds K (queries 4 rg .. 4 rg + 3)
    float dq[4][DE];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int e = 0; e < DE; ++e) dq[x][e] = 0.f;
#pragma unroll 4
    for (int j = 0; j < kBT; ++j) {
      const float4 dsv = lds4(&sm.dst[j][4 * rg]);
      float kr[DE];
      lds_dims(sm.k[j], dg, kr);
      const float dw[4] = {dsv.x, dsv.y, dsv.z, dsv.w};
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int e = 0; e < DE; ++e) dq[x][e] = fmaf(dw[x], kr[e], dq[x][e]);
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int i = i0 + 4 * rg + x;
      if (i < n) {
#pragma unroll
        for (int e = 0; e < DE; ++e) dq[x][e] *= a.alpha;
        red_add_dims(b.dq + ((size_t)(q0 + i) * a.H + head) * D, dg, dq[x]);
      }
    }
  }
  // this CTA owns d_k and d_v of its keys
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int j = j0 + 4 * rg + x;
    if (j < n) {
      float* pk = b.dk + ((size_t)(q0 + j) * a.H + head) * D;
      float* pv = b.dv + ((size_t)(q0 + j) * a.H + head) * D;
#pragma unroll
      for (int e = 0; e < DE; ++e) {
        pk[dim_of<DE>(dg, e)] = a.alpha * dk[x][e];
        pv[dim_of<DE>(dg, e)] = dv[x][e];
      }
    }
  }
  __syncthreads();
  for (int x = tid; x < a.nb; x += kBwdThreads)
    if (sm.drt[x] != 0.f) atomicAdd(b.d_rt + x, sm.drt[x]);
}

}  // namespace

cudaError_t launch_attn_bwd(const AttnArgs& a, const BucketTable& thr, const float* d_o, float* dq, float* dk,
                            float* dv, float* d_rp, float* d_rt, cudaStream_t s) {
  BwdOut b{d_o, dq, dk, dv, d_rp, d_rt};
  if ((a.d == 32 || a.d == 64 || a.d == 128) && a.T_q > 0) {
    if (cudaMemsetAsync(dq, 0, sizeof(float) * (size_t)a.T_q * a.H * a.d, s) != cudaSuccess) return cudaGetLastError();
    const int max_blocks = (a.n_max + kBT - 1) / kBT;  // key blocks of the longest user
    const dim3 grid(a.B * a.H, max_blocks);            // block 0 of every user first: the longest CTAs lead
    auto go = [&](auto kern, size_t smem) {
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      kern<<<grid, kBwdThreads, smem, s>>>(a, thr, b);
    };
    if (a.d == 32) {
      if (a.in_bf16) go(attn_bwd_tiled_kernel<32, __nv_bfloat16>, sizeof(BwdSmem<32>));
      else go(attn_bwd_tiled_kernel<32, float>, sizeof(BwdSmem<32>));
    } else if (a.d == 64) {
      if (a.in_bf16) go(attn_bwd_tiled_kernel<64, __nv_bfloat16>, sizeof(BwdSmem<64>));
      else go(attn_bwd_tiled_kernel<64, float>, sizeof(BwdSmem<64>));
    } else {
      if (a.in_bf16) go(attn_bwd_tiled_kernel<128, __nv_bfloat16>, sizeof(BwdSmem<128>));
      else go(attn_bwd_tiled_kernel<128, float>, sizeof(BwdSmem<128>));
    }
    return cudaGetLastError();
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long warps = (long long)a.T_q * a.H;
  const int blocks = (int)std::min<long long>((warps + 7) / 8, (long long)sms * 16);
  if (blocks <= 0) return cudaSuccess;
  if (a.in_bf16) {
    attn_bwd_q_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(a, thr, b);
    attn_bwd_kv_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(a, thr, b);
  } else {
    attn_bwd_q_kernel<float><<<blocks, 256, 0, s>>>(a, thr, b);
    attn_bwd_kv_kernel<float><<<blocks, 256, 0, s>>>(a, thr, b);
  }
  return cudaGetLastError();
}

}  // namespace hstu
