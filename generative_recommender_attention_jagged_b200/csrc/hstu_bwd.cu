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
// (exact integer time buckets, expf).  The bias gradients are summed with
// atomics: a warp first folds runs of equal indices of its own row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

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

}  // namespace

cudaError_t launch_attn_bwd(const AttnArgs& a, const BucketTable& thr, const float* d_o, float* dq, float* dk,
                            float* dv, float* d_rp, float* d_rt, cudaStream_t s) {
  BwdOut b{d_o, dq, dk, dv, d_rp, d_rt};
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
