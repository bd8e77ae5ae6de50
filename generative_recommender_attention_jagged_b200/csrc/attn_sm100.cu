// HSTU pointwise attention on the sm_100a tensor cores (bf16 in, fp32 accumulate).
//
// One CTA computes one work item: 128 query rows of one (user, head) against
// a range of 128-key tiles (all the tiles the rows need, or one split of them
// in paged mode).  Per key tile:
//
//   S  = Q K^T            tcgen05.mma, A = Q (smem, K-major), B = K (smem, K-major),
//                         fp32 accumulator in tensor memory (128 lanes x 128 columns)
//   P  = SiLU(alpha S + rab_pos[p_i - p_j + N - 1] + rab_ts[bucket(t_i - t_j)]),
//        0 outside the allowed set; computed by four elementwise warps that read
//        S with tcgen05.ld and write P as bf16 pairs back over S (tcgen05.st)
//   O += P V              tcgen05.mma, A = P (tensor memory), B = V (smem, MN-major)
//
// There is no softmax, no row maximum and no rescaling: the weights are
// pointwise ("Generative Recommenders at Scale", Inside NVIDIA's GPU-native
// stack: SiLU weighting instead of softmax, relative attention bias).  The
// 1/N_max factor and the LayerNorm gate are applied by the epilogue kernel;
// for M-FALCON candidates ("HSTU Generative Recommenders: Deploy on GPU
// Cloud", M-FALCON section) the key range stops at the end of the history and
// the candidate's own term a_ii v_i is added by the epilogue, so no tile of
// the candidate x candidate block is ever issued.
//
// Warp roles (192 threads): warps 0-3 elementwise (thread = query row = TMEM
// lane), warp 4 TMA producer (Q once, K/V through a 2-stage ring, paged
// prefix gathered page by page), warp 5 MMA issuer and TMEM owner.  S is
// double-buffered in tensor memory so QK^T of tile t+1 runs while the
// elementwise warps turn tile t into P.  Every wait is bounded (about 2 s),
// after which the kernel reports HSTU_ERR_TIMEOUT and winds down.
//
// Time buckets are exact: the elementwise thread finds the bucket of its
// row's first key by a binary search over integer edges, then walks down the
// edges as the keys get closer in time (timestamps are non-decreasing inside
// a user, so |t_i - t_j| only shrinks along a row); warps whose rows stay in
// one bucket over the whole tile skip the walk.
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "device_common.cuh"

namespace hstu {

namespace {

constexpr int kThreads = 192;
constexpr int kStages = 2;
constexpr int kTileBytes = kTile * 128 * 2;  // 128 rows x 128 bf16 = 32 KB
constexpr int kHalfBytes = kTile * 128;      // 128 rows x 64 bf16: one 128B-swizzled box
constexpr uint32_t kTmemCols = 512;          // S0 [0,128) S1 [128,256) O [256,384)
constexpr int kHeadDim = 128;

struct __align__(1024) Smem {
  uint8_t q[kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  long long thr[kMaxBuckets];
  float rab_ts_half[kMaxBuckets];
  long long ts_tile[2][kTile];
  float win[2][256];
  uint64_t bar_q;
  uint64_t bar_k_full[kStages];
  uint64_t bar_v_full[kStages];
  uint64_t bar_kv_empty[kStages];
  uint64_t bar_s_full[2];
  uint64_t bar_p_full[2];
  uint64_t bar_o_full;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;  // + alignment slack

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void sts_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// elementwise warps agree on a flag (bar.red.and over the 128 threads)
__device__ __forceinline__ bool ew_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const AttnArgs a, const BucketTable tab, const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_kpool,
                      const __grid_constant__ CUtensorMap tm_vpool) {
  const int item_idx = blockIdx.x;
  if (item_idx >= a.hdr->n_items) return;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const WorkItem it = a.items[item_idx];
  // a work list not written by this call's scheduler must not send us out of bounds
  if (it.user < 0 || it.user >= a.B || it.head < 0 || it.head >= a.H || it.split < 0 ||
      it.split >= a.num_splits || it.qtile < 0 ||
      it.qtile * kTile >= a.q_offsets[it.user + 1] - a.q_offsets[it.user])
    return;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const TileGeom g = tile_geom(a, it.user, it.qtile);
  int tb, te;
  split_range(g.n_tiles, it.split, a.num_splits, tb, te);
  const int nt = te - tb;

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.bar_k_full[s], 1);
      mbar_init(&sm.bar_v_full[s], 1);
      mbar_init(&sm.bar_kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.bar_s_full[b], 1);
      mbar_init(&sm.bar_p_full[b], kTile);
    }
    mbar_init(&sm.bar_o_full, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  for (int x = threadIdx.x; x < kMaxBuckets; x += kThreads) {
    sm.thr[x] = tab.thr[x];
    sm.rab_ts_half[x] = x < a.nb ? 0.5f * a.rab_ts[x] : 0.f;
  }
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    if (a.paged) {
      prefetch_tmap(&tm_kpool);
      prefetch_tmap(&tm_vpool);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort;

  if (warp == 4) {
    // ------------------------------------------------------------------ producer
    const int head = it.head;
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.bar_q, kTileBytes);
      tma_load_3d(sm.q, &tm_q, &sm.bar_q, 0, head, g.qrow0);
      tma_load_3d(sm.q + kHalfBytes, &tm_q, &sm.bar_q, 64, head, g.qrow0);
    }
    const int row_base = a.q_offsets[it.user] - g.L;  // row of key position p is row_base + p (p >= L)
    int issued = 0;
    for (int t = 0; t < nt; ++t) {
      const int s = t % kStages;
      const uint32_t ph = (t / kStages) & 1;
      int k0, width;
      key_tile(g, tb + t, k0, width);
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&sm.bar_kv_empty[s], ph ^ 1, abort_flag, a.hdr, 1);
      ok = __shfl_sync(~0u, ok, 0);
      if (!ok) break;
      uint8_t* kd = sm.k[s];
      uint8_t* vd = sm.v[s];
      if (k0 >= g.L) {
        if (lane == 0) {
          const int row = row_base + k0;
          mbar_arrive_expect_tx(&sm.bar_k_full[s], kTileBytes);
          tma_load_3d(kd, &tm_k, &sm.bar_k_full[s], 0, head, row);
          tma_load_3d(kd + kHalfBytes, &tm_k, &sm.bar_k_full[s], 64, head, row);
          mbar_arrive_expect_tx(&sm.bar_v_full[s], kTileBytes);
          tma_load_3d(vd, &tm_v, &sm.bar_v_full[s], 0, head, row);
          tma_load_3d(vd + kHalfBytes, &tm_v, &sm.bar_v_full[s], 64, head, row);
        }
      } else {
        // paged prefix: whole pages by TMA, a partial last page and the rows
        // past the prefix by 16-byte loads / zero stores
        const int P = a.page_size;
        const int full_pages = width / P;
        const int man_lo = full_pages * P;
        const int first_page = k0 / P;
        const int32_t* prow = a.page_table + (size_t)it.user * a.max_pages + first_page;
        if (man_lo < kTile) {
          const int pid = (width > man_lo) ? prow[full_pages] : 0;
          const uint8_t* kpage = static_cast<const uint8_t*>(a.k_pool) + ((size_t)pid * a.H + head) * P * kHeadDim * 2;
          const uint8_t* vpage = static_cast<const uint8_t*>(a.v_pool) + ((size_t)pid * a.H + head) * P * kHeadDim * 2;
          const uint32_t kbase = smem_u32(kd), vbase = smem_u32(vd);
          for (int idx = lane; idx < (kTile - man_lo) * 16; idx += 32) {
            const int r = man_lo + (idx >> 4);
            const int ch = idx & 15;  // 16-byte chunk of the 256-byte row
            const uint32_t off = (ch >> 3) * kHalfBytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
            uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
            if (r < width) {
              const size_t goff = (size_t)(r - man_lo) * kHeadDim * 2 + ch * 16;
              kv = ldg_nc_v4(kpage + goff);
              vv = ldg_nc_v4(vpage + goff);
            }
            sts_v4(kbase + off, kv);
            sts_v4(vbase + off, vv);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          const uint32_t bytes = (uint32_t)full_pages * P * kHeadDim * 2;
          mbar_arrive_expect_tx(&sm.bar_k_full[s], bytes);
          for (int pg = 0; pg < full_pages; ++pg) {
            const int pid = prow[pg];
            tma_load_4d(kd + pg * P * 128, &tm_kpool, &sm.bar_k_full[s], 0, 0, head, pid);
            tma_load_4d(kd + kHalfBytes + pg * P * 128, &tm_kpool, &sm.bar_k_full[s], 64, 0, head, pid);
          }
          mbar_arrive_expect_tx(&sm.bar_v_full[s], bytes);
          for (int pg = 0; pg < full_pages; ++pg) {
            const int pid = prow[pg];
            tma_load_4d(vd + pg * P * 128, &tm_vpool, &sm.bar_v_full[s], 0, 0, head, pid);
            tma_load_4d(vd + kHalfBytes + pg * P * 128, &tm_vpool, &sm.bar_v_full[s], 64, 0, head, pid);
          }
        }
      }
      issued = t + 1;
    }
    // no copy may still be landing in shared memory when the CTA exits
    if (lane == 0) {
      mbar_wait(&sm.bar_q, 0, nullptr, a.hdr, 9);
      for (int t = max(0, issued - kStages); t < issued; ++t) {
        const uint32_t ph = (t / kStages) & 1;
        mbar_wait(&sm.bar_k_full[t % kStages], ph, nullptr, a.hdr, 9);
        mbar_wait(&sm.bar_v_full[t % kStages], ph, nullptr, a.hdr, 9);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 128, 0, 1);
      const uint32_t q_base = smem_u32(sm.q);
      const uint32_t o_tmem = tmem + 256;
      bool ok = nt == 0 || mbar_wait(&sm.bar_q, 0, abort_flag, a.hdr, 2);
      tc_fence_after();
      for (int t = 0; ok && t <= nt; ++t) {
        if (t < nt) {
          const int s = t % kStages;
          const int buf = t & 1;
          ok = mbar_wait(&sm.bar_k_full[s], (t / kStages) & 1, abort_flag, a.hdr, 3);
          if (!ok) break;
          tc_fence_after();
          const uint32_t k_base = smem_u32(sm.k[s]);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            mma_ss(tmem + buf * 128, sw128_desc(q_base + off, 16, 1024), sw128_desc(k_base + off, 16, 1024),
                   idesc_qk, kk > 0);
          }
          mma_commit(&sm.bar_s_full[buf]);
        }
        if (t > 0) {
          const int tp = t - 1;
          const int sp = tp % kStages;
          const int bp = tp & 1;
          ok = mbar_wait(&sm.bar_p_full[bp], (tp >> 1) & 1, abort_flag, a.hdr, 4);
          if (!ok) break;
          ok = mbar_wait(&sm.bar_v_full[sp], (tp / kStages) & 1, abort_flag, a.hdr, 5);
          if (!ok) break;
          tc_fence_after();
          const uint32_t v_base = smem_u32(sm.v[sp]);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(o_tmem, tmem + bp * 128 + kk * 8, sw128_desc(v_base + kk * 2048, kHalfBytes, 1024), idesc_pv,
                   (tp > 0 || kk > 0));
          mma_commit(&sm.bar_kv_empty[sp]);
        }
      }
      mma_commit(&sm.bar_o_full);
      // tensor memory is freed below only after every issued MMA completed
      mbar_wait(&sm.bar_o_full, 0, nullptr, a.hdr, 8);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ elementwise
    const int r = threadIdx.x;  // query row of the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const bool valid = r < g.nq_rows;
    const int i = min(g.qs + r, g.n - 1);  // rows past the user repeat its last row (discarded)
    const int jmax = i < g.h ? i : g.h - 1;
    const int pr = min(i, g.h);
    const int pr_min = min(g.qs, g.h);
    const int xoff = pr - pr_min + 127;
    const long long t_i = a.ts[g.tso + i];
    const float alpha_half = 0.5f * a.alpha;
    const int n_rab = 2 * a.n_max - 1;
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const int buf = t & 1;
      int k0, width;
      key_tile(g, tb + t, k0, width);
      sm.ts_tile[buf][r] = a.ts[g.tso + k0 + min(r, width - 1)];
      const int wb = pr_min - k0 - 127 + a.n_max - 1;
      for (int x = r; x < 256; x += kTile) {
        const int idx = wb + x;
        sm.win[buf][x] = (idx >= 0 && idx < n_rab) ? 0.5f * a.rab_pos[idx] : 0.f;
      }
      ok = mbar_wait(&sm.bar_s_full[buf], (t >> 1) & 1, abort_flag, a.hdr, 6);
      ok = ew_all(ok);  // also publishes ts_tile / win to the other elementwise warps
      if (!ok) break;
      tc_fence_after();
      const int climit = min(jmax - k0, width - 1);  // columns c <= climit are allowed
      const bool need_mask = !__all_sync(~0u, climit >= kTile - 1);
      int b = 0;
      bool uni = true;
      if (climit >= 0) {
        b = bucket_of_dt(sm.thr, t_i - sm.ts_tile[buf][0]);
        uni = b == bucket_of_dt(sm.thr, t_i - sm.ts_tile[buf][climit]);
      }
      const bool walk = !__all_sync(~0u, uni);
      float tsb = sm.rab_ts_half[b];
      long long tlim = t_i + 1 - sm.thr[b];  // bucket drops once t_j > tlim
      const long long* tst = sm.ts_tile[buf];
      const float* win = sm.win[buf];
      const uint32_t s_tmem = tmem + lane_base + buf * 128;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t sr[32];
        tmem_ld32(s_tmem + ch * 32, sr);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float pv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int col = ch * 32 + c + e;
            if (walk) {
              const long long tj = tst[col];
              while (b > 0 && tj > tlim) {
                --b;
                tlim = t_i + 1 - sm.thr[b];
                tsb = sm.rab_ts_half[b];
              }
            }
            const float hb = fmaf(__uint_as_float(sr[c + e]), alpha_half, win[xoff - col] + tsb);
            const float th = tanh_approx(hb);
            float p = fmaf(hb, th, hb);  // SiLU(s) with hb = s/2: hb (1 + tanh hb)
            if (need_mask) p = (col <= climit) ? p : 0.f;
            pv[e] = p;
          }
          pk[c >> 1] = pack_bf16x2(pv[0], pv[1]);
        }
        tmem_st16(s_tmem + ch * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.bar_p_full[buf]);
    }
    if (ok && nt > 0) {
      ok = ew_all(mbar_wait(&sm.bar_o_full, 0, abort_flag, a.hdr, 7));
      tc_fence_after();
    }
    if (ok) {
      float* orow = a.o_ws + (((size_t)it.split * a.T_q + (g.qrow0 + r)) * a.H + it.head) * kHeadDim;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t orr[32];
        if (nt > 0) {
          tmem_ld32(tmem + lane_base + 256 + ch * 32, orr);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) orr[x] = 0u;
        }
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(orow + ch * 32);
#pragma unroll
          for (int x = 0; x < 8; ++x)
            dst[x] = make_float4(__uint_as_float(orr[4 * x]), __uint_as_float(orr[4 * x + 1]),
                                 __uint_as_float(orr[4 * x + 2]), __uint_as_float(orr[4 * x + 3]));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_attn_sm100(const AttnArgs& a, const BucketTable& thr, const CUtensorMap& tm_q,
                              const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_kpool,
                              const CUtensorMap& tm_vpool, cudaStream_t s) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (a.max_items <= 0) return cudaSuccess;
  attn_sm100_kernel<<<a.max_items, kThreads, kSmemBytes, s>>>(a, thr, tm_q, tm_k, tm_v, tm_kpool, tm_vpool);
  return cudaGetLastError();
}

}  // namespace hstu
