// Backward of the attention core o = A V on the sm_100a tensor cores (bf16
// operands, fp32 accumulate), for bf16 inputs with d = 128.
//
// ("Generative Recommenders at Scale", Inside NVIDIA's GPU-native stack:
// SiLU weighting with relative attention bias; "How Generative Recommenders
// Are Redefining RecSys at Scale", Summary: the models are trained.)  With
// g = dL/do, on the allowed set:
//   a_ij  = SiLU(s_ij) / N_max,  ds_ij = (g_i . v_j) SiLU'(s_ij) / N_max,
//   SiLU'(x) = sig(x) (1 + x (1 - sig(x)))
//   dv_j = sum_i a_ij g_i,  dk_j = alpha sum_i ds_ij q_i,  dq_i = alpha sum_j ds_ij k_j,
//   d rab_pos[p(i) - p(j) + N_max - 1] += ds_ij,  d rab_ts[b(i, j)] += ds_ij.
//
// One CTA per (user, head, block of 128 keys) walks the 128-row query blocks
// that see the keys (all later blocks for history keys; only its own block
// when every key is a candidate).  Tensor memory, lane = key of the block:
//   [0, 128)    S^T = K Q_i^T, then P^T (bf16 pairs) over the columns read
//   [128, 256)  dP^T = V G_i^T, then dS^T (bf16 pairs), then dQ_i = dS K
//               (lane = query row for that product)
//   [256, 384)  dV += P^T G_i        [384, 512)  dK += dS^T Q_i
// G is d_o rounded to bf16 (converted into the workspace first).  Per query
// block: the issuer computes S^T and dP^T (tcgen05 SS, K / V K-major as A,
// Q_i / G_i K-major as B); the elementwise warps (thread = key, warpgroup =
// 32 query columns) form a and ds with the exact bucket and mask, write P^T
// and dS^T back as bf16 and accumulate the bias-table gradients; the issuer
// adds P^T G_i and dS^T Q_i (TS, P^T / dS^T from tensor memory); once those
// have read Q_i, the elementwise warps store dS^T as bf16 over Q_i in
// shared memory (128B-swizzled, query-contiguous), the issuer computes
// dS K (A = dS from shared memory, MN-major), and the elementwise warps add
// that tile to d_q with vector atomics (d_q is zeroed first).  Q_i and G_i
// are double-buffered; K and V stay resident.  Every wait is bounded (about
// 2 s), after which the kernel reports HSTU_ERR_TIMEOUT and winds down.
#include <cuda_bf16.h>
#include <stdint.h>

#include "attn_common.cuh"

namespace hstu {

namespace {

constexpr int kBwEwWarps = 16;
constexpr int kBwProducerWarp = kBwEwWarps;
constexpr int kBwMmaWarp = kBwEwWarps + 1;   // MMA issuer, TMEM owner
constexpr int kBwThreads = 32 * (kBwEwWarps + 2);
constexpr uint32_t kBwTmemCols = 512;
constexpr uint32_t kColDp = 128, kColDv = 256, kColDk = 384;
constexpr int kDrpWin = 256;                 // position differences of one block pair: at most 255

struct __align__(1024) BwdSmemTc {
  uint8_t k[kTileBytes];       // K of the key block [key][d], two 128B-swizzled boxes (d 0-63, 64-127)
  uint8_t v[kTileBytes];
  uint8_t q[2][kTileBytes];    // Q_i; once dK(i) has read it, dS^T(i) [key][query] in the same layout
  uint8_t g[2][kTileBytes];    // G_i = bf16 d_o
  long long thr[kMaxBuckets];
  float rab_ts[kMaxBuckets];
  float drt[kMaxBuckets];      // d rab_ts of this CTA
  float drp[kDrpWin];          // d rab_pos of the current block pair, from its smallest difference
  long long tq[kTile];         // timestamps of the current query block
  float rpw[kDrpWin];          // rab_pos of the current block pair, from its smallest difference
  uint64_t bar_kv;
  uint64_t bar_qg_full[2];     // Q_i and G_i landed in buffer b
  uint64_t bar_qg_free[2];     // every GEMM that read buffer b (and the dS^T written into it) completed
  uint64_t bar_s_full;         // S^T(i), dP^T(i) written
  uint64_t bar_p_full;         // P^T(i), dS^T(i) in tensor memory (16 elementwise warps)
  uint64_t bar_dk_done;        // dV(i), dK(i) completed: Q_i's buffer may take dS^T(i)
  uint64_t bar_ds_full;        // dS^T(i) in shared memory (16 elementwise warps)
  uint64_t bar_dq_full;        // dQ_i part in tensor memory
  uint64_t bar_dq_read;        // dQ_i part read (16 elementwise warps)
  uint64_t bar_acc_full;       // every GEMM completed
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kBwSmemBytes = sizeof(BwdSmemTc) + 1024;
static_assert(kBwSmemBytes <= 227 * 1024, "shared memory budget");

// 32 lanes x 16 columns of 32-bit
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// wait for tcgen05.ld whose destinations are a and b (keeps their uses after the wait)
__device__ __forceinline__ void tmem_wait_ld2(uint32_t (&a)[16], uint32_t (&b)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]),
                 "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]), "+r"(a[13]), "+r"(a[14]),
                 "+r"(a[15]), "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]),
                 "+r"(b[6]), "+r"(b[7]), "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]), "+r"(b[12]),
                 "+r"(b[13]), "+r"(b[14]), "+r"(b[15])
               :
               : "memory");
}
// 32 lanes x 8 columns of 32-bit store
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// the 512 elementwise threads agree on a flag (barrier 1), so that they leave
// the loop together and never split across a later barrier
__device__ __forceinline__ bool bw_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 512, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

struct BwdTcOut {
  const __nv_bfloat16* g;  // d_o as bf16 [T, H, 128]
  float *dq, *dk, *dv, *d_rp, *d_rt;
};

__global__ void __launch_bounds__(kBwThreads, 1)
    attn_bwd_sm100_kernel(const AttnArgs a, const BucketTable tab, const BwdTcOut b,
                          const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g) {
  if (a.hdr->status != 0) return;  // the inputs failed validation
  const int u = blockIdx.x / a.H;
  const int head = blockIdx.x - u * a.H;
  const int q0 = a.q_offsets[u];
  const int n = a.q_offsets[u + 1] - q0;
  const int k0 = blockIdx.y * kTile;  // first key of the block
  if (k0 >= n) return;
  const int h = n - (a.num_cand ? a.num_cand[u] : 0);
  // query blocks from the key block on; a block of candidate keys is seen only by itself
  const int nsteps = k0 >= h ? 1 : (n - k0 + kTile - 1) / kTile;
  extern __shared__ uint8_t smem_raw[];
  BwdSmemTc& sm = aligned_smem<BwdSmemTc>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_kv, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.bar_qg_full[x], 1);
      mbar_init(&sm.bar_qg_free[x], 1);
    }
    mbar_init(&sm.bar_s_full, 1);
    mbar_init(&sm.bar_p_full, kBwEwWarps);
    mbar_init(&sm.bar_dk_done, 1);
    mbar_init(&sm.bar_ds_full, kBwEwWarps);
    mbar_init(&sm.bar_dq_full, 1);
    mbar_init(&sm.bar_dq_read, kBwEwWarps);
    mbar_init(&sm.bar_acc_full, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  for (int x = threadIdx.x; x < kMaxBuckets; x += kBwThreads) {
    sm.thr[x] = tab.thr[x];
    sm.rab_ts[x] = x < a.nb ? a.rab_ts[x] : 0.f;
    sm.drt[x] = 0.f;
  }
  for (int x = threadIdx.x; x < kDrpWin; x += kBwThreads) sm.drp[x] = 0.f;
  if (warp == kBwMmaWarp) {
    tmem_alloc(&sm.tmem_base, kBwTmemCols);
    tmem_relinquish();
  }
  if (warp == kBwProducerWarp && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_g);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort;

  if (warp == kBwProducerWarp) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.bar_kv, 2 * kTileBytes);
      tma_load_3d(sm.k, &tm_k, &sm.bar_kv, 0, head, q0 + k0);
      tma_load_3d(sm.k + kHalfBytes, &tm_k, &sm.bar_kv, 64, head, q0 + k0);
      tma_load_3d(sm.v, &tm_v, &sm.bar_kv, 0, head, q0 + k0);
      tma_load_3d(sm.v + kHalfBytes, &tm_v, &sm.bar_kv, 64, head, q0 + k0);
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        const int bb = i & 1;
        // buffer bb was last used by block i - 2
        if (i >= 2 && !mbar_wait(&sm.bar_qg_free[bb], ((i >> 1) & 1) ^ 1, abort_flag, a.hdr, 40)) break;
        const int row = q0 + k0 + kTile * i;
        mbar_arrive_expect_tx(&sm.bar_qg_full[bb], 2 * kTileBytes);
        tma_load_3d(sm.q[bb], &tm_q, &sm.bar_qg_full[bb], 0, head, row);
        tma_load_3d(sm.q[bb] + kHalfBytes, &tm_q, &sm.bar_qg_full[bb], 64, head, row);
        tma_load_3d(sm.g[bb], &tm_g, &sm.bar_qg_full[bb], 0, head, row);
        tma_load_3d(sm.g[bb] + kHalfBytes, &tm_g, &sm.bar_qg_full[bb], 64, head, row);
        issued = i + 1;
      }
      // no copy may still be landing in shared memory when the CTA exits
      mbar_wait(&sm.bar_kv, 0, nullptr, a.hdr, 41);
      for (int i = max(0, issued - 2); i < issued; ++i)
        mbar_wait(&sm.bar_qg_full[i & 1], (i >> 1) & 1, nullptr, a.hdr, 41);
    }
    __syncwarp();
  } else if (warp == kBwMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_ss = idesc_bf16(kTile, kTile, 0, 0);  // A, B K-major
      constexpr uint32_t idesc_ts = idesc_bf16(kTile, kTile, 0, 1);  // B MN-major
      constexpr uint32_t idesc_dq = idesc_bf16(kTile, kTile, 1, 1);  // A, B MN-major
      const uint32_t k_base = smem_u32(sm.k), v_base = smem_u32(sm.v);
      bool ok = mbar_wait(&sm.bar_kv, 0, abort_flag, a.hdr, 43);
      for (int i = 0; ok && i < nsteps; ++i) {
        const int bb = i & 1;
        const uint32_t qb = smem_u32(sm.q[bb]), gb = smem_u32(sm.g[bb]);
        ok = mbar_wait(&sm.bar_qg_full[bb], (i >> 1) & 1, abort_flag, a.hdr, 44);
        if (!ok) break;
        tc_fence_after();
        // S^T = K Q_i^T (lane = key, column = query)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_ss(tmem, sw128_desc(k_base + off, 16, 1024), sw128_desc(qb + off, 16, 1024), idesc_ss, kk > 0);
        }
        // columns 128.. hold the previous block's dQ part until it was read
        if (i > 0) {
          ok = mbar_wait(&sm.bar_dq_read, (i - 1) & 1, abort_flag, a.hdr, 45);
          if (!ok) break;
          tc_fence_after();
        }
        // dP^T = V G_i^T
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_ss(tmem + kColDp, sw128_desc(v_base + off, 16, 1024), sw128_desc(gb + off, 16, 1024), idesc_ss,
                 kk > 0);
        }
        mma_commit(&sm.bar_s_full);
        ok = mbar_wait(&sm.bar_p_full, i & 1, abort_flag, a.hdr, 46);
        if (!ok) break;
        tc_fence_after();
        // dV += P^T G_i and dK += dS^T Q_i: the bf16 pairs of queries
        // 16 kk .. 16 kk + 15 sit at column 32 (kk >> 1) + 8 (kk & 1)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + kColDv, tmem + 32 * (kk >> 1) + 8 * (kk & 1),
                 sw128_desc(gb + kk * 2048, kHalfBytes, 1024), idesc_ts, (i > 0 || kk > 0));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + kColDk, tmem + kColDp + 32 * (kk >> 1) + 8 * (kk & 1),
                 sw128_desc(qb + kk * 2048, kHalfBytes, 1024), idesc_ts, (i > 0 || kk > 0));
        mma_commit(&sm.bar_dk_done);
        ok = mbar_wait(&sm.bar_ds_full, i & 1, abort_flag, a.hdr, 46);
        if (!ok) break;
        tc_fence_after();
        // dQ_i part = dS K: A = dS^T in Q_i's buffer read query-contiguous
        // (keys 16 kk .. 16 kk + 15), B = K read with d contiguous
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + kColDp, sw128_desc(qb + kk * 2048, kHalfBytes, 1024),
                 sw128_desc(k_base + kk * 2048, kHalfBytes, 1024), idesc_dq, kk > 0);
        mma_commit(&sm.bar_dq_full);
        mma_commit(&sm.bar_qg_free[bb]);
      }
      mma_commit(&sm.bar_acc_full);
      // tensor memory is freed below only after every issued MMA completed
      mbar_wait(&sm.bar_acc_full, 0, nullptr, a.hdr, 48);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ elementwise (thread = key)
    const int grp = warp >> 2;                // query columns 32 grp .. 32 grp + 31 of each block
    const int r = threadIdx.x & (kTile - 1);  // TMEM lane: key k0 + r (query qs + r for dQ)
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int j = k0 + r;
    const bool jv = j < n;
    const int jc = min(j, n - 1);
    const long long t_j = a.ts[q0 + jc];
    const int p_j = min(jc, h);
    const float alpha = a.alpha;
    const float inv_n = 1.f / (float)a.n_max;
    // time bucket of the key's next allowed query: queries only grow later,
    // so the walk only moves up (wb < 0: not started)
    int wb = -1;
    unsigned long long wlim = 0;
    float wrt = 0.f;
    int run_b = -1;  // a run of equal buckets not yet added to d rab_ts
    float run_v = 0.f;
    bool ok = true;
    for (int i = 0; i < nsteps; ++i) {
      const int qs = k0 + kTile * i;
      const int lo = min(qs, h) - min(k0 + kTile - 1, h);  // smallest p(i) - p(j) of the block pair
      // the block's query timestamps and the pair's position-bias window into
      // shared memory (the previous block's were last read before the
      // barrier that followed its elementwise step)
      if (threadIdx.x < kTile) {
        sm.tq[threadIdx.x] = a.ts[q0 + min(qs + (int)threadIdx.x, n - 1)];
      } else if (threadIdx.x < kTile + kDrpWin - 1) {
        const int idx = lo + ((int)threadIdx.x - kTile) + a.n_max - 1;
        sm.rpw[threadIdx.x - kTile] = (idx >= 0 && idx <= 2 * a.n_max - 2) ? __ldg(a.rab_pos + idx) : 0.f;
      }
      ok = mbar_wait(&sm.bar_s_full, i & 1, abort_flag, a.hdr, 49);
      ok = bw_all(ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t dsk[16];  // dS^T of this thread's 32 queries, bf16 pairs
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t sr[16], dp[16];
        tmem_ld16(tmem + lane_base + 32 * grp + 16 * hf, sr);
        tmem_ld16(tmem + lane_base + kColDp + 32 * grp + 16 * hf, dp);
        tmem_wait_ld2(sr, dp);
        uint32_t pk[8];
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          float pv[2], dv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int qi = qs + 32 * grp + 16 * hf + c + e;
            const bool allowed = jv && qi < n && (qi < h ? j <= qi : (j < h || j == qi));
            pv[e] = 0.f;
            dv[e] = 0.f;
            if (allowed) {
              const long long t_i = sm.tq[qi - qs];
              const unsigned long long udt = (unsigned long long)t_i - (unsigned long long)t_j;
              if (wb < 0) {
                wb = min(bucket_of_dt(sm.thr, t_i - t_j), a.nb - 1);
                wlim = (unsigned long long)(sm.thr[min(wb + 1, kMaxBuckets - 1)] - 1);
                wrt = sm.rab_ts[wb];
              }
              while (wb < a.nb - 1 && udt >= wlim) {
                ++wb;
                wlim = (unsigned long long)(sm.thr[min(wb + 1, kMaxBuckets - 1)] - 1);
                wrt = sm.rab_ts[wb];
              }
              const int pi = min(qi, h);
              const float s = fmaf(alpha, __uint_as_float(sr[c + e]), sm.rpw[pi - p_j - lo] + wrt);
              const float sg = fmaf(0.5f, tanh_approx(0.5f * s), 0.5f);  // sigmoid(s)
              pv[e] = s * sg * inv_n;
              dv[e] = __uint_as_float(dp[c + e]) * sg * fmaf(s, 1.f - sg, 1.f) * inv_n;
              atomicAdd(&sm.drp[pi - p_j - lo], dv[e]);
              if (wb != run_b) {
                if (run_b >= 0) atomicAdd(&sm.drt[run_b], run_v);
                run_b = wb;
                run_v = 0.f;
              }
              run_v += dv[e];
            }
          }
          pk[c >> 1] = pack_bf16x2(pv[0], pv[1]);
          dsk[8 * hf + (c >> 1)] = pack_bf16x2(dv[0], dv[1]);
        }
        // P^T over S^T, dS^T over dP^T: columns this warpgroup has read
        tmem_st8(tmem + lane_base + 32 * grp + 8 * hf, pk);
        tmem_st8(tmem + lane_base + kColDp + 32 * grp + 8 * hf, &dsk[8 * hf]);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar_p_full);
      ok = mbar_wait(&sm.bar_dk_done, i & 1, abort_flag, a.hdr, 50);
      ok = bw_all(ok);  // every thread's d rab_pos atomics of the pair are done too
      if (!ok) break;
      if (threadIdx.x < kDrpWin - 1) {
        const float x = sm.drp[threadIdx.x];
        if (x != 0.f) {
          atomicAdd(b.d_rp + (lo + (int)threadIdx.x + a.n_max - 1), x);
          sm.drp[threadIdx.x] = 0.f;
        }
      }
      // dS^T into Q_i's buffer (dK has read Q_i): row = key, 128 queries as
      // two 128B-swizzled halves, 16-byte chunk c of a row at c ^ (row & 7)
      const uint32_t qrow = smem_u32(sm.q[i & 1]) + (grp >> 1) * kHalfBytes + r * 128;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        sts_v4(qrow + (((4 * (grp & 1) + e) ^ (r & 7)) << 4),
               make_uint4(dsk[4 * e], dsk[4 * e + 1], dsk[4 * e + 2], dsk[4 * e + 3]));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar_ds_full);
      ok = mbar_wait(&sm.bar_dq_full, i & 1, abort_flag, a.hdr, 51);
      ok = bw_all(ok);
      if (!ok) break;
      tc_fence_after();
      // dQ part: lane = query row qs + r, columns = d
      uint32_t dq[32];
      tmem_ld32(tmem + lane_base + kColDp + 32 * grp, dq);
      tmem_wait_ld(dq);
      if (qs + r < n) {
        float* dst = b.dq + ((size_t)(q0 + qs + r) * a.H + head) * kHeadDim + 32 * grp;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          red_add_v4(dst + 4 * e, alpha * __uint_as_float(dq[4 * e]), alpha * __uint_as_float(dq[4 * e + 1]),
                     alpha * __uint_as_float(dq[4 * e + 2]), alpha * __uint_as_float(dq[4 * e + 3]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar_dq_read);
    }
    if (run_b >= 0) atomicAdd(&sm.drt[run_b], run_v);
    if (ok) ok = mbar_wait(&sm.bar_acc_full, 0, abort_flag, a.hdr, 52);
    ok = bw_all(ok);
    if (ok) {
      tc_fence_after();
      // dV and dK rows of the block's keys (fp32)
      uint32_t acc[32];
      tmem_ld32(tmem + lane_base + kColDv + 32 * grp, acc);
      tmem_wait_ld(acc);
      if (jv) {
        float4* dst = reinterpret_cast<float4*>(b.dv + ((size_t)(q0 + j) * a.H + head) * kHeadDim + 32 * grp);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dst[e] = make_float4(__uint_as_float(acc[4 * e]), __uint_as_float(acc[4 * e + 1]),
                               __uint_as_float(acc[4 * e + 2]), __uint_as_float(acc[4 * e + 3]));
      }
      tmem_ld32(tmem + lane_base + kColDk + 32 * grp, acc);
      tmem_wait_ld(acc);
      if (jv) {
        float4* dst = reinterpret_cast<float4*>(b.dk + ((size_t)(q0 + j) * a.H + head) * kHeadDim + 32 * grp);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dst[e] = make_float4(alpha * __uint_as_float(acc[4 * e]), alpha * __uint_as_float(acc[4 * e + 1]),
                               alpha * __uint_as_float(acc[4 * e + 2]), alpha * __uint_as_float(acc[4 * e + 3]));
      }
    }
    bw_all(true);  // every run is in the CTA's d rab_ts histogram
    if (threadIdx.x < a.nb) {
      const float x = sm.drt[threadIdx.x];
      if (x != 0.f) atomicAdd(b.d_rt + threadIdx.x, x);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kBwMmaWarp) tmem_dealloc(tmem, kBwTmemCols);
}

__global__ void d_o_to_bf16_kernel(const float4* __restrict__ src, uint2* __restrict__ dst, long long n4) {
  for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < n4; x += (long long)gridDim.x * blockDim.x) {
    const float4 v = src[x];
    dst[x] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

}  // namespace

bool attn_bwd_sm100_supported(const AttnArgs& a) { return a.in_bf16 && a.d == kHeadDim; }

cudaError_t launch_attn_bwd_sm100(const AttnArgs& a, const BucketTable& thr, const float* d_o, void* g_bf16,
                                  const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                  const CUtensorMap& tm_g, float* dq, float* dk, float* dv, float* d_rp,
                                  float* d_rt, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static unsigned long long attr_set = 0;  // one bit per device
  if (dev < 64 && !(attr_set & (1ull << dev))) {
    cudaError_t e =
        cudaFuncSetAttribute(attn_bwd_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBwSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  if (a.T_q <= 0) return cudaSuccess;
  const long long n4 = (long long)a.T_q * a.H * kHeadDim / 4;
  const int cblocks = (int)std::min<long long>((n4 + 255) / 256, (long long)sms * 8);
  d_o_to_bf16_kernel<<<cblocks, 256, 0, s>>>(reinterpret_cast<const float4*>(d_o), static_cast<uint2*>(g_bf16), n4);
  if (cudaMemsetAsync(dq, 0, sizeof(float) * (size_t)a.T_q * a.H * kHeadDim, s) != cudaSuccess)
    return cudaGetLastError();
  BwdTcOut b{static_cast<const __nv_bfloat16*>(g_bf16), dq, dk, dv, d_rp, d_rt};
  // key block 0 of every (user, head) first: the CTAs with the most query blocks lead
  const dim3 grid(a.B * a.H, (a.n_max + kTile - 1) / kTile);
  attn_bwd_sm100_kernel<<<grid, kBwThreads, kBwSmemBytes, s>>>(a, thr, b, tm_q, tm_k, tm_v, tm_g);
  return cudaGetLastError();
}

}  // namespace hstu
