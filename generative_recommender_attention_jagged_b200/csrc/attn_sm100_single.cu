// HSTU pointwise attention on the sm_100a tensor cores, one query tile per CTA.
//
// The same arithmetic as attn_sm100.cu (S = Q K^T by tcgen05.mma, bias +
// SiLU + mask in registers, O += P V with P in tensor memory, exact time
// buckets), organised for work items of a single 128-row query tile against a
// long key range: the paged incremental mode, where a request's few new
// actions and candidates attend to a cached prefix of thousands of keys
// ("Recomendador generativo HSTU com Dynamo-Triton", KV cache section: only
// the new tokens are computed against the paged GPU cache).  That workload is
// bound by reading the cached K and V from HBM, so the kernel keeps as many
// pages in flight per SM as shared memory allows and keeps every warp on the
// one tile:
//
//   - S is double-buffered in tensor memory (S0, S1, O: 3 x 128 columns):
//     S(t + 1) is computed while the elementwise warps turn S(t) into P(t),
//     so the tensor core and the elementwise warps overlap within one tile.
//   - the four elementwise warpgroups each take one 32-key chunk of every key
//     tile (thread = query row = TMEM lane), so all 16 warps work on the tile.
//   - K and V have separate rings (3 and 2 stages) and separate producer
//     warps: a K stage is refilled as soon as the S GEMM that read it
//     completed, a V stage once its A.V GEMM completed, which gives each page
//     read two or more key tiles of lead time.  The key tiles' metadata (timestamps and
//     position window) has its own 3-stage ring and producer warp, released
//     by the elementwise warps, so it never waits behind a page read.
//
// Warp roles (640 threads): warps 0-15 elementwise (warpgroup g = chunk g),
// warp 16 the K producer (Q once, then K tiles: whole pages by TMA, a partial
// last page and the rows past the prefix by 16-byte loads), warp 17 the V
// producer (V tiles likewise), warp 18 the MMA issuer (and the owner of
// tensor memory), warp 19 the metadata producer.  Warpgroup g packs its P
// into the first 16 of its own 32 S columns (no other group reads them).  The
// issuer's order per key tile t: wait P(t), O += P(t) V(t), then S(t + 2)
// into the buffer P(t) occupied (tcgen05 MMAs of one thread run in order, so
// the A.V GEMM has read P(t) before S(t + 2) overwrites it).  Every wait is
// bounded (about 2 s), after which the kernel reports HSTU_ERR_TIMEOUT and
// winds down.
#include <cuda_bf16.h>
#include <stdint.h>

#include "attn_common.cuh"

namespace hstu {

namespace {

constexpr int kEwWarps = 16;              // 4 warpgroups: one 32-key chunk of every key tile each
constexpr int kKProducerWarp = kEwWarps;
constexpr int kVProducerWarp = kEwWarps + 1;
constexpr int kMmaWarp = kEwWarps + 2;    // MMA issuer, TMEM owner
constexpr int kMetaWarp = kEwWarps + 3;
constexpr int kThreads = 32 * (kEwWarps + 4);
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kMetaStages = 3;
constexpr uint32_t kTmemCols = 512;       // S0 [0,128) S1 [128,256) O [256,384)

struct __align__(1024) SmemSingle {
  uint8_t q[kTileBytes];
  uint8_t k[kKStages][kTileBytes];
  uint8_t v[kVStages][kTileBytes];
  Meta meta[kMetaStages];
  long long thr[kMaxBuckets];
  float rab_ts_half[kMaxBuckets];
  uint4 oct[32];
  uint32_t win_rs[kWinLoads * 16];  // metadata producer scratch: R as 416 bf16
  uint64_t bar_q;
  uint64_t bar_k_full[kKStages];
  uint64_t bar_v_full[kVStages];
  uint64_t bar_meta_full[kMetaStages];   // 32 producer lanes
  uint64_t bar_meta_empty[kMetaStages];  // released by the 16 elementwise warps
  uint64_t bar_k_empty[kKStages];   // released by the S GEMM that read it
  uint64_t bar_v_empty[kVStages];   // released by the A.V GEMM that read it
  uint64_t bar_s_full[2];           // S buffer b written
  uint64_t bar_p_full[2];           // P in buffer b written (all 512 elementwise threads)
  uint64_t bar_o_full;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytesSingle = sizeof(SmemSingle) + 1024;  // + alignment slack
static_assert(kSmemBytesSingle <= 227 * 1024, "shared memory budget");

// Page ids of key tile t of the item for a producer warp: lane l holds the
// id of the tile's page l (the tile spans at most 128 / 8 = 16 pages), loaded
// one tile ahead so that no page-id load sits in front of a TMA copy.
__device__ __forceinline__ int tile_page_id(const AttnArgs& a, const TileGeom& g, int user, int t, int lane) {
  int k0, width;
  key_tile(g, t, k0, width);
  if (k0 >= g.L) return 0;
  const int pages = (width + a.page_size - 1) / a.page_size;
  return lane < pages ? a.page_table[(size_t)user * a.max_pages + k0 / a.page_size + lane] : 0;
}

// One key tile's K or V rows into a stage: whole pages by TMA (4-D boxes of
// one page x 64 elements of one head), a partial last page and the rows past
// the prefix by 16-byte loads and zero stores, new-token tiles by TMA.
// Called by all lanes of a producer warp (lane l holding page id l);
// lane 0 issues the TMA copies.
__device__ __forceinline__ void load_kv_tile(const AttnArgs& a, const TileGeom& g, int head, int row_base, int k0,
                                             int width, int my_pid, const CUtensorMap* tm_rows,
                                             const CUtensorMap* tm_pool, const void* pool, uint8_t* dst,
                                             uint64_t* bar, int lane) {
  if (k0 >= g.L) {
    if (lane == 0) {
      const int row = row_base + k0;
      mbar_arrive_expect_tx(bar, kTileBytes);
      tma_load_3d(dst, tm_rows, bar, 0, head, row);
      tma_load_3d(dst + kHalfBytes, tm_rows, bar, 64, head, row);
    }
    return;
  }
  const int P = a.page_size;
  const int full_pages = width / P;
  const int man_lo = full_pages * P;
  if (man_lo < kTile) {
    const int pid = __shfl_sync(~0u, my_pid, min(full_pages, 31));  // id 0 when no partial page
    const uint8_t* page = static_cast<const uint8_t*>(pool) + ((size_t)pid * a.H + head) * P * kHeadDim * 2;
    const uint32_t base = smem_u32(dst);
    for (int idx = lane; idx < (kTile - man_lo) * 16; idx += 32) {
      const int r = man_lo + (idx >> 4);
      const int ch = idx & 15;  // 16-byte chunk of the 256-byte row
      const uint32_t off = (ch >> 3) * kHalfBytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
      uint4 val = make_uint4(0, 0, 0, 0);
      if (r < width) val = ldg_nc_v4(page + (size_t)(r - man_lo) * kHeadDim * 2 + ch * 16);
      sts_v4(base + off, val);
    }
    fence_proxy_async_smem();
  }
  __syncwarp();
  if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)full_pages * P * kHeadDim * 2);
  for (int pg = 0; pg < full_pages; ++pg) {
    const int pid = __shfl_sync(~0u, my_pid, pg);
    if (lane == 0) {
      tma_load_4d(dst + pg * P * 128, tm_pool, bar, 0, 0, head, pid);
      tma_load_4d(dst + kHalfBytes + pg * P * 128, tm_pool, bar, 64, 0, head, pid);
    }
  }
}

template <bool PRECISE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_single_kernel(const AttnArgs a, const BucketTable tab, const __grid_constant__ CUtensorMap tm_q,
                             const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                             const __grid_constant__ CUtensorMap tm_kpool,
                             const __grid_constant__ CUtensorMap tm_vpool) {
  const int item_idx = blockIdx.x;
  if (item_idx >= a.hdr->n_items) return;
  extern __shared__ uint8_t smem_raw[];
  SmemSingle& sm = aligned_smem<SmemSingle>(smem_raw);

  const WorkItem it = a.items[item_idx];
  // a work list not written by this call's scheduler must not send us out of bounds
  if (it.user < 0 || it.user >= a.B || it.head < 0 || it.head >= a.H || it.split < 0 ||
      it.split >= a.num_splits || it.qtile < 0 || it.qtile * kTile >= a.q_offsets[it.user + 1] - a.q_offsets[it.user])
    return;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const TileGeom g = tile_geom(a, it.user, it.qtile);
  int tb, te;
  split_range(g.n_tiles, it.split, a.num_splits, tb, te);
  const int cnt = max(0, te - tb);            // key tiles of this item
  const int prmin = min(g.qs, g.h);           // smallest query position of the tile

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&sm.bar_k_full[s], 1);
      mbar_init(&sm.bar_k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&sm.bar_v_full[s], 1);
      mbar_init(&sm.bar_v_empty[s], 1);
    }
    for (int s = 0; s < kMetaStages; ++s) {
      mbar_init(&sm.bar_meta_full[s], 32);
      mbar_init(&sm.bar_meta_empty[s], kEwWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.bar_s_full[b], 1);
      mbar_init(&sm.bar_p_full[b], 32 * kEwWarps);
    }
    mbar_init(&sm.bar_o_full, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kKProducerWarp && lane == 0) {
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
  const int head = it.head;
  const int row_base = a.q_offsets[it.user] - g.L;  // row of key position p is row_base + p (p >= L)

  if (warp == kKProducerWarp) {
    // ------------------------------------------------------------------ K producer
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.bar_q, kTileBytes);
      tma_load_3d(sm.q, &tm_q, &sm.bar_q, 0, head, g.qrow0);
      tma_load_3d(sm.q + kHalfBytes, &tm_q, &sm.bar_q, 64, head, g.qrow0);
    }
    int issued = 0;
    int pid = cnt > 0 && a.paged ? tile_page_id(a, g, it.user, tb, lane) : 0;
    for (int t = 0; t < cnt; ++t) {
      const int s = t % kKStages;
      bool ok = true;
      // the stage's previous tile (t - 3) is released by its S GEMM
      if (lane == 0 && t >= kKStages)
        ok = mbar_wait(&sm.bar_k_empty[s], ((t / kKStages) & 1) ^ 1, abort_flag, a.hdr, 1);
      ok = __shfl_sync(~0u, ok, 0);
      if (!ok) break;
      int k0, width;
      key_tile(g, tb + t, k0, width);
      load_kv_tile(a, g, head, row_base, k0, width, pid, &tm_k, &tm_kpool, a.k_pool, sm.k[s], &sm.bar_k_full[s],
                   lane);
      if (t + 1 < cnt && a.paged) pid = tile_page_id(a, g, it.user, tb + t + 1, lane);
      issued = t + 1;
    }
    // no copy may still be landing in shared memory when the CTA exits
    if (lane == 0) {
      mbar_wait(&sm.bar_q, 0, nullptr, a.hdr, 9);
      for (int t = max(0, issued - kKStages); t < issued; ++t)
        mbar_wait(&sm.bar_k_full[t % kKStages], (t / kKStages) & 1, nullptr, a.hdr, 9);
    }
    __syncwarp();
  } else if (warp == kVProducerWarp) {
    // ------------------------------------------------------------------ V producer
    int issued = 0;
    int pid = cnt > 0 && a.paged ? tile_page_id(a, g, it.user, tb, lane) : 0;
    for (int t = 0; t < cnt; ++t) {
      const int s = t % kVStages;
      bool ok = true;
      // the stage's previous tile (t - 2) is released by its A.V GEMM
      if (lane == 0 && t >= kVStages)
        ok = mbar_wait(&sm.bar_v_empty[s], ((t / kVStages) & 1) ^ 1, abort_flag, a.hdr, 1);
      ok = __shfl_sync(~0u, ok, 0);
      if (!ok) break;
      int k0, width;
      key_tile(g, tb + t, k0, width);
      load_kv_tile(a, g, head, row_base, k0, width, pid, &tm_v, &tm_vpool, a.v_pool, sm.v[s], &sm.bar_v_full[s],
                   lane);
      if (t + 1 < cnt && a.paged) pid = tile_page_id(a, g, it.user, tb + t + 1, lane);
      issued = t + 1;
    }
    if (lane == 0)
      for (int t = max(0, issued - kVStages); t < issued; ++t)
        mbar_wait(&sm.bar_v_full[t % kVStages], (t / kVStages) & 1, nullptr, a.hdr, 9);
    __syncwarp();
  } else if (warp == kMetaWarp) {
    // ------------------------------------------------------------------ metadata producer
    const int n_rab = 2 * a.n_max - 1;
    // Per-tile metadata (key timestamps, position-bias window) is loaded into
    // registers one tile ahead, so its global-load latency hides behind the
    // wait for a free stage.  Lane l holds timestamps of columns l + 32k and
    // window values R[l + 32k].
    long long mts[4];
    float mwin[kWinLoads];
    auto load_meta = [&](int t) {
      int k0, width;
      key_tile(g, tb + t, k0, width);
#pragma unroll
      for (int k = 0; k < 4; ++k) mts[k] = a.ts[g.tso + k0 + min(lane + 32 * k, width - 1)];
      const int g0 = prmin + 255 - k0 + a.n_max - 1;  // rab_pos index of R[0]
#pragma unroll
      for (int k = 0; k < kWinLoads; ++k) {
        const int idx = g0 - (lane + 32 * k);
        mwin[k] = (idx >= 0 && idx < n_rab) ? 0.5f * __ldg(a.rab_pos + idx) : 0.f;
      }
    };
    if (cnt > 0) load_meta(0);
    for (int t = 0; t < cnt; ++t) {
      const int s = t % kMetaStages;
      bool ok = true;
      // the stage's previous tile (t - 3) is released by the elementwise warps
      if (lane == 0 && t >= kMetaStages)
        ok = mbar_wait(&sm.bar_meta_empty[s], ((t / kMetaStages) & 1) ^ 1, abort_flag, a.hdr, 1);
      ok = __shfl_sync(~0u, ok, 0);
      if (!ok) break;
      Meta& m = sm.meta[s];
#pragma unroll
      for (int k = 0; k < 4; ++k) m.ts[lane + 32 * k] = mts[k];
      // window: R as bf16 into the scratch row, then the eight shifted copies
      // (16-byte chunk f of copy p = R[8f + p .. 8f + p + 7]) by funnel shifts
      __syncwarp();
      uint16_t* rs16 = reinterpret_cast<uint16_t*>(sm.win_rs);
#pragma unroll
      for (int k = 0; k < kWinLoads; ++k) rs16[lane + 32 * k] = __bfloat16_as_ushort(__float2bfloat16_rn(mwin[k]));
      __syncwarp();
      for (int q = lane; q < kWinChunks * 8; q += 32) {
        const int f = q >> 3, p = q & 7;
        const int wb = 4 * f + (p >> 1);
        const uint32_t sh = 16u * (p & 1);
        const uint32_t x0 = sm.win_rs[wb], x1 = sm.win_rs[wb + 1], x2 = sm.win_rs[wb + 2],
                       x3 = sm.win_rs[wb + 3], x4 = sm.win_rs[wb + 4];
        m.win[f][p] = make_uint4(__funnelshift_r(x0, x1, sh), __funnelshift_r(x1, x2, sh),
                                 __funnelshift_r(x2, x3, sh), __funnelshift_r(x3, x4, sh));
      }
      mbar_arrive(&sm.bar_meta_full[s]);
      if (t + 1 < cnt) load_meta(t + 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 128, 0, 1);
      // S(t) = Q K(t)^T over 128 keys into buffer t & 1; its K stage is
      // released when it completes
      auto issue_s = [&](int t) {
        const uint32_t q_base = smem_u32(sm.q);
        const uint32_t k_base = smem_u32(sm.k[t % kKStages]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_ss(tmem + (t & 1) * 128, sw128_desc(q_base + off, 16, 1024), sw128_desc(k_base + off, 16, 1024),
                 idesc_qk, kk > 0);
        }
        mma_commit(&sm.bar_s_full[t & 1]);
        mma_commit(&sm.bar_k_empty[t % kKStages]);
      };
      // O += P(t) V(t): the P of keys 16 kk .. 16 kk + 15 sits at column
      // 32 (kk >> 1) + 8 (kk & 1) of buffer t & 1 (warpgroup kk >> 1 packed
      // its 32 keys into the first 16 of its own 32 columns)
      auto issue_pv = [&](int t) {
        const uint32_t v_base = smem_u32(sm.v[t % kVStages]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + 256, tmem + (t & 1) * 128 + (kk >> 1) * 32 + (kk & 1) * 8,
                 sw128_desc(v_base + kk * 2048, kHalfBytes, 1024), idesc_pv, (t > 0 || kk > 0));
        mma_commit(&sm.bar_v_empty[t % kVStages]);
      };
      bool ok = cnt == 0 || mbar_wait(&sm.bar_q, 0, abort_flag, a.hdr, 2);
      for (int t = 0; ok && t < min(cnt, 2); ++t) {
        ok = mbar_wait(&sm.bar_k_full[t], 0, abort_flag, a.hdr, 3);
        if (!ok) break;
        tc_fence_after();
        issue_s(t);
      }
      for (int t = 0; ok && t < cnt; ++t) {
        ok = mbar_wait(&sm.bar_p_full[t & 1], (t >> 1) & 1, abort_flag, a.hdr, 4);
        if (ok) ok = mbar_wait(&sm.bar_v_full[t % kVStages], (t / kVStages) & 1, abort_flag, a.hdr, 5);
        if (!ok) break;
        tc_fence_after();
        issue_pv(t);
        if (t + 2 < cnt) {
          ok = mbar_wait(&sm.bar_k_full[(t + 2) % kKStages], ((t + 2) / kKStages) & 1, abort_flag, a.hdr, 3);
          if (!ok) break;
          tc_fence_after();
          issue_s(t + 2);
        }
      }
      mma_commit(&sm.bar_o_full);
      // tensor memory is freed below only after every issued MMA completed
      mbar_wait(&sm.bar_o_full, 0, nullptr, a.hdr, 8);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ elementwise
    // the bucket tables are read only here: copied while the producers start
    // their loads, then the 512 elementwise threads meet at barrier 5
    for (int x = threadIdx.x; x < kMaxBuckets; x += 32 * kEwWarps) {
      sm.thr[x] = tab.thr[x];
      sm.rab_ts_half[x] = x < a.nb ? 0.5f * a.rab_ts[x] : 0.f;
    }
    if (threadIdx.x < 32)
      sm.oct[threadIdx.x] = make_uint4(tab.oct[threadIdx.x][0], tab.oct[threadIdx.x][1], tab.oct[threadIdx.x][2],
                                       tab.oct[threadIdx.x][3]);
    named_bar_sync(5, 32 * kEwWarps);
    const int grp = warp >> 2;                // warpgroup = 32-key chunk of every key tile
    const int r = threadIdx.x & (kTile - 1);  // query row of the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int i = min(g.qs + r, g.n - 1);     // rows past the user repeat its last row (discarded)
    const int jmax = i < g.h ? i : g.h - 1;
    const int pr = min(i, g.h);
    const int zb = prmin + 255 - pr;          // window element of column 0 (see Meta)
    const float alpha_half = 0.5f * a.alpha;
    const int col0 = 32 * grp;
    Walk w;
    w.t_i = a.ts[g.tso + i];
    w.b = 0;
    w.tlim = 0;
    w.tsb = 0.f;
    bool ok = true;
    for (int t = 0; t < cnt; ++t) {
      const int s = t % kMetaStages;
      const int b = t & 1;
      int k0, width;
      key_tile(g, tb + t, k0, width);
      ok = mbar_wait(&sm.bar_meta_full[s], (t / kMetaStages) & 1, abort_flag, a.hdr, 6);
      ok = ok && mbar_wait(&sm.bar_s_full[b], (t >> 1) & 1, abort_flag, a.hdr, 6);
      ok = ew_all(ok, grp);
      if (!ok) break;
      tc_fence_after();
      const Meta& m = sm.meta[s];
      const int climit = min(jmax - k0, width - 1);  // columns c <= climit are allowed
      const uint32_t s_tmem = tmem + lane_base + b * 128;
      uint32_t sr[32];
      tmem_ld32(s_tmem + col0, sr);
      if (t == 0) {
        // the walk starts at this warpgroup's first column and only moves right
        w.b = bucket_of_dt(sm.thr, w.t_i - m.ts[min(col0, width - 1)]);
        w.tlim = w.t_i + 1 - sm.thr[w.b];
        w.tsb = sm.rab_ts_half[w.b];
      }
      const bool need_mask = !__all_sync(~0u, climit >= col0 + 31);
      int pos;
      float tsb_lo;
      const int mode = chunk_mode(w, m.ts, col0, climit, sm.thr, sm.rab_ts_half, pos, tsb_lo);
      const int z0 = zb + col0;
      const uint32_t wbase = smem_u32(&m.win[z0 >> 3][z0 & 7]);
      uint32_t pw[16];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint4 v4 = lds_v4(wbase + k * 8 * 16);
        pw[4 * k] = v4.x;
        pw[4 * k + 1] = v4.y;
        pw[4 * k + 2] = v4.z;
        pw[4 * k + 3] = v4.w;
      }
      tmem_wait_ld(sr);
      uint32_t pk[16];
      if (need_mask)
        silu_chunk_mode<true, PRECISE>(mode, sr, pw, pk, m.ts, col0, climit, pos, tsb_lo, alpha_half, w, sm.thr,
                                       sm.rab_ts_half, sm.oct);
      else
        silu_chunk_mode<false, PRECISE>(mode, sr, pw, pk, m.ts, col0, climit, pos, tsb_lo, alpha_half, w, sm.thr,
                                        sm.rab_ts_half, sm.oct);
      // P of keys col0 .. col0 + 31 packs into columns col0 .. col0 + 15 of
      // the buffer, this group's own (already read) S columns
      tmem_st16(s_tmem + col0, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.bar_p_full[b]);
      __syncwarp();  // every lane of the warp is done with the stage's metadata
      if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.bar_meta_empty[s]);
    }
    if (ok && cnt > 0) {
      ok = ew_all(mbar_wait(&sm.bar_o_full, 0, abort_flag, a.hdr, 7), grp);
      tc_fence_after();
    }
    // with no key tile nothing waited for Q; it lands in a staging area below
    if (ok && cnt == 0) ok = ew_all(mbar_wait(&sm.bar_q, 0, abort_flag, a.hdr, 7), grp);
    if (ok) {
      // O columns 32 grp .. 32 grp + 31 go out through shared memory: 128 rows
      // x 128 bytes, 16-byte chunk c of row r at c ^ (r & 7), in the Q buffer
      // (groups 0, 1) or the first K stage (groups 2, 3), both idle once every
      // GEMM completed; each warp then writes whole 128-byte row segments
      const uint32_t stage = (grp < 2 ? smem_u32(sm.q) : smem_u32(sm.k[0])) + (grp & 1) * (kTileBytes / 2);
      const int wq = warp & 3;  // warp rank in the warpgroup
      uint32_t orr[32];
      if (cnt > 0) {
        tmem_ld32(tmem + lane_base + 256 + col0, orr);
        tmem_wait_ld(orr);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) orr[e] = 0u;
      }
#pragma unroll
      for (int c = 0; c < 8; ++c)
        sts_v4(stage + r * 128 + ((c ^ (r & 7)) << 4),
               make_uint4(orr[4 * c], orr[4 * c + 1], orr[4 * c + 2], orr[4 * c + 3]));
      named_bar_sync(1 + grp, kTile);
      // lanes 8 i .. 8 i + 7 of a warp write row rr's 8 chunks
#pragma unroll 1
      for (int rr = 4 * wq + (lane >> 3); rr < kTile; rr += 16) {
        const int c = lane & 7;
        if (rr < g.nq_rows) {
          const uint4 val = lds_v4(stage + rr * 128 + ((c ^ (rr & 7)) << 4));
          float* orow = a.o_ws + (((size_t)it.split * a.T_q + (g.qrow0 + rr)) * a.H + it.head) * kHeadDim;
          *reinterpret_cast<uint4*>(orow + col0 + 4 * c) = val;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_attn_sm100_single(const AttnArgs& a, const BucketTable& thr, const CUtensorMap& tm_q,
                                     const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_kpool,
                                     const CUtensorMap& tm_vpool, cudaStream_t s) {
  int dev = 0;
  cudaGetDevice(&dev);
  static unsigned long long attr_set = 0;  // one bit per device
  if (dev < 64 && !(attr_set & (1ull << dev))) {
    cudaError_t e = cudaFuncSetAttribute(attn_sm100_single_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytesSingle);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_sm100_single_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSmemBytesSingle);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  if (a.max_items <= 0) return cudaSuccess;
  if (a.precise_silu)
    attn_sm100_single_kernel<true>
        <<<a.max_items, kThreads, kSmemBytesSingle, s>>>(a, thr, tm_q, tm_k, tm_v, tm_kpool, tm_vpool);
  else
    attn_sm100_single_kernel<false>
        <<<a.max_items, kThreads, kSmemBytesSingle, s>>>(a, thr, tm_q, tm_k, tm_v, tm_kpool, tm_vpool);
  return cudaGetLastError();
}

}  // namespace hstu
