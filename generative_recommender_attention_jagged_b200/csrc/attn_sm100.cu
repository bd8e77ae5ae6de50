// HSTU pointwise attention on the sm_100a tensor cores (bf16 in, fp32 accumulate).
//
// One CTA computes one work item: two 128-row query tiles A and B (rows
// qs..qs+255 of one user and head) against a range of 128-key tiles (all the
// tiles the rows need, or one split of them in paged mode).  Per key tile and
// query tile X:
//
//   S_X  = Q_X K^T          tcgen05.mma, A = Q_X (smem, K-major), B = K (smem,
//                           K-major), fp32 accumulator in tensor memory
//   P_X  = SiLU(alpha S_X + rab_pos[p_i - p_j + N - 1] + rab_ts[bucket(t_i - t_j)]),
//          0 outside the allowed set; computed by the two elementwise
//          warpgroups of X (64 keys each), which read S_X with tcgen05.ld and
//          write P_X as bf16 pairs back over their own half of S_X (tcgen05.st)
//   O_X += P_X V            tcgen05.mma, A = P_X (tensor memory), B = V (smem, MN-major)
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
// Warp roles (608 threads): warps 0-15 elementwise in four warpgroups, one
// per (query tile, 64-key half of every key tile) (thread = query row = TMEM
// lane; a warp reaches the lanes of its rank in the warpgroup), warp 16
// producer (Q once; K/V through a 2-stage ring by TMA, the paged prefix page
// by page; per key tile it also stages the keys' timestamps and a window of
// 0.5*rab_pos in shared memory), warps 17 and 18 the MMA issuers of query
// tiles A and B (warp 17 owns tensor memory).  Tensor memory holds S_A, S_B,
// O_A, O_B (4 x 128 columns).  Each tile's issuer follows its own two
// warpgroups: as soon as one 64-key half of P is written it issues that
// half's A.V GEMM and then the next key tile's S for the same 64 columns
// (N = 64), so a warpgroup waits only for its own half, and neither tile's
// GEMMs queue behind the other tile's waits.  A K/V stage is released once
// both tiles' GEMMs that read it completed.  At the end each warpgroup stages
// its O columns in its tile's (then idle) Q buffer and writes whole 128-byte
// row segments of the fp32 partial.  Every wait is bounded (about 2 s), after
// which the kernel reports HSTU_ERR_TIMEOUT and winds down.
//
// Elementwise work per score: hb = s/2 = (alpha/2) S + 0.5 (rab_pos + rab_ts)
// with packed f32x2 FMA, then SiLU(s) = hb (1 + tanh hb): by default hb is
// rounded to bf16 and one packed bf16x2 tanh and one bf16x2 FMA produce two
// scores of P at once (P is bf16 for the A.V GEMM anyway); with the precise
// option tanh and the FMA run in fp32 and P is rounded once.  Time
// buckets are exact: a thread finds the bucket of its row's first key once per
// work item by a binary search over integer edges, then walks down the edges
// as the keys come closer in time (timestamps are non-decreasing inside a
// user, so |t_i - t_j| only shrinks along a row).  Per 32-column chunk one
// compare tells whether a row stays in its bucket; a chunk where every row of
// the warp does uses a constant, a chunk with at most one edge per row finds
// it by a 5-step search and selects, and only chunks with more edges (next to
// the diagonal) take each column's bucket from an octave table (the bit length
// of |dt| + 1 picks four integer edges).  The SiLU loop itself is branch-free.
// The producer loads each tile's metadata into registers one tile ahead, so
// its global-load latency hides behind the wait for a free stage.
#include <cuda_bf16.h>
#include <stdint.h>

#include "attn_common.cuh"

namespace hstu {

namespace {

constexpr int kQTiles = 2;
constexpr int kEwWarps = 16;                 // 4 warpgroups: (query tile, 64-column half)
constexpr int kThreads = 32 * (kEwWarps + 3);
constexpr int kProducerWarp = kEwWarps;
constexpr int kMmaWarp = kEwWarps + 1;   // MMA issuer of tile A, TMEM owner
constexpr int kMmaWarpB = kEwWarps + 2;  // MMA issuer of tile B
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;          // S_A [0,128) S_B [128,256) O_A [256,384) O_B [384,512)
struct __align__(1024) Smem {
  uint8_t q[kQTiles][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  Meta meta[kStages];
  long long thr[kMaxBuckets];
  float rab_ts_half[kMaxBuckets];
  uint4 oct[32];
  uint32_t win_rs[kWinLoads * 16];  // producer scratch: R as 416 bf16
  uint64_t bar_q;
  uint64_t bar_k_full[kStages];
  uint64_t bar_v_full[kStages];
  uint64_t bar_meta_full[kStages];
  uint64_t bar_kv_empty[kQTiles][kStages];  // stage released by tile X's GEMMs
  uint64_t bar_s_full[kQTiles][2];  // S of keys 0-63 / 64-127 written
  uint64_t bar_p_lo[kQTiles];  // P of keys 0-63 written
  uint64_t bar_p_hi[kQTiles];  // P of keys 64-127 written
  uint64_t bar_o_full[kQTiles];
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;  // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

template <bool PRECISE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const AttnArgs a, const BucketTable tab, const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_kpool,
                      const __grid_constant__ CUtensorMap tm_vpool) {
  const int item_idx = blockIdx.x;
  if (item_idx >= a.hdr->n_items) return;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = aligned_smem<Smem>(smem_raw);

  const WorkItem it = a.items[item_idx];
  // a work list not written by this call's scheduler must not send us out of bounds
  if (it.user < 0 || it.user >= a.B || it.head < 0 || it.head >= a.H || it.split < 0 ||
      it.split >= a.num_splits || it.qtile < 0 ||
      it.qtile * kQTiles * kTile >= a.q_offsets[it.user + 1] - a.q_offsets[it.user])
    return;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const TileGeom gA = tile_geom(a, it.user, it.qtile * kQTiles);
  const bool hasB = (it.qtile * kQTiles + 1) * kTile < a.q_offsets[it.user + 1] - a.q_offsets[it.user];
  const TileGeom gB = hasB ? tile_geom(a, it.user, it.qtile * kQTiles + 1) : gA;
  const int nA = gA.n_tiles;
  const int nB = hasB ? gB.n_tiles : 0;
  int tb, te;
  split_range(max(nA, nB), it.split, a.num_splits, tb, te);
  const int cA = max(0, min(te, nA) - tb);  // key tiles of this item for tile A
  const int cB = max(0, min(te, nB) - tb);
  const int cT = max(cA, cB);
  const int prmin = min(gA.qs, gA.h);       // smallest query position of the item

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.bar_k_full[s], 1);
      mbar_init(&sm.bar_v_full[s], 1);
      mbar_init(&sm.bar_meta_full[s], 32);
      mbar_init(&sm.bar_kv_empty[0][s], 1);
      mbar_init(&sm.bar_kv_empty[1][s], 1);
    }
    for (int x = 0; x < kQTiles; ++x) {
      mbar_init(&sm.bar_s_full[x][0], 1);
      mbar_init(&sm.bar_s_full[x][1], 1);
      mbar_init(&sm.bar_p_lo[x], kTile);
      mbar_init(&sm.bar_p_hi[x], kTile);
    }
    mbar_init(&sm.bar_o_full[0], 1);
    mbar_init(&sm.bar_o_full[1], 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  for (int x = threadIdx.x; x < kMaxBuckets; x += kThreads) {
    sm.thr[x] = tab.thr[x];
    sm.rab_ts_half[x] = x < a.nb ? 0.5f * a.rab_ts[x] : 0.f;
  }
  if (threadIdx.x < 32)
    sm.oct[threadIdx.x] = make_uint4(tab.oct[threadIdx.x][0], tab.oct[threadIdx.x][1], tab.oct[threadIdx.x][2],
                                     tab.oct[threadIdx.x][3]);
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
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

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ producer
    const int head = it.head;
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.bar_q, (hasB ? 2 : 1) * kTileBytes);
      tma_load_3d(sm.q[0], &tm_q, &sm.bar_q, 0, head, gA.qrow0);
      tma_load_3d(sm.q[0] + kHalfBytes, &tm_q, &sm.bar_q, 64, head, gA.qrow0);
      if (hasB) {
        tma_load_3d(sm.q[1], &tm_q, &sm.bar_q, 0, head, gB.qrow0);
        tma_load_3d(sm.q[1] + kHalfBytes, &tm_q, &sm.bar_q, 64, head, gB.qrow0);
      }
    }
    const int row_base = a.q_offsets[it.user] - gA.L;  // row of key position p is row_base + p (p >= L)
    const int n_rab = 2 * a.n_max - 1;
    // Per-tile metadata (key timestamps, position-bias window) is loaded into
    // registers one tile ahead, so its global-load latency hides behind the
    // wait for a free stage.  Lane l holds timestamps of columns l + 32k and
    // window entries x = l + 32k - 3 (x in [-3, 384)).
    long long mts[4];
    float mwin[kWinLoads];
    auto load_meta = [&](int t) {
      int k0, width;
      key_tile(gA, tb + t, k0, width);
#pragma unroll
      for (int k = 0; k < 4; ++k) mts[k] = a.ts[gA.tso + k0 + min(lane + 32 * k, width - 1)];
      const int g0 = prmin + 255 - k0 + a.n_max - 1;  // rab_pos index of R[0]
#pragma unroll
      for (int k = 0; k < kWinLoads; ++k) {
        const int idx = g0 - (lane + 32 * k);
        mwin[k] = (idx >= 0 && idx < n_rab) ? 0.5f * __ldg(a.rab_pos + idx) : 0.f;
      }
    };
    if (cT > 0) load_meta(0);
    int issued = 0;
    for (int t = 0; t < cT; ++t) {
      const int s = t % kStages;
      const uint32_t ph = (t / kStages) & 1;
      int k0, width;
      key_tile(gA, tb + t, k0, width);
      bool ok = true;
      // the stage's previous tile (t - kStages) is released by each query tile that used it
      if (lane == 0 && t - kStages < cA) ok = mbar_wait(&sm.bar_kv_empty[0][s], ph ^ 1, abort_flag, a.hdr, 1);
      if (lane == 0 && ok && t - kStages < cB) ok = mbar_wait(&sm.bar_kv_empty[1][s], ph ^ 1, abort_flag, a.hdr, 1);
      ok = __shfl_sync(~0u, ok, 0);
      if (!ok) break;
      uint8_t* kd = sm.k[s];
      uint8_t* vd = sm.v[s];
      if (k0 >= gA.L) {
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
          const uint8_t* kpage =
              static_cast<const uint8_t*>(a.k_pool) + ((size_t)pid * a.H + head) * P * kHeadDim * 2;
          const uint8_t* vpage =
              static_cast<const uint8_t*>(a.v_pool) + ((size_t)pid * a.H + head) * P * kHeadDim * 2;
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
      // publish this tile's metadata, then start loading the next tile's
      Meta& m = sm.meta[s];
#pragma unroll
      for (int k = 0; k < 4; ++k) m.ts[lane + 32 * k] = mts[k];
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
      if (t + 1 < cT) load_meta(t + 1);
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
  } else if (warp == kMmaWarp || warp == kMmaWarpB) {
    // ------------------------------------------------------------------ MMA issuers, one per query tile
    if (lane == 0) {
      const int x = warp == kMmaWarp ? 0 : 1;
      const int c = x == 0 ? cA : cB;
      constexpr uint32_t idesc_pv = idesc_bf16(128, 128, 0, 1);
      constexpr uint32_t idesc_qk_half = idesc_bf16(128, 64, 0, 0);
      // S_X over keys [64 h, 64 h + 64) of tile t into columns 64 h .. 64 h + 63:
      // issued per half so that each half follows its own half of P into the
      // A.V GEMM (the half's columns hold that P until then)
      auto issue_s_half = [&](int t, int h) {
        const uint32_t q_base = smem_u32(sm.q[x]);
        const uint32_t k_base = smem_u32(sm.k[t % kStages]) + h * 64 * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_ss(tmem + x * 128 + 64 * h, sw128_desc(q_base + off, 16, 1024), sw128_desc(k_base + off, 16, 1024),
                 idesc_qk_half, kk > 0);
        }
        mma_commit(&sm.bar_s_full[x][h]);
      };
      // O_X += P_X V over keys [64 h, 64 h + 64): P at columns 64 h .. 64 h + 31 of
      // S_X (16 keys per 8 columns), V rows 64 h..
      auto issue_pv_half = [&](int t, int h) {
        const uint32_t v_base = smem_u32(sm.v[t % kStages]);
#pragma unroll
        for (int kk = 4 * h; kk < 4 * h + 4; ++kk)
          mma_ts(tmem + 256 + x * 128, tmem + x * 128 + 64 * h + (kk - 4 * h) * 8,
                 sw128_desc(v_base + kk * 2048, kHalfBytes, 1024), idesc_pv, (t > 0 || kk > 0));
      };
      bool ok = c == 0 || mbar_wait(&sm.bar_q, 0, abort_flag, a.hdr, 2);
      if (ok && c > 0) ok = mbar_wait(&sm.bar_k_full[0], 0, abort_flag, a.hdr, 3);
      tc_fence_after();
      if (ok && c > 0) {
        issue_s_half(0, 0);
        issue_s_half(0, 1);
      }
      for (int t = 0; ok && t < c; ++t) {
        const int s = t % kStages;
        ok = mbar_wait(&sm.bar_p_lo[x], t & 1, abort_flag, a.hdr, 4);
        if (ok) ok = mbar_wait(&sm.bar_v_full[s], (t / kStages) & 1, abort_flag, a.hdr, 5);
        if (!ok) break;
        tc_fence_after();
        issue_pv_half(t, 0);
        const bool next = t + 1 < c;
        if (next) {
          ok = mbar_wait(&sm.bar_k_full[(t + 1) % kStages], ((t + 1) / kStages) & 1, abort_flag, a.hdr, 3);
          if (!ok) break;
          tc_fence_after();
          issue_s_half(t + 1, 0);
        }
        ok = mbar_wait(&sm.bar_p_hi[x], t & 1, abort_flag, a.hdr, 4);
        if (!ok) break;
        tc_fence_after();
        issue_pv_half(t, 1);
        if (next) issue_s_half(t + 1, 1);
        mma_commit(&sm.bar_kv_empty[x][s]);
      }
      mma_commit(&sm.bar_o_full[x]);
      // tensor memory is freed below only after every issued MMA completed
      mbar_wait(&sm.bar_o_full[x], 0, nullptr, a.hdr, 8);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ elementwise
    const int x = warp >> 3;                 // query tile of this warpgroup
    const int half = (warp >> 2) & 1;        // key columns 64*half .. 64*half + 63 of every tile
    const int group = warp >> 2;             // warpgroup index 0..3
    const int r = threadIdx.x & (kTile - 1); // query row of the tile == TMEM lane
    const TileGeom& g = x == 0 ? gA : gB;
    const int cnt = x == 0 ? cA : cB;
    const bool exists = x == 0 || hasB;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int i = min(g.qs + r, g.n - 1);  // rows past the user repeat its last row (discarded)
    const int jmax = i < g.h ? i : g.h - 1;
    const int pr = min(i, g.h);
    const int zb = prmin + 255 - pr;       // window element of column 0
    const float alpha_half = 0.5f * a.alpha;
    const uint32_t s_tmem = tmem + lane_base + x * 128;
    Walk w;
    w.t_i = a.ts[g.tso + i];
    w.b = 0;
    w.tlim = 0;
    w.tsb = 0.f;
    bool ok = true;
    for (int t = 0; t < cnt; ++t) {
      const int s = t % kStages;
      int k0, width;
      key_tile(g, tb + t, k0, width);
      ok = mbar_wait(&sm.bar_meta_full[s], (t / kStages) & 1, abort_flag, a.hdr, 6);
      ok = ok && mbar_wait(&sm.bar_s_full[x][half], t & 1, abort_flag, a.hdr, 6);
      ok = ew_all(ok, group);
      if (!ok) break;
      tc_fence_after();
      const Meta& m = sm.meta[s];
      const int climit = min(jmax - k0, width - 1);  // columns c <= climit are allowed
      if (t == 0) {
        w.b = bucket_of_dt(sm.thr, w.t_i - m.ts[0]);
        w.tlim = w.t_i + 1 - sm.thr[w.b];
        w.tsb = sm.rab_ts_half[w.b];
      }
      const bool need_mask = !__all_sync(~0u, climit >= kTile - 1);
#pragma unroll 1
      for (int ch = 2 * half; ch < 2 * half + 2; ++ch) {
        uint32_t sr[32];
        tmem_ld32(s_tmem + ch * 32, sr);
        const int col0 = ch * 32;
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
          silu_chunk_mode<true, PRECISE>(mode, sr, pw, pk, m.ts, col0, climit, pos, tsb_lo, alpha_half, w,
                                         sm.thr, sm.rab_ts_half, sm.oct);
        else
          silu_chunk_mode<false, PRECISE>(mode, sr, pw, pk, m.ts, col0, climit, pos, tsb_lo, alpha_half, w,
                                          sm.thr, sm.rab_ts_half, sm.oct);
        // P of this chunk packs into the warpgroup's own (already read) S columns:
        // keys 0-63 at columns 0-31, keys 64-127 at columns 64-95
        tmem_st16(s_tmem + half * 64 + (ch & 1) * 16, pk);
      }
      // this warpgroup's 64-key half of P goes to the A.V GEMM
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(half == 0 ? &sm.bar_p_lo[x] : &sm.bar_p_hi[x]);
    }
    if (ok && cT > 0) {
      ok = ew_all(mbar_wait(&sm.bar_o_full[x], 0, abort_flag, a.hdr, 7), group);
      tc_fence_after();
    }
    // a tile with no key tile of this split (the whole item, or only this
    // tile when the other has some) issued no GEMM, so nothing waited for its
    // Q copy; that copy lands in the staging area used below
    if (ok && cnt == 0 && exists) ok = ew_all(mbar_wait(&sm.bar_q, 0, abort_flag, a.hdr, 7), group);
    if (ok && exists && a.o_bf16) {
      // O of this warpgroup's 64 columns as bf16 (one split feeding the
      // LayerNorm gate): 128 rows x 128 bytes staged in its half of the tile's
      // Q buffer, 16-byte chunk c of row r at c ^ (r & 7), then whole 128-byte
      // row segments per warp
      const uint32_t stage = smem_u32(sm.q[x]) + half * (kTileBytes / 2);
      const int wq = warp & 3;
      uint32_t pk[32];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t orr[32];
        if (cnt > 0) {
          tmem_ld32(tmem + lane_base + 256 + x * 128 + half * 64 + h2 * 32, orr);
          tmem_wait_ld(orr);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = 0u;
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[16 * h2 + e] = pack_bf16x2(__uint_as_float(orr[2 * e]), __uint_as_float(orr[2 * e + 1]));
      }
#pragma unroll
      for (int c = 0; c < 8; ++c)
        sts_v4(stage + r * 128 + ((c ^ (r & 7)) << 4), make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]));
      named_bar_sync(1 + group, kTile);
#pragma unroll 1
      for (int rr = 4 * wq + (lane >> 3); rr < kTile; rr += 16) {
        const int c = lane & 7;
        if (rr < g.nq_rows) {
          const uint4 val = lds_v4(stage + rr * 128 + ((c ^ (rr & 7)) << 4));
          __nv_bfloat16* orow =
              reinterpret_cast<__nv_bfloat16*>(a.o_ws) + ((size_t)(g.qrow0 + rr) * a.H + it.head) * kHeadDim;
          *reinterpret_cast<uint4*>(orow + half * 64 + 8 * c) = val;
        }
      }
    } else if (ok && exists) {
      // O of this warpgroup's 64 columns goes out through shared memory, 32
      // columns at a time: its half of the tile's Q buffer (free once the
      // tile's GEMMs completed) holds 128 rows x 128 bytes, 16-byte chunk c of
      // row r at c ^ (r & 7), and each warp then writes whole 128-byte row
      // segments (a thread's own row would be 32 scattered 16-byte pieces)
      const uint32_t stage = smem_u32(sm.q[x]) + half * (kTileBytes / 2);
      const int wq = warp & 3;  // warp rank in the warpgroup
#pragma unroll 1
      for (int ch = 2 * half; ch < 2 * half + 2; ++ch) {
        uint32_t orr[32];
        if (cnt > 0) {
          tmem_ld32(tmem + lane_base + 256 + x * 128 + ch * 32, orr);
          tmem_wait_ld(orr);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = 0u;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c)
          sts_v4(stage + r * 128 + ((c ^ (r & 7)) << 4),
                 make_uint4(orr[4 * c], orr[4 * c + 1], orr[4 * c + 2], orr[4 * c + 3]));
        named_bar_sync(1 + group, kTile);
        // lanes 8 i .. 8 i + 7 of a warp write row rr's 8 chunks
#pragma unroll 1
        for (int rr = 4 * wq + (lane >> 3); rr < kTile; rr += 16) {
          const int c = lane & 7;
          if (rr < g.nq_rows) {
            const uint4 val = lds_v4(stage + rr * 128 + ((c ^ (rr & 7)) << 4));
            float* orow = a.o_ws + (((size_t)it.split * a.T_q + (g.qrow0 + rr)) * a.H + it.head) * kHeadDim;
            *reinterpret_cast<uint4*>(orow + ch * 32 + 4 * c) = val;
          }
        }
        named_bar_sync(1 + group, kTile);  // the staging area is reused by the next chunk
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_attn_sm100(const AttnArgs& a, const BucketTable& thr, const CUtensorMap& tm_q,
                              const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_kpool,
                              const CUtensorMap& tm_vpool, cudaStream_t s) {
  int dev = 0;
  cudaGetDevice(&dev);
  static unsigned long long attr_set = 0;  // one bit per device
  if (dev < 64 && !(attr_set & (1ull << dev))) {
    cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_sm100_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  if (a.max_items <= 0) return cudaSuccess;
  if (a.precise_silu)
    attn_sm100_kernel<true><<<a.max_items, kThreads, kSmemBytes, s>>>(a, thr, tm_q, tm_k, tm_v, tm_kpool, tm_vpool);
  else
    attn_sm100_kernel<false><<<a.max_items, kThreads, kSmemBytes, s>>>(a, thr, tm_q, tm_k, tm_v, tm_kpool, tm_vpool);
  return cudaGetLastError();
}

}  // namespace hstu
