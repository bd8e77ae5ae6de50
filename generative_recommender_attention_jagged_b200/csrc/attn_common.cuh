// Shared parts of the tensor-core attention kernels (attn_sm100.cu: two
// query tiles per CTA; attn_sm100_single.cu: one query tile per CTA): tile
// sizes, the per-key-tile metadata staged in shared memory, small PTX
// helpers, and the elementwise step that turns a 32-column chunk of S into
// bf16 P (time bucket modes, SiLU).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "device_common.cuh"

namespace hstu {
namespace {

constexpr int kTileBytes = kTile * 128 * 2;  // 128 rows x 128 bf16 = 32 KB
constexpr int kHalfBytes = kTile * 128;      // 128 rows x 64 bf16: one 128B-swizzled box
constexpr int kHeadDim = 128;
// Position-bias window of a 256-row x 128-key block, as bf16 (a one-tile
// item uses the first 128 rows).  R[z] = 0.5 * rab_pos[prmin + 255 - k0 +
// N_max - 1 - z] (0 outside the table), where prmin is the item's smallest
// query position and k0 the tile's first key: row position pr, chunk column
// col0 + c needs R[z0 + c] with z0 = prmin + 255 - pr + col0, and the pair of
// columns (c, c + 1) is the bf16 pair (R[z0 + c], R[z0 + c + 1]).  Eight
// copies shifted by 0..7 let every row read the 32 values of a chunk as four
// 16-byte loads: copy p holds R[e + p] at element e, and its 16-byte chunk f
// sits at win[f][p], so the eight rows of a quarter-warp (eight different p)
// hit eight different bank groups.
constexpr int kWinChunks = 49;               // elements 0..391 of each copy
constexpr int kWinLoads = 13;                // producer: R[l + 32 k], k < 13
struct Meta {
  long long ts[kTile];                       // key timestamps (the last one repeated past the tile's width)
  uint4 win[kWinChunks][8];                  // 8 copies x 392 bf16, interleaved by 16-byte chunk
};

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


__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr)
               : "memory");
  return r;
}

// the threads of one elementwise warpgroup wait for each other (barrier 1 + group)
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// the 128 threads of one elementwise warpgroup (0..3) agree on a flag
__device__ __forceinline__ bool ew_all(bool ok, int group) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok), "r"(1 + group)
      : "memory");
  return r != 0;
}

// packed fp32 pairs (sm_100): lo in the low half
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint32_t add_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Row state of the exact time-bucket walk.
struct Walk {
  long long t_i;   // the row's timestamp
  long long tlim;  // bucket b still holds while t_j <= tlim  (tlim = t_i + 1 - thr[b])
  int b;
  float tsb;       // 0.5 * rab_ts[b]
};

__device__ __forceinline__ void walk_to(Walk& w, long long tj, const long long* thr, const float* rts) {
  while (w.b > 0 && tj > w.tlim) {
    --w.b;
    w.tlim = w.t_i + 1 - thr[w.b];
    w.tsb = rts[w.b];
  }
}

// Time-bias modes of a 32-column chunk.
enum BiasMode { kBiasConst = 0, kBiasEdge = 1, kBiasOct = 2, kBiasWalk = 3 };

// 32 scores of one row: S (fp32 bits, sr[0..31]) -> P (bf16 pairs).  pw[k] is
// the bf16 pair 0.5 * (rab_pos of column 2k, of column 2k + 1).
//   kBiasConst: the row's time bucket is the same over the chunk (w.tsb)
//   kBiasEdge:  one bucket edge: columns before `pos` use tsb_lo, the rest w.tsb
//   kBiasOct:   every column's bucket from the octave table (|dt| + 1 < 2^32)
//   kBiasWalk:  per-column walk over the bucket edges (wider gaps)
// MASK zeroes the columns past climit.
template <int MODE, bool MASK, bool PRECISE>
__device__ __forceinline__ void silu_chunk(const uint32_t* sr, const uint32_t (&pw)[16], uint32_t (&pk)[16],
                                           const long long* ts, int col0, int climit, int pos, float tsb_lo,
                                           float alpha_half, Walk& w, const long long* thr, const float* rts,
                                           const uint4* oct) {
  const uint64_t ah2 = pk2(alpha_half, alpha_half);
  const uint64_t tsb2 = pk2(w.tsb, w.tsb);
  const unsigned int ti1 = (unsigned int)(w.t_i + 1);  // octave mode: differences fit in 32 bits
  int b_last = 0;
  // time bias of column col (0.5 * rab_ts[bucket]) in the chunk's mode
  auto ts_bias = [&](int col) -> float {
    if constexpr (MODE == kBiasEdge) {
      return col < pos ? tsb_lo : w.tsb;
    } else if constexpr (MODE == kBiasOct) {
      const unsigned int x = max(ti1 - (unsigned int)ts[col], 1u);  // later keys only in masked columns
      b_last = bucket_oct(oct, x);
      return rts[b_last];
    } else {
      walk_to(w, ts[col], thr, rts);
      return w.tsb;
    }
  };
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    uint64_t tb2 = tsb2;
    if constexpr (MODE != kBiasConst) tb2 = pk2(ts_bias(col0 + c), ts_bias(col0 + c + 1));
    const uint64_t h2 = fma2(pk2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), ah2, tb2);
    float h0, h1;
    upk2(h2, h0, h1);
    const uint32_t pb = pw[c >> 1];
    if constexpr (PRECISE) {
      // fp32: P = hb (1 + tanh hb), one MUFU tanh per score, rounded once to bf16
      h0 += __uint_as_float(pb << 16);
      h1 += __uint_as_float(pb & 0xFFFF0000u);
      if constexpr (MASK) {  // SiLU(0) = 0 exactly: masking hb masks P
        h0 = (col0 + c <= climit) ? h0 : 0.f;
        h1 = (col0 + c + 1 <= climit) ? h1 : 0.f;
      }
      const uint64_t p2 = fma2(pk2(h0, h1), pk2(tanh_approx(h0), tanh_approx(h1)), pk2(h0, h1));
      float p0, p1;
      upk2(p2, p0, p1);
      pk[c >> 1] = pack_bf16x2(p0, p1);
    } else {
      // packed bf16: one MUFU tanh per two scores; P = hb (1 + tanh hb) as one bf16x2 FMA
      uint32_t hb = add_bf16x2(pack_bf16x2(h0, h1), pb);
      if constexpr (MASK)
        hb &= (col0 + c <= climit ? 0x0000FFFFu : 0u) | (col0 + c + 1 <= climit ? 0xFFFF0000u : 0u);
      pk[c >> 1] = fma_bf16x2(hb, tanh_bf16x2(hb), hb);
    }
  }
  if constexpr (MODE == kBiasOct) {  // the walk state continues from the chunk's last column
    w.b = b_last;
    w.tlim = w.t_i + 1 - thr[b_last];
    w.tsb = rts[b_last];
  }
}

template <bool MASK, bool PRECISE>
__device__ __forceinline__ void silu_chunk_mode(int mode, const uint32_t* sr, const uint32_t (&pw)[16],
                                                uint32_t (&pk)[16], const long long* ts, int col0, int climit,
                                                int pos, float tsb_lo, float alpha_half, Walk& w,
                                                const long long* thr, const float* rts, const uint4* oct) {
  if (mode == kBiasConst)
    silu_chunk<kBiasConst, MASK, PRECISE>(sr, pw, pk, ts, col0, climit, pos, tsb_lo, alpha_half, w, thr, rts, oct);
  else if (mode == kBiasEdge)
    silu_chunk<kBiasEdge, MASK, PRECISE>(sr, pw, pk, ts, col0, climit, pos, tsb_lo, alpha_half, w, thr, rts, oct);
  else if (mode == kBiasOct)
    silu_chunk<kBiasOct, MASK, PRECISE>(sr, pw, pk, ts, col0, climit, pos, tsb_lo, alpha_half, w, thr, rts, oct);
  else
    silu_chunk<kBiasWalk, MASK, PRECISE>(sr, pw, pk, ts, col0, climit, pos, tsb_lo, alpha_half, w, thr, rts, oct);
}

// Time-bias mode of the chunk starting at col0 for this row, decided by the
// warp (the walk state describes the last column processed so far).  May step
// the walk over one edge (edge mode); returns the mode, the edge column `pos`
// and the bias before the edge `tsb_lo`.
__device__ __forceinline__ int chunk_mode(Walk& w, const long long* ts, int col0, int climit,
                                          const long long* thr, const float* rts, int& pos, float& tsb_lo) {
  const int col_last = min(col0 + 31, climit);
  const bool none = col_last < col0;                    // chunk fully masked for this row
  const long long t_last = ts[max(col_last, 0)];
  const bool uni = none || t_last <= w.tlim;            // no bucket edge in the chunk
  int mode = kBiasConst;
  pos = col0 + 32;
  tsb_lo = w.tsb;
  if (!__all_sync(~0u, uni)) {
    const long long tlim2 = w.b > 0 ? w.t_i + 1 - thr[w.b - 1] : LLONG_MIN;
    const bool one = uni || t_last <= tlim2;              // at most one edge in the chunk
    // octave mode needs |dt| + 1 < 2^32 at the chunk's first allowed column
    const bool narrow = uni || (w.t_i + 1 - ts[col0]) < (1ll << 32);
    if (__all_sync(~0u, one)) {
      mode = kBiasEdge;
      if (!uni) {
        // first column of the chunk past the edge (timestamps are sorted)
        pos = col0;
#pragma unroll
        for (int step = 16; step >= 1; step >>= 1)
          if (ts[pos + step - 1] <= w.tlim) pos += step;
        --w.b;
        w.tlim = tlim2;
        w.tsb = rts[w.b];
      }
    } else {
      mode = __all_sync(~0u, narrow) ? kBiasOct : kBiasWalk;
    }
  }
  return mode;
}


}  // namespace
}  // namespace hstu
