// Device-side helpers shared by the kernels: sm_100a inline PTX wrappers
// (mbarrier, TMA, tcgen05 / tensor memory), bounded waits, the exact time
// bucket search and the per-tile geometry of the jagged / paged sequence.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include <climits>

#include "hstu_internal.h"

namespace hstu {

// status codes (mirror include/hstu.h)
constexpr int32_t kErrLength = -4;
constexpr int32_t kErrTimeout = -7;
constexpr int32_t kErrUnsorted = -8;
constexpr int32_t kErrPage = -9;

__device__ __forceinline__ void report_error(WsHeader* hdr, int32_t code, int32_t detail) {
  if (atomicCAS(&hdr->status, 0, code) == 0) hdr->detail = detail;
}

// ---------------------------------------------------------------------------
// time bucket: largest b with thr[b] <= x (x = |dt| + 1 >= 1, thr[0] = 1)
// ---------------------------------------------------------------------------
__device__ __forceinline__ int bucket_search(const long long* thr, long long x) {
  // before the step of size s, b <= 128 - 2s, so b + s <= 127 stays in range
  int b = 0;
#pragma unroll
  for (int step = 64; step >= 1; step >>= 1)
    if (thr[b + step] <= x) b += step;
  return b;
}

// |dt| + 1 as an unsigned 64-bit value, saturating (|INT64_MIN| + 1 fits in u64)
__device__ __forceinline__ unsigned long long abs_dt_plus1(long long dt) {
  unsigned long long m = dt < 0 ? 0ull - (unsigned long long)dt : (unsigned long long)dt;
  return m == ~0ull ? m : m + 1;
}

// bucket of a 32-bit x >= 1 from the octave table (see BucketTable::oct)
__device__ __forceinline__ int bucket_oct(const uint4* oct, unsigned int x) {
  unsigned int e;
  asm("bfind.u32 %0, %1;" : "=r"(e) : "r"(x));
  const uint4 t = oct[e];
  return (int)t.x + (x >= t.y) + (x >= t.z) + (x >= t.w);
}

__device__ __forceinline__ int bucket_of_dt(const long long* thr, long long dt) {
  unsigned long long x = abs_dt_plus1(dt);
  // thresholds are < 2^63, so any x >= 2^63 lies above every finite edge
  if (x >= (1ull << 63)) return bucket_search(thr, LLONG_MAX);
  return bucket_search(thr, (long long)x);
}

// ---------------------------------------------------------------------------
// geometry of a query tile (see TileGeom)
// ---------------------------------------------------------------------------
// key tiles needed by query tile `qtile` of a user with cached prefix L,
// sequence length n and history h (pure arithmetic, no memory access)
__host__ __device__ __forceinline__ int key_tiles_of(int L, int n, int h, int qtile) {
  const int qs = L + qtile * kTile;
  const int q_last = min(qs + kTile, n) - 1;
  const int kv_end = max(0, min(q_last + 1, h));
  return ceil_div(min(L, kv_end), kTile) + (kv_end > L ? ceil_div(kv_end - L, kTile) : 0);
}

__device__ __forceinline__ TileGeom tile_geom(const AttnArgs& a, int user, int qtile) {
  TileGeom g;
  const int q0 = a.q_offsets[user];
  const int nq = a.q_offsets[user + 1] - q0;
  g.L = a.paged ? a.cached_lens[user] : 0;
  g.n = g.L + nq;
  const int c = a.num_cand ? a.num_cand[user] : 0;
  g.h = g.n - c;
  g.qs = g.L + qtile * kTile;
  g.nq_rows = min(kTile, g.n - g.qs);
  const int q_last = g.qs + g.nq_rows - 1;
  g.kv_end = max(0, min(q_last + 1, g.h));
  g.n_pre = ceil_div(min(g.L, g.kv_end), kTile);
  g.n_tiles = g.n_pre + (g.kv_end > g.L ? ceil_div(g.kv_end - g.L, kTile) : 0);
  g.qrow0 = q0 + qtile * kTile;
  g.tso = a.paged ? a.ts_offsets[user] : q0;
  return g;
}

// key tile t of a query tile: first key position and number of keys
__device__ __forceinline__ void key_tile(const TileGeom& g, int t, int& k0, int& width) {
  if (t < g.n_pre) {
    k0 = t * kTile;
    width = min(kTile, g.L - k0);
  } else {
    k0 = g.L + (t - g.n_pre) * kTile;
    width = min(kTile, g.n - k0);
  }
}

// key tiles [tb, te) of split s out of S
__device__ __forceinline__ void split_range(int n_tiles, int s, int S, int& tb, int& te) {
  tb = (int)(((long long)n_tiles * s) / S);
  te = (int)(((long long)n_tiles * (s + 1)) / S);
}

// ---------------------------------------------------------------------------
// sm_100a PTX: shared-memory addresses, mbarriers, TMA, tcgen05
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// The 1024-byte aligned start of the dynamic shared memory, derived from the
// __shared__ array by pointer arithmetic so that the compiler keeps the shared
// address space (a round trip through an integer turns every access through
// the result into a generic one: generic atomics and loads take the L1TEX
// path instead of the shared-memory pipe).
template <typename T>
__device__ __forceinline__ T& aligned_smem(uint8_t* smem_raw) {
  return *reinterpret_cast<T*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase of the given parity to complete.  Gives up after about
// 2 s (or at once when another warp already gave up and raised *abort),
// reporting HSTU_ERR_TIMEOUT; returns false then.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          WsHeader* hdr, int where) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (abort != nullptr && *abort) return false;
      const uint64_t now = global_timer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > 2000000000ull) {
        if (abort != nullptr) *abort = 1;
        report_error(hdr, kErrTimeout, where);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled TMA load (no multicast): box lands in smem, completes tx on bar
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// 3-D tiled TMA load (no multicast): box lands in smem, completes tx on bar
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0,
                                            int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// ---- tcgen05 / tensor memory ----
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D(tmem) (+)= A(smem desc) * B(smem desc)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D(tmem) (+)= A(tmem) * B(smem desc)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on bar once every tcgen05.mma issued so far by this thread completes
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 columns of 32-bit: thread t of the warp receives lane (base+t)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// wait for a tcgen05.ld whose 32 destination registers are r: naming them as
// operands keeps every use of r after the wait
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// 32 lanes x 16 columns of 32-bit store
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for a 128-byte-swizzled operand
// (Blackwell descriptor version 1): start address, leading and stride byte
// offsets (all in 16-byte units), swizzle mode 2 = 128B.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulate.
// a_mn / b_mn: operand stored MN-major (transposed) instead of K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17)     // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t tanh_bf16x2(uint32_t x) {
  uint32_t y;
  asm("tanh.approx.bf16x2 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t fma_bf16x2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace hstu
