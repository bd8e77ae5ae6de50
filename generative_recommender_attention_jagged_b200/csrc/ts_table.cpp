// Exact bucket edges for the HSTU time bias.
//
// The time bucket of a gap dt is floor(ln(|dt| + 1) / 0.301) clamped to the
// table ("Generative Recommenders at Scale": HSTU adds a relative attention
// bias; the bucket rule is the one the attention definition fixes).  For an
// integer x = |dt| + 1 >= 1 that floor is the largest b with
// ln(x) >= 0.301 b, i.e. with x >= ceil(e^(0.301 b)).  This file finds those
// integer edges once, in binary128 arithmetic, and then confirms each one by
// checking ln(x) on both sides of it, so the device can bucket with integer
// compares only and be bit-exact.
#include <quadmath.h>

#include <climits>
#include <mutex>

#include "hstu_internal.h"

namespace hstu {

namespace {

// smallest integer x >= 1 with logq(x) >= 0.301*b (as binary128)
long long edge_for(int b) {
  // the decimal 0.301 rounded once to binary128
  const __float128 step = strtoflt128("0.301", nullptr);
  const __float128 target = step * (__float128)b;
  if (target > logq((__float128)LLONG_MAX)) return LLONG_MAX;
  __float128 e = expq(target);
  long long x = (long long)ceilq(e);
  if (x < 1) x = 1;
  // confirm by the definition (ln on both sides), stepping at most a few times
  for (int it = 0; it < 4 && x > 1 && logq((__float128)(x - 1)) >= target; ++it) --x;
  for (int it = 0; it < 4 && logq((__float128)x) < target; ++it) ++x;
  return x;
}

BucketTable g_tables[kMaxBuckets + 1];
std::once_flag g_once[kMaxBuckets + 1];

}  // namespace

const BucketTable& bucket_table(int num_buckets) {
  std::call_once(g_once[num_buckets], [num_buckets] {
    BucketTable& t = g_tables[num_buckets];
    for (int b = 0; b < kMaxBuckets; ++b) t.thr[b] = b < num_buckets ? edge_for(b) : LLONG_MAX;
    // octave table: the bucket of 2^e and the (at most three) edges inside [2^e, 2^(e+1))
    for (int e = 0; e < 32; ++e) {
      const long long lo = 1ll << e, hi = (2ll << e) - 1;
      int b_lo = 0;
      for (int b = 0; b < kMaxBuckets; ++b)
        if (t.thr[b] <= lo) b_lo = b;
      t.oct[e][0] = (unsigned int)b_lo;
      for (int k = 1; k <= 3; ++k) {
        const int b = b_lo + k;
        t.oct[e][k] = (b < kMaxBuckets && t.thr[b] <= hi) ? (unsigned int)t.thr[b] : 0xFFFFFFFFu;
      }
    }
  });
  return g_tables[num_buckets];
}

}  // namespace hstu
