// Host side of libhstu.so: the C ABI declared in include/hstu.h.
//
// Checks arguments, lays out the caller's workspace, builds the TMA tensor
// maps for the tensor-core path and launches the kernels.  It never
// allocates device memory and never synchronises (except in
// hstu_check_device_error, whose job is to read the device status word).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "hstu.h"
#include "hstu_internal.h"

using namespace hstu;

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// ---- driver entry point for tensor-map encoding (no -lcuda needed) ----
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

// [rows, H, d] bf16 with a token stride: box = 128 rows x 64 elements of one head
bool encode_rows(CUtensorMap* m, const void* base, int rows, int H, int d, int stride_elems) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)stride_elems * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kTile};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// pool [num_pages, H, page_size, d] bf16: box = one page x 64 elements of one head
bool encode_pool(CUtensorMap* m, const void* base, int num_pages, int H, int P, int d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)P, (cuuint64_t)H, (cuuint64_t)num_pages};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)P * d * 2, (cuuint64_t)H * P * d * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)P, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool device_is_sm100() {
  static int cached[64];  // 0 unknown, 1 yes, 2 no
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev < 0 || dev >= 64) return false;
  if (cached[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return cached[dev] == 1;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_params(const hstu_attn_params* p) {
  if (!p) return HSTU_ERR_INVALID_ARG;
  if (p->batch <= 0 || p->num_heads <= 0 || p->head_dim <= 0 || p->n_max <= 0 || p->total_tokens < 0 ||
      p->max_seq_len < 0)
    return HSTU_ERR_INVALID_ARG;
  if (p->num_ts_buckets <= 0 || p->num_ts_buckets > kMaxBuckets) return HSTU_ERR_UNSUPPORTED;
  if (p->dtype != HSTU_DT_F32 && p->dtype != HSTU_DT_BF16) return HSTU_ERR_INVALID_ARG;
  const uint32_t known = HSTU_F_FORCE_SIMT | HSTU_F_OUTPUT_RAW_AV | HSTU_F_PRECISE_SILU | HSTU_F_STAGE_PLAN |
                         HSTU_F_STAGE_ATTN | HSTU_F_STAGE_EPILOGUE;
  if (p->flags & ~known) return HSTU_ERR_INVALID_ARG;
  if (p->head_dim > 256 || (long long)p->num_heads * p->head_dim > 1024) return HSTU_ERR_UNSUPPORTED;
  const int qs = p->qkv_stride ? p->qkv_stride : p->num_heads * p->head_dim;
  const int us = p->u_stride ? p->u_stride : p->num_heads * p->head_dim;
  if (qs < p->num_heads * p->head_dim || us < p->num_heads * p->head_dim) return HSTU_ERR_INVALID_ARG;
  const int vec = p->dtype == HSTU_DT_BF16 ? 8 : 4;
  if (qs % vec || us % vec) return HSTU_ERR_ALIGNMENT;
  return HSTU_OK;
}

bool use_tensor_cores(const hstu_attn_params* p) {
  return !(p->flags & HSTU_F_FORCE_SIMT) && p->dtype == HSTU_DT_BF16 && p->head_dim == 128 && device_is_sm100();
}

// Query tiles per tensor-core work item.  A paged call whose users have on
// average at most one tile of new rows (incremental serving: a few actions and
// candidates against a long cached prefix) runs the one-tile kernel, which
// keeps all its warps on that tile and double-buffers S; everything else runs
// the two-tile kernel, which reads each K/V tile once for 256 query rows.
int item_tiles_for(const hstu_attn_params* p, bool paged) {
  return paged && (long long)p->total_tokens <= (long long)kTile * p->batch ? 1 : 2;
}

struct Layout {
  size_t items_off, o_off, total;
  int max_items;
};

Layout layout_for(const hstu_attn_params* p, int splits, bool tc, int item_tiles) {
  Layout l;
  const long long T = p->total_tokens;
  const long long rows = (long long)item_tiles * kTile;
  const long long qtiles = (T + rows - 1) / rows + p->batch;  // sum_u ceil(n_u/rows) <= T/rows + B
  const long long items = tc ? qtiles * p->num_heads * splits : 0;
  l.max_items = (int)items;
  l.items_off = sizeof(WsHeader);
  l.o_off = align_up(l.items_off + (size_t)items * sizeof(WorkItem));
  l.total = align_up(l.o_off + (size_t)splits * T * p->num_heads * p->head_dim * sizeof(float));
  return l;
}

struct Common {
  const void *q, *k, *v, *u;
  const int32_t* q_offsets;
  const int64_t* ts;
  const int32_t* ts_offsets;
  const int32_t* num_cand;
  const float *rab_pos, *rab_ts, *gamma, *beta;
  const void *k_pool, *v_pool;
  int32_t num_pages;
  const int32_t* page_table;
  int32_t max_pages, page_size;
  const int32_t* cached_lens;
  int32_t splits;
  void* out;
  void* ws;
  size_t ws_bytes;
  cudaStream_t stream;
  bool paged;
};

int run(const hstu_attn_params* p, const Common& c) {
  if (int rc = check_params(p)) return rc;
  // arrays indexed by token may be null when there are no tokens (an empty
  // tensor need not have storage); paged timestamps also cover the prefix
  const bool rows = p->total_tokens > 0;
  if ((rows && (!c.q || !c.k || !c.v || !c.u || !c.out)) || (!c.ts && (rows || c.paged)) || !c.q_offsets ||
      !c.rab_pos || !c.rab_ts || !c.ws)
    return HSTU_ERR_INVALID_ARG;
  if (c.paged && (!c.ts_offsets || !c.cached_lens || !c.page_table || !c.k_pool || !c.v_pool || c.page_size <= 0 ||
                  c.num_pages <= 0 || c.max_pages <= 0))
    return HSTU_ERR_INVALID_ARG;
  if (c.splits < 1 || c.splits > kMaxSplits) return HSTU_ERR_INVALID_ARG;
  const void* ptrs[] = {c.q, c.k, c.v, c.u, c.out, c.ws, c.k_pool, c.v_pool, c.gamma, c.beta};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return HSTU_ERR_ALIGNMENT;
  const bool tc = use_tensor_cores(p);
  // tensor-core path: whole pages land as 1024-byte-aligned swizzled boxes
  if (tc && c.paged && (c.page_size < 8 || c.page_size > kTile || kTile % c.page_size)) return HSTU_ERR_UNSUPPORTED;
  const int item_tiles = item_tiles_for(p, c.paged);
  const Layout l = layout_for(p, tc ? c.splits : 1, tc, item_tiles);
  if (c.ws_bytes < l.total) return HSTU_ERR_WORKSPACE;

  uint32_t stages = p->flags & (HSTU_F_STAGE_PLAN | HSTU_F_STAGE_ATTN | HSTU_F_STAGE_EPILOGUE);
  if (!stages) stages = HSTU_F_STAGE_PLAN | HSTU_F_STAGE_ATTN | HSTU_F_STAGE_EPILOGUE;

  AttnArgs a;
  std::memset(&a, 0, sizeof a);
  a.B = p->batch;
  a.H = p->num_heads;
  a.d = p->head_dim;
  a.n_max = p->n_max;
  a.nb = p->num_ts_buckets;
  a.T_q = p->total_tokens;
  a.qkv_stride = p->qkv_stride ? p->qkv_stride : p->num_heads * p->head_dim;
  a.u_stride = p->u_stride ? p->u_stride : p->num_heads * p->head_dim;
  a.alpha = p->alpha;
  a.ln_eps = p->ln_eps;
  a.paged = c.paged ? 1 : 0;
  a.num_splits = tc ? c.splits : 1;
  a.page_size = c.page_size;
  a.num_pages = c.num_pages;
  a.max_pages = c.max_pages;
  a.max_items = l.max_items;
  a.item_tiles = item_tiles;
  a.out_raw = (p->flags & HSTU_F_OUTPUT_RAW_AV) ? 1 : 0;
  // one split of A.V partials feeding the LayerNorm gate is rounded to bf16
  // once (y is bf16 and normalised right after): half the bytes written and read
  a.o_bf16 = (tc && item_tiles == 2 && !c.paged && a.num_splits == 1 && !a.out_raw &&
              (p->num_heads * p->head_dim) % 128 == 0)
                 ? 1
                 : 0;
  a.self_term = tc ? 1 : 0;
  a.out_bf16 = p->dtype == HSTU_DT_BF16 ? 1 : 0;
  a.in_bf16 = p->dtype == HSTU_DT_BF16 ? 1 : 0;
  a.precise_silu = (p->flags & HSTU_F_PRECISE_SILU) ? 1 : 0;
  a.q = c.q;
  a.k = c.k;
  a.v = c.v;
  a.u = c.u;
  a.q_offsets = c.q_offsets;
  a.ts = c.ts;
  a.ts_offsets = c.paged ? c.ts_offsets : c.q_offsets;
  a.num_cand = c.num_cand;
  a.rab_pos = c.rab_pos;
  a.rab_ts = c.rab_ts;
  a.ln_gamma = c.gamma;
  a.ln_beta = c.beta;
  a.k_pool = c.k_pool;
  a.v_pool = c.v_pool;
  a.page_table = c.page_table;
  a.cached_lens = c.cached_lens;
  a.out = c.out;
  a.hdr = static_cast<WsHeader*>(c.ws);
  a.items = reinterpret_cast<WorkItem*>(static_cast<char*>(c.ws) + l.items_off);
  a.o_ws = reinterpret_cast<float*>(static_cast<char*>(c.ws) + l.o_off);

  const BucketTable& thr = bucket_table(a.nb);
  cudaError_t e = cudaSuccess;
  if (stages & HSTU_F_STAGE_PLAN) {
    if ((e = cudaMemsetAsync(c.ws, 0, sizeof(WsHeader), c.stream)) != cudaSuccess) return HSTU_ERR_CUDA;
    if ((e = launch_plan(a, tc, p->max_seq_len, c.stream)) != cudaSuccess) return HSTU_ERR_CUDA;
  }
  if (a.T_q == 0) return HSTU_OK;
  if (stages & HSTU_F_STAGE_ATTN) {
    if (tc) {
      CUtensorMap tq, tk, tv, tkp, tvp;
      std::memset(&tkp, 0, sizeof tkp);
      std::memset(&tvp, 0, sizeof tvp);
      if (!encode_rows(&tq, c.q, a.T_q, a.H, a.d, a.qkv_stride) ||
          !encode_rows(&tk, c.k, a.T_q, a.H, a.d, a.qkv_stride) ||
          !encode_rows(&tv, c.v, a.T_q, a.H, a.d, a.qkv_stride))
        return HSTU_ERR_CUDA;
      if (c.paged && (!encode_pool(&tkp, c.k_pool, c.num_pages, a.H, c.page_size, a.d) ||
                      !encode_pool(&tvp, c.v_pool, c.num_pages, a.H, c.page_size, a.d)))
        return HSTU_ERR_CUDA;
      e = item_tiles == 1 ? launch_attn_sm100_single(a, thr, tq, tk, tv, tkp, tvp, c.stream)
                          : launch_attn_sm100(a, thr, tq, tk, tv, tkp, tvp, c.stream);
    } else {
      e = launch_attn_simt(a, thr, c.stream);
    }
    if (e != cudaSuccess) return HSTU_ERR_CUDA;
  }
  if (stages & HSTU_F_STAGE_EPILOGUE) {
    if ((e = launch_epilogue(a, c.stream)) != cudaSuccess) return HSTU_ERR_CUDA;
  }
  return HSTU_OK;
}

}  // namespace

extern "C" {

size_t hstu_attn_workspace_size(const hstu_attn_params* p) {
  if (check_params(p) != HSTU_OK) return 0;
  return layout_for(p, 1, use_tensor_cores(p), item_tiles_for(p, false)).total;
}

size_t hstu_attn_paged_workspace_size(const hstu_attn_params* p, int32_t num_splits) {
  if (check_params(p) != HSTU_OK || num_splits < 1 || num_splits > kMaxSplits) return 0;
  const bool tc = use_tensor_cores(p);
  return layout_for(p, tc ? num_splits : 1, tc, item_tiles_for(p, true)).total;
}

int32_t hstu_attn_paged_default_splits(const hstu_attn_params* p, int32_t max_cached_len) {
  if (check_params(p) != HSTU_OK) return 1;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // work items before splitting: every user has at least one block of query rows
  const long long rows = (long long)item_tiles_for(p, true) * kTile;
  const long long qblocks = std::max<long long>(p->batch, (p->total_tokens + rows - 1) / rows);
  const long long units = std::max<long long>(1, qblocks * p->num_heads);
  const long long key_tiles = std::max(1, (max_cached_len + kTile - 1) / kTile);
  long long s = std::max<long long>(1, sms / units);  // fill one wave of CTAs, not more
  s = std::min<long long>(s, std::max<long long>(1, key_tiles / 2));  // >= 2 key tiles per split
  return (int32_t)std::max<long long>(1, std::min<long long>(s, kMaxSplits));
}

int hstu_attn_fwd(const hstu_attn_params* p, const void* q, const void* k, const void* v, const void* u,
                  const int32_t* seq_offsets, const int64_t* timestamps, const int32_t* num_candidates,
                  const float* rab_pos, const float* rab_ts, const float* ln_gamma, const float* ln_beta,
                  void* out, void* workspace, size_t workspace_bytes, hstu_stream_t stream) {
  Common c;
  std::memset(&c, 0, sizeof c);
  c.q = q;
  c.k = k;
  c.v = v;
  c.u = u;
  c.q_offsets = seq_offsets;
  c.ts = timestamps;
  c.num_cand = num_candidates;
  c.rab_pos = rab_pos;
  c.rab_ts = rab_ts;
  c.gamma = ln_gamma;
  c.beta = ln_beta;
  c.splits = 1;
  c.out = out;
  c.ws = workspace;
  c.ws_bytes = workspace_bytes;
  c.stream = reinterpret_cast<cudaStream_t>(stream);
  c.paged = false;
  return run(p, c);
}

int hstu_attn_fwd_paged(const hstu_attn_params* p, const void* q_new, const void* k_new, const void* v_new,
                        const void* u_new, const int32_t* new_offsets, const int64_t* timestamps,
                        const int32_t* ts_offsets, const int32_t* num_candidates, const float* rab_pos,
                        const float* rab_ts, const float* ln_gamma, const float* ln_beta, const void* k_pool,
                        const void* v_pool, int32_t num_pages, const int32_t* kv_page_table,
                        int32_t max_pages_per_user, int32_t page_size, const int32_t* cached_lens,
                        int32_t num_splits, void* out, void* workspace, size_t workspace_bytes,
                        hstu_stream_t stream) {
  Common c;
  std::memset(&c, 0, sizeof c);
  c.q = q_new;
  c.k = k_new;
  c.v = v_new;
  c.u = u_new;
  c.q_offsets = new_offsets;
  c.ts = timestamps;
  c.ts_offsets = ts_offsets;
  c.num_cand = num_candidates;
  c.rab_pos = rab_pos;
  c.rab_ts = rab_ts;
  c.gamma = ln_gamma;
  c.beta = ln_beta;
  c.k_pool = k_pool;
  c.v_pool = v_pool;
  c.num_pages = num_pages;
  c.page_table = kv_page_table;
  c.max_pages = max_pages_per_user;
  c.page_size = page_size;
  c.cached_lens = cached_lens;
  c.splits = num_splits;
  c.out = out;
  c.ws = workspace;
  c.ws_bytes = workspace_bytes;
  c.stream = reinterpret_cast<cudaStream_t>(stream);
  c.paged = true;
  return run(p, c);
}

// the tensor-core backward applies: bf16, d = 128, sm_100, not forced onto CUDA cores
bool bwd_on_tensor_cores(const hstu_attn_params* p) {
  return p->dtype == HSTU_DT_BF16 && p->head_dim == 128 && !(p->flags & HSTU_F_FORCE_SIMT) && device_is_sm100();
}

// bytes of the bf16 copy of d_o the tensor-core backward stages after the status header
size_t bwd_g_bytes(const hstu_attn_params* p) {
  return bwd_on_tensor_cores(p) ? (size_t)p->total_tokens * p->num_heads * p->head_dim * 2 : 0;
}

size_t hstu_attn_bwd_workspace_size(const hstu_attn_params* p) {
  if (check_params(p) != HSTU_OK) return 0;
  return align_up(sizeof(WsHeader)) + bwd_g_bytes(p);
}

int hstu_attn_bwd(const hstu_attn_params* p, const void* q, const void* k, const void* v,
                  const int32_t* seq_offsets, const int64_t* timestamps, const int32_t* num_candidates,
                  const float* rab_pos, const float* rab_ts, const float* d_o, float* d_q, float* d_k, float* d_v,
                  float* d_rab_pos, float* d_rab_ts, void* workspace, size_t workspace_bytes,
                  hstu_stream_t stream) {
  if (int rc = check_params(p)) return rc;
  // arrays indexed by token may be null when there are no tokens
  const bool rows = p->total_tokens > 0;
  if ((rows && (!q || !k || !v || !timestamps || !d_o || !d_q || !d_k || !d_v)) || !seq_offsets || !rab_pos ||
      !rab_ts || !d_rab_pos || !d_rab_ts || !workspace)
    return HSTU_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, d_o, d_q, d_k, d_v, workspace};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return HSTU_ERR_ALIGNMENT;
  const size_t g_bytes = bwd_g_bytes(p);
  if (workspace_bytes < sizeof(WsHeader) || (g_bytes && workspace_bytes < align_up(sizeof(WsHeader)) + g_bytes))
    return HSTU_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  AttnArgs a;
  std::memset(&a, 0, sizeof a);
  a.B = p->batch;
  a.H = p->num_heads;
  a.d = p->head_dim;
  a.n_max = p->n_max;
  a.nb = p->num_ts_buckets;
  a.T_q = p->total_tokens;
  a.qkv_stride = p->qkv_stride ? p->qkv_stride : p->num_heads * p->head_dim;
  a.u_stride = a.qkv_stride;
  a.alpha = p->alpha;
  a.num_splits = 1;
  a.in_bf16 = p->dtype == HSTU_DT_BF16 ? 1 : 0;
  a.q = q;
  a.k = k;
  a.v = v;
  a.q_offsets = seq_offsets;
  a.ts = timestamps;
  a.ts_offsets = seq_offsets;
  a.num_cand = num_candidates;
  a.rab_pos = rab_pos;
  a.rab_ts = rab_ts;
  a.hdr = static_cast<WsHeader*>(workspace);
  if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), s) != cudaSuccess ||
      cudaMemsetAsync(d_rab_pos, 0, sizeof(float) * (2 * (size_t)p->n_max - 1), s) != cudaSuccess ||
      cudaMemsetAsync(d_rab_ts, 0, sizeof(float) * (size_t)p->num_ts_buckets, s) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (a.T_q == 0) return HSTU_OK;
  // the forward's checks of offsets, lengths, candidate counts and timestamps
  if (launch_plan(a, false, p->max_seq_len, s) != cudaSuccess) return HSTU_ERR_CUDA;
  const BucketTable& thr = bucket_table(a.nb);
  if (g_bytes) {
    void* g = static_cast<char*>(workspace) + align_up(sizeof(WsHeader));
    CUtensorMap tq, tk, tv, tg;
    if (!encode_rows(&tq, q, a.T_q, a.H, a.d, a.qkv_stride) || !encode_rows(&tk, k, a.T_q, a.H, a.d, a.qkv_stride) ||
        !encode_rows(&tv, v, a.T_q, a.H, a.d, a.qkv_stride) || !encode_rows(&tg, g, a.T_q, a.H, a.d, a.H * a.d))
      return HSTU_ERR_CUDA;
    return launch_attn_bwd_sm100(a, thr, d_o, g, tq, tk, tv, tg, d_q, d_k, d_v, d_rab_pos, d_rab_ts, s) ==
                   cudaSuccess
               ? HSTU_OK
               : HSTU_ERR_CUDA;
  }
  return launch_attn_bwd(a, thr, d_o, d_q, d_k, d_v, d_rab_pos, d_rab_ts, s) == cudaSuccess ? HSTU_OK
                                                                                            : HSTU_ERR_CUDA;
}

int hstu_ts_bucket(const int64_t* dt, int64_t n, int32_t num_buckets, int32_t* out, hstu_stream_t stream) {
  if (n < 0 || num_buckets <= 0 || num_buckets > kMaxBuckets) return HSTU_ERR_INVALID_ARG;
  if (n > 0 && (!dt || !out)) return HSTU_ERR_INVALID_ARG;
  const cudaError_t e = launch_ts_bucket(dt, n, out, bucket_table(num_buckets), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

int hstu_check_device_error(const void* workspace, hstu_stream_t stream) {
  if (!workspace) return HSTU_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return HSTU_ERR_CUDA;
  int32_t status = 0;
  if (cudaMemcpy(&status, workspace, sizeof status, cudaMemcpyDeviceToHost) != cudaSuccess) return HSTU_ERR_CUDA;
  return status;
}

const char* hstu_status_string(int status) {
  switch (status) {
    case HSTU_OK: return "HSTU_OK";
    case HSTU_ERR_INVALID_ARG: return "HSTU_ERR_INVALID_ARG: invalid argument";
    case HSTU_ERR_UNSUPPORTED: return "HSTU_ERR_UNSUPPORTED: shape not supported";
    case HSTU_ERR_ALIGNMENT: return "HSTU_ERR_ALIGNMENT: pointer or stride not 16-byte aligned";
    case HSTU_ERR_LENGTH: return "HSTU_ERR_LENGTH: bad offsets, lengths or candidate counts";
    case HSTU_ERR_WORKSPACE: return "HSTU_ERR_WORKSPACE: workspace too small";
    case HSTU_ERR_CUDA: return "HSTU_ERR_CUDA: CUDA call failed";
    case HSTU_ERR_TIMEOUT: return "HSTU_ERR_TIMEOUT: a device wait ran out";
    case HSTU_ERR_UNSORTED: return "HSTU_ERR_UNSORTED: timestamps decrease within a user or exceed 2^61";
    case HSTU_ERR_PAGE: return "HSTU_ERR_PAGE: page id out of range";
    case HSTU_ERR_POOL: return "HSTU_ERR_POOL: free-page stack or page-table row too small";
    default: return "unknown status";
  }
}

int hstu_version(void) { return 100; }

}  // extern "C"
