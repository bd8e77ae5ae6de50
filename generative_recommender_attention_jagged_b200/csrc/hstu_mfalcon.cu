// M-FALCON: a large candidate set scored against the cached history in
// microbatches, each one pass of the paged forward.
//
// ("HSTU Generative Recommenders: Deploy on GPU Cloud", M-FALCON section.)
// Per microbatch m every user contributes exactly `mb` rows: its candidates
// m*mb .. m*mb+mb-1 where they exist, zero rows past its last candidate.  A
// gather kernel packs those rows (and the user's history timestamps followed
// by the rows' timestamps) into the workspace; the paged forward runs with
// every row a candidate, so each row attends to the history and to itself;
// a scatter kernel copies the real rows' outputs back.  With exactly mb rows
// per user the microbatch's offsets are u*mb, known without a device scan.
//
// Workspace: [0, 256) the status word kept across microbatches, then the
// paged forward's own workspace, then the packed rows, timestamps and offsets.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "hstu.h"
#include "hstu_internal.h"

namespace hstu {
namespace {

constexpr size_t kAlignMf = 256;
size_t up(size_t x) { return (x + kAlignMf - 1) / kAlignMf * kAlignMf; }

struct MfLayout {
  size_t paged_off, paged_bytes;
  size_t q_off, k_off, v_off, u_off, out_off, ts_off, off_off;
  size_t total;
};

MfLayout layout_mf(const hstu_attn_params* p, int mb, int splits, long long hist_tokens, hstu_attn_params* pp) {
  MfLayout l;
  std::memset(&l, 0, sizeof l);
  *pp = *p;
  const long long rows = (long long)p->batch * mb;
  pp->total_tokens = (int32_t)rows;
  pp->qkv_stride = 0;
  pp->u_stride = 0;
  pp->flags = p->flags & (HSTU_F_PRECISE_SILU | HSTU_F_FORCE_SIMT);
  const size_t es = p->dtype == HSTU_DT_BF16 ? 2 : 4;
  const size_t row_bytes = (size_t)p->num_heads * p->head_dim * es;
  l.paged_off = sizeof(WsHeader);
  l.paged_bytes = hstu_attn_paged_workspace_size(pp, splits);
  if (l.paged_bytes == 0) return l;
  l.q_off = up(l.paged_off + l.paged_bytes);
  l.k_off = up(l.q_off + rows * row_bytes);
  l.v_off = up(l.k_off + rows * row_bytes);
  l.u_off = up(l.v_off + rows * row_bytes);
  l.out_off = up(l.u_off + rows * row_bytes);
  l.ts_off = up(l.out_off + rows * row_bytes);
  l.off_off = up(l.ts_off + (size_t)(hist_tokens + rows) * sizeof(int64_t));
  l.total = up(l.off_off + 3 * (size_t)(p->batch + 1) * sizeof(int32_t));
  return l;
}

struct MfArgs {
  int B, mb, m, H, d, esize, T_c, max_cand;
  long long hist_tokens;
  WsHeader* hdr;  // outer status word; pad[0] = 1 once the inputs were found consistent
  long long qkv_stride, u_stride;  // elements between candidate rows of q/k/v and of u
  const uint8_t *q, *k, *v, *u;
  const int32_t* cand_offsets;
  const int64_t* hist_ts;
  const int32_t* hist_off;
  const int64_t* cand_ts;
  const int32_t* cached_lens;
  uint8_t *q_mb, *k_mb, *v_mb, *u_mb, *out_mb;
  int64_t* ts_mb;
  int32_t *new_off, *ts_off, *ncand;
  uint8_t* out;
};

// checks the caller's offsets (the gather and scatter read through them), then
// the offsets of the packed microbatch: every user has mb rows, all candidates
__global__ void __launch_bounds__(1024) mf_meta_kernel(MfArgs a) {
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  for (int u = threadIdx.x; u < a.B; u += blockDim.x) {
    const int c0 = a.cand_offsets[u], c1 = a.cand_offsets[u + 1];
    const int h0 = a.hist_off[u], h1 = a.hist_off[u + 1];
    bool bad = c0 < 0 || c1 < c0 || c1 > a.T_c || c1 - c0 > a.max_cand || h0 < 0 || h1 < h0 ||
               (long long)h1 > a.hist_tokens || h1 - h0 != a.cached_lens[u];
    if (u == 0) bad = bad || c0 != 0 || h0 != 0;
    if (u == a.B - 1) bad = bad || c1 != a.T_c;
    if (bad) atomicCAS(&s_bad, 0, u + 1);
  }
  __syncthreads();
  if (s_bad) {
    if (threadIdx.x == 0 && atomicCAS(&a.hdr->status, 0, HSTU_ERR_LENGTH) == 0) a.hdr->detail = s_bad - 1;
    // offsets the paged forward rejects at once (the last user's rows do not reach
    // T), so that it reads nothing through the caller's offsets or stale scratch
    for (int u = threadIdx.x; u <= a.B; u += blockDim.x) {
      a.new_off[u] = 0;
      a.ts_off[u] = 0;
      if (u < a.B) a.ncand[u] = 0;
    }
    return;
  }
  for (int u = threadIdx.x; u <= a.B; u += blockDim.x) {
    a.new_off[u] = u * a.mb;
    a.ts_off[u] = a.hist_off[u] + u * a.mb;
    if (u < a.B) a.ncand[u] = a.mb;
  }
  if (threadIdx.x == 0) a.hdr->pad[0] = 1;
}

// rows (16-byte pieces; zero past the user's candidates) and timestamps of user blockIdx.x
__global__ void __launch_bounds__(256) mf_gather_kernel(MfArgs a) {
  if (a.hdr->pad[0] != 1) return;
  const int u = blockIdx.x;
  const int c0 = a.cand_offsets[u], C = a.cand_offsets[u + 1] - c0;
  const int first = a.m * a.mb;
  const int row_chunks = a.H * a.d * a.esize / 16;
  // a warp copies whole rows (tensor, row) of the microbatch, its lanes
  // striding over the row's 16-byte chunks: one division per row
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int wr = blockIdx.y * wpb + (threadIdx.x >> 5); wr < 4 * a.mb; wr += gridDim.y * wpb) {
    const int arr = wr / a.mb;
    const int j = wr - arr * a.mb;
    const int c = first + j;
    const uint8_t* src = arr == 0 ? a.q : arr == 1 ? a.k : arr == 2 ? a.v : a.u;
    uint8_t* dst = arr == 0 ? a.q_mb : arr == 1 ? a.k_mb : arr == 2 ? a.v_mb : a.u_mb;
    const long long stride = arr == 3 ? a.u_stride : a.qkv_stride;
    const uint8_t* srow = src + (size_t)(c0 + c) * stride * a.esize;
    uint8_t* drow = dst + ((size_t)u * a.mb + j) * row_chunks * 16;
    for (int ch = lane; ch < row_chunks; ch += 32) {
      uint4 val = make_uint4(0, 0, 0, 0);
      if (c < C) val = *reinterpret_cast<const uint4*>(srow + (size_t)ch * 16);
      *reinterpret_cast<uint4*>(drow + (size_t)ch * 16) = val;
    }
  }
  // timestamps: the history, then the rows' (a padding row repeats the latest one)
  const int L = a.cached_lens[u];
  const int h0 = a.hist_off[u];
  int64_t* dst_ts = a.ts_mb + a.ts_off[u];
  const int64_t pad_ts = C > 0 ? a.cand_ts[c0 + C - 1] : (L > 0 ? a.hist_ts[h0 + L - 1] : 0);
  for (int t = blockIdx.y * blockDim.x + threadIdx.x; t < L + a.mb; t += gridDim.y * blockDim.x) {
    if (t < L) dst_ts[t] = a.hist_ts[h0 + t];
    else dst_ts[t] = (first + t - L < C) ? a.cand_ts[c0 + first + t - L] : pad_ts;
  }
}

// outputs of the real rows back to their places
__global__ void __launch_bounds__(256) mf_scatter_kernel(MfArgs a) {
  if (a.hdr->pad[0] != 1) return;
  const int u = blockIdx.x;
  const int c0 = a.cand_offsets[u], C = a.cand_offsets[u + 1] - c0;
  const int first = a.m * a.mb;
  const int n = min(a.mb, C - first);
  if (n <= 0) return;
  const int row_chunks = a.H * a.d * a.esize / 16;
  for (long long x = blockIdx.y * (long long)blockDim.x + threadIdx.x; x < (long long)n * row_chunks;
       x += (long long)gridDim.y * blockDim.x) {
    const int j = (int)(x / row_chunks), ch = (int)(x - (long long)j * row_chunks);
    *reinterpret_cast<uint4*>(a.out + ((size_t)(c0 + first + j) * row_chunks) * 16 + (size_t)ch * 16) =
        *reinterpret_cast<const uint4*>(a.out_mb + ((size_t)u * a.mb + j) * row_chunks * 16 + (size_t)ch * 16);
  }
}

// keep the first error of any microbatch in the outer status word
__global__ void mf_status_kernel(WsHeader* outer, const WsHeader* inner) {
  if (threadIdx.x == 0 && inner->status != 0 && outer->status == 0) {
    outer->status = inner->status;
    outer->detail = inner->detail;
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace hstu

using namespace hstu;

extern "C" {

size_t hstu_mfalcon_workspace_size(const hstu_attn_params* p, int32_t microbatch, int32_t num_splits,
                                   int64_t hist_tokens) {
  if (!p || p->batch <= 0 || microbatch <= 0 || hist_tokens < 0) return 0;
  if ((long long)p->batch * microbatch > INT32_MAX) return 0;
  hstu_attn_params pp;
  return layout_mf(p, microbatch, num_splits, hist_tokens, &pp).total;
}

int hstu_mfalcon_fwd(const hstu_attn_params* p, const void* q_c, const void* k_c, const void* v_c,
                     const void* u_c, const int32_t* cand_offsets, const int64_t* hist_timestamps,
                     const int32_t* hist_ts_offsets, int64_t hist_tokens, const int64_t* cand_timestamps,
                     const float* rab_pos, const float* rab_ts, const float* ln_gamma, const float* ln_beta,
                     const void* k_pool, const void* v_pool, int32_t num_pages, const int32_t* kv_page_table,
                     int32_t max_pages_per_user, int32_t page_size, const int32_t* cached_lens,
                     int32_t max_candidates, int32_t microbatch, int32_t num_splits, void* out, void* workspace,
                     size_t workspace_bytes, hstu_stream_t stream) {
  if (!p || p->batch <= 0 || p->num_heads <= 0 || p->head_dim <= 0 || microbatch <= 0 || max_candidates < 0 ||
      hist_tokens < 0 || p->total_tokens < 0)
    return HSTU_ERR_INVALID_ARG;
  if (p->dtype != HSTU_DT_BF16 && p->dtype != HSTU_DT_F32) return HSTU_ERR_INVALID_ARG;
  if (!q_c || !k_c || !v_c || !u_c || !cand_offsets || !hist_timestamps || !hist_ts_offsets || !cand_timestamps ||
      !out || !workspace || !cached_lens)
    return HSTU_ERR_INVALID_ARG;
  if ((long long)p->batch * microbatch > INT32_MAX) return HSTU_ERR_INVALID_ARG;
  const int esize = p->dtype == HSTU_DT_BF16 ? 2 : 4;
  const long long hd = (long long)p->num_heads * p->head_dim;
  const long long qs = p->qkv_stride ? p->qkv_stride : hd, us = p->u_stride ? p->u_stride : hd;
  if (qs < hd || us < hd) return HSTU_ERR_INVALID_ARG;
  if ((hd * esize) % 16 || (qs * esize) % 16 || (us * esize) % 16 || !aligned16(q_c) || !aligned16(k_c) ||
      !aligned16(v_c) || !aligned16(u_c) || !aligned16(out) || !aligned16(workspace))
    return HSTU_ERR_ALIGNMENT;
  hstu_attn_params pp;
  const MfLayout l = layout_mf(p, microbatch, num_splits, hist_tokens, &pp);
  if (l.paged_bytes == 0) return HSTU_ERR_INVALID_ARG;
  if (workspace_bytes < l.total) return HSTU_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), s) != cudaSuccess) return HSTU_ERR_CUDA;
  if (p->total_tokens == 0 || max_candidates == 0) return HSTU_OK;
  MfArgs a;
  a.B = p->batch;
  a.mb = microbatch;
  a.H = p->num_heads;
  a.d = p->head_dim;
  a.esize = esize;
  a.T_c = p->total_tokens;
  a.max_cand = max_candidates;
  a.hist_tokens = hist_tokens;
  a.hdr = reinterpret_cast<WsHeader*>(ws);
  a.qkv_stride = qs;
  a.u_stride = us;
  a.q = static_cast<const uint8_t*>(q_c);
  a.k = static_cast<const uint8_t*>(k_c);
  a.v = static_cast<const uint8_t*>(v_c);
  a.u = static_cast<const uint8_t*>(u_c);
  a.cand_offsets = cand_offsets;
  a.hist_ts = hist_timestamps;
  a.hist_off = hist_ts_offsets;
  a.cand_ts = cand_timestamps;
  a.cached_lens = cached_lens;
  a.q_mb = reinterpret_cast<uint8_t*>(ws + l.q_off);
  a.k_mb = reinterpret_cast<uint8_t*>(ws + l.k_off);
  a.v_mb = reinterpret_cast<uint8_t*>(ws + l.v_off);
  a.u_mb = reinterpret_cast<uint8_t*>(ws + l.u_off);
  a.out_mb = reinterpret_cast<uint8_t*>(ws + l.out_off);
  a.ts_mb = reinterpret_cast<int64_t*>(ws + l.ts_off);
  a.new_off = reinterpret_cast<int32_t*>(ws + l.off_off);
  a.ts_off = a.new_off + (p->batch + 1);
  a.ncand = a.ts_off + (p->batch + 1);
  a.out = static_cast<uint8_t*>(out);
  a.m = 0;
  mf_meta_kernel<<<1, 1024, 0, s>>>(a);
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  const int n_mb = (max_candidates + microbatch - 1) / microbatch;
  // enough blocks per user that each thread moves about four 16-byte pieces
  const long long row_chunks = hd * esize / 16;
  const int gy_gather = (int)std::max(1ll, std::min(256ll, (4ll * microbatch * row_chunks + 1023) / 1024));
  const int gy_scatter = (int)std::max(1ll, std::min(256ll, ((long long)microbatch * row_chunks + 1023) / 1024));
  for (int m = 0; m < n_mb; ++m) {
    a.m = m;
    mf_gather_kernel<<<dim3(p->batch, gy_gather), 256, 0, s>>>(a);
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
    const int rc = hstu_attn_fwd_paged(&pp, a.q_mb, a.k_mb, a.v_mb, a.u_mb, a.new_off, a.ts_mb, a.ts_off, a.ncand,
                                       rab_pos, rab_ts, ln_gamma, ln_beta, k_pool, v_pool, num_pages,
                                       kv_page_table, max_pages_per_user, page_size, cached_lens, num_splits,
                                       a.out_mb, ws + l.paged_off, l.paged_bytes, stream);
    if (rc != HSTU_OK) return rc;
    mf_status_kernel<<<1, 32, 0, s>>>(reinterpret_cast<WsHeader*>(ws),
                                      reinterpret_cast<const WsHeader*>(ws + l.paged_off));
    mf_scatter_kernel<<<dim3(p->batch, gy_scatter), 256, 0, s>>>(a);
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  }
  return HSTU_OK;
}

}  // extern "C"
