// Paged KV cache, write side: append new actions' K/V behind the cached
// prefix (pages from a device free-page stack) and evict users.
//
// ("Recomendador generativo HSTU com Dynamo-Triton", KV cache section: a
// stable prefix of each user is kept in a paged GPU table so that a request
// only computes its new actions and candidates; the table is looked up,
// allocated, appended to and evicted.)
//
// Append runs as two kernels on the caller's stream:
//   1. plan (one block): per user the pages the append needs, a block-wide
//      prefix sum, the all-or-nothing check against the free stack and the
//      page-table rows, then the new page ids, the new cached lengths and the
//      new stack height.  It leaves the users' old lengths in the workspace.
//   2. copy (a block row per user): 16-byte moves of every appended token's
//      K and V rows (all heads) into their page slots, reading the old lengths.
// Evict is one block: prefix sum of the users' page counts, pages pushed back
// in page-table order, rows cleared to -1, lengths zeroed.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "hstu.h"
#include "hstu_internal.h"
#include "device_common.cuh"

namespace hstu {
namespace {

constexpr int kPlanThreads = 1024;
constexpr int32_t kErrPool = -10;

struct KvArgs {
  int32_t B, H, d, P, num_pages, max_pages, esize, total_new;
  long long kv_stride;  // elements between tokens of k_new / v_new
  const uint8_t* k_new;
  const uint8_t* v_new;
  const int32_t* new_offsets;
  const int32_t* num_append;
  uint8_t* k_pool;
  uint8_t* v_pool;
  int32_t* page_table;
  int32_t* cached_lens;
  int32_t* free_pages;
  int32_t* free_count;
  WsHeader* hdr;     // status word; pad[0] = 1 once the plan was applied
  int32_t* l_old;    // [B] lengths before the append
  int32_t* n_app;    // [B] tokens appended
};

// Exclusive prefix sum of v over the block (all threads call it), with the total.
__device__ int block_exclusive_scan(int v, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(~0u, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int ws = lane < nwarps ? warp_sums[lane] : 0;
    int wi = ws;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(~0u, wi, o);
      if (lane >= o) wi += y;
    }
    warp_sums[lane] = wi - ws;        // exclusive sum of the warps before
    if (lane == 31) warp_sums[32] = wi;  // block total
  }
  __syncthreads();
  const int excl = warp_sums[warp] + incl - v;
  total = warp_sums[32];
  __syncthreads();
  return excl;
}

__global__ void __launch_bounds__(kPlanThreads) kv_append_plan_kernel(const KvArgs a) {
  __shared__ int warp_sums[33];
  __shared__ int s_err, s_total;
  if (threadIdx.x == 0) {
    s_err = 0;
    s_total = 0;
  }
  __syncthreads();
  // pass 1: validate and count pages (total over users, in chunks of the block)
  for (int base = 0; base < a.B; base += blockDim.x) {
    const int u = base + threadIdx.x;
    int need = 0;
    if (u < a.B) {
      const int L = a.cached_lens[u];
      const int r0 = a.new_offsets[u], r1 = a.new_offsets[u + 1];
      const int n_new = r1 - r0;
      const int app = a.num_append ? a.num_append[u] : n_new;
      if (L < 0 || r0 < 0 || r1 > a.total_new || n_new < 0 || app < 0 || app > n_new) {
        atomicCAS(&s_err, 0, kErrLength);
      } else {
        const long long have = ((long long)L + a.P - 1) / a.P;
        const long long want = ((long long)L + app + a.P - 1) / a.P;
        if (want > a.max_pages) {
          atomicCAS(&s_err, 0, kErrPool);
        } else {
          need = (int)(want - have);
          // a partly filled last page receives tokens: its id must be a pool page
          if (app > 0 && L % a.P != 0) {
            const int pid = a.page_table[(size_t)u * a.max_pages + L / a.P];
            if (pid < 0 || pid >= a.num_pages) atomicCAS(&s_err, 0, kErrPage);
          }
        }
      }
    }
    int total;
    block_exclusive_scan(need, warp_sums, total);
    if (threadIdx.x == 0) s_total += total;
    __syncthreads();
  }
  const int fc = *a.free_count;
  if (threadIdx.x == 0 && s_err == 0 && (s_total > fc || fc > a.num_pages)) s_err = kErrPool;
  __syncthreads();
  if (s_err == 0)  // the pages about to be taken must be pool pages
    for (int x = fc - s_total + threadIdx.x; x < fc; x += blockDim.x) {
      const int pid = a.free_pages[x];
      if (pid < 0 || pid >= a.num_pages) atomicCAS(&s_err, 0, kErrPage);
    }
  __syncthreads();
  if (s_err != 0) {  // all or nothing
    if (threadIdx.x == 0) report_error(a.hdr, s_err, 0);
    return;
  }
  // pass 2: take the pages (users in order from the top of the stack)
  int carry = 0;
  for (int base = 0; base < a.B; base += blockDim.x) {
    const int u = base + threadIdx.x;
    int need = 0, L = 0, app = 0;
    long long have = 0;
    if (u < a.B) {
      L = a.cached_lens[u];
      app = a.num_append ? a.num_append[u] : a.new_offsets[u + 1] - a.new_offsets[u];
      have = ((long long)L + a.P - 1) / a.P;
      need = (int)(((long long)L + app + a.P - 1) / a.P - have);
    }
    int total;
    const int pre = carry + block_exclusive_scan(need, warp_sums, total);
    if (u < a.B) {
      int32_t* row = a.page_table + (size_t)u * a.max_pages;
      for (int j = 0; j < need; ++j) row[have + j] = a.free_pages[fc - 1 - pre - j];
      a.l_old[u] = L;
      a.n_app[u] = app;
      a.cached_lens[u] = L + app;
    }
    carry += total;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    *a.free_count = fc - s_total;
    a.hdr->pad[0] = 1;  // applied: the copy kernel may run
  }
}

// K and V rows of the appended tokens of user blockIdx.x, 16 bytes per step.
__global__ void __launch_bounds__(256) kv_append_copy_kernel(const KvArgs a) {
  if (a.hdr->pad[0] != 1) return;
  const int u = blockIdx.x;
  const int app = a.n_app[u];
  if (app <= 0) return;
  const int L = a.l_old[u];
  const int row0 = a.new_offsets[u];
  const int chunks = a.d * a.esize / 16;           // 16-byte pieces of one head's row
  const long long per_token = (long long)a.H * chunks;
  const long long items = (long long)app * per_token;
  const int32_t* prow = a.page_table + (size_t)u * a.max_pages;
  for (long long x = blockIdx.y * (long long)blockDim.x + threadIdx.x; x < 2 * items;
       x += (long long)gridDim.y * blockDim.x) {
    const bool is_v = x >= items;
    const long long y = is_v ? x - items : x;
    const int j = (int)(y / per_token);
    const int rem = (int)(y - (long long)j * per_token);
    const int h = rem / chunks, c = rem - h * chunks;
    const int pos = L + j;
    const int page = prow[pos / a.P];
    const int slot = pos % a.P;
    const uint8_t* src = (is_v ? a.v_new : a.k_new) +
                         (((size_t)(row0 + j) * a.kv_stride + (size_t)h * a.d) * a.esize) + (size_t)c * 16;
    uint8_t* dst = (is_v ? a.v_pool : a.k_pool) +
                   ((((size_t)page * a.H + h) * a.P + slot) * a.d) * a.esize + (size_t)c * 16;
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
  }
}

__global__ void __launch_bounds__(kPlanThreads) kv_evict_kernel(KvArgs a, const int32_t* mask) {
  __shared__ int warp_sums[33];
  __shared__ int s_err, s_total;
  if (threadIdx.x == 0) {
    s_err = 0;
    s_total = 0;
  }
  __syncthreads();
  for (int base = 0; base < a.B; base += blockDim.x) {
    const int u = base + threadIdx.x;
    int cnt = 0;
    if (u < a.B && mask[u]) {
      const int L = a.cached_lens[u];
      if (L < 0) {
        atomicCAS(&s_err, 0, kErrLength);
      } else {
        const long long pages = ((long long)L + a.P - 1) / a.P;
        if (pages > a.max_pages) atomicCAS(&s_err, 0, kErrLength);
        cnt = (int)(pages < a.max_pages ? pages : a.max_pages);
        for (int j = 0; j < cnt; ++j) {
          const int pid = a.page_table[(size_t)u * a.max_pages + j];
          if (pid < 0 || pid >= a.num_pages) atomicCAS(&s_err, 0, kErrPage);
        }
      }
    }
    int total;
    block_exclusive_scan(cnt, warp_sums, total);
    if (threadIdx.x == 0) s_total += total;
    __syncthreads();
  }
  const int fc = *a.free_count;
  if (threadIdx.x == 0 && s_err == 0 && (fc < 0 || fc + s_total > a.num_pages)) s_err = kErrPool;
  __syncthreads();
  if (s_err != 0) {
    if (threadIdx.x == 0) report_error(a.hdr, s_err, 0);
    return;
  }
  int carry = 0;
  for (int base = 0; base < a.B; base += blockDim.x) {
    const int u = base + threadIdx.x;
    const bool ev = u < a.B && mask[u];
    const int cnt = ev ? (int)(((long long)a.cached_lens[u] + a.P - 1) / a.P) : 0;
    int total;
    const int pre = carry + block_exclusive_scan(cnt, warp_sums, total);
    if (ev) {
      int32_t* row = a.page_table + (size_t)u * a.max_pages;
      for (int j = 0; j < cnt; ++j) {
        a.free_pages[fc + pre + j] = row[j];
        row[j] = -1;
      }
      a.cached_lens[u] = 0;
    }
    carry += total;
  }
  __syncthreads();
  if (threadIdx.x == 0) *a.free_count = fc + s_total;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t ws_bytes_for(const hstu_kv_params* p) {
  return sizeof(WsHeader) + ((size_t)p->batch * 2 * sizeof(int32_t) + 255) / 256 * 256;
}

int check(const hstu_kv_params* p) {
  if (!p || p->batch <= 0 || p->num_heads <= 0 || p->head_dim <= 0 || p->page_size <= 0 || p->num_pages <= 0 ||
      p->max_pages_per_user <= 0 || p->kv_stride < 0 || p->total_new < 0)
    return HSTU_ERR_INVALID_ARG;
  if (p->dtype != HSTU_DT_BF16 && p->dtype != HSTU_DT_F32) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

}  // namespace
}  // namespace hstu

using namespace hstu;

extern "C" {

size_t hstu_kv_workspace_size(const hstu_kv_params* p) { return check(p) == HSTU_OK ? ws_bytes_for(p) : 0; }

int hstu_kv_append(const hstu_kv_params* p, const void* k_new, const void* v_new, const int32_t* new_offsets,
                   const int32_t* num_append, void* k_pool, void* v_pool, int32_t* page_table,
                   int32_t* cached_lens, int32_t* free_pages, int32_t* free_count, void* workspace,
                   size_t workspace_bytes, hstu_stream_t stream) {
  if (int rc = check(p)) return rc;
  if (!k_new || !v_new || !new_offsets || !k_pool || !v_pool || !page_table || !cached_lens || !free_pages ||
      !free_count || !workspace)
    return HSTU_ERR_INVALID_ARG;
  const int esize = p->dtype == HSTU_DT_BF16 ? 2 : 4;
  const long long stride = p->kv_stride ? p->kv_stride : (long long)p->num_heads * p->head_dim;
  if (stride < (long long)p->num_heads * p->head_dim) return HSTU_ERR_INVALID_ARG;
  if ((p->head_dim * esize) % 16 || (stride * esize) % 16 || !aligned16(k_new) || !aligned16(v_new) ||
      !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(workspace))
    return HSTU_ERR_ALIGNMENT;
  if (workspace_bytes < ws_bytes_for(p)) return HSTU_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  KvArgs a;
  a.B = p->batch;
  a.H = p->num_heads;
  a.d = p->head_dim;
  a.P = p->page_size;
  a.num_pages = p->num_pages;
  a.max_pages = p->max_pages_per_user;
  a.esize = esize;
  a.total_new = p->total_new;
  a.kv_stride = stride;
  a.k_new = static_cast<const uint8_t*>(k_new);
  a.v_new = static_cast<const uint8_t*>(v_new);
  a.new_offsets = new_offsets;
  a.num_append = num_append;
  a.k_pool = static_cast<uint8_t*>(k_pool);
  a.v_pool = static_cast<uint8_t*>(v_pool);
  a.page_table = page_table;
  a.cached_lens = cached_lens;
  a.free_pages = free_pages;
  a.free_count = free_count;
  a.hdr = static_cast<WsHeader*>(workspace);
  a.l_old = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + sizeof(WsHeader));
  a.n_app = a.l_old + p->batch;
  if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), s) != cudaSuccess) return HSTU_ERR_CUDA;
  kv_append_plan_kernel<<<1, kPlanThreads, 0, s>>>(a);
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  kv_append_copy_kernel<<<dim3(p->batch, 8), 256, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

int hstu_kv_evict(const hstu_kv_params* p, const int32_t* evict_mask, int32_t* page_table, int32_t* cached_lens,
                  int32_t* free_pages, int32_t* free_count, void* workspace, size_t workspace_bytes,
                  hstu_stream_t stream) {
  if (int rc = check(p)) return rc;
  if (!evict_mask || !page_table || !cached_lens || !free_pages || !free_count || !workspace)
    return HSTU_ERR_INVALID_ARG;
  if (workspace_bytes < ws_bytes_for(p)) return HSTU_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  KvArgs a{};
  a.B = p->batch;
  a.P = p->page_size;
  a.num_pages = p->num_pages;
  a.max_pages = p->max_pages_per_user;
  a.page_table = page_table;
  a.cached_lens = cached_lens;
  a.free_pages = free_pages;
  a.free_count = free_count;
  a.hdr = static_cast<WsHeader*>(workspace);
  if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), s) != cudaSuccess) return HSTU_ERR_CUDA;
  kv_evict_kernel<<<1, kPlanThreads, 0, s>>>(a, evict_mask);
  return cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

}  // extern "C"
