// Internal declarations shared by the host API (hstu_api.cpp) and the CUDA
// kernels.  Nothing here is part of the public C ABI (include/hstu.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hstu {

constexpr int kMaxBuckets = 128;   // rab_ts entries supported
constexpr int kTile = 128;         // query rows / key rows per tensor-core tile
constexpr int kItemRows = 256;     // query rows per work item of the two-tile kernel
constexpr int kMaxSplits = 64;

// Bucket edges: thr[b] = smallest integer x with ln(x) >= 0.301*b, for
// b < num_buckets; entries at or above num_buckets hold INT64_MAX so that a
// search over all 128 entries clamps to num_buckets-1.  bucket(x) = the
// largest b with thr[b] <= x, x = |dt| + 1.
struct BucketTable {
  long long thr[kMaxBuckets];
  // For x in [2^e, 2^(e+1)), e = 0..31: bucket(x) = oct[e][0] + #{k = 1..3 : x >= oct[e][k]}
  // (an octave spans ln2/0.301 = 2.3 buckets, so it holds at most 3 edges);
  // edges that are not reached are 0xFFFFFFFF.
  unsigned int oct[32][4];
};

// Layer glue GEMM on the tensor cores (gemm_sm100.cu): out = act(x W + bias),
// bf16, on pairs of SMs (tcgen05 cta_group::2) with 256 x 256 output tiles per
// pair; K a multiple of 64, N a multiple of 256; hdr = a workspace status header.
bool gemm_sm100_supported(int K, int N);
cudaError_t launch_gemm_sm100(const void* x, long long T, int K, long long x_stride, const void* w, int N,
                              const float* bias, void* out, long long out_stride, bool silu, void* hdr,
                              cudaStream_t s);

// Built once per process in exact binary128 arithmetic (ts_table.cpp).
const BucketTable& bucket_table(int num_buckets);

// Workspace header (first 256 bytes of every workspace).
struct WsHeader {
  int32_t status;      // first device-detected error (hstu_status), 0 = OK
  int32_t detail;      // user index or item that raised it
  int32_t n_items;     // work items written by the scheduler
  int32_t blocks_done; // plan kernel: validation blocks finished (the last one schedules)
  int32_t pad[60];
};
static_assert(sizeof(WsHeader) == 256, "header size");

// Work item: one (user, block of item_tiles * kTile query rows, head, key split).
struct WorkItem {
  int32_t user;
  int32_t qtile;  // index of the block of query rows inside the user's query rows
  int32_t head;
  int32_t split;
};

// Everything the device needs for one attention call.
struct AttnArgs {
  int32_t B, H, d, n_max, nb;
  int32_t T_q;          // query rows
  int32_t qkv_stride;   // elements between tokens in q/k/v
  int32_t u_stride;     // elements between tokens in u
  float alpha;
  float ln_eps;
  int32_t paged;        // 0 = jagged full sequence, 1 = paged prefix + new tokens
  int32_t num_splits;
  int32_t page_size, num_pages, max_pages;
  int32_t max_items;
  int32_t item_tiles;   // query tiles per work item: 2 (two-tile kernel) or 1 (one-tile kernel)
  int32_t out_raw;      // write o (fp32 [T,H,d]) instead of y
  int32_t self_term;    // epilogue adds a_ii v_i for candidate rows (tensor-core path)
  int32_t out_bf16;     // out dtype
  int32_t in_bf16;      // q/k/v/u/pool dtype
  int32_t precise_silu; // tensor-core path: fp32 tanh per score instead of packed bf16x2
  int32_t o_bf16;       // o_ws holds one split of bf16 partials (two-tile kernel, y output)
  const void* q;
  const void* k;
  const void* v;
  const void* u;
  const int32_t* q_offsets;   // [B+1] over query rows
  const int64_t* ts;          // timestamps of full sequences
  const int32_t* ts_offsets;  // [B+1] over full sequences (== q_offsets when not paged)
  const int32_t* num_cand;    // [B] or null
  const float* rab_pos;
  const float* rab_ts;
  const float* ln_gamma;
  const float* ln_beta;
  const void* k_pool;
  const void* v_pool;
  const int32_t* page_table;
  const int32_t* cached_lens; // [B] or null (not paged)
  void* out;
  WsHeader* hdr;
  WorkItem* items;
  float* o_ws;                // [num_splits][T_q][H][d]
};

// Geometry of one query tile: all indices are positions inside the user's
// full sequence (prefix + new tokens in paged mode).
struct TileGeom {
  int32_t L;        // cached prefix length (0 when not paged)
  int32_t n;        // full sequence length
  int32_t h;        // history length (n - candidates)
  int32_t qs;       // first query position of the tile
  int32_t nq_rows;  // valid query rows in the tile
  int32_t kv_end;   // keys [0, kv_end) are needed by some row (candidate self term excluded)
  int32_t n_pre;    // key tiles over the paged prefix
  int32_t n_tiles;  // all key tiles
  int32_t qrow0;    // row of the tile's first query in q/u/out
  int32_t tso;      // offset of the user's timestamps
};

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Launchers implemented in the .cu files.  All return a cudaError_t.
// Validation of offsets, lengths, page ids and timestamps; with `schedule`
// the last block to finish also builds the tensor-core work list.
cudaError_t launch_plan(const AttnArgs& a, bool schedule, int max_seq_len, cudaStream_t s);
cudaError_t launch_attn_sm100(const AttnArgs& a, const BucketTable& thr, const CUtensorMap& tm_q,
                              const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                              const CUtensorMap& tm_kpool, const CUtensorMap& tm_vpool,
                              cudaStream_t s);
// One query tile per CTA (items of kTile rows), S double-buffered in tensor
// memory: for calls whose users have few query rows against long key ranges
// (the paged incremental mode).
cudaError_t launch_attn_sm100_single(const AttnArgs& a, const BucketTable& thr, const CUtensorMap& tm_q,
                                     const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                     const CUtensorMap& tm_kpool, const CUtensorMap& tm_vpool, cudaStream_t s);
cudaError_t launch_attn_simt(const AttnArgs& a, const BucketTable& thr, cudaStream_t s);

// Backward of the attention core on CUDA cores (hstu_bwd.cu); gradients fp32,
// d_rp / d_rt must be zeroed by the caller.
cudaError_t launch_attn_bwd(const AttnArgs& a, const BucketTable& thr, const float* d_o, float* dq, float* dk,
                            float* dv, float* d_rp, float* d_rt, cudaStream_t s);
// Backward on the tensor cores (attn_bwd_sm100.cu): bf16 inputs, d = 128.
// g_bf16: scratch for d_o rounded to bf16 ([T, H, 128]); tm_g maps it.
bool attn_bwd_sm100_supported(const AttnArgs& a);
cudaError_t launch_attn_bwd_sm100(const AttnArgs& a, const BucketTable& thr, const float* d_o, void* g_bf16,
                                  const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                  const CUtensorMap& tm_g, float* dq, float* dk, float* dv, float* d_rp,
                                  float* d_rt, cudaStream_t s);
cudaError_t launch_epilogue(const AttnArgs& a, cudaStream_t s);
cudaError_t launch_ts_bucket(const int64_t* dt, int64_t n, int32_t* out, const BucketTable& thr,
                             cudaStream_t s);

}  // namespace hstu
