/*
 * hstu.h - C ABI of libhstu.so: HSTU pointwise attention over jagged
 * per-user sequences on NVIDIA B200 (sm_100a).
 *
 * The operation (one definition for every entry point below):
 *
 *   For user u with n tokens of which the last c are candidates (h = n - c),
 *   local token indices i, j in [0, n):
 *     position      p(i)   = min(i, h)
 *     allowed       M(i,j) = j <= i                 for history rows (i < h)
 *                            j < h  or  j == i      for candidate rows (i >= h)
 *     time bucket   b(i,j) = clamp(floor(ln(|t_i - t_j| + 1) / 0.301), 0, NB - 1)
 *     score         s(i,j) = alpha * <q_i, k_j> + rab_pos[p(i) - p(j) + n_max - 1]
 *                            + rab_ts[b(i,j)]
 *     weight        a(i,j) = SiLU(s(i,j)) / n_max on M(i,j), 0 elsewhere
 *     per head      o_i    = sum_j a(i,j) v_j
 *     output        y_i    = (LayerNorm(o_i) * gamma + beta) * u_i
 *                            (LayerNorm over the H*d concatenated head features,
 *                             biased variance, epsilon ln_eps)
 *
 * Sources (web pages on HSTU generative recommenders):
 *   "Generative Recommenders at Scale" - Inside NVIDIA's GPU-native stack, and FAQ:
 *       HSTU swaps softmax attention for SiLU weighting, a relative attention
 *       bias and elementwise gating.
 *   "How Generative Recommenders Are Redefining RecSys at Scale" - Summary and
 *       Takeaways: timestamp-ordered interleaved items/actions; gating is
 *       applied before the output projection.
 *   "HSTU Generative Recommenders: Deploy on GPU Cloud" - M-FALCON section:
 *       candidates scored in one pass with mask and relative bias modified so
 *       that they share the history computation.
 *   "Recomendador generativo HSTU com Dynamo-Triton" - KV cache section: the
 *       cache keeps attention state of a stable prefix in a paged GPU table so
 *       that only new actions and candidates are computed.
 *
 * Conventions
 *   - The caller owns every buffer.  The library never allocates device or
 *     host memory; scratch space is the caller's `workspace` (the one
 *     exception, cuBLASLt's per-device handle, is described at hstu_linear).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  The return value covers host-side argument checks and
 *     launch errors only.  Errors the device detects (bad offsets, lengths
 *     above n_max, unsorted timestamps, page ids out of range, a wait that ran
 *     out) are written to a status word inside the workspace and read with
 *     hstu_check_device_error().
 *   - Device pointers (including ln_gamma, ln_beta) must be 16-byte aligned;
 *     q/k/v/u row strides must be
 *     multiples of 8 elements (bf16) or 4 elements (fp32).
 *   - `out` must not alias any input.
 *   - Within one user, timestamps must be non-decreasing (the pages' inputs
 *     are timestamp-ordered); the device reports HSTU_ERR_UNSORTED otherwise.
 *   - No state is kept between calls; calls on different streams with
 *     different workspaces may run concurrently.
 */
#ifndef HSTU_H_
#define HSTU_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#ifndef HSTU_STREAM_T_DEFINED
#define HSTU_STREAM_T_DEFINED
typedef struct CUstream_st* hstu_stream_t; /* same object as cudaStream_t */
#endif

typedef enum {
  HSTU_OK = 0,
  HSTU_ERR_INVALID_ARG = -1,   /* a NULL pointer, a non-positive size, an unknown flag      */
  HSTU_ERR_UNSUPPORTED = -2,   /* a shape this build does not implement                     */
  HSTU_ERR_ALIGNMENT = -3,     /* a pointer or stride breaks the 16-byte rule               */
  HSTU_ERR_LENGTH = -4,        /* device: offsets not monotone, n > n_max, c > n, T mismatch */
  HSTU_ERR_WORKSPACE = -5,     /* workspace too small                                        */
  HSTU_ERR_CUDA = -6,          /* a CUDA runtime/driver call failed                          */
  HSTU_ERR_TIMEOUT = -7,       /* device: a bounded wait inside a kernel ran out             */
  HSTU_ERR_UNSORTED = -8,      /* device: timestamps decrease inside a user                  */
  HSTU_ERR_PAGE = -9,          /* device: a page-table entry outside [0, num_pages)          */
  HSTU_ERR_POOL = -10          /* device: KV append found the free-page stack or a page-table
                                  row too small; nothing was changed                         */
} hstu_status;

typedef enum { HSTU_DT_F32 = 0, HSTU_DT_BF16 = 1 } hstu_dtype;

/* flags */
#define HSTU_F_FORCE_SIMT     0x1u  /* use the CUDA-core kernel even where the tensor-core one applies */
#define HSTU_F_OUTPUT_RAW_AV  0x2u  /* write o = A.V as fp32 [T,H,d] to `out` instead of y            */
#define HSTU_F_PRECISE_SILU   0x4u  /* tensor-core path: SiLU with an fp32 tanh per score (slower);
                                       default: packed bf16x2 tanh/FMA, P is bf16 either way         */
#define HSTU_F_STAGE_PLAN     0x10u /* run only the validate + tile-schedule kernels                    */
#define HSTU_F_STAGE_ATTN     0x20u /* run only the attention kernel (needs a plan in the workspace)    */
#define HSTU_F_STAGE_EPILOGUE 0x40u /* run only the LayerNorm-gate epilogue (needs the attention part)  */
/* With none of the HSTU_F_STAGE_* bits set a call runs all three stages.  The
 * split lets a caller time each kernel with events on its own stream; the
 * stages must run in order on one stream with one workspace. */

typedef struct {
  int32_t batch;           /* B users                                                        */
  int32_t num_heads;       /* H                                                              */
  int32_t head_dim;        /* d = d_qk = d_v; tensor-core path: 128 (bf16); CUDA-core: 1..256 */
  int32_t n_max;           /* N_max: rab_pos has 2*n_max-1 entries; every n <= n_max         */
  int32_t num_ts_buckets;  /* NB entries of rab_ts, 1..128                                   */
  int32_t total_tokens;    /* T: query rows (all tokens, or new tokens in paged mode)        */
  int32_t max_seq_len;     /* host upper bound of n over users (paged: cached + new)          */
  int32_t qkv_stride;      /* elements between consecutive tokens in q, k, v; 0 = H*d       */
  int32_t u_stride;        /* elements between consecutive tokens in u; 0 = H*d             */
  float alpha;             /* score scale, usually 1/sqrt(d)                                 */
  float ln_eps;            /* LayerNorm epsilon, usually 1e-5                                */
  hstu_dtype dtype;        /* type of q, k, v, u, the pool and out (raw-AV output is fp32)   */
  uint32_t flags;          /* HSTU_F_*                                                       */
} hstu_attn_params;

/* Bytes of workspace hstu_attn_fwd needs for these parameters. */
size_t hstu_attn_workspace_size(const hstu_attn_params* p);

/*
 * Jagged full-sequence forward (prefill / training-style forward, M-FALCON
 * ranking when num_candidates is given).
 *   q, k, v        [T, H, d] dtype, token stride qkv_stride
 *   u              [T, H*d]  dtype, token stride u_stride
 *   seq_offsets    [B+1] int32, seq_offsets[0] = 0, seq_offsets[B] = T
 *   timestamps     [T] int64 seconds, non-decreasing inside each user
 *   num_candidates [B] int32 or NULL (no candidates); the last c tokens of a
 *                  user are its candidates
 *   rab_pos        [2*n_max-1] fp32;  rab_ts [num_ts_buckets] fp32
 *   ln_gamma, ln_beta  [H*d] fp32 or NULL (= 1 and = 0)
 *   out            [T, H*d] dtype (fp32 [T,H,d] o with HSTU_F_OUTPUT_RAW_AV)
 *   workspace      device scratch of at least hstu_attn_workspace_size() bytes
 * With T = 0 the arrays indexed by token (q, k, v, u, timestamps, out) may be
 * NULL; the call then only checks seq_offsets.
 * Returns HSTU_OK or a negative hstu_status.
 */
int hstu_attn_fwd(const hstu_attn_params* p, const void* q, const void* k, const void* v,
                  const void* u, const int32_t* seq_offsets, const int64_t* timestamps,
                  const int32_t* num_candidates, const float* rab_pos, const float* rab_ts,
                  const float* ln_gamma, const float* ln_beta, void* out, void* workspace,
                  size_t workspace_bytes, hstu_stream_t stream);

/*
 * hstu_attn_fwd without a workspace argument, for callers that cannot
 * allocate device memory where they run attention (for example a server whose
 * memory plan forbids allocation on the request path, or a plug-in whose host
 * runtime owns the allocator).  The pages have no counterpart: this is an
 * interface convenience of this library.  Same arguments and result as
 * hstu_attn_fwd minus workspace/workspace_bytes (invalid parameters give the
 * codes hstu_attn_fwd gives).  Scratch lives in one 16 MiB device array of
 * the library, held on every GPU that loads it until exit; problems whose
 * hstu_attn_workspace_size() exceeds 16 MiB (about 8,000 tokens at
 * H*d = 512) return HSTU_ERR_WORKSPACE before any launch.  All calls share
 * that array: calls whose kernels overlap on the GPU race, so order them
 * (e.g. one stream).  Every call clears the part that must start at zero.
 * The first call in a CUDA context looks the array's address up and keeps it
 * for that context; a call in another context (another device, or the same
 * device after cudaDeviceReset) looks it up again.  Make each context's first
 * call before any stream capture.  Nothing is allocated.  The device status
 * word sits in that internal array: read it with
 * hstu_static_ws_check_device_error().
 */
int hstu_attn_fwd_static_ws(const hstu_attn_params* p, const void* q, const void* k, const void* v,
                            const void* u, const int32_t* seq_offsets, const int64_t* timestamps,
                            const int32_t* num_candidates, const float* rab_pos, const float* rab_ts,
                            const float* ln_gamma, const float* ln_beta, void* out, hstu_stream_t stream);

/* Synchronises `stream`, then returns the status word the device wrote during
 * the last hstu_attn_fwd_static_ws call on the current device (HSTU_OK if
 * none); HSTU_ERR_CUDA if the array's address cannot be looked up. */
int hstu_static_ws_check_device_error(hstu_stream_t stream);

/* Bytes of workspace hstu_attn_fwd_paged needs with `num_splits` key splits. */
size_t hstu_attn_paged_workspace_size(const hstu_attn_params* p, int32_t num_splits);

/* A split count that fills the GPU for this problem (1..64). */
int32_t hstu_attn_paged_default_splits(const hstu_attn_params* p, int32_t max_cached_len);

/*
 * Incremental forward over a paged K/V cache.  User u has cached_lens[u]
 * prefix tokens whose K/V sit in the pools, plus new tokens given densely.
 * The result for every new token equals the full-recompute result over
 * prefix + new tokens (positions and timestamps count the prefix).
 *   q_new, k_new, v_new [T_new, H, d]; u_new [T_new, H*d]   (T_new = p->total_tokens)
 *   new_offsets   [B+1] int32 over the new tokens
 *   timestamps    int64, per user cached_lens[u] + new tokens (prefix first),
 *                 jagged by ts_offsets [B+1]
 *   num_candidates [B] int32 or NULL: the last new tokens of a user are candidates
 *   k_pool, v_pool [num_pages, H, page_size, d] dtype; slot s of page g holds
 *                 token g_index*page_size + s of the user that owns the page
 *   kv_page_table [B, max_pages_per_user] int32 physical page ids; entry
 *                 (u, x) for x < ceil(cached_lens[u]/page_size) must be in
 *                 [0, num_pages); other entries are not read
 *   page_size     8, 16, 32, 64 or 128 (tensor-core path); any positive value (CUDA-core path)
 *   num_splits    key splits per (user, head, query tile), 1..64
 *   out           [T_new, H*d] dtype
 */
int hstu_attn_fwd_paged(const hstu_attn_params* p, const void* q_new, const void* k_new,
                        const void* v_new, const void* u_new, const int32_t* new_offsets,
                        const int64_t* timestamps, const int32_t* ts_offsets,
                        const int32_t* num_candidates, const float* rab_pos,
                        const float* rab_ts, const float* ln_gamma, const float* ln_beta,
                        const void* k_pool, const void* v_pool, int32_t num_pages,
                        const int32_t* kv_page_table, int32_t max_pages_per_user,
                        int32_t page_size, const int32_t* cached_lens, int32_t num_splits,
                        void* out, void* workspace, size_t workspace_bytes,
                        hstu_stream_t stream);

/*
 * Time buckets of n time differences: out[i] = clamp(floor(ln(|dt[i]|+1)/0.301),
 * 0, num_buckets-1), bit-exact for every int64 input.
 *   dt [n] int64 device; out [n] int32 device; num_buckets 1..128.
 */
int hstu_ts_bucket(const int64_t* dt, int64_t n, int32_t num_buckets, int32_t* out,
                   hstu_stream_t stream);

/* ---- Layer glue around the attention ------------------------------------
 *
 * One HSTU layer is  x -> f1 -> attention -> f2  (no residual, no input norm):
 *   f1:  [U | V | Q | K] = SiLU(x W1 + b1)       d_model -> 4*H*d
 *   f2:  x_next          = y W2 + b2             H*d -> d_model
 * ("Generative Recommenders at Scale", Inside NVIDIA's GPU-native stack: the
 * pointwise projection with SiLU feeding the attention; "How Generative
 * Recommenders Are Redefining RecSys at Scale", Takeaways: gating before the
 * output projection.)  f1's output columns are ordered [U | V | Q | K], each
 * block H*d wide and head-major inside (column = block*H*d + head*d + e), so
 * the four blocks of one [T, 4*H*d] buffer are directly the u, v, q, k
 * arguments of hstu_attn_fwd (token stride 4*H*d).
 *
 * bf16 calls with d_in a multiple of 64, d_out a multiple of 256 and either
 * SiLU (f1) or d_out >= 1024 run the library's own tcgen05 GEMM on pairs of
 * SMs (256 x 256 output tiles, fp32 accumulate in tensor memory) with the
 * fp32 bias and the SiLU in its epilogue: one pass over the output.  Other
 * calls (f2's narrow 512-column output, where cuBLASLt is faster; other
 * shapes, fp32, HSTU_LIN_CUBLAS) use cuBLASLt (fp32 accumulate, bias
 * rounded to bf16 for bf16 calls and added in its epilogue) and, for SiLU, an
 * in-place SiLU kernel.  The first cuBLASLt call on a device
 * creates that device's handle (host memory owned by cuBLASLt); nothing else
 * is allocated.  The workspace begins with a status word
 * (hstu_check_device_error) that reports a timed-out wait of the GEMM.
 */
#define HSTU_LIN_SILU 0x1u    /* hstu_linear only: apply SiLU to the output (f1)             */
#define HSTU_LIN_CUBLAS 0x2u  /* use the cuBLASLt GEMM even where the library's own applies  */

typedef struct {
  int64_t rows;        /* T (0 is allowed: nothing to do)                              */
  int32_t d_in;        /* K: columns of x, rows of w                                   */
  int32_t d_out;       /* N: columns of w and of out; a multiple of 8                   */
  int64_t x_stride;    /* elements between rows of x; 0 = d_in; a multiple of 8        */
  int64_t out_stride;  /* elements between rows of out; 0 = d_out; a multiple of 8     */
  hstu_dtype dtype;    /* x, w, out: bf16 (fp32 accumulate) or fp32                     */
  uint32_t flags;      /* HSTU_LIN_SILU, HSTU_LIN_CUBLAS                                */
} hstu_linear_params;

/* Bytes of workspace the linear entry points use: a 256-byte status header,
 * cuBLASLt scratch (32 MiB) and room for a bf16 copy of the bias. */
size_t hstu_linear_workspace_size(const hstu_linear_params* p);

/* out[r, :] = act(x[r, :] W + bias), act = SiLU with HSTU_LIN_SILU, else identity.
 *   x    [rows, d_in]  dtype, row stride x_stride, device, 16-byte aligned
 *   w    [d_in, d_out] dtype, row-major, contiguous, device, 16-byte aligned
 *   bias [d_out] fp32 device or NULL (= 0), added to the fp32 accumulator in the
 *        GEMM epilogue (on the cuBLASLt route of a bf16 call: rounded to bf16
 *        into the workspace first)
 *   out  [rows, d_out] dtype, row stride out_stride; must not overlap x or w
 * Returns HSTU_OK, HSTU_ERR_INVALID_ARG / _ALIGNMENT / _WORKSPACE for bad
 * arguments (nothing launched), HSTU_ERR_CUDA if cuBLASLt or a launch fails. */
int hstu_linear(const hstu_linear_params* p, const void* x, const void* w, const float* bias, void* out,
                void* workspace, size_t workspace_bytes, hstu_stream_t stream);

/* f1 of the layer: hstu_linear with HSTU_LIN_SILU forced on (w = W1 [d_model, 4*H*d]). */
int hstu_layer_f1(const hstu_linear_params* p, const void* x, const void* w1, const float* b1, void* uvqk,
                  void* workspace, size_t workspace_bytes, hstu_stream_t stream);

/* f2 of the layer: hstu_linear without activation (w = W2 [H*d, d_model]). */
int hstu_layer_f2(const hstu_linear_params* p, const void* y, const void* w2, const float* b2, void* x_next,
                  void* workspace, size_t workspace_bytes, hstu_stream_t stream);

/* ---- Backward of the attention core ----------------------------------------
 *
 * For training ("How Generative Recommenders Are Redefining RecSys at Scale",
 * Summary: the models are trained at scale): given d_o = dL/do for the raw
 * per-head output o = A V (before the LayerNorm gate; the gate's backward is
 * elementwise and not part of this call), the gradients of q, k, v and of the
 * two bias tables over jagged users (no paged prefix):
 *   ds_ij = (d_o_i . v_j) SiLU'(s_ij) / n_max on the allowed set,
 *           SiLU'(x) = sig(x) (1 + x (1 - sig(x)))
 *   d_q_i = alpha sum_j ds_ij k_j,   d_k_j = alpha sum_i ds_ij q_i,
 *   d_v_j = sum_i a_ij d_o_i,        d_rab_pos[p(i)-p(j)+n_max-1] += ds_ij,
 *   d_rab_ts[b(i,j)] += ds_ij
 * bf16 inputs with d = 128 run on the tensor cores (tcgen05): d_o is rounded
 * to bf16 into the workspace, the weights a and the score gradients ds are
 * rounded to bf16 as GEMM operands, all sums accumulate in fp32 (the bf16
 * tolerance of the forward applies).  Other inputs, or HSTU_F_FORCE_SIMT in
 * p->flags, run on CUDA cores in fp32.  Scores are recomputed as in the
 * forward (exact time buckets).
 *   q, k, v     [T, H, d] dtype with token stride p->qkv_stride
 *   d_o         [T, H, d] fp32 contiguous
 *   d_q, d_k, d_v [T, H, d] fp32 contiguous (written)
 *   d_rab_pos   [2*n_max-1] fp32, d_rab_ts [num_ts_buckets] fp32 (zeroed, then summed)
 *   workspace   hstu_attn_bwd_workspace_size(p) bytes: the status header and,
 *               on the tensor-core path, T*H*d*2 bytes for the bf16 copy of d_o
 * With T = 0 the arrays indexed by token may be NULL (the bias-table
 * gradients are still zeroed).
 * Device checks as in hstu_attn_fwd (status word in the workspace).
 */
size_t hstu_attn_bwd_workspace_size(const hstu_attn_params* p);
int hstu_attn_bwd(const hstu_attn_params* p, const void* q, const void* k, const void* v,
                  const int32_t* seq_offsets, const int64_t* timestamps, const int32_t* num_candidates,
                  const float* rab_pos, const float* rab_ts, const float* d_o, float* d_q, float* d_k, float* d_v,
                  float* d_rab_pos, float* d_rab_ts, void* workspace, size_t workspace_bytes,
                  hstu_stream_t stream);

/* ---- M-FALCON: a large candidate set against the cached history -----------
 *
 * ("HSTU Generative Recommenders: Deploy on GPU Cloud", M-FALCON section:
 * candidates are scored in microbatches in one pass over the shared history,
 * the mask and relative bias modified so that each candidate sees the history
 * and itself only.)  Candidate i of user u attends to the user's cached
 * history (positions 0 .. L_u-1, read through the paged pool) and to itself;
 * all of a user's candidates sit at position L_u.  Candidates never see one
 * another, so the split into microbatches does not change any output.
 *
 * Each microbatch takes `microbatch` candidates of every user (users with
 * fewer left are padded with zero rows whose outputs are dropped) and runs
 * the paged forward once: microbatch + L_u must not exceed n_max.
 *   q_c, k_c, v_c [T_c, H, d], u_c [T_c, H*d] dtype: candidates, user after
 *                 user by cand_offsets [B+1] (p->total_tokens = T_c);
 *                 row strides p->qkv_stride / p->u_stride as in hstu_attn_fwd
 *   hist_timestamps [hist_tokens] int64, jagged by hist_ts_offsets [B+1]:
 *                 each user's cached_lens[u] history timestamps
 *   cand_timestamps [T_c] int64, non-decreasing per user and not before the
 *                 user's last history timestamp
 *   pool, page table, cached_lens as in hstu_attn_fwd_paged
 *   max_candidates  host bound of candidates per user (sets the microbatch count)
 *   out [T_c, H*d] dtype
 * Device errors of any microbatch stay in the workspace's status word.
 */
size_t hstu_mfalcon_workspace_size(const hstu_attn_params* p, int32_t microbatch, int32_t num_splits,
                                   int64_t hist_tokens);
int hstu_mfalcon_fwd(const hstu_attn_params* p, const void* q_c, const void* k_c, const void* v_c,
                     const void* u_c, const int32_t* cand_offsets, const int64_t* hist_timestamps,
                     const int32_t* hist_ts_offsets, int64_t hist_tokens, const int64_t* cand_timestamps,
                     const float* rab_pos, const float* rab_ts, const float* ln_gamma, const float* ln_beta,
                     const void* k_pool, const void* v_pool, int32_t num_pages, const int32_t* kv_page_table,
                     int32_t max_pages_per_user, int32_t page_size, const int32_t* cached_lens,
                     int32_t max_candidates, int32_t microbatch, int32_t num_splits, void* out, void* workspace,
                     size_t workspace_bytes, hstu_stream_t stream);

/* ---- Paged KV cache: the write side --------------------------------------
 *
 * ("Recomendador generativo HSTU com Dynamo-Triton", KV cache section: the
 * attention state of a user's stable prefix is kept in a paged GPU table, so
 * that a request only computes its new actions and candidates.)  These calls
 * maintain that table after a request: the new actions' K and V are appended
 * behind the cached prefix (candidates are never cached), pages come from a
 * free-page stack on the device, and evicting a user returns its pages.
 *
 * Pool and table have the layout hstu_attn_fwd_paged reads:
 *   k_pool, v_pool  [num_pages, H, page_size, d] dtype
 *   page_table      [batch, max_pages_per_user] int32; entries past a user's
 *                   last page are -1 (append writes new ids, evict writes -1)
 *   cached_lens     [batch] int32 tokens cached per user
 *   free_pages      [num_pages] int32 stack of free page ids; the top
 *                   free_count[0] entries (indices 0 .. free_count-1) are free
 *   free_count      [1] int32 device
 * Allocation policy (deterministic): users take pages in user order from the
 * top of the stack; user u's j-th new page is
 *   free_pages[free_count - 1 - (pages taken by users < u) - j].
 * Both calls are all-or-nothing: if the stack or a page-table row is too
 * small for the whole batch, the device writes HSTU_ERR_POOL to the status
 * word of `workspace` (hstu_check_device_error) and changes nothing.
 */
typedef struct {
  int32_t batch;               /* users in page_table / cached_lens                        */
  int32_t num_heads, head_dim; /* H, d of the pool                                         */
  int32_t page_size;           /* tokens per page (any positive value)                     */
  int32_t num_pages;           /* pages in the pool                                        */
  int32_t max_pages_per_user;  /* columns of page_table                                    */
  int32_t kv_stride;           /* elements between tokens of k_new / v_new; 0 = H*d         */
  int32_t total_new;           /* rows of k_new / v_new (new_offsets[batch] must not exceed) */
  hstu_dtype dtype;            /* element type of the pool and of k_new / v_new            */
} hstu_kv_params;

/* Bytes of workspace hstu_kv_append / hstu_kv_evict need (status word + per-user scratch). */
size_t hstu_kv_workspace_size(const hstu_kv_params* p);

/* Append: for user u the first num_append[u] of its new tokens (rows
 * new_offsets[u] .. of k_new / v_new [T_new, H, d]) go to positions
 * cached_lens[u] .. of its sequence; then cached_lens[u] += num_append[u].
 * num_append NULL = all new tokens.  Pointers are device pointers; k_new,
 * v_new, the pools and kv_stride * element size must be 16-byte aligned. */
int hstu_kv_append(const hstu_kv_params* p, const void* k_new, const void* v_new, const int32_t* new_offsets,
                   const int32_t* num_append, void* k_pool, void* v_pool, int32_t* page_table,
                   int32_t* cached_lens, int32_t* free_pages, int32_t* free_count, void* workspace,
                   size_t workspace_bytes, hstu_stream_t stream);

/* Evict: every user u with evict_mask[u] != 0 pushes its pages back onto the
 * free stack (in page-table order), gets a row of -1 and cached_lens[u] = 0.
 * The pool contents are left as they are. */
int hstu_kv_evict(const hstu_kv_params* p, const int32_t* evict_mask, int32_t* page_table, int32_t* cached_lens,
                  int32_t* free_pages, int32_t* free_count, void* workspace, size_t workspace_bytes,
                  hstu_stream_t stream);

/* Synchronises `stream`, then returns the status word the device wrote into
 * `workspace` during the last call that used it (HSTU_OK if none). */
int hstu_check_device_error(const void* workspace, hstu_stream_t stream);

/* Human-readable name of a status code (static string). */
const char* hstu_status_string(int status);

/* Library version, e.g. 100 for 0.1.0. */
int hstu_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_H_ */
