// hstu_attn_fwd_static_ws: the jagged forward without a caller-provided
// workspace.
//
// Who needs this: callers that cannot allocate device memory at the point
// where they run attention.  Examples are an inference server whose memory
// plan is fixed at start-up and forbids allocation on the request path, and
// a plug-in running inside a host runtime that owns the device allocator and
// exposes none to the plug-in.  Such callers still pass their inputs and
// output; the scratch space the forward needs (status word, tile work list,
// fp32 partial sums of A.V) lives in one file-scope device array of this
// library instead of in a caller workspace.
//
// Properties a user must know:
//   - The array holds kStaticWsBytes (16 MiB) on every GPU that loads the
//     library, until the process exits.  hstu_attn_workspace_size(p) must
//     not exceed it (about 8,000 tokens at H*d = 512); larger problems are
//     rejected with HSTU_ERR_WORKSPACE before anything is launched.
//   - All calls share the array.  Two calls whose kernels overlap on the
//     GPU (different streams without ordering between them) race on it and
//     produce garbage; order such calls, e.g. on one stream.
//   - The array keeps the previous call's contents.  The only part that
//     must start at zero, the status/work-count header, is cleared by every
//     call; the work list and partial sums are fully rewritten before use.
//   - The first call on a device looks the array's device address up (one
//     cudaGetSymbolAddress per device, cached).  Make that first call before
//     any stream capture that includes this entry point.
//   - No cudaMalloc, cudaFree or other allocating routine is called.
#include <cuda_runtime.h>

#include <mutex>

#include "hstu.h"

namespace {

constexpr size_t kStaticWsBytes = 16u << 20;

// The scratch array.  In host code this name is only a stand-in for the
// device object; the kernels receive its device address, looked up below.
static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

constexpr int kMaxDevices = 64;
void* g_ws_ptr[kMaxDevices];
std::mutex g_ws_mutex;

// Device address of g_static_ws on the current device (nullptr on failure).
void* static_ws_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  if (!g_ws_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_ws) != cudaSuccess) return nullptr;
    g_ws_ptr[dev] = ptr;
  }
  return g_ws_ptr[dev];
}

}  // namespace

extern "C" int hstu_attn_fwd_static_ws(const hstu_attn_params* p, const void* q, const void* k, const void* v,
                                       const void* u, const int32_t* seq_offsets, const int64_t* timestamps,
                                       const int32_t* num_candidates, const float* rab_pos, const float* rab_ts,
                                       const float* ln_gamma, const float* ln_beta, void* out,
                                       hstu_stream_t stream) {
  const size_t need = hstu_attn_workspace_size(p);
  if (need == 0) return HSTU_ERR_INVALID_ARG;
  if (need > kStaticWsBytes) return HSTU_ERR_WORKSPACE;  // problem too large for the static scratch
  void* ws = static_ws_address();
  if (!ws) return HSTU_ERR_CUDA;
  return hstu_attn_fwd(p, q, k, v, u, seq_offsets, timestamps, num_candidates, rab_pos, rab_ts, ln_gamma, ln_beta,
                       out, ws, kStaticWsBytes, stream);
}
