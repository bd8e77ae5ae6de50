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
//   - The first call in a CUDA context looks the array's device address up
//     (cudaGetSymbolAddress with that context current) and keeps it for that
//     context.  A later call in a different context (another device, or the
//     same device after cudaDeviceReset re-created its primary context, which
//     reloads the module and may move the array) looks it up again.  Make
//     each context's first call before any stream capture that includes this
//     entry point.
//   - The device status word sits in the array; hstu_static_ws_check_device_error
//     reads it (it synchronises the stream, like hstu_check_device_error).
//   - No cudaMalloc, cudaFree or other allocating routine is called.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "hstu.h"

namespace {

constexpr size_t kStaticWsBytes = 16u << 20;

// The scratch array.  In host code this name is only a stand-in for the
// device object; the kernels receive its device address, looked up below.
static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

constexpr int kMaxDevices = 64;
struct CachedAddress {
  unsigned long long ctx_id;  // context the address belongs to (0 = none yet)
  void* ptr;
};
CachedAddress g_ws[kMaxDevices];
std::mutex g_ws_mutex;

// cuCtxGetCurrent / cuCtxGetId through the runtime's driver entry points (no -lcuda).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Unique id of the context current on this thread for device `dev`; 0 on failure.
unsigned long long current_context_id(int dev) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return 0;
  if (!ctx) {
    // no context yet on this thread: cudaSetDevice makes the device's primary
    // context current (creating it if needed), as the next runtime call would
    if (cudaSetDevice(dev) != cudaSuccess || get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_static_ws in the current context (nullptr on failure).
void* static_ws_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  const unsigned long long ctx = current_context_id(dev);
  if (ctx == 0) return nullptr;
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  if (g_ws[dev].ctx_id != ctx || !g_ws[dev].ptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_ws) != cudaSuccess || !ptr) return nullptr;
    g_ws[dev].ctx_id = ctx;
    g_ws[dev].ptr = ptr;
  }
  return g_ws[dev].ptr;
}

}  // namespace

extern "C" int hstu_attn_fwd_static_ws(const hstu_attn_params* p, const void* q, const void* k, const void* v,
                                       const void* u, const int32_t* seq_offsets, const int64_t* timestamps,
                                       const int32_t* num_candidates, const float* rab_pos, const float* rab_ts,
                                       const float* ln_gamma, const float* ln_beta, void* out,
                                       hstu_stream_t stream) {
  const size_t need = hstu_attn_workspace_size(p);
  // invalid parameters: hstu_attn_fwd checks them before it looks at the
  // workspace, so it returns the same code it would give with one
  if (need == 0)
    return hstu_attn_fwd(p, q, k, v, u, seq_offsets, timestamps, num_candidates, rab_pos, rab_ts, ln_gamma,
                         ln_beta, out, nullptr, 0, stream);
  if (need > kStaticWsBytes) return HSTU_ERR_WORKSPACE;  // problem too large for the static scratch
  void* ws = static_ws_address();
  if (!ws) return HSTU_ERR_CUDA;
  return hstu_attn_fwd(p, q, k, v, u, seq_offsets, timestamps, num_candidates, rab_pos, rab_ts, ln_gamma, ln_beta,
                       out, ws, kStaticWsBytes, stream);
}

extern "C" int hstu_static_ws_check_device_error(hstu_stream_t stream) {
  void* ws = static_ws_address();
  if (!ws) return HSTU_ERR_CUDA;
  return hstu_check_device_error(ws, stream);
}
