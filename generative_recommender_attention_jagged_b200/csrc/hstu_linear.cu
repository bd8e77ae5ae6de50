// Layer glue around the attention: f1 = SiLU(x W1 + b1) and f2 = y W2 + b2.
//
// Both are plain GEMMs and go to cuBLASLt (fp32 accumulate, bias in the GEMM
// epilogue).  cuBLASLt has no SiLU epilogue, so f1's activation runs in place
// right after the GEMM in one vectorised pass over the output (16 bytes per
// thread and step; the [T, 4*H*d] bf16 output of f1 is read and written once).
//
// Row-major out[T, N] = x[T, K] W[K, N] is the column-major product
// out^T[N, T] = W^T[N, K] x^T[K, T] with no transposes: W row-major is a
// column-major N x K matrix with leading dimension N, and x row-major is a
// column-major K x T matrix with leading dimension x_stride.
#include <cublasLt.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "hstu.h"
#include "hstu_internal.h"

namespace {

constexpr size_t kLinearWorkspace = 32u << 20;  // cuBLASLt scratch for large-N GEMMs on sm_100
constexpr size_t kHeaderBytes = 256;             // status word of the library's own GEMM

// ---- SiLU in place ----------------------------------------------------------
__device__ __forceinline__ float silu_f(float x) { return x / (1.f + __expf(-x)); }

// bf16, 8 elements (16 bytes) per thread and step; cols and stride multiples of 8
__global__ void silu_bf16_kernel(__nv_bfloat16* out, long long rows, int cols, long long stride) {
  const int vec_per_row = cols / 8;
  const long long total = rows * vec_per_row;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long r = idx / vec_per_row;
    const int c = (int)(idx - r * vec_per_row) * 8;
    uint4* p = reinterpret_cast<uint4*>(out + r * stride + c);
    uint4 v = *p;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      h[e] = __floats2bfloat162_rn(silu_f(f.x), silu_f(f.y));
    }
    *p = v;
  }
}

// fp32, 4 elements per thread and step (accurate expf: the fp32 path is checked at 1e-5)
__global__ void silu_f32_kernel(float* out, long long rows, int cols, long long stride) {
  const int vec_per_row = cols / 4;
  const long long total = rows * vec_per_row;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long r = idx / vec_per_row;
    const int c = (int)(idx - r * vec_per_row) * 4;
    float4* p = reinterpret_cast<float4*>(out + r * stride + c);
    float4 v = *p;
    v.x = v.x / (1.f + expf(-v.x));
    v.y = v.y / (1.f + expf(-v.y));
    v.z = v.z / (1.f + expf(-v.z));
    v.w = v.w / (1.f + expf(-v.w));
    *p = v;
  }
}

// fp32 bias -> bf16 copy in the workspace, for the bf16 GEMM epilogue
__global__ void bias_to_bf16_kernel(const float* in, __nv_bfloat16* out, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    out[i] = __float2bfloat16_rn(in[i]);
}

// ---- cuBLASLt plans -----------------------------------------------------------
struct Plan {
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t a = nullptr, b = nullptr, c = nullptr;
  cublasLtMatmulAlgo_t algo;
  bool ok = false;
};

using PlanKey = std::tuple<int, long long, int, int, long long, long long, int, bool>;

constexpr int kMaxDevices = 64;
constexpr size_t kMaxCachedPlans = 1024;  // shapes beyond this get a plan per call
cublasLtHandle_t g_handle[kMaxDevices];
std::map<PlanKey, Plan> g_plans;
std::mutex g_mutex;  // guards the handles, the cache and each plan's bias-pointer attribute

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void destroy_plan(Plan& pl) {
  if (pl.a) cublasLtMatrixLayoutDestroy(pl.a);
  if (pl.b) cublasLtMatrixLayoutDestroy(pl.b);
  if (pl.c) cublasLtMatrixLayoutDestroy(pl.c);
  if (pl.op) cublasLtMatmulDescDestroy(pl.op);
  pl = Plan();
}

// Descriptors of one GEMM shape and the heuristic's first algorithm.
bool make_plan(Plan& pl, cublasLtHandle_t handle, const hstu_linear_params& p, long long xs, long long os,
               bool bias) {
  const cudaDataType_t dt = p.dtype == HSTU_DT_BF16 ? CUDA_R_16BF : CUDA_R_32F;
  bool ok = cublasLtMatmulDescCreate(&pl.op, CUBLAS_COMPUTE_32F, CUDA_R_32F) == CUBLAS_STATUS_SUCCESS;
  if (ok && bias) {  // the bias has the output's type (bf16 GEMMs take no fp32 bias)
    const cublasLtEpilogue_t epi = CUBLASLT_EPILOGUE_BIAS;
    ok = cublasLtMatmulDescSetAttribute(pl.op, CUBLASLT_MATMUL_DESC_EPILOGUE, &epi, sizeof epi) ==
         CUBLAS_STATUS_SUCCESS;
  }
  // column-major views: W^T is N x K (ld N), x^T is K x T (ld xs), out^T is N x T (ld os)
  ok = ok && cublasLtMatrixLayoutCreate(&pl.a, dt, p.d_out, p.d_in, p.d_out) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&pl.b, dt, p.d_in, p.rows, xs) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&pl.c, dt, p.d_out, p.rows, os) == CUBLAS_STATUS_SUCCESS;
  if (ok) {
    cublasLtMatmulPreference_t pref = nullptr;
    size_t ws = kLinearWorkspace;
    ok = cublasLtMatmulPreferenceCreate(&pref) == CUBLAS_STATUS_SUCCESS &&
         cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws, sizeof ws) ==
             CUBLAS_STATUS_SUCCESS;
    cublasLtMatmulHeuristicResult_t res;
    int n = 0;
    ok = ok &&
         cublasLtMatmulAlgoGetHeuristic(handle, pl.op, pl.a, pl.b, pl.c, pl.c, pref, 1, &res, &n) ==
             CUBLAS_STATUS_SUCCESS &&
         n > 0;
    if (ok) pl.algo = res.algo;
    if (pref) cublasLtMatmulPreferenceDestroy(pref);
  }
  pl.ok = ok;
  return ok;
}

// Enqueues the GEMM (plan from the cache, or a temporary one past the cache's size).
int enqueue_gemm(int dev, const hstu_linear_params& p, long long xs, long long os, const void* x, const void* w,
                 const void* bias, void* out, void* ws, cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_handle[dev] && cublasLtCreate(&g_handle[dev]) != CUBLAS_STATUS_SUCCESS) {
    g_handle[dev] = nullptr;
    return HSTU_ERR_CUDA;
  }
  const PlanKey key{dev, (long long)p.rows, p.d_in, p.d_out, xs, os, (int)p.dtype, bias != nullptr};
  Plan temp;
  Plan* pl = nullptr;
  auto it = g_plans.find(key);
  if (it != g_plans.end()) {
    pl = &it->second;
  } else if (g_plans.size() < kMaxCachedPlans) {
    pl = &g_plans[key];
    make_plan(*pl, g_handle[dev], p, xs, os, bias != nullptr);
  } else {
    pl = &temp;
    make_plan(temp, g_handle[dev], p, xs, os, bias != nullptr);
  }
  int rc = pl->ok ? HSTU_OK : HSTU_ERR_CUDA;
  if (rc == HSTU_OK && bias &&
      cublasLtMatmulDescSetAttribute(pl->op, CUBLASLT_MATMUL_DESC_BIAS_POINTER, &bias, sizeof bias) !=
          CUBLAS_STATUS_SUCCESS)
    rc = HSTU_ERR_CUDA;
  const float one = 1.f, zero = 0.f;
  if (rc == HSTU_OK && cublasLtMatmul(g_handle[dev], pl->op, &one, w, pl->a, x, pl->b, &zero, out, pl->c, out, pl->c,
                                      &pl->algo, ws, kLinearWorkspace, stream) != CUBLAS_STATUS_SUCCESS)
    rc = HSTU_ERR_CUDA;
  if (pl == &temp) destroy_plan(temp);
  return rc;
}

// status header, cuBLASLt scratch, then (bf16) the bias converted to bf16
size_t workspace_bytes(const hstu_linear_params& p) {
  return kHeaderBytes + kLinearWorkspace + (p.d_out > 0 ? ((size_t)p.d_out * 2 + 255) / 256 * 256 : 0);
}

bool device_is_sm100(int dev) {
  static int cached[64];  // 0 unknown, 1 yes, 2 no
  if (dev < 0 || dev >= 64) return false;
  if (cached[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return cached[dev] == 1;
}

int run_linear(const hstu_linear_params* p, const void* x, const void* w, const float* bias, void* out,
               void* ws, size_t ws_bytes, cudaStream_t stream, bool silu) {
  if (!p || p->rows < 0 || p->d_in <= 0 || p->d_out <= 0) return HSTU_ERR_INVALID_ARG;
  if (p->dtype != HSTU_DT_BF16 && p->dtype != HSTU_DT_F32) return HSTU_ERR_INVALID_ARG;
  if (p->flags & ~(HSTU_LIN_SILU | HSTU_LIN_CUBLAS)) return HSTU_ERR_INVALID_ARG;
  const long long xs = p->x_stride ? p->x_stride : p->d_in;
  const long long os = p->out_stride ? p->out_stride : p->d_out;
  if (xs < p->d_in || os < p->d_out) return HSTU_ERR_INVALID_ARG;
  if (p->rows == 0) return HSTU_OK;
  if (!x || !w || !out || !ws) return HSTU_ERR_INVALID_ARG;
  if (p->d_out % 8 || xs % 8 || os % 8) return HSTU_ERR_ALIGNMENT;
  if (!aligned16(x) || !aligned16(w) || !aligned16(out) || !aligned16(ws) || (bias && !aligned16(bias)))
    return HSTU_ERR_ALIGNMENT;
  if (ws_bytes < workspace_bytes(*p)) return HSTU_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HSTU_ERR_CUDA;
  char* wsc = static_cast<char*>(ws);
  // the library's own GEMM (SM pairs, bias and activation in the epilogue)
  // where it is the faster one: SiLU (the activation pass it saves is a full
  // read + write of the output) or an output of 1024+ columns; a narrow plain
  // projection (f2) has too few output tiles per SM pair and goes to cuBLASLt
  if (p->dtype == HSTU_DT_BF16 && !(p->flags & HSTU_LIN_CUBLAS) && device_is_sm100(dev) &&
      hstu::gemm_sm100_supported(p->d_in, p->d_out) && (silu || p->d_out >= 1024)) {
    if (cudaMemsetAsync(wsc, 0, kHeaderBytes, stream) != cudaSuccess) return HSTU_ERR_CUDA;
    return hstu::launch_gemm_sm100(x, p->rows, p->d_in, xs, w, p->d_out, bias, out, os, silu, wsc, stream) ==
                   cudaSuccess
               ? HSTU_OK
               : HSTU_ERR_CUDA;
  }
  ws = wsc + kHeaderBytes;
  const void* gemm_bias = bias;
  if (bias && p->dtype == HSTU_DT_BF16) {
    __nv_bfloat16* b16 = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(ws) + kLinearWorkspace);
    bias_to_bf16_kernel<<<(p->d_out + 255) / 256, 256, 0, stream>>>(bias, b16, p->d_out);
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
    gemm_bias = b16;
  }
  if (int rc = enqueue_gemm(dev, *p, xs, os, x, w, gemm_bias, out, ws, stream)) return rc;
  if (silu) {
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int per = p->dtype == HSTU_DT_BF16 ? 8 : 4;
    const long long vecs = p->rows * (p->d_out / per);
    const int blocks = (int)std::min<long long>((vecs + 255) / 256, (long long)sms * 8);
    if (p->dtype == HSTU_DT_BF16)
      silu_bf16_kernel<<<blocks, 256, 0, stream>>>(static_cast<__nv_bfloat16*>(out), p->rows, p->d_out, os);
    else
      silu_f32_kernel<<<blocks, 256, 0, stream>>>(static_cast<float*>(out), p->rows, p->d_out, os);
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  }
  return HSTU_OK;
}

}  // namespace

extern "C" {

size_t hstu_linear_workspace_size(const hstu_linear_params* p) { return p ? workspace_bytes(*p) : 0; }

int hstu_linear(const hstu_linear_params* p, const void* x, const void* w, const float* bias, void* out,
                void* workspace, size_t workspace_bytes, hstu_stream_t stream) {
  return run_linear(p, x, w, bias, out, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream),
                    p && (p->flags & HSTU_LIN_SILU));
}

int hstu_layer_f1(const hstu_linear_params* p, const void* x, const void* w1, const float* b1, void* uvqk,
                  void* workspace, size_t workspace_bytes, hstu_stream_t stream) {
  return run_linear(p, x, w1, b1, uvqk, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), true);
}

int hstu_layer_f2(const hstu_linear_params* p, const void* y, const void* w2, const float* b2, void* x_next,
                  void* workspace, size_t workspace_bytes, hstu_stream_t stream) {
  return run_linear(p, y, w2, b2, x_next, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream),
                    false);
}

}  // extern "C"
