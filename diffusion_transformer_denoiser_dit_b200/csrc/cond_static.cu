// dit_condition_static: the condition-vector computation (timestep sinusoid ->
// SiLU MLP -> + class row or text vector) for callers that cannot allocate device
// memory — for example code running inside an allocator callback, a host that
// hands the library a fixed memory budget, or an embedding where every cudaMalloc
// must happen up front.  Its intermediate buffers live in a fixed, file-scope
// device array instead of a handle's workspace.
#include <mutex>

#include "common.cuh"
#include "internal.h"

// Scratch capacity, in floats, shared by every call on a device:
//   E   [rows, freq_dim]   timestep sinusoid
//   hid [rows, hidden]     first MLP layer after SiLU
//   sc  [rows, hidden]     SiLU(c), written by the same kernel that writes c
constexpr int kMaxRows = 128;
constexpr int kMaxFreq = 512;
constexpr int kMaxHidden = 1536;
constexpr size_t kScratchFloats = (size_t)kMaxRows * kMaxFreq + 2 * (size_t)kMaxRows * kMaxHidden;  // 1.75 MiB

// Lives on every GPU that loads the library, until the process exits.
static __device__ __align__(256) float g_cond_scratch[kScratchFloats];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Device address of g_cond_scratch, per device, and the context it was resolved in: a
// device reset tears the primary context down and a new one may place the array
// elsewhere, so the address is looked up again whenever the current context changes.
float* g_scratch_dev[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

typedef CUresult (*PFN_ctxGetCurrent_t)(CUcontext*);

CUcontext current_context() {
  static PFN_ctxGetCurrent_t fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<PFN_ctxGetCurrent_t>(p);
  }
  CUcontext c = nullptr;
  return fn(&c) == CUDA_SUCCESS ? c : nullptr;
}

// Resolves the device address of the scratch array on the current device (once per
// device and context).  Host code must not use the array's name as a pointer: on the
// host it is only a stand-in symbol.
cudaError_t scratch_address(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  const CUcontext ctx = current_context();
  if (g_scratch_dev[dev] == nullptr || ctx == nullptr || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_cond_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_dev[dev] = static_cast<float*>(p);
    g_scratch_ctx[dev] = current_context();
  }
  *out = g_scratch_dev[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" dit_status dit_condition_static(const float* t, const void* y, int B, int guided, const float* w1,
                                           const float* b1, const float* w2, const float* b2, const float* table,
                                           int cond_kind, int num_classes, int freq_dim, int hidden, float t_scale,
                                           float* c_out, int* status, dit_stream_t stream) {
  if (t == nullptr || y == nullptr || w1 == nullptr || b1 == nullptr || w2 == nullptr || b2 == nullptr ||
      c_out == nullptr || B < 1 || hidden < 4 || (hidden & 3) || freq_dim < 4 || (freq_dim & 3))
    return DIT_ERR_INVALID_ARG;
  if (cond_kind != DIT_COND_CLASS && cond_kind != DIT_COND_VECTOR) return DIT_ERR_INVALID_ARG;
  if (cond_kind == DIT_COND_CLASS && (table == nullptr || num_classes < 1)) return DIT_ERR_INVALID_ARG;
  if (guided && cond_kind != DIT_COND_CLASS) return DIT_ERR_INVALID_ARG;
  const int R = guided ? 2 * B : B;
  // sizes beyond the fixed scratch are refused before anything is launched
  if (R > kMaxRows || freq_dim > kMaxFreq || hidden > kMaxHidden) return DIT_ERR_INVALID_ARG;

  float* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return DIT_ERR_CUDA;
  dit::CondArgs a;
  a.t = t;
  a.y = y;
  a.B = B;
  a.R = R;
  a.d = hidden;
  a.freq = freq_dim;
  a.cond_kind = cond_kind;
  a.num_classes = num_classes;
  a.guided = guided ? 1 : 0;
  a.t_scale = t_scale;
  a.w1 = w1;
  a.b1 = b1;
  a.w2 = w2;
  a.b2 = b2;
  a.table = table;
  a.E = base;                                   // fully rewritten by every call
  a.hid = base + (size_t)kMaxRows * kMaxFreq;   // fully rewritten by every call
  a.sc = a.hid + (size_t)kMaxRows * kMaxHidden;  // written, never read back here
  a.sc_bf16 = 0;
  a.c = c_out;
  a.status = status;
  if (dit::launch_condition(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return DIT_ERR_CUDA;
  return DIT_OK;
}
