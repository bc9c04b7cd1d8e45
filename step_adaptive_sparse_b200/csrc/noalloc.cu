// area_window_attn_noalloc: windowed attention without a caller-provided
// workspace, for callers that cannot allocate device memory.
//
// The fp32 merge workspace of area_window_attn lives here in a fixed
// file-scope device array instead of a buffer the caller allocates.  Every
// GPU that loads libarea holds this array (kNoallocWsBytes) until the
// process exits.  The computation is exactly that of area_window_attn: the
// same launches, given this array as workspace.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "area_internal.cuh"

namespace area {
namespace {

constexpr size_t kNoallocWsBytes = size_t(32) << 20;   // 32 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_noalloc_ws[kNoallocWsBytes / sizeof(float)];

// Address of g_noalloc_ws as seen from one CUDA context.  The module holding
// the array is loaded per context, so an address is only valid in the context
// it was looked up in: after cudaDeviceReset, or when the caller switches to
// another context on the same device, the array may sit elsewhere.  The cache
// is therefore keyed on the context's unique id (cuCtxGetId), not on the
// device number alone.
struct CachedAddress {
  unsigned long long ctx_id = 0;
  bool valid = false;
  float* ptr = nullptr;
};

std::mutex g_setup_mutex;
CachedAddress g_cache[kMaxDevices];

cudaError_t current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  if (!get_current || !get_id) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess) return cudaErrorNotSupported;
    get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    e = cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess) return cudaErrorNotSupported;
    get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
  if (get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  return cudaSuccess;
}

// Device address of g_noalloc_ws in the current context, looked up once per
// (device, context).  In host code the symbol is only a host-side stand-in;
// the address a kernel may use comes from cudaGetSymbolAddress with the
// device (and its context) current.
cudaError_t workspace_for_current_context(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  CachedAddress& c = g_cache[dev];
  unsigned long long id = 0;
  if (current_context_id(&id) == cudaSuccess && c.valid && c.ctx_id == id) {
    *out = c.ptr;
    return cudaSuccess;
  }
  // First call in this context (or no context bound yet: the lookup makes the
  // runtime bind the device's primary context, then its id is read).
  void* p = nullptr;
  if ((e = cudaGetSymbolAddress(&p, g_noalloc_ws)) != cudaSuccess) return e;
  if ((e = current_context_id(&id)) != cudaSuccess) return e;
  c.ptr = static_cast<float*>(p);
  c.ctx_id = id;
  c.valid = true;
  *out = c.ptr;
  return cudaSuccess;
}

}  // namespace
}  // namespace area

extern "C" int area_window_attn_noalloc(const void* q, const void* k, const void* v,
                                        const area_plan_cfg* cfg, const void* plan,
                                        size_t plan_bytes, void* o, int H, int D, float scale,
                                        int dtype, cudaStream_t stream) {
  // The same checks, in the same order, as area_window_attn up to the
  // workspace, so both calls give the same status for the same bad input.
  if (!plan) return AREA_EINVAL;
  area::PlanLayout L;
  const int st = area::plan_layout(cfg, &L);
  if (st != AREA_OK) return st;
  if (!q || !k || !v || !o || H < 1) return AREA_EINVAL;
  if (dtype != AREA_DTYPE_F32 && dtype != AREA_DTYPE_BF16) return AREA_EUNSUPPORTED;
  if (D != 64 && D != 128) return AREA_EUNSUPPORTED;
  size_t need = 0;
  const int sz = area_window_attn_ws_bytes(cfg, H, D, &need);
  if (sz != AREA_OK) return sz;
  if (need > area::kNoallocWsBytes) return AREA_ENOSPACE;   // beyond the static workspace
  float* ws = nullptr;
  const cudaError_t e = area::workspace_for_current_context(&ws);
  if (e != cudaSuccess) return area::fail_cuda(e);
  return area_window_attn(q, k, v, cfg, plan, plan_bytes, o, ws, need, H, D, scale, dtype,
                          stream);
}
