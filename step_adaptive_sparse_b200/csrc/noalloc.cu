// area_window_attn_noalloc: windowed attention without a caller-provided
// workspace, for callers that cannot allocate device memory.
//
// The fp32 merge workspace of area_window_attn lives here in a fixed
// file-scope device array instead of a buffer the caller allocates.  Every
// GPU that loads libarea holds this array (kNoallocWsBytes) until the
// process exits.  The computation is exactly that of area_window_attn: the
// same zero / attention / finalise launches, given this array as workspace.
#include <mutex>

#include "area_internal.cuh"

namespace area {
namespace {

constexpr size_t kNoallocWsBytes = size_t(32) << 20;   // 32 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_noalloc_ws[kNoallocWsBytes / sizeof(float)];

std::mutex g_setup_mutex;
float* g_ws_ptr[kMaxDevices] = {};

// Device address of g_noalloc_ws on the current device, looked up once per
// device.  In host code the symbol is only a host-side stand-in; the address
// a kernel may use comes from cudaGetSymbolAddress with that device current.
cudaError_t workspace_for_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_ws_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_ws);
    if (e != cudaSuccess) return e;
    g_ws_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_ws_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace area

extern "C" int area_window_attn_noalloc(const void* q, const void* k, const void* v,
                                        const area_plan_cfg* cfg, const void* plan,
                                        size_t plan_bytes, void* o, int H, int D, float scale,
                                        int dtype, cudaStream_t stream) {
  if (!q || !k || !v || !o || !plan || H < 1 || (D != 64 && D != 128)) return AREA_EINVAL;
  if (dtype != AREA_DTYPE_F32 && dtype != AREA_DTYPE_BF16) return AREA_EINVAL;
  area::PlanLayout L;
  const int st = area::plan_layout(cfg, &L);
  if (st != AREA_OK) return st;
  const size_t need = (size_t)(L.B * H * L.N * D) * sizeof(float);
  if (need > area::kNoallocWsBytes) return AREA_ENOSPACE;   // beyond the static workspace
  float* ws = nullptr;
  if (area::workspace_for_current_device(&ws) != cudaSuccess) return AREA_ECUDA;
  return area_window_attn(q, k, v, cfg, plan, plan_bytes, o, ws, need, H, D, scale, dtype,
                          stream);
}
