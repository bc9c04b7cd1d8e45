// extern "C" entry points of libarea: argument validation and dispatch.
// Every function is stateless and asynchronous on the caller's stream; see
// include/area.h for the contract of each call.
#include <stdio.h>

#include "area_internal.cuh"

namespace {
thread_local int g_last_cuda_error = 0;
}  // namespace

namespace area {
int fail_cuda(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return AREA_ECUDA;
}
}  // namespace area

namespace {
using area::fail_cuda;

int finish(cudaError_t e) { return e == cudaSuccess ? AREA_OK : fail_cuda(e); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
// outputs and the merge workspace are written 32 bytes (one L2 sector) per
// thread and instruction
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31) == 0; }

bool valid_dtype(int dtype) { return dtype == AREA_DTYPE_F32 || dtype == AREA_DTYPE_BF16; }

// Common checks of the attention calls.
int check_attn(const void* q, const void* k, const void* v, const void* o, int B, int H, int N,
               int Nk, int D, int dtype) {
  if (!q || !k || !v || !o) return AREA_EINVAL;
  if (B < 1 || H < 1 || N < 1 || Nk < 1) return AREA_EINVAL;
  if (!valid_dtype(dtype)) return AREA_EUNSUPPORTED;
  if (D != 64 && D != 128) return AREA_EUNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned32(o)) return AREA_EINVAL;
  if ((int64_t)B * H > 65535 * 64) return AREA_EINVAL;
  return AREA_OK;
}

int dense_attn(const void* q, const void* k, const void* v, const void* kt, const void* vt,
               int T, void* o, int B, int H, int N, int Nk, int D, float scale, int dtype,
               cudaStream_t s) {
  int st = check_attn(q, k, v, o, B, H, N, Nk, D, dtype);
  if (st != AREA_OK) return st;
  if (B > 65535 || H > 65535) return AREA_EINVAL;
  if (T < 0 || (T > 0 && (!kt || !vt || !aligned16(kt) || !aligned16(vt)))) return AREA_EINVAL;
  if (dtype == AREA_DTYPE_BF16)       // tensor cores, head_dim 64 or 128
    return finish(area::launch_dense_attn_tc(q, k, v, kt, vt, o, B, H, N, Nk, T, D, scale, s));
  return finish(
      area::launch_dense_attn_simt(q, k, v, kt, vt, o, B, H, N, Nk, T, D, scale, dtype, s));
}

int window_attn(const void* q, const void* k, const void* v, const void* kt, const void* vt,
                int T, const int* cand, int R, const area_plan_cfg* cfg, const void* plan,
                size_t plan_bytes, void* o, void* ws, size_t ws_bytes, int H, int D, float scale,
                int dtype, cudaStream_t stream) {
  if (!plan || !ws) return AREA_EINVAL;
  area::PlanLayout L;
  int st = area::plan_layout(cfg, &L);
  if (st != AREA_OK) return st;
  st = check_attn(q, k, v, o, (int)L.B, H, (int)L.N, (int)L.N, D, dtype);
  if (st != AREA_OK) return st;
  if (T < 0 || (T > 0 && (!kt || !vt || !aligned16(kt) || !aligned16(vt)))) return AREA_EINVAL;
  if (cand && R < 1) return AREA_EINVAL;
  if (plan_bytes < (size_t)L.total) return AREA_ENOSPACE;
  const size_t ws_need = (size_t)area::window_ws_bytes(L, H, D);
  if (ws_bytes < ws_need) return AREA_ENOSPACE;
  // room for the staging area: the plan's global-KV rows are copied once per
  // call and loaded as tiles (tensor-core path, plan lists only)
  // (the plan's lists, or the bridged call's per-head candidate rows)
  const size_t stage_need = cand ? (size_t)4 * L.B * H * R * D
                                 : (size_t)area::window_stage_bytes(L, H, D);
  const bool staged = dtype == AREA_DTYPE_BF16 && (cand ? R >= 128 : L.G > 0) &&
                      L.B * H <= 65535 && ws_bytes >= ws_need + stage_need;
  if (!aligned32(ws) || (reinterpret_cast<uintptr_t>(plan) & 255) != 0) return AREA_EINVAL;
  if (H > 65535 || L.B > 65535) return AREA_EINVAL;
  if (dtype == AREA_DTYPE_BF16)       // tensor cores, head_dim 64 or 128
    return finish(area::launch_window_attn_tc(q, k, v, kt, vt, T, cand, R, L, plan, o, ws,
                                              staged, H, D, scale, stream));
  return finish(area::launch_window_attn_simt(q, k, v, kt, vt, T, cand, R, L, plan, o, ws, H, D,
                                              scale, dtype, stream));
}

}  // namespace

extern "C" {

const char* area_status_string(int status) {
  switch (status) {
    case AREA_OK: return "AREA_OK: success";
    case AREA_EINVAL: return "AREA_EINVAL: invalid argument (null pointer, size or enum)";
    case AREA_EUNSUPPORTED: return "AREA_EUNSUPPORTED: dtype, head_dim or shape not supported";
    case AREA_ENOSPACE: return "AREA_ENOSPACE: plan or workspace buffer too small";
    case AREA_ECUDA: return "AREA_ECUDA: CUDA launch error (see area_last_cuda_error)";
    default: return "unknown libarea status";
  }
}

int area_last_cuda_error(void) { return g_last_cuda_error; }

const char* area_version(void) { return "libarea 0.1.0 sm_100a"; }

int area_kernel_error(int* code) {
  if (!code) return AREA_EINVAL;
  int tc = 0, pl = 0;
  int st = finish(area::read_and_clear_tc_error(&tc));
  if (st != AREA_OK) return st;
  st = finish(area::read_and_clear_plan_error(&pl));
  if (st != AREA_OK) return st;
  *code = tc | (pl ? AREA_KERR_PLAN_BARRIER : 0);
  return AREA_OK;
}

int area_pool_kv(const void* k, const void* v, void* kp, void* vp, int B, int H, int Hg, int Wg,
                 int D, int f, int mode, int dtype, cudaStream_t stream) {
  if (!k || !v || !kp || !vp) return AREA_EINVAL;
  if (B < 1 || H < 1 || Hg < 1 || Wg < 1 || D < 1 || f < 1) return AREA_EINVAL;
  if (Hg % f || Wg % f) return AREA_EINVAL;
  if (mode != AREA_POOL_MEAN && mode != AREA_POOL_CENTER) return AREA_EINVAL;
  if (!valid_dtype(dtype)) return AREA_EINVAL;
  if (D % 8) return AREA_EUNSUPPORTED;
  if (!aligned16(k) || !aligned16(v) || !aligned16(kp) || !aligned16(vp)) return AREA_EINVAL;
  return finish(area::launch_pool_kv(k, v, kp, vp, B, H, Hg, Wg, D, f, mode, dtype, stream));
}

int area_coarse_attn(const void* q, const void* kp, const void* vp, void* o, int B, int H, int N,
                     int Nk, int D, float scale, int dtype, cudaStream_t stream) {
  return dense_attn(q, kp, vp, nullptr, nullptr, 0, o, B, H, N, Nk, D, scale, dtype, stream);
}

int area_coarse_attn_text(const void* q, const void* kp, const void* vp, const void* kt,
                          const void* vt, void* o, int B, int H, int N, int Nk, int T, int D,
                          float scale, int dtype, cudaStream_t stream) {
  return dense_attn(q, kp, vp, kt, vt, T, o, B, H, N, Nk, D, scale, dtype, stream);
}

int area_full_attn(const void* q, const void* k, const void* v, void* o, int B, int H, int N,
                   int D, float scale, int dtype, cudaStream_t stream) {
  return dense_attn(q, k, v, nullptr, nullptr, 0, o, B, H, N, N, D, scale, dtype, stream);
}

int area_dwt_detail(const void* src, int src_dtype, int C, float* energy, int B, int Hg, int Wg,
                    int mode, cudaStream_t stream) {
  if (!src || !energy) return AREA_EINVAL;
  if (B < 1 || C < 1 || Hg < 2 || Wg < 2 || (Hg & 1) || (Wg & 1)) return AREA_EINVAL;
  if (mode != AREA_DETAIL_HH && mode != AREA_DETAIL_ALL3) return AREA_EINVAL;
  if (!valid_dtype(src_dtype)) return AREA_EINVAL;
  return finish(area::launch_dwt_detail(src, src_dtype, C, energy, B, Hg, Wg, mode, stream));
}

int area_window_plan_bytes(const area_plan_cfg* cfg, size_t* plan_bytes) {
  if (!plan_bytes) return AREA_EINVAL;
  area::PlanLayout L;
  const int st = area::plan_layout(cfg, &L);
  if (st != AREA_OK) return st;
  *plan_bytes = (size_t)L.total;
  return AREA_OK;
}

int area_window_plan(const float* energy, const area_plan_cfg* cfg, void* plan,
                     size_t plan_bytes, cudaStream_t stream) {
  if (!energy || !plan) return AREA_EINVAL;
  area::PlanLayout L;
  const int st = area::plan_layout(cfg, &L);
  if (st != AREA_OK) return st;
  if (plan_bytes < (size_t)L.total) return AREA_ENOSPACE;
  if ((reinterpret_cast<uintptr_t>(plan) & 255) != 0) return AREA_EINVAL;
  return finish(area::launch_window_plan(energy, cfg, L, plan, stream));
}

int area_dwt_window_plan(const void* src, int src_dtype, int C, int mode, float* energy,
                         const area_plan_cfg* cfg, void* plan, size_t plan_bytes,
                         cudaStream_t stream) {
  if (!src || !energy || !plan) return AREA_EINVAL;
  if (C < 1 || (mode != AREA_DETAIL_HH && mode != AREA_DETAIL_ALL3)) return AREA_EINVAL;
  if (!valid_dtype(src_dtype)) return AREA_EINVAL;
  area::PlanLayout L;
  const int st = area::plan_layout(cfg, &L);
  if (st != AREA_OK) return st;
  if (plan_bytes < (size_t)L.total) return AREA_ENOSPACE;
  if ((reinterpret_cast<uintptr_t>(plan) & 255) != 0) return AREA_EINVAL;
  return finish(area::launch_dwt_window_plan(src, src_dtype, C, mode, energy, cfg, L, plan,
                                             stream));
}

int area_test_plan_barrier_expiry(const void* src, int src_dtype, int C, float* energy,
                                  const area_plan_cfg* cfg, void* plan, size_t plan_bytes,
                                  cudaStream_t stream) {
  if (!src || !energy || !plan || C < 1 || !valid_dtype(src_dtype)) return AREA_EINVAL;
  area::PlanLayout L;
  const int st = area::plan_layout(cfg, &L);
  if (st != AREA_OK) return st;
  if (plan_bytes < (size_t)L.total) return AREA_ENOSPACE;
  if ((reinterpret_cast<uintptr_t>(plan) & 255) != 0) return AREA_EINVAL;
  // every grid-barrier target one above the grid: no barrier can complete,
  // and each wait gives up after 1 ms
  return finish(area::launch_dwt_window_plan(src, src_dtype, C, AREA_DETAIL_HH, energy, cfg, L,
                                             plan, stream, 1u, 1000000ull));
}

int area_window_attn_ws_bytes(const area_plan_cfg* cfg, int H, int D, size_t* ws_bytes) {
  if (!ws_bytes || H < 1 || D < 1) return AREA_EINVAL;
  area::PlanLayout L;
  const int st = area::plan_layout(cfg, &L);
  if (st != AREA_OK) return st;
  *ws_bytes = (size_t)area::window_ws_bytes(L, H, D);
  return AREA_OK;
}

int area_window_attn_stage_bytes(const area_plan_cfg* cfg, int H, int D, size_t* stage_bytes) {
  if (!stage_bytes || H < 1 || D < 1) return AREA_EINVAL;
  area::PlanLayout L;
  const int st = area::plan_layout(cfg, &L);
  if (st != AREA_OK) return st;
  *stage_bytes = (size_t)area::window_stage_bytes(L, H, D);
  return AREA_OK;
}

int area_window_attn(const void* q, const void* k, const void* v, const area_plan_cfg* cfg,
                     const void* plan, size_t plan_bytes, void* o, void* ws, size_t ws_bytes,
                     int H, int D, float scale, int dtype, cudaStream_t stream) {
  return window_attn(q, k, v, nullptr, nullptr, 0, nullptr, 0, cfg, plan, plan_bytes, o, ws,
                     ws_bytes, H, D, scale, dtype, stream);
}

int area_window_attn_text(const void* q, const void* k, const void* v, const void* kt,
                          const void* vt, int T, const area_plan_cfg* cfg, const void* plan,
                          size_t plan_bytes, void* o, void* ws, size_t ws_bytes, int H, int D,
                          float scale, int dtype, cudaStream_t stream) {
  return window_attn(q, k, v, kt, vt, T, nullptr, 0, cfg, plan, plan_bytes, o, ws, ws_bytes, H,
                     D, scale, dtype, stream);
}

int area_bridge_select_ws_bytes(int B, int H, int Hg, int Wg, int D, size_t* ws_bytes) {
  if (!ws_bytes || B < 1 || H < 1 || Hg < 1 || Wg < 1 || D < 1) return AREA_EINVAL;
  if ((int64_t)Hg * Wg > INT32_MAX) return AREA_EUNSUPPORTED;
  *ws_bytes = area::bridge_ws_bytes(B, H, Hg, Wg, D);
  return AREA_OK;
}

int area_bridge_select(const void* k, int dtype, int B, int H, int Hg, int Wg, int D, int ry,
                       int rx, int* cand, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!k || !cand || !ws) return AREA_EINVAL;
  if (B < 1 || H < 1 || Hg < 1 || Wg < 1 || ry < 1 || rx < 1 || ry > Hg || rx > Wg)
    return AREA_EINVAL;
  if (!valid_dtype(dtype)) return AREA_EINVAL;
  if (D != 64 && D != 128) return AREA_EUNSUPPORTED;
  const int64_t N = (int64_t)Hg * Wg;
  if (N > INT32_MAX) return AREA_EUNSUPPORTED;
  if (((N + 1023) / 1024) * D * 4 > 227 * 1024) return AREA_EUNSUPPORTED;   // chunk sums in smem
  if (rx > 16384) return AREA_EUNSUPPORTED;                                  // cell keys in smem
  if (ws_bytes < area::bridge_ws_bytes(B, H, Hg, Wg, D)) return AREA_ENOSPACE;
  if (!aligned16(k) || !aligned16(ws)) return AREA_EINVAL;
  return finish(area::launch_bridge_select(k, dtype, B, H, Hg, Wg, D, ry, rx, cand,
                                           static_cast<float*>(ws), stream));
}

int area_window_attn_bridge_stage_bytes(int B, int H, int R, int D, size_t* stage_bytes) {
  if (!stage_bytes || B < 1 || H < 1 || R < 1 || D < 1) return AREA_EINVAL;
  *stage_bytes = (size_t)4 * B * H * R * D;
  return AREA_OK;
}

int area_window_attn_bridge(const void* q, const void* k, const void* v, const int* cand, int R,
                            const area_plan_cfg* cfg, const void* plan, size_t plan_bytes,
                            void* o, void* ws, size_t ws_bytes, int H, int D, float scale,
                            int dtype, cudaStream_t stream) {
  if (!cand) return AREA_EINVAL;
  return window_attn(q, k, v, nullptr, nullptr, 0, cand, R, cfg, plan, plan_bytes, o, ws,
                     ws_bytes, H, D, scale, dtype, stream);
}

}  // extern "C"
