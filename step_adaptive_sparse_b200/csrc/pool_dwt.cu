// Phase I K/V pooling and the Phase II Haar detail map: HBM-bound kernels.
//
// Pooling (AReA summary pages: ai.info "Methodology in Plain English", Phase I;
// gpt-diffusion.com "Las dos fases de AReA", Fase I): one representative K/V
// token per f x f block of the token grid.
//
// Detail map (same pages, Phase II): one-level Haar transform of each 2x2
// token cell per channel, energy averaged over channels, in exact-order fp32
// so that split decisions downstream are reproducible bit for bit.
#include "area_internal.cuh"
#include "detail_cell.cuh"

namespace area {
namespace {

// 16-byte vector of 8 bf16 or 4 fp32 values.
template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* out) {
    uint4 r = __ldcs(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      out[2 * i] = f.x;
      out[2 * i + 1] = f.y;
    }
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float* in) {
    uint4 r;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = r;
  }
};
template <> struct Vec<float> {
  static constexpr int n = 4;
  __device__ __forceinline__ static void load(const float* p, float* out) {
    float4 r = __ldcs(reinterpret_cast<const float4*>(p));
    out[0] = r.x; out[1] = r.y; out[2] = r.z; out[3] = r.w;
  }
  __device__ __forceinline__ static void store(float* p, const float* in) {
    *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
  }
};

// One thread = one 16-byte vector of one pooled token of K or V.
// Consecutive threads walk the vectors of a pooled row, then the pooled
// tokens along x, so each warp reads whole 128-byte lines of the input.
template <typename T, int MODE>
__global__ void __launch_bounds__(256) pool_kv_kernel(const T* __restrict__ k,
                                                      const T* __restrict__ v,
                                                      T* __restrict__ kp, T* __restrict__ vp,
                                                      int64_t n_vec_per_tensor, int Wg, int f,
                                                      int Wp, int Np, int vec_per_row) {
  constexpr int NV = Vec<T>::n;
  const float inv = 1.0f / (float)(f * f);
  for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < 2 * n_vec_per_tensor;
       g += (int64_t)gridDim.x * blockDim.x) {
    const bool is_v = g >= n_vec_per_tensor;
    const int64_t e = is_v ? g - n_vec_per_tensor : g;
    const int vec = (int)(e % vec_per_row);
    const int64_t row = e / vec_per_row;          // (b*H + h) * Np + pidx
    const int pidx = (int)(row % Np);
    const int64_t bh = row / Np;
    const int py = pidx / Wp, px = pidx % Wp;
    const T* src = is_v ? v : k;
    T* dst = is_v ? vp : kp;
    const int64_t N = (int64_t)Np * f * f;
    const T* base = src + (bh * N) * (int64_t)(vec_per_row * NV) + vec * NV;
    float acc[NV];
    if (MODE == AREA_POOL_CENTER) {
      const int64_t tok = (int64_t)(py * f + f / 2) * Wg + (px * f + f / 2);
      Vec<T>::load(base + tok * (vec_per_row * NV), acc);
    } else {
#pragma unroll
      for (int c = 0; c < NV; ++c) acc[c] = 0.f;
      for (int i = 0; i < f; ++i) {
        const int64_t tok0 = (int64_t)(py * f + i) * Wg + px * f;
        for (int j = 0; j < f; ++j) {
          float t[NV];
          Vec<T>::load(base + (tok0 + j) * (vec_per_row * NV), t);
#pragma unroll
          for (int c = 0; c < NV; ++c) acc[c] += t[c];
        }
      }
#pragma unroll
      for (int c = 0; c < NV; ++c) acc[c] *= inv;
    }
    Vec<T>::store(dst + row * (int64_t)(vec_per_row * NV) + vec * NV, acc);
  }
}

// One thread per 2x2 cell (the cell arithmetic is in detail_cell.cuh).
template <typename T, int MODE, bool VEC>
__global__ void __launch_bounds__(256) dwt_detail_kernel(const T* __restrict__ src, int C,
                                                         float* __restrict__ energy, int B,
                                                         int Hg, int Wg) {
  const int64_t ncell = (int64_t)B * (Hg / 2) * (Wg / 2);
  const float inv = __frcp_rn((float)C);
  for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < ncell;
       g += (int64_t)gridDim.x * blockDim.x)
    energy[g] = detail_cell<T, MODE, VEC>(src, C, g, Hg, Wg, inv);
}

int grid_for(int64_t work, int block) {
  int64_t g = (work + block - 1) / block;
  const int64_t cap = 148LL * 64;  // grid-stride beyond this
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

cudaError_t launch_pool_kv(const void* k, const void* v, void* kp, void* vp, int B, int H,
                           int Hg, int Wg, int D, int f, int mode, int dtype, cudaStream_t s) {
  const int Wp = Wg / f, Np = (Hg / f) * Wp;
  const int nv = dtype == AREA_DTYPE_BF16 ? 8 : 4;
  const int vec_per_row = D / nv;
  const int64_t nvec = (int64_t)B * H * Np * vec_per_row;
  const int grid = grid_for(2 * nvec, 256);
  if (dtype == AREA_DTYPE_BF16) {
    auto* kk = static_cast<const __nv_bfloat16*>(k);
    auto* vv = static_cast<const __nv_bfloat16*>(v);
    auto* ko = static_cast<__nv_bfloat16*>(kp);
    auto* vo = static_cast<__nv_bfloat16*>(vp);
    if (mode == AREA_POOL_MEAN)
      pool_kv_kernel<__nv_bfloat16, AREA_POOL_MEAN><<<grid, 256, 0, s>>>(kk, vv, ko, vo, nvec, Wg, f, Wp, Np, vec_per_row);
    else
      pool_kv_kernel<__nv_bfloat16, AREA_POOL_CENTER><<<grid, 256, 0, s>>>(kk, vv, ko, vo, nvec, Wg, f, Wp, Np, vec_per_row);
  } else {
    auto* kk = static_cast<const float*>(k);
    auto* vv = static_cast<const float*>(v);
    auto* ko = static_cast<float*>(kp);
    auto* vo = static_cast<float*>(vp);
    if (mode == AREA_POOL_MEAN)
      pool_kv_kernel<float, AREA_POOL_MEAN><<<grid, 256, 0, s>>>(kk, vv, ko, vo, nvec, Wg, f, Wp, Np, vec_per_row);
    else
      pool_kv_kernel<float, AREA_POOL_CENTER><<<grid, 256, 0, s>>>(kk, vv, ko, vo, nvec, Wg, f, Wp, Np, vec_per_row);
  }
  return cudaGetLastError();
}

cudaError_t launch_dwt_detail(const void* src, int src_dtype, int C, float* energy, int B,
                              int Hg, int Wg, int mode, cudaStream_t s) {
  const int64_t ncell = (int64_t)B * (Hg / 2) * (Wg / 2);
  const int grid = grid_for(ncell, 256);
#define AREA_DWT_LAUNCH(T, M, V) \
  dwt_detail_kernel<T, M, V><<<grid, 256, 0, s>>>(static_cast<const T*>(src), C, energy, B, Hg, Wg)
  if (src_dtype == AREA_DTYPE_BF16) {
    const bool vec = C % 8 == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0;
    if (mode == AREA_DETAIL_HH) {
      if (vec) AREA_DWT_LAUNCH(__nv_bfloat16, AREA_DETAIL_HH, true);
      else AREA_DWT_LAUNCH(__nv_bfloat16, AREA_DETAIL_HH, false);
    } else {
      if (vec) AREA_DWT_LAUNCH(__nv_bfloat16, AREA_DETAIL_ALL3, true);
      else AREA_DWT_LAUNCH(__nv_bfloat16, AREA_DETAIL_ALL3, false);
    }
  } else {
    const bool vec = C % 4 == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0;
    if (mode == AREA_DETAIL_HH) {
      if (vec) AREA_DWT_LAUNCH(float, AREA_DETAIL_HH, true);
      else AREA_DWT_LAUNCH(float, AREA_DETAIL_HH, false);
    } else {
      if (vec) AREA_DWT_LAUNCH(float, AREA_DETAIL_ALL3, true);
      else AREA_DWT_LAUNCH(float, AREA_DETAIL_ALL3, false);
    }
  }
#undef AREA_DWT_LAUNCH
  return cudaGetLastError();
}

}  // namespace area
