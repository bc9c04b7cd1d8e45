// Haar detail energy of one 2x2 token cell (AReA summary pages: ai.info
// "Methodology in Plain English", Phase II: a DWT map of the current hidden
// states measures fine detail).  One level of the 2-D Haar transform per
// channel, energy averaged over the channels, in exact-order fp32 (explicit
// round-to-nearest operations, no contraction) so that the split decisions
// downstream are reproducible bit for bit.  Used by the stand-alone detail
// kernel and by the fused detail + planner kernel.
#pragma once

#include "area_internal.cuh"

namespace area {
namespace detail_map {

// 16 bytes of 8 bf16 or 4 fp32 channel values, widened to fp32.
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
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
};
template <> struct Vec16<float> {
  static constexpr int n = 4;
  __device__ __forceinline__ static void load(const float* p, float* out) {
    float4 r = __ldcs(reinterpret_cast<const float4*>(p));
    out[0] = r.x; out[1] = r.y; out[2] = r.z; out[3] = r.w;
  }
};

template <int MODE>
__device__ __forceinline__ float cell_energy(float a, float b, float c, float d) {
  const float amb = __fsub_rn(a, b), cmd = __fsub_rn(c, d);
  const float hh = __fmul_rn(__fsub_rn(amb, cmd), 0.5f);
  if (MODE == AREA_DETAIL_HH) return __fmul_rn(hh, hh);
  const float lh = __fmul_rn(__fsub_rn(__fadd_rn(a, b), __fadd_rn(c, d)), 0.5f);
  const float hl = __fmul_rn(__fadd_rn(amb, cmd), 0.5f);
  return __fadd_rn(__fadd_rn(__fmul_rn(lh, lh), __fmul_rn(hl, hl)), __fmul_rn(hh, hh));
}

}  // namespace detail_map

// Energy of flat cell g = (b * Hg/2 + cy) * Wg/2 + cx of a channels-last
// source [B, Hg*Wg, C]; the C channels of each of the four tokens are read as
// 16-byte vectors when C fills whole vectors (VEC), else one by one.
// inv = fl32(1 / C).
template <typename T, int MODE, bool VEC>
__device__ __forceinline__ float detail_cell(const T* __restrict__ src, int C, int64_t g, int Hg,
                                             int Wg, float inv) {
  const int Hc = Hg / 2, Wc = Wg / 2;
  const int cx = (int)(g % Wc);
  const int64_t r = g / Wc;
  const int cy = (int)(r % Hc);
  const int64_t b = r / Hc;
  const int64_t t00 = (b * Hg + 2 * cy) * (int64_t)Wg + 2 * cx;
  const T* pa = src + t00 * C;
  const T* pb = pa + C;
  const T* pc = pa + (int64_t)Wg * C;
  const T* pd = pc + C;
  float acc = 0.f;
  if (VEC) {
    constexpr int NV = detail_map::Vec16<T>::n;
    for (int c0 = 0; c0 < C; c0 += NV) {
      float a[NV], bb[NV], c[NV], d[NV];
      detail_map::Vec16<T>::load(pa + c0, a);
      detail_map::Vec16<T>::load(pb + c0, bb);
      detail_map::Vec16<T>::load(pc + c0, c);
      detail_map::Vec16<T>::load(pd + c0, d);
#pragma unroll
      for (int i = 0; i < NV; ++i)
        acc = __fadd_rn(acc, detail_map::cell_energy<MODE>(a[i], bb[i], c[i], d[i]));
    }
  } else {
    for (int c = 0; c < C; ++c)
      acc = __fadd_rn(acc, detail_map::cell_energy<MODE>(load_as_float(pa, c), load_as_float(pb, c),
                                                         load_as_float(pc, c), load_as_float(pd, c)));
  }
  return __fmul_rn(acc, inv);
}

}  // namespace area
