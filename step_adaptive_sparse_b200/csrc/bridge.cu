// The global-KV bridge of the AReA pages: per head, distinctive keys by their
// deviation from the global mean key, spread spatially over the grid
// (ai.info summary, "Methodology in Plain English", Phase II: R = (rho w)^2
// tokens drawn from the rest of the grid, selected by deviation from the
// global mean key and spread spatially, rho = 0.5).
//
// Reading (shared with the oracle, bit-exact):
//   mean_d  = (sum over 1024-token chunks, in order, of the in-order chunk
//             sums of K[t, d]) * fl32(1 / N);
//   dev(t)  = (((0 + e_0) + e_1) + ...) with e_d = (K[t, d] - mean_d)^2;
//   the grid is cut into ry x rx cells; each cell gives its token of largest
//   deviation, the lowest token index among equals.
// All fp32 operations are explicit round-to-nearest (no contraction).
#include "area_internal.cuh"

namespace area {
namespace {

constexpr int kChunk = 1024;

// One block per (b, h): threads (chunk lane, dim); partial sums in shared
// memory, then one thread per dim adds the chunk sums in order.
template <typename T>
__global__ void __launch_bounds__(1024) bridge_mean_kernel(const T* __restrict__ k, int N, int D,
                                                          float* __restrict__ mean) {
  extern __shared__ float s_part[];              // [nchunk][D]
  const int bh = blockIdx.x;
  const int lanes = blockDim.x / D;
  const int cl = threadIdx.x / D, d = threadIdx.x % D;
  const int nchunk = (N + kChunk - 1) / kChunk;
  const T* kb = k + (int64_t)bh * N * D;
  if (cl < lanes) {
    for (int c = cl; c < nchunk; c += lanes) {
      float part = 0.f;
      const int t1 = min(N, (c + 1) * kChunk);
      for (int t = c * kChunk; t < t1; ++t) part = __fadd_rn(part, load_as_float(kb, (int64_t)t * D + d));
      s_part[c * D + d] = part;
    }
  }
  __syncthreads();
  if (threadIdx.x < D) {
    float total = 0.f;
    for (int c = 0; c < nchunk; ++c) total = __fadd_rn(total, s_part[c * D + threadIdx.x]);
    mean[(int64_t)bh * D + threadIdx.x] = __fmul_rn(total, __frcp_rn((float)N));
  }
}

// One warp per cell: lanes compute the deviation of the cell's tokens, then a
// warp reduction keeps the largest (the lowest index among equals).
template <typename T>
__global__ void __launch_bounds__(256) bridge_cell_kernel(const T* __restrict__ k,
                                                         const float* __restrict__ mean,
                                                         int Hg, int Wg, int D, int ry, int rx,
                                                         int ncell_total, int* __restrict__ cand) {
  const int warp_g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp_g >= ncell_total) return;
  const int R = ry * rx;
  const int bh = warp_g / R, cell = warp_g % R;
  const int cy = cell / rx, cx = cell % rx;
  const int y0 = (int)(((int64_t)cy * Hg) / ry), y1 = (int)(((int64_t)(cy + 1) * Hg) / ry);
  const int x0 = (int)(((int64_t)cx * Wg) / rx), x1 = (int)(((int64_t)(cx + 1) * Wg) / rx);
  const int cw = x1 - x0, n = (y1 - y0) * cw;
  const int64_t N = (int64_t)Hg * Wg;
  const T* kb = k + (int64_t)bh * N * D;
  const float* mu = mean + (int64_t)bh * D;
  float best = -1.f;
  int bt = 0x7fffffff;
  for (int i = lane; i < n; i += 32) {
    const int tok = (y0 + i / cw) * Wg + x0 + i % cw;
    const T* row = kb + (int64_t)tok * D;
    float dev = 0.f;
    for (int d = 0; d < D; ++d) {
      const float e = __fsub_rn(load_as_float(row, d), mu[d]);
      dev = __fadd_rn(dev, __fmul_rn(e, e));
    }
    if (dev > best || (dev == best && tok < bt)) {
      best = dev;
      bt = tok;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, off);
    const int ot = __shfl_xor_sync(0xffffffffu, bt, off);
    if (ob > best || (ob == best && ot < bt)) {
      best = ob;
      bt = ot;
    }
  }
  if (lane == 0) cand[(int64_t)bh * R + cell] = bt;
}

}  // namespace

cudaError_t launch_bridge_select(const void* k, int dtype, int B, int H, int Hg, int Wg, int D,
                                 int ry, int rx, int* cand, float* mean, cudaStream_t s) {
  const int N = Hg * Wg;
  const int nchunk = (N + kChunk - 1) / kChunk;
  const int smem = nchunk * D * (int)sizeof(float);
  const int BH = B * H;
  const int ncell = BH * ry * rx;
  const int grid2 = (ncell * 32 + 255) / 256;
  if (dtype == AREA_DTYPE_BF16) {
    auto fn = bridge_mean_kernel<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    fn<<<BH, 1024, smem, s>>>(static_cast<const __nv_bfloat16*>(k), N, D, mean);
    bridge_cell_kernel<__nv_bfloat16><<<grid2, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(k), mean, Hg, Wg, D, ry, rx, ncell, cand);
  } else {
    auto fn = bridge_mean_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    fn<<<BH, 1024, smem, s>>>(static_cast<const float*>(k), N, D, mean);
    bridge_cell_kernel<float><<<grid2, 256, 0, s>>>(static_cast<const float*>(k), mean, Hg, Wg,
                                                    D, ry, rx, ncell, cand);
  }
  return cudaGetLastError();
}

}  // namespace area
