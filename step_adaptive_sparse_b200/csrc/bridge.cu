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
//
// The path reads K twice, the least a two-pass statistic allows (the mean
// has to be complete before the first deviation):
//   1. bridge_chunk_kernel  -- one thread per (chunk, 16-byte column slice),
//      coalesced 16-byte cp.async copies, the chunk's rows summed in order;
//   2. bridge_mean_kernel   -- per (b, h), the chunk sums added in order;
//   3. bridge_cell_kernel   -- one block per (b, h, band of cell rows):
//      double-buffered cp.async tiles of whole token rows in padded shared
//      memory, one thread per token for dev(t), and a 64-bit shared atomicMax
//      per cell on (bits(dev) << 32 | ~token) -- dev >= +0, so its bits order
//      like its value, and the complemented index makes the lowest token win
//      among equal deviations.  Heads run in reverse order so that the heads
//      pass 1 read last are still in L2.
#include "area_internal.cuh"

namespace area {
namespace {

constexpr int kChunk = 1024;
constexpr int kChunkThreads = 128;
constexpr int kCellTokens = 64;     // tokens per shared tile = threads per block
constexpr int kStage = 16;          // rows per thread per cp.async batch in pass 1

template <typename T>
struct Vec;                         // 16 bytes of K widened to fp32
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ __forceinline__ static void widen(const uint4& r, float* f) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <>
struct Vec<float> {
  static constexpr int n = 4;
  __device__ __forceinline__ static void widen(const uint4& r, float* f) {
    f[0] = __uint_as_float(r.x);
    f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z);
    f[3] = __uint_as_float(r.w);
  }
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_one() {
  asm volatile("cp.async.wait_group 1;\n" ::: "memory");
}

// Pass 1: part[bh][c][d] = in-order sum of K[t, d] over the rows t of chunk c.
// Each thread stages its own next kStage rows of its slice with cp.async
// (double-buffered), so a batch of loads is in flight per thread without
// holding it in registers; it reads back only what it copied, so no block
// barrier is needed.
template <typename T>
__global__ void __launch_bounds__(kChunkThreads) bridge_chunk_kernel(const T* __restrict__ k,
                                                                     int N, int D, int nchunk,
                                                                     float* __restrict__ part) {
  constexpr int V = Vec<T>::n;
  extern __shared__ __align__(16) uint4 s_rows[];      // [2][kStage][kChunkThreads]
  const int tpr = D / V;                               // 16-byte slices per row
  const int cpb = kChunkThreads / tpr;                 // chunks per block
  const int bpb = (nchunk + cpb - 1) / cpb;            // blocks per (b, h)
  const int bh = blockIdx.x / bpb;
  const int c = (blockIdx.x % bpb) * cpb + threadIdx.x / tpr;
  const int sl = threadIdx.x % tpr;
  if (c >= nchunk) return;
  const int t0 = c * kChunk, n = min(N - t0, kChunk);
  const uint4* src = reinterpret_cast<const uint4*>(k + ((int64_t)bh * N + t0) * D) + sl;
  auto slot = [&](int b, int u) { return s_rows + ((b & 1) * kStage + u) * kChunkThreads + threadIdx.x; };
  auto issue = [&](int b) {
#pragma unroll
    for (int u = 0; u < kStage; ++u) {
      const int t = b * kStage + u;
      if (t < n) cp_async16(slot(b, u), src + (int64_t)t * tpr);
    }
  };
  float acc[V];
#pragma unroll
  for (int j = 0; j < V; ++j) acc[j] = 0.f;
  const int nb = (n + kStage - 1) / kStage;
  issue(0);
  cp_async_commit();
  for (int b = 0; b < nb; ++b) {
    if (b + 1 < nb) issue(b + 1);
    cp_async_commit();
    cp_async_wait_one();
    const int rows = min(kStage, n - b * kStage);
    for (int u = 0; u < rows; ++u) {
      float f[V];
      Vec<T>::widen(*slot(b, u), f);
#pragma unroll
      for (int j = 0; j < V; ++j) acc[j] = __fadd_rn(acc[j], f[j]);
    }
  }
  float* dst = part + ((int64_t)bh * nchunk + c) * D + sl * V;
#pragma unroll
  for (int j = 0; j < V; ++j) dst[j] = acc[j];
}

// Pass 2: one block per (b, h): stage its chunk sums in shared memory, then
// one thread per dim adds them in chunk order.
__global__ void __launch_bounds__(1024) bridge_mean_kernel(const float* __restrict__ part, int N,
                                                          int D, int nchunk,
                                                          float* __restrict__ mean) {
  extern __shared__ float s_part[];                    // [nchunk][D]
  const int bh = blockIdx.x;
  const float* src = part + (int64_t)bh * nchunk * D;
  const int n = nchunk * D;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s_part[i] = src[i];
  __syncthreads();
  if (threadIdx.x < D) {
    float total = 0.f;
    for (int c = 0; c < nchunk; ++c) total = __fadd_rn(total, s_part[c * D + threadIdx.x]);
    mean[(int64_t)bh * D + threadIdx.x] = __fmul_rn(total, __frcp_rn((float)N));
  }
}

// Pass 3: one block per (b, h, cell row cy); the band of grid rows
// [y0, y1) is contiguous in K.  Shared memory: two tiles of kCellTokens rows
// (row stride D*sizeof(T) + 16 bytes, so the 16-byte reads of eight
// consecutive rows fall in distinct banks), the mean key, one 64-bit key per
// cell of the band.
template <typename T>
__global__ void __launch_bounds__(kCellTokens) bridge_cell_kernel(const T* __restrict__ k,
                                                                  const float* __restrict__ mean,
                                                                  int BH, int Hg, int Wg, int D,
                                                                  int ry, int rx,
                                                                  int* __restrict__ cand) {
  constexpr int V = Vec<T>::n;
  extern __shared__ __align__(16) unsigned char smem[];
  const int rb = D * (int)sizeof(T);                   // bytes per token row
  const int rs = rb + 16;                              // padded stride in shared memory
  const int spr = rb / 16;                             // 16-byte slices per row
  float* s_mu = reinterpret_cast<float*>(smem + 2 * kCellTokens * rs);
  unsigned long long* s_key = reinterpret_cast<unsigned long long*>(s_mu + D);

  const int cy = blockIdx.x % ry;
  const int bh = BH - 1 - blockIdx.x / ry;
  const int y0 = (int)(((int64_t)cy * Hg) / ry), y1 = (int)(((int64_t)(cy + 1) * Hg) / ry);
  const int n = (y1 - y0) * Wg;                        // tokens in the band
  const int tok0 = y0 * Wg;
  const int64_t N = (int64_t)Hg * Wg;
  const unsigned char* src =
      reinterpret_cast<const unsigned char*>(k + ((int64_t)bh * N + tok0) * D);
  for (int i = threadIdx.x; i < D; i += kCellTokens) s_mu[i] = mean[(int64_t)bh * D + i];
  for (int i = threadIdx.x; i < rx; i += kCellTokens) s_key[i] = 0ull;

  const int ntile = (n + kCellTokens - 1) / kCellTokens;
  auto issue = [&](int tile) {
    const int rows = min(kCellTokens, n - tile * kCellTokens);
    const unsigned char* g = src + (int64_t)tile * kCellTokens * rb;
    unsigned char* s = smem + (tile & 1) * kCellTokens * rs;
    for (int p = threadIdx.x; p < rows * spr; p += kCellTokens)
      cp_async16(s + (p / spr) * rs + (p % spr) * 16, g + (int64_t)p * 16);
  };
  issue(0);
  cp_async_commit();
  for (int it = 0; it < ntile; ++it) {
    if (it + 1 < ntile) issue(it + 1);
    cp_async_commit();                                 // possibly empty: keeps the count uniform
    cp_async_wait_one();                               // this thread's copies of tile `it`
    __syncthreads();                                   // everyone's copies of tile `it`
    const int i = it * kCellTokens + threadIdx.x;
    if (i < n) {
      const uint4* row =
          reinterpret_cast<const uint4*>(smem + ((it & 1) * kCellTokens + threadIdx.x) * rs);
      float dev = 0.f;
      for (int s = 0; s < spr; ++s) {
        float f[V];
        Vec<T>::widen(row[s], f);
#pragma unroll
        for (int j = 0; j < V; ++j) {
          const float e = __fsub_rn(f[j], s_mu[s * V + j]);
          dev = __fadd_rn(dev, __fmul_rn(e, e));
        }
      }
      const int tok = tok0 + i;
      const int x = i % Wg;                            // the band starts at column 0
      const int cx = (int)((((int64_t)x + 1) * rx - 1) / Wg);
      const unsigned long long key =
          ((unsigned long long)__float_as_uint(dev) << 32) | (0xffffffffu - (uint32_t)tok);
      atomicMax(&s_key[cx], key);
    }
    __syncthreads();                                   // tile `it` fully read before reuse
  }
  int* out = cand + (int64_t)bh * ry * rx + (int64_t)cy * rx;
  for (int i = threadIdx.x; i < rx; i += kCellTokens)
    out[i] = (int)(0xffffffffu - (uint32_t)(s_key[i] & 0xffffffffull));
}

template <typename T>
cudaError_t launch_typed(const T* k, int B, int H, int Hg, int Wg, int D, int ry, int rx,
                         int* cand, float* ws, cudaStream_t s) {
  const int N = Hg * Wg;
  const int BH = B * H;
  const int nchunk = (N + kChunk - 1) / kChunk;
  float* mean = ws;
  float* part = ws + (int64_t)BH * D;
  const int cpb = kChunkThreads / (D / Vec<T>::n);
  const int64_t grid1 = (int64_t)BH * ((nchunk + cpb - 1) / cpb);
  const int smem1 = 2 * kStage * kChunkThreads * 16;
  cudaError_t e = cudaFuncSetAttribute(bridge_chunk_kernel<T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem1);
  if (e != cudaSuccess) return e;
  bridge_chunk_kernel<T><<<(unsigned)grid1, kChunkThreads, smem1, s>>>(k, N, D, nchunk, part);
  const int smem2 = nchunk * D * (int)sizeof(float);
  e = cudaFuncSetAttribute(bridge_mean_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem2);
  if (e != cudaSuccess) return e;
  bridge_mean_kernel<<<BH, 1024, smem2, s>>>(part, N, D, nchunk, mean);
  const int smem3 = 2 * kCellTokens * (D * (int)sizeof(T) + 16) + D * 4 + rx * 8;
  e = cudaFuncSetAttribute(bridge_cell_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem3);
  if (e != cudaSuccess) return e;
  bridge_cell_kernel<T><<<(unsigned)((int64_t)BH * ry), kCellTokens, smem3, s>>>(
      k, mean, BH, Hg, Wg, D, ry, rx, cand);
  return cudaGetLastError();
}

}  // namespace

size_t bridge_ws_bytes(int B, int H, int Hg, int Wg, int D) {
  const int64_t N = (int64_t)Hg * Wg;
  const int64_t nchunk = (N + kChunk - 1) / kChunk;
  return (size_t)((int64_t)B * H * D * (1 + nchunk) * (int64_t)sizeof(float));
}

cudaError_t launch_bridge_select(const void* k, int dtype, int B, int H, int Hg, int Wg, int D,
                                 int ry, int rx, int* cand, float* ws, cudaStream_t s) {
  if (dtype == AREA_DTYPE_BF16)
    return launch_typed(static_cast<const __nv_bfloat16*>(k), B, H, Hg, Wg, D, ry, rx, cand, ws,
                        s);
  return launch_typed(static_cast<const float*>(k), B, H, Hg, Wg, D, ry, rx, cand, ws, s);
}

}  // namespace area
