// CUDA-core attention: the fp32 path (the tiny configuration, tolerance 1e-4;
// bf16 runs on the tensor-core kernel).  Same semantics as the tensor-core
// kernels:
//   dense  : O = softmax(scale * Q K^T) V over all Nk keys (coarse and full
//            attention, AReA Phase I / the speedup denominator);
//   window : per plan work item (window W, 256-query block), keys S = Halo
//            rectangle of W followed by its global-KV tokens.  A token inside
//            one window only takes that window's output; a token in an overlap
//            has one fp32 accumulator row, written by its lowest parity class
//            of windows, added to by the higher ones and normalised by the
//            per-token weight sum by the highest (AReA Phase II,
//            centre-weighted blending of overlaps).  One launch per parity
//            class keeps that order; windows of one class never overlap.
// Pages: ai.info "Methodology in Plain English" (Phase I, Phase II).
#include "area_internal.cuh"

namespace area {
namespace {

constexpr int kSimtQ = 32;        // queries per block
constexpr int kSimtTPQ = 8;       // threads per query
constexpr int kSimtKV = 64;       // keys per shared-memory chunk
constexpr int kSimtThreads = kSimtQ * kSimtTPQ;

struct DenseRows {
  int N, Nk;
};

template <typename T, int D, bool WINDOW>
__global__ void __launch_bounds__(kSimtThreads) attn_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const T* __restrict__ kt, const T* __restrict__ vt, int ntext, const int* __restrict__ cand,
    int R, T* __restrict__ o, float* acc, int H, DenseRows dr, PlanView P, float scale, int cls,
    int nx2, long long n_ov) {
  constexpr int DPT = D / kSimtTPQ;
  extern __shared__ float smem[];
  float* Ks = smem;                       // [kSimtKV][D]
  float* Vs = smem + kSimtKV * D;         // [kSimtKV][D]
  __shared__ int s_kvtok[kSimtKV];
  __shared__ bool s_kvtxt[kSimtKV];
  __shared__ bool s_kvok[kSimtKV];

  const int b = blockIdx.z, h = blockIdx.y;
  const int tid = threadIdx.x;
  const int ql = tid / kSimtTPQ, part = tid % kSimtTPQ;

  // ---- query rows and key/value set of this block
  int N, nkv, wi = 0, r = 0;
  int4 win = make_int4(0, 0, 0, 0), ext = make_int4(0, 0, 0, 0);
  const int* glist = nullptr;
  bool qvalid;
  int qtok;
  if (WINDOW) {
    N = P.N;
    const int ic = blockIdx.x / (kQTile / kSimtQ);       // item within the class
    const int sub = blockIdx.x % (kQTile / kSimtQ);
    if (ic >= P.nclass[b * 4 + cls]) return;
    int item = ic;
    for (int c = 0; c < cls; ++c) item += P.nclass[b * 4 + c];
    const int2 it = P.items[(int64_t)b * P.nitem_max + item];
    wi = it.x;
    const int64_t wo = (int64_t)b * P.nw + wi;
    win = P.win[wo];
    ext = P.ext[wo];
    nkv = ext.z * ext.w + (cand ? R : P.gcount[wo]);
    glist = cand ? cand + ((int64_t)b * H + h) * R : P.gidx + wo * P.G;
    r = it.y * kQTile + sub * kSimtQ + ql;
    qvalid = r < win.z * win.w;
    qtok = qvalid ? (win.x + r / win.w) * P.Wg + win.y + r % win.w : 0;
  } else {
    N = dr.N;
    nkv = dr.Nk;
    r = blockIdx.x * kSimtQ + ql;
    qvalid = r < N;
    qtok = qvalid ? r : 0;
  }
  const int64_t bh = (int64_t)b * H + h;
  const int Nkv_rows = WINDOW ? N : dr.Nk;  // rows of the K/V tensors per (b, h)
  const T* qrow = q + (bh * N + qtok) * D;
  const T* kb = k + bh * Nkv_rows * D;
  const T* vb = v + bh * Nkv_rows * D;
  const T* ktb = kt ? kt + bh * ntext * D : nullptr;   // text keys after the image keys
  const T* vtb = vt ? vt + bh * ntext * D : nullptr;
  const int nimg = nkv;
  nkv += ntext;

  float qv[DPT], acc_v[DPT];
#pragma unroll
  for (int i = 0; i < DPT; ++i) {
    qv[i] = load_as_float(qrow, part + kSimtTPQ * i) * scale;
    acc_v[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  for (int c0 = 0; c0 < nkv; c0 += kSimtKV) {
    const int cn = min(kSimtKV, nkv - c0);
    if (tid < kSimtKV) {
      int tok = 0;
      bool txt = false, ok = true;
      const int j = c0 + tid;
      if (tid < cn) {
        if (j >= nimg) {
          tok = j - nimg;
          txt = true;
        } else if (WINDOW) {
          const int ne = ext.z * ext.w;
          tok = j < ne ? (ext.x + j / ext.w) * P.Wg + ext.y + j % ext.w : glist[j - ne];
          if (cand && j >= ne) {     // bridge candidates inside the rectangle are skipped
            const int ty = tok / P.Wg, tx = tok % P.Wg;
            ok = !(ty >= ext.x && ty < ext.x + ext.z && tx >= ext.y && tx < ext.y + ext.w);
          }
        } else {
          tok = j;
        }
      }
      s_kvtok[tid] = tok;
      s_kvtxt[tid] = txt;
      s_kvok[tid] = ok;
    }
    __syncthreads();
    // cooperative load: thread -> (row, quarter of the row)
    for (int e = tid; e < kSimtKV * 4; e += kSimtThreads) {
      const int row = e >> 2, qd = e & 3;
      const int64_t src = (int64_t)s_kvtok[row] * D;
      const T* ks = s_kvtxt[row] ? ktb : kb;
      const T* vs = s_kvtxt[row] ? vtb : vb;
#pragma unroll 4
      for (int d = qd * (D / 4); d < (qd + 1) * (D / 4); ++d) {
        const bool ok = row < cn;
        Ks[row * D + d] = ok ? load_as_float(ks, src + d) : 0.f;
        Vs[row * D + d] = ok ? load_as_float(vs, src + d) : 0.f;
      }
    }
    __syncthreads();
    float s[kSimtKV];
    float mc = -INFINITY;
#pragma unroll
    for (int j = 0; j < kSimtKV; ++j) {
      float part_dot = 0.f;
#pragma unroll
      for (int i = 0; i < DPT; ++i) part_dot += qv[i] * Ks[j * D + part + kSimtTPQ * i];
      part_dot += __shfl_xor_sync(0xffffffffu, part_dot, 1);
      part_dot += __shfl_xor_sync(0xffffffffu, part_dot, 2);
      part_dot += __shfl_xor_sync(0xffffffffu, part_dot, 4);
      s[j] = (j < cn && s_kvok[j]) ? part_dot : -INFINITY;
      mc = fmaxf(mc, s[j]);
    }
    const float mn = fmaxf(m, mc);
    const float corr = expf(m - mn);
    l *= corr;
#pragma unroll
    for (int i = 0; i < DPT; ++i) acc_v[i] *= corr;
#pragma unroll
    for (int j = 0; j < kSimtKV; ++j) {
      const float p = expf(s[j] - mn);
      l += p;
#pragma unroll
      for (int i = 0; i < DPT; ++i) acc_v[i] += p * Vs[j * D + part + kSimtTPQ * i];
    }
    m = mn;
    __syncthreads();
  }
  if (!qvalid) return;
  const float inv = 1.f / l;
  T* dst = o + (bh * N + qtok) * D;
  if (WINDOW) {
    const int parent = P.parent[(int64_t)b * P.nw + wi];
    const int4 my = axis_merge(parent / P.nbx, P.nby, P.Hg, P.hy, P.sy);
    const int4 mx = axis_merge(parent % P.nbx, P.nbx, P.Wg, P.wx, P.sx);
    const int y = qtok / P.Wg, x = qtok % P.Wg;
    const MergeRole mr = merge_role(y, x, cls, my, mx, P.Wg, nx2);
    if (mr.ov) {
      // overlap: this class's share goes to the token's accumulator row
      const float t = (float)(min(y - win.x + 1, win.x + win.z - y) *
                              min(x - win.y + 1, win.y + win.w - x));
      float* arow = acc + (bh * n_ov + mr.rank) * D;
      const float winv = 1.f / P.wsum[(int64_t)b * P.N + qtok];
#pragma unroll
      for (int i = 0; i < DPT; ++i) {
        const int d = part + kSimtTPQ * i;
        float a = acc_v[i] * (t * inv);
        if (!mr.first) a += arow[d];
        if (mr.last) store_from_float(dst, d, a * winv);
        else arow[d] = a;
      }
      return;
    }
  }
  // the only window containing this token (or dense attention): the output
#pragma unroll
  for (int i = 0; i < DPT; ++i) store_from_float(dst, part + kSimtTPQ * i, acc_v[i] * inv);
}

struct MergeArgs {
  float* acc;       // accumulator rows [B*H][n_ov][D]
  int nx2;
  long long n_ov;
};

template <typename T, int D, bool WINDOW>
cudaError_t launch_simt(dim3 grid, const void* q, const void* k, const void* v, const void* kt,
                        const void* vt, int ntext, const int* cand, int R, void* o,
                        const MergeArgs& ma, int H, DenseRows dr, PlanView P, float scale,
                        cudaStream_t s) {
  const int smem = 2 * kSimtKV * D * (int)sizeof(float);
  auto fn = attn_simt_kernel<T, D, WINDOW>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // window mode: one launch per parity class, in class order
  for (int cls = 0; cls < (WINDOW ? 4 : 1); ++cls) {
    fn<<<grid, kSimtThreads, smem, s>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                        static_cast<const T*>(v), static_cast<const T*>(kt),
                                        static_cast<const T*>(vt), ntext, cand, R,
                                        static_cast<T*>(o), ma.acc, H, dr, P, scale, cls, ma.nx2,
                                        ma.n_ov);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_dense_attn_simt(const void* q, const void* k, const void* v, const void* kt,
                                   const void* vt, void* o, int B, int H, int N, int Nk, int T,
                                   int D, float scale, int dtype, cudaStream_t s) {
  dim3 grid((N + kSimtQ - 1) / kSimtQ, H, B);
  DenseRows dr{N, Nk};
  PlanView P{};
  if (dtype == AREA_DTYPE_F32) {
    if (D == 64) return launch_simt<float, 64, false>(grid, q, k, v, kt, vt, T, nullptr, 0, o, MergeArgs{}, H, dr, P, scale, s);
    return launch_simt<float, 128, false>(grid, q, k, v, kt, vt, T, nullptr, 0, o, MergeArgs{}, H, dr, P, scale, s);
  }
  return cudaErrorNotSupported;           // bf16 runs on the tensor-core kernel
}

cudaError_t launch_window_attn_simt(const void* q, const void* k, const void* v, const void* kt,
                                    const void* vt, int T, const int* cand, int R,
                                    const PlanLayout& L, const void* plan, void* o, void* ws,
                                    int H, int D, float scale, int dtype, cudaStream_t s) {
  PlanView P = plan_view(L, const_cast<void*>(plan));
  const MergeArgs ma{reinterpret_cast<float*>(static_cast<char*>(ws) +
                                              window_ws_header_bytes(L.B, H)),
                     (int)L.nx2, (long long)L.n_ov};
  dim3 grid((unsigned)(L.nitem_max * (kQTile / kSimtQ)), H, (unsigned)L.B);
  DenseRows dr{(int)L.N, (int)L.N};
  if (dtype == AREA_DTYPE_F32) {
    if (D == 64) return launch_simt<float, 64, true>(grid, q, k, v, kt, vt, T, cand, R, o, ma, H, dr, P, scale, s);
    return launch_simt<float, 128, true>(grid, q, k, v, kt, vt, T, cand, R, o, ma, H, dr, P, scale, s);
  }
  return cudaErrorNotSupported;           // bf16 runs on the tensor-core kernel
}

}  // namespace area
