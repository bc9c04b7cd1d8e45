// Internal declarations shared by the libarea translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "area.h"

namespace area {

constexpr int kQTile = 256;          // queries per work item (two 128-row MMA tiles)
constexpr int kMaxG = 4096;          // largest global-KV count per window
constexpr int kMaxGrid = 1 << 15;    // largest grid side accepted (tokens)

// ---------------------------------------------------------------------------
// plan layout: computed identically by every entry point from the config
// ---------------------------------------------------------------------------
struct PlanLayout {
  int64_t B, Hg, Wg, w, halo, G;
  uint64_t seed;                // border jitter and Halo widths (0: none)
  int64_t sy, sx;               // border shift of this plan per axis
  int64_t nby, nbx, hy, wx;     // base tiling: counts (this plan) and window sides
  int64_t nb_cap;               // base-window capacity per element (section strides)
  int64_t nb, nw;               // base windows of this plan / final-window capacity
  int64_t nitem_max;            // work-item capacity per element
  int64_t N;                    // tokens per element
  int64_t ntile_sort;           // 256-element tiles of the radix sort
  int64_t ny2, nx2;             // positions covered by two base windows, per axis
  int64_t n_ov;                 // tokens covered by more than one window (per element)
  int64_t off[AREA_PLAN_NSEC];  // byte offsets of the sections
  int64_t scratch_keys_a, scratch_keys_b, scratch_vals_a, scratch_vals_b,
          scratch_hist,         // byte offsets inside the buffer
          scratch_bar;          // grid-barrier words of the fused planner
  int64_t total;                // bytes
};

int plan_layout(const area_plan_cfg* cfg, PlanLayout* L);

// Device view of a plan (pointers into the plan buffer).
struct PlanView {
  int B, Hg, Wg, w, halo, G;
  unsigned long long seed;
  int sy, sx;
  int nby, nbx, hy, wx, nb, nb_cap, nw, nitem_max, N;
  int4* base;          // [B][nb]
  float* score;        // [B][nb]
  uint8_t* split;      // [B][nb]
  int* nwin;           // [B]
  int4* win;           // [B][nw]
  int* parent;         // [B][nw]
  int4* ext;           // [B][nw]
  int* gcount;         // [B][nw]
  int* gidx;           // [B][nw][G]
  float* wsum;         // [B][N]
  int* cover;          // [B][N] number of final windows containing the token
  int* order;          // [B][N]
  int* nitem;          // [B+1]
  int2* items;         // [B][nitem_max]
  int* nclass;         // [B+1][4] work items per parity class (row B: totals)
};

PlanView plan_view(const PlanLayout& L, void* plan);

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float load_as_float(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_as_float(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_from_float(float* p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void store_from_float(__nv_bfloat16* p, int64_t i, float v) {
  p[i] = __float2bfloat16_rn(v);
}

// Start of the i-th of n evenly spaced windows of side we on an axis of length L.
__host__ __device__ __forceinline__ int tile_start(int i, int n, int L, int we) {
  return n > 1 ? (int)(((int64_t)i * (L - we)) / (n - 1)) : 0;
}

// Window i of an axis of length L under a border shift: the even tiling of
// the extended axis [-shift, L) (n windows of side we), clipped to [0, L).
__host__ __device__ __forceinline__ void axis_window(int i, int n, int L, int we, int shift,
                                                     int* start, int* size) {
  const int a = tile_start(i, n, L + shift, we) - shift;
  const int lo = a > 0 ? a : 0;
  const int hi = a + we < L ? a + we : L;
  *start = lo;
  *size = hi - lo;
}

// Merge geometry of base window i along one axis (n windows, shift as in
// axis_window).  Consecutive windows may overlap; windows two apart never do
// (their spacing exceeds half a window), so a position is covered by one or
// two windows of an axis.  Returns
//   x = start of window i, y = end of the overlap with window i-1 (x when
//   none), z = start of the overlap with window i+1 (end of window i when
//   none), w = number of twice-covered positions before the start of i.
__host__ __device__ inline int4 axis_merge(int i, int n, int L, int we, int shift) {
  int a, s;
  axis_window(i, n, L, we, shift, &a, &s);
  int lo_end = a, hi_start = a + s;
  if (i > 0) {
    int ap, sp;
    axis_window(i - 1, n, L, we, shift, &ap, &sp);
    lo_end = ap + sp > a ? ap + sp : a;
  }
  if (i + 1 < n) {
    int an, sn;
    axis_window(i + 1, n, L, we, shift, &an, &sn);
    hi_start = an < a + s ? an : a + s;
  }
  int cnt = 0, ak, sk;
  axis_window(0, n, L, we, shift, &ak, &sk);
  for (int k = 0; k + 1 <= i - 1; ++k) {       // overlaps of windows (k, k+1) before a
    int an, sn;
    axis_window(k + 1, n, L, we, shift, &an, &sn);
    cnt += ak + sk > an ? ak + sk - an : 0;
    ak = an;
    sk = sn;
  }
  return make_int4(a, lo_end, hi_start, cnt);
}

// Number of positions of an axis covered by two windows.
__host__ __device__ inline int axis_twice_total(int n, int L, int we, int shift) {
  int cnt = 0, ak, sk;
  axis_window(0, n, L, we, shift, &ak, &sk);
  for (int k = 0; k + 1 < n; ++k) {
    int an, sn;
    axis_window(k + 1, n, L, we, shift, &an, &sn);
    cnt += ak + sk > an ? ak + sk - an : 0;
    ak = an;
    sk = sn;
  }
  return cnt;
}

// Parity class of a base window: windows of one class never overlap.
__host__ __device__ inline int window_class(int parent, int nbx) {
  return (((parent / nbx) & 1) << 1) | ((parent % nbx) & 1);
}

// Role of one output row in the centre-weighted merge.  A token inside one
// window stores its output directly.  A token covered by several windows
// (one per parity class at most) has one fp32 accumulator row: the window of
// its lowest class stores, the middle ones add, the highest class adds and
// normalises.  my/mx: axis_merge of the base window along y and x.
struct MergeRole {
  bool ov, first, last;
  int64_t rank;        // accumulator row among the overlapped tokens of the element
};
__host__ __device__ inline MergeRole merge_role(int y, int x, int cls, int4 my, int4 mx,
                                                int Wg, int nx2) {
  MergeRole r;
  const bool ty = y < my.y || y >= my.z;
  const bool tx = x < mx.y || x >= mx.z;
  r.ov = ty || tx;
  const int py = cls >> 1, px = cls & 1;
  const int minc = ((ty ? 0 : py) << 1) | (tx ? 0 : px);
  const int maxc = ((ty ? 1 : py) << 1) | (tx ? 1 : px);
  r.first = cls == minc;
  r.last = cls == maxc;
  const int by = my.w + ((y < my.y ? y : my.y) - my.x) + (y >= my.z ? y - my.z : 0);
  const int bx = mx.w + ((x < mx.y ? x : mx.y) - mx.x) + (x >= mx.z ? x - mx.z : 0);
  r.rank = (int64_t)by * Wg + (int64_t)(y - by) * nx2 + (ty ? x : bx);
  return r;
}

// Window keys: the Halo rectangle is covered by full patches of kPW x kPH
// grid tokens (one 128-key tile, one 3-D tiled TMA box per 64-column half),
// and its right and bottom strips left over by the patches by cells of
// kCW x kCH tokens, kCells cells per tile, one box each (the tokens of one
// grid row are contiguous).  Only the last tile of a rectangle whose sides
// are multiples of 4 has unused rows.  Patches alone (16 x 8, masked at the
// edges) computed 6% more (query, key) pairs than valid ones over the
// FLUX-shaped 6144^2 schedule and 21% more at 2048^2; cells alone cost TMA
// throughput (8 boxes per half tile: 11% slower tiles on a 256 x 256 window,
// measured).  Queries of a window whose sides are multiples of 4 come in
// cells too; other windows' queries are gathered row by row.  The global-KV
// list is copied row by row.
constexpr int kPW = 16, kPH = 8;
constexpr int kCW = 4, kCH = 4;
constexpr int kCellKeys = kCW * kCH;         // rows of one cell
constexpr int kCells = 128 / kCellKeys;      // cells per tile
static_assert(kPW * kPH == 128 && kPW % kCW == 0 && kPH % kCH == 0, "patch of whole cells");

// Tiling of a Halo rectangle of eh x ew tokens: npx x npy patches (row-major),
// then the cells of the right strip (x >= kPW * npx, all rows; c1x per row)
// and of the bottom strip (x < kPW * npx, y >= kPH * npy; c2x per row).
struct RectTiling {
  int npx, npy, npatch;   // patches per row, patch rows, patches (= patch tiles)
  int c1x, n1;            // right strip: cells per row, cells
  int c2x;                // bottom strip: cells per row
  int ncell;              // cells of both strips
};
__host__ __device__ __forceinline__ RectTiling rect_tiling(int eh, int ew) {
  RectTiling t;
  t.npx = ew / kPW;
  t.npy = eh / kPH;
  t.npatch = t.npx * t.npy;
  t.c1x = (ew - kPW * t.npx + kCW - 1) / kCW;
  t.n1 = t.c1x * ((eh + kCH - 1) / kCH);
  t.c2x = kPW * t.npx / kCW;
  t.ncell = t.n1 + t.c2x * ((eh - kPH * t.npy + kCH - 1) / kCH);
  return t;
}
// Rectangle tiles: the patches, then the cells kCells by kCells.
__host__ __device__ __forceinline__ int rect_tiles(const RectTiling& t) {
  return t.npatch + (t.ncell + kCells - 1) / kCells;
}
// Offset (y, x) inside the rectangle of the top-left token of strip cell c.
__host__ __device__ __forceinline__ int2 strip_cell(const RectTiling& t, int c) {
  if (c < t.n1) return make_int2((c / t.c1x) * kCH, kPW * t.npx + (c % t.c1x) * kCW);
  c -= t.n1;
  return make_int2(kPH * t.npy + (c / t.c2x) * kCH, (c % t.c2x) * kCW);
}

// Cells per row of a window (y0, x0, hy, wx) whose queries are taken in cells
// (both sides multiples of the cell's), else 0: its queries are row-major.
__host__ __device__ __forceinline__ int query_cells_per_row(int4 win) {
  return (win.z % kCH == 0 && win.w % kCW == 0) ? win.w / kCW : 0;
}
// Query token of position p of a window (positions past nq read position 0).
// With qcx > 0 the window is enumerated cell by cell (cells row-major, qcx per
// row; inside a cell row-major), else row-major.
__host__ __device__ __forceinline__ int window_query_token(const int4& win, int qcx, int nq, int p,
                                                  int Wg) {
  if (p >= nq) p = 0;
  if (qcx > 0) {
    const int c = p / kCellKeys, k = p % kCellKeys;
    return (win.x + (c / qcx) * kCH + k / kCW) * Wg + win.y + (c % qcx) * kCW + k % kCW;
  }
  return (win.x + p / win.w) * Wg + win.y + p % win.w;
}

// Window-attention workspace: a header of uint32 counters (the dynamic unit
// counter, then one completion counter per (element, head, parity class)),
// rounded up to 256 bytes, then one fp32 accumulator row per (element, head,
// overlapped token).
constexpr int kWsUnitCounter = 0, kWsClassDone = 1;
__host__ __device__ inline int64_t window_ws_header_bytes(int64_t B, int64_t H) {
  return ((4 * (1 + 4 * B * H)) + 255) & ~int64_t(255);
}

// Counter-based draws: output number (stream * 2^32 + index) of the SplitMix64
// sequence (Steele, Lea, Flood 2014) seeded with `seed`.
__host__ __device__ __forceinline__ unsigned long long splitmix64(unsigned long long s) {
  unsigned long long z = s + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__host__ __device__ __forceinline__ unsigned long long counter_random(unsigned long long seed,
                                                                     unsigned long long stream,
                                                                     unsigned long long index) {
  return splitmix64(seed + 0x9E3779B97F4A7C15ull * ((stream << 32) + index));
}
constexpr unsigned long long kStreamJitter = 1, kStreamHalo = 2;

// Records a CUDA error for area_last_cuda_error (per host thread) and
// returns AREA_ECUDA.
int fail_cuda(cudaError_t e);

// ---------------------------------------------------------------------------
// launchers (return cudaError_t of the launch)
// ---------------------------------------------------------------------------
cudaError_t launch_pool_kv(const void* k, const void* v, void* kp, void* vp, int B, int H,
                           int Hg, int Wg, int D, int f, int mode, int dtype, cudaStream_t s);
cudaError_t launch_dwt_detail(const void* src, int src_dtype, int C, float* energy, int B,
                              int Hg, int Wg, int mode, cudaStream_t s);
cudaError_t launch_window_plan(const float* energy, const area_plan_cfg* cfg,
                               const PlanLayout& L, void* plan, cudaStream_t s);

// CUDA-core attention (fp32, D = 64 or 128).
cudaError_t launch_dense_attn_simt(const void* q, const void* k, const void* v, const void* kt,
                                   const void* vt, void* o, int B, int H, int N, int Nk, int T,
                                   int D, float scale, int dtype, cudaStream_t s);
// Window attention on CUDA cores: one launch per parity class, so that the
// merge of overlapped tokens runs in class order.  ws: the window workspace
// (header + accumulator rows).
cudaError_t launch_window_attn_simt(const void* q, const void* k, const void* v, const void* kt,
                                    const void* vt, int T, const int* cand, int R,
                                    const PlanLayout& L, const void* plan, void* o, void* ws,
                                    int H, int D, float scale, int dtype, cudaStream_t s);

// tcgen05 tensor-core attention (bf16, D = 64 or 128).  kt, vt: [B, H, T, D]
// text keys appended after the image keys of every query (T = 0: none).
cudaError_t launch_dense_attn_tc(const void* q, const void* k, const void* v, const void* kt,
                                 const void* vt, void* o, int B, int H, int N, int Nk, int T,
                                 int D, float scale, cudaStream_t s);
cudaError_t read_and_clear_tc_error(int* code);
// cand (may be null): per-head bridge candidates [B*H][R]; when given they
// replace the plan's global-KV lists, candidates inside a window's Halo
// rectangle are skipped.
// staged: the workspace extends window_stage_bytes past window_ws_bytes, and
// the global-KV rows of each window are first copied there (one launch) so
// that the attention kernel loads whole list tiles with tiled TMA.
cudaError_t launch_window_attn_tc(const void* q, const void* k, const void* v, const void* kt,
                                  const void* vt, int T, const int* cand, int R,
                                  const PlanLayout& L, const void* plan, void* o, void* ws,
                                  bool staged, int H, int D, float scale, cudaStream_t s);
// Bytes of the window workspace for H heads of head_dim D.
int64_t window_ws_bytes(const PlanLayout& L, int H, int D);
// Bytes of the optional staging area of the global-KV rows (bf16 K then V,
// [B][H][nw][G][D] each), appended to the workspace.
int64_t window_stage_bytes(const PlanLayout& L, int H, int D);
// Detail map and planner in one cooperative launch (one memset of the
// barrier words first); a barrier timeout raises the planner error flag.
// target_extra (0 in every product call) raises each grid-barrier target so
// that the first barrier cannot complete; wait_ns bounds each barrier wait
// (0: the default of 2 s).  Both exist for the expiry test hook.
cudaError_t launch_dwt_window_plan(const void* src, int src_dtype, int C, int mode, float* energy,
                                   const area_plan_cfg* cfg, const PlanLayout& L, void* plan,
                                   cudaStream_t s, unsigned target_extra = 0,
                                   uint64_t wait_ns = 0);
cudaError_t read_and_clear_plan_error(int* code);

// Scratch of area_bridge_select: the mean keys [B*H][D] then the chunk sums
// [B*H][ceil(N/1024)][D], fp32.
size_t bridge_ws_bytes(int B, int H, int Hg, int Wg, int D);
cudaError_t launch_bridge_select(const void* k, int dtype, int B, int H, int Hg, int Wg, int D,
                                 int ry, int rx, int* cand, float* mean, cudaStream_t s);

}  // namespace area
