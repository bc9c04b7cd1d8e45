// Phase II planner on the device: base tiling, DWT-guided quadrant splits,
// Halo rectangles, the global-KV bridge, merge-weight sums and the work list.
//
// Method (AReA summary pages: ai.info "Methodology in Plain English",
// Phase II; gpt-diffusion.com "Las dos fases de AReA", Fase II): windows cover
// the grid in an evenly spaced base tiling; windows over smooth regions of a
// DWT detail map split into four quadrants; each window's keys are extended
// by a Halo ring and by global-KV tokens from the rest of the image; the
// overlapping outputs are blended with centre weights.
//
// Index lists, split decisions and scores are bit-exact by construction:
// integer arithmetic, plus fp32 sums in a fixed order with explicit
// round-to-nearest operations.  The global-KV ranking is a stable LSD radix
// sort of the energy bits (descending), which keeps token order among ties.
#include "area_internal.cuh"
#include "detail_cell.cuh"

namespace area {

__device__ int g_plan_error = 0;   // set when a fused-planner grid barrier times out

static int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

// Radix-sort tile: 256 threads x 16 ordered rounds of one element each.
constexpr int kSortRounds = 16;
constexpr int kSortTile = 256 * kSortRounds;

int plan_layout(const area_plan_cfg* cfg, PlanLayout* L) {
  if (!cfg || !L) return AREA_EINVAL;
  if (cfg->B < 1 || cfg->Hg < 2 || cfg->Wg < 2 || (cfg->Hg & 1) || (cfg->Wg & 1) ||
      cfg->Hg > kMaxGrid || cfg->Wg > kMaxGrid || cfg->w < 1 || cfg->halo < 0 || cfg->G < 0 ||
      cfg->G > kMaxG || cfg->B > (1 << 11))
    return AREA_EINVAL;
  const int64_t N = (int64_t)cfg->Hg * cfg->Wg;
  if (N > (int64_t(1) << 26)) return AREA_EINVAL;
  L->B = cfg->B; L->Hg = cfg->Hg; L->Wg = cfg->Wg; L->w = cfg->w; L->halo = cfg->halo;
  L->G = cfg->G; L->N = N;
  L->hy = cfg->w < cfg->Hg ? cfg->w : cfg->Hg;
  L->wx = cfg->w < cfg->Wg ? cfg->w : cfg->Wg;
  L->seed = cfg->jitter_seed;
  // border shift of this plan (0 without a seed or when the window spans the axis)
  L->sy = (L->seed && L->hy < L->Hg)
              ? (int64_t)(counter_random(L->seed, kStreamJitter, 0) % (unsigned long long)L->hy)
              : 0;
  L->sx = (L->seed && L->wx < L->Wg)
              ? (int64_t)(counter_random(L->seed, kStreamJitter, 1) % (unsigned long long)L->wx)
              : 0;
  L->nby = (cfg->Hg + L->sy + L->hy - 1) / L->hy;
  L->nbx = (cfg->Wg + L->sx + L->wx - 1) / L->wx;
  L->nb = L->nby * L->nbx;
  // capacity covers every shift in [0, side): one more window per axis at most
  const int64_t cy = L->seed && L->hy < L->Hg ? (cfg->Hg + 2 * L->hy - 2) / L->hy
                                              : (cfg->Hg + L->hy - 1) / L->hy;
  const int64_t cx = L->seed && L->wx < L->Wg ? (cfg->Wg + 2 * L->wx - 2) / L->wx
                                              : (cfg->Wg + L->wx - 1) / L->wx;
  L->nb_cap = cy * cx;
  L->nw = 4 * L->nb_cap;
  L->nitem_max = L->nb_cap * ((L->hy * L->wx + kQTile - 1) / kQTile + 3);
  L->ntile_sort = (N + kSortTile - 1) / kSortTile;
  L->ny2 = axis_twice_total((int)L->nby, (int)L->Hg, (int)L->hy, (int)L->sy);
  L->nx2 = axis_twice_total((int)L->nbx, (int)L->Wg, (int)L->wx, (int)L->sx);
  L->n_ov = L->ny2 * L->Wg + (L->Hg - L->ny2) * L->nx2;
  const int64_t B = L->B;
  const int64_t sizes[AREA_PLAN_NSEC] = {
      B * L->nb_cap * 16, B * L->nb_cap * 4, B * L->nb_cap, B * 4,
      B * L->nw * 16, B * L->nw * 4, B * L->nw * 16, B * L->nw * 4,
      B * L->nw * L->G * 4, B * N * 4, B * N * 4, (B + 1) * 4,
      B * L->nitem_max * 8, B * N * 4, (B + 1) * 16, 0};
  int64_t off = 256;  // header
  for (int s = 0; s < AREA_PLAN_NSEC; ++s) {
    L->off[s] = off;
    off = align256(off + (sizes[s] > 0 ? sizes[s] : 1));
  }
  // scratch of one radix sort (batch elements are sorted one after another)
  off = L->off[AREA_PLAN_SEC_SCRATCH];
  L->scratch_keys_a = off; off = align256(off + N * 4);
  L->scratch_keys_b = off; off = align256(off + N * 4);
  L->scratch_vals_a = off; off = align256(off + N * 4);
  L->scratch_vals_b = off; off = align256(off + N * 4);
  L->scratch_hist = off;   off = align256(off + 256 * L->ntile_sort * 4);
  L->scratch_bar = off;    off = align256(off + 8);   // grid barrier of the fused planner
  L->total = off;
  return AREA_OK;
}

PlanView plan_view(const PlanLayout& L, void* plan) {
  char* p = static_cast<char*>(plan);
  PlanView v;
  v.B = (int)L.B; v.Hg = (int)L.Hg; v.Wg = (int)L.Wg; v.w = (int)L.w; v.halo = (int)L.halo;
  v.G = (int)L.G; v.nby = (int)L.nby; v.nbx = (int)L.nbx; v.hy = (int)L.hy; v.wx = (int)L.wx;
  v.seed = L.seed; v.sy = (int)L.sy; v.sx = (int)L.sx; v.nb_cap = (int)L.nb_cap;
  v.nb = (int)L.nb; v.nw = (int)L.nw; v.nitem_max = (int)L.nitem_max; v.N = (int)L.N;
  v.base = reinterpret_cast<int4*>(p + L.off[AREA_PLAN_SEC_BASE]);
  v.score = reinterpret_cast<float*>(p + L.off[AREA_PLAN_SEC_SCORE]);
  v.split = reinterpret_cast<uint8_t*>(p + L.off[AREA_PLAN_SEC_SPLIT]);
  v.nwin = reinterpret_cast<int*>(p + L.off[AREA_PLAN_SEC_NWIN]);
  v.win = reinterpret_cast<int4*>(p + L.off[AREA_PLAN_SEC_WIN]);
  v.parent = reinterpret_cast<int*>(p + L.off[AREA_PLAN_SEC_PARENT]);
  v.ext = reinterpret_cast<int4*>(p + L.off[AREA_PLAN_SEC_EXT]);
  v.gcount = reinterpret_cast<int*>(p + L.off[AREA_PLAN_SEC_GCOUNT]);
  v.gidx = reinterpret_cast<int*>(p + L.off[AREA_PLAN_SEC_GIDX]);
  v.wsum = reinterpret_cast<float*>(p + L.off[AREA_PLAN_SEC_WSUM]);
  v.cover = reinterpret_cast<int*>(p + L.off[AREA_PLAN_SEC_COVER]);
  v.order = reinterpret_cast<int*>(p + L.off[AREA_PLAN_SEC_ORDER]);
  v.nitem = reinterpret_cast<int*>(p + L.off[AREA_PLAN_SEC_NITEM]);
  v.items = reinterpret_cast<int2*>(p + L.off[AREA_PLAN_SEC_ITEMS]);
  v.nclass = reinterpret_cast<int*>(p + L.off[AREA_PLAN_SEC_NCLASS]);
  return v;
}

namespace {

struct HeaderArgs {
  int64_t v[32];
};

// ---------------------------------------------------------------------------
// Planner stages.  Each stage is a device function over one work item (a
// base window, a batch element, a block of tokens, a sort tile, a final
// window) run by a whole thread block; the separate kernels below launch one
// block per item, the fused kernel loops its blocks over the items and
// separates the stages with grid barriers.  Thread counts are any multiple of
// 32 up to 1024, except the sort histogram and scatter (256 threads).
// No stage pointer is __restrict__: in the fused kernel a stage reads what
// other blocks wrote before the last grid barrier, which must not go through
// the non-coherent read-only load path.
// ---------------------------------------------------------------------------

// Exclusive block-wide scan of one int per thread (blockDim.x multiple of 32,
// at most 1024).  Returns the exclusive prefix; *total receives the sum.
__device__ int block_exclusive_scan(int x, int* total) {
  __shared__ int s_warp[33];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarp = blockDim.x >> 5;
  int inc = x;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += t;
  }
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int wv = lane < nwarp ? s_warp[lane] : 0;
    int wi = wv;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int t = __shfl_up_sync(0xffffffffu, wi, d);
      if (lane >= d) wi += t;
    }
    if (lane < nwarp) s_warp[lane] = wi - wv;  // exclusive warp offsets
    if (lane == 31) s_warp[32] = wi;
  }
  __syncthreads();
  const int res = s_warp[warp] + inc - x;
  *total = s_warp[32];
  __syncthreads();
  return res;
}

// Header; zeroes the totals that stage_windows accumulates (the work-item
// total and the per-class totals, row B of NCLASS).
__device__ void stage_header(int64_t* hdr, const HeaderArgs& a, int* nitem_total,
                             int* nclass_total) {
  if (threadIdx.x < 32) hdr[threadIdx.x] = a.v[threadIdx.x];
  if (threadIdx.x == 0) *nitem_total = 0;
  if (threadIdx.x < 4) nclass_total[threadIdx.x] = 0;
}

// Split score of base window `item` = b * nb_cap + bi.
__device__ void stage_base(const float* E, const PlanView& P, float thr, int item,
                           float* s_rows) {
  const int b = item / P.nb_cap, bi = item % P.nb_cap;
  if (bi >= P.nb) return;
  const int iy = bi / P.nbx, ix = bi % P.nbx;
  int y0, hy, x0, wx;
  axis_window(iy, P.nby, P.Hg, P.hy, P.sy, &y0, &hy);
  axis_window(ix, P.nbx, P.Wg, P.wx, P.sx, &x0, &wx);
  const int Wc = P.Wg / 2;
  const float* Eb = E + (int64_t)b * (P.Hg / 2) * Wc;
  for (int y = threadIdx.x; y < hy; y += blockDim.x) {
    const float* er = Eb + (int64_t)((y0 + y) >> 1) * Wc;
    float acc = 0.f;
    for (int x = x0; x < x0 + wx; ++x) acc = __fadd_rn(acc, er[x >> 1]);
    s_rows[y] = acc;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float S = 0.f;
    for (int y = 0; y < hy; ++y) S = __fadd_rn(S, s_rows[y]);
    const float T = __fmul_rn(thr, (float)(hy * wx));
    const bool split = hy >= 2 && wx >= 2 && S < T;
    const int64_t o = (int64_t)b * P.nb_cap + bi;
    P.base[o] = make_int4(y0, x0, hy, wx);
    P.score[o] = S;
    P.split[o] = split ? 1 : 0;
  }
  __syncthreads();                             // s_rows is reused by the next item
}

__device__ __forceinline__ int4 halo_rect(int4 w, int h, int Hg, int Wg) {
  const int ey0 = max(0, w.x - h), ex0 = max(0, w.y - h);
  const int ey1 = min(Hg, w.x + w.z + h), ex1 = min(Wg, w.y + w.w + h);
  return make_int4(ey0, ex0, ey1 - ey0, ex1 - ex0);
}

// Final windows, Halo rectangles, G_W and the work list of batch element b.
__device__ void stage_windows(const PlanView& P, int b) {
  const int4* base = P.base + (int64_t)b * P.nb_cap;
  const uint8_t* split = P.split + (int64_t)b * P.nb_cap;
  int4* win = P.win + (int64_t)b * P.nw;
  int* parent = P.parent + (int64_t)b * P.nw;
  int4* ext = P.ext + (int64_t)b * P.nw;
  int* gcount = P.gcount + (int64_t)b * P.nw;
  int running = 0, total;
  for (int c0 = 0; c0 < P.nb; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    const bool valid = i < P.nb;
    const bool sp = valid && split[i];
    const int cnt = valid ? (sp ? 4 : 1) : 0;
    const int at = running + block_exclusive_scan(cnt, &total);
    if (valid) {
      const int4 bw = base[i];
      int4 q[4];
      int nq = 1;
      if (sp) {
        const int ht = bw.z / 2, wl = bw.w / 2;
        q[0] = make_int4(bw.x, bw.y, ht, wl);
        q[1] = make_int4(bw.x, bw.y + wl, ht, bw.w - wl);
        q[2] = make_int4(bw.x + ht, bw.y, bw.z - ht, wl);
        q[3] = make_int4(bw.x + ht, bw.y + wl, bw.z - ht, bw.w - wl);
        nq = 4;
      } else {
        q[0] = bw;
      }
      for (int j = 0; j < nq; ++j) {
        // Halo width: fixed, or drawn in [0, halo] per final window with a seed
        const int h = P.seed ? (int)(counter_random(P.seed, kStreamHalo,
                                                    ((unsigned long long)b << 20) + at + j) %
                                     (unsigned long long)(P.halo + 1))
                             : P.halo;
        const int4 e = halo_rect(q[j], h, P.Hg, P.Wg);
        const int64_t rest = (int64_t)P.N - (int64_t)e.z * e.w;
        win[at + j] = q[j];
        parent[at + j] = i;
        ext[at + j] = e;
        gcount[at + j] = (int)(rest < P.G ? rest : P.G);
      }
    }
    running += total;
  }
  const int nwin = running;
  if (threadIdx.x == 0) P.nwin[b] = nwin;
  __syncthreads();
  // Work items, grouped by the parity class of the base window (windows of
  // one class never overlap, so the merge can run class after class); within
  // a class, windows whose parent kept its size first (largest KV sets), then
  // the quadrants, each in window order.
  int2* items = P.items + (int64_t)b * P.nitem_max;
  running = 0;
  for (int pc = 0; pc < 4; ++pc) {
    const int start = running;
    for (int sc = 0; sc < 2; ++sc) {
      for (int c0 = 0; c0 < nwin; c0 += blockDim.x) {
        const int wi = c0 + threadIdx.x;
        int nq = 0;
        if (wi < nwin && (int)split[parent[wi]] == sc && window_class(parent[wi], P.nbx) == pc) {
          const int4 w = win[wi];
          nq = (w.z * w.w + kQTile - 1) / kQTile;
        }
        const int at = running + block_exclusive_scan(nq, &total);
        for (int t = 0; t < nq; ++t) items[at + t] = make_int2(wi, t);
        running += total;
      }
    }
    if (threadIdx.x == 0) {
      P.nclass[b * 4 + pc] = running - start;
      atomicAdd(P.nclass + P.B * 4 + pc, running - start);
    }
  }
  if (threadIdx.x == 0) {
    P.nitem[b] = running;
    atomicAdd(P.nitem + P.B, running);
  }
}

// ---- stable LSD radix sort of (~energy bits, token) ------------------------
// Keys and values of the tokens t in [t0, t0 + blockDim.x).
__device__ void stage_sort_init(const float* E, int b, const PlanView& P,
                                uint32_t* keys, int* vals, int t0) {
  const int t = t0 + threadIdx.x;
  if (t >= P.N) return;
  const int y = t / P.Wg, x = t % P.Wg;
  const int Wc = P.Wg / 2;
  const float e = E[((int64_t)b * (P.Hg / 2) + (y >> 1)) * Wc + (x >> 1)];
  keys[t] = ~__float_as_uint(e);   // ascending order of ~bits = descending energy
  vals[t] = t;
}

// Digit histogram of sort tile `tile` (256 threads).
__device__ void stage_sort_hist(const uint32_t* keys, int n, int shift,
                                uint32_t* hist, int ntile, int tile) {
  __shared__ uint32_t s_h[256];
  s_h[threadIdx.x] = 0;
  __syncthreads();
  const int base = tile * kSortTile;
#pragma unroll 4
  for (int r = 0; r < kSortRounds; ++r) {
    const int i = base + r * 256 + threadIdx.x;
    if (i < n) atomicAdd(&s_h[(keys[i] >> shift) & 255u], 1u);
  }
  __syncthreads();
  hist[(int64_t)threadIdx.x * ntile + tile] = s_h[threadIdx.x];
  __syncthreads();
}

// Exclusive scan, in place, of the digit-major histogram (one block).
__device__ void stage_sort_scan(uint32_t* hist, int m) {
  const int per = (m + blockDim.x - 1) / blockDim.x;
  const int lo = threadIdx.x * per, hi = min(m, lo + per);
  int sum = 0;
  for (int i = lo; i < hi; ++i) sum += (int)hist[i];
  int total;
  int run = block_exclusive_scan(sum, &total);
  for (int i = lo; i < hi; ++i) {
    const int h = (int)hist[i];
    hist[i] = (uint32_t)run;
    run += h;
  }
}

// Stable scatter of sort tile `tile` (256 threads): elements are taken in
// index order (round r, then warp, then lane); each element's rank among
// equal digits is its rank within its warp, plus the equal digits of earlier
// warps of the same round, plus those of earlier rounds.
__device__ void tile_offsets_from_hist(const uint32_t* hist, int ntile, int tile, int* s_run);

// With raw = true the histogram is the unscanned one and the tile's offsets
// are derived from it in the block.
__device__ void stage_sort_scatter(const uint32_t* kin, const int* vin,
                                   uint32_t* kout, int* vout, int n, int shift,
                                   const uint32_t* hist, int ntile, int tile, bool raw = false) {
  __shared__ int s_cnt[8][257];
  __shared__ int s_run[256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (raw) tile_offsets_from_hist(hist, ntile, tile, s_run);
  else s_run[threadIdx.x] = (int)hist[(int64_t)threadIdx.x * ntile + tile];
  for (int r = 0; r < kSortRounds; ++r) {
    for (int j = threadIdx.x; j < 8 * 257; j += 256) (&s_cnt[0][0])[j] = 0;
    __syncthreads();
    const int i = tile * kSortTile + r * 256 + threadIdx.x;
    const bool valid = i < n;
    const uint32_t key = valid ? kin[i] : 0u;
    const int val = valid ? vin[i] : 0;
    const int d = valid ? (int)((key >> shift) & 255u) : 256;
    const unsigned peers = __match_any_sync(0xffffffffu, d);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (lane == __ffs(peers) - 1) s_cnt[warp][d] = __popc(peers);
    __syncthreads();
    // exclusive prefix over warps for digit dd; the round total advances s_run
    const int dd = threadIdx.x;
    int run = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const int c = s_cnt[w][dd];
      s_cnt[w][dd] = run;
      run += c;
    }
    __syncthreads();
    if (valid) {
      const int pos = s_run[d] + s_cnt[warp][d] + rank;
      kout[pos] = key;
      vout[pos] = val;
    }
    __syncthreads();
    s_run[dd] += run;
  }
  __syncthreads();
}

// Digit offsets of sort tile `tile` straight from the raw (unscanned)
// digit-major histogram: s_run[d] = (keys of all tiles with a smaller digit)
// + (keys of earlier tiles with digit d).  The same integers the scan stage
// produces, so the fused kernel can skip that stage and its barriers.
__device__ void tile_offsets_from_hist(const uint32_t* hist, int ntile, int tile, int* s_run) {
  const int d = threadIdx.x;                   // 256 threads, one digit each
  const uint32_t* row = hist + (int64_t)d * ntile;
  int before = 0, all = 0;
  for (int t = 0; t < ntile; ++t) {
    const int h = (int)row[t];
    before += t < tile ? h : 0;
    all += h;
  }
  int total;
  const int smaller = block_exclusive_scan(all, &total);
  s_run[d] = smaller + before;
  __syncthreads();
}

// Global-KV bridge of final window `item` = b * nw + wi: the first G_W
// tokens of the ranked order outside ext(W).
__device__ void stage_global(const PlanView& P, int item) {
  const int b = item / P.nw, wi = item % P.nw;
  if (wi >= P.nwin[b] || P.G == 0) return;
  const int64_t o = (int64_t)b * P.nw + wi;
  const int4 e = P.ext[o];
  const int gw = P.gcount[o];
  int* out = P.gidx + o * P.G;
  const int* order = P.order + (int64_t)b * P.N;
  int count = 0, total;
  for (int c0 = 0; c0 < P.N && count < gw; c0 += blockDim.x) {
    const int p = c0 + threadIdx.x;
    int tok = -1, flag = 0;
    if (p < P.N) {
      tok = order[p];
      const int y = tok / P.Wg, x = tok % P.Wg;
      flag = (y >= e.x && y < e.x + e.z && x >= e.y && x < e.y + e.w) ? 0 : 1;
    }
    const int at = count + block_exclusive_scan(flag, &total);
    if (flag && at < gw) out[at] = tok;
    count += total;
  }
  for (int j = gw + threadIdx.x; j < P.G; j += blockDim.x) out[j] = -1;
}

// Sum of tent weights, and count, of the final windows that contain each of
// the tokens g in [g0, g0 + blockDim.x) (g = b * N + t).
__device__ void stage_wsum(const PlanView& P, int64_t g0) {
  const int64_t g = g0 + threadIdx.x;
  if (g >= (int64_t)P.B * P.N) return;
  const int b = (int)(g / P.N);
  const int t = (int)(g % P.N);
  const int y = t / P.Wg, x = t % P.Wg;
  int total = 0, count = 0;
  for (int iy = 0; iy < P.nby; ++iy) {
    int y0, hy;
    axis_window(iy, P.nby, P.Hg, P.hy, P.sy, &y0, &hy);
    if (y < y0 || y >= y0 + hy) continue;
    for (int ix = 0; ix < P.nbx; ++ix) {
      int x0, wx;
      axis_window(ix, P.nbx, P.Wg, P.wx, P.sx, &x0, &wx);
      if (x < x0 || x >= x0 + wx) continue;
      int qy0 = y0, qhy = hy, qx0 = x0, qwx = wx;
      if (P.split[(int64_t)b * P.nb_cap + iy * P.nbx + ix]) {
        const int ht = hy / 2, wl = wx / 2;
        if (y < y0 + ht) { qhy = ht; } else { qy0 = y0 + ht; qhy = hy - ht; }
        if (x < x0 + wl) { qwx = wl; } else { qx0 = x0 + wl; qwx = wx - wl; }
      }
      total += min(y - qy0 + 1, qy0 + qhy - y) * min(x - qx0 + 1, qx0 + qwx - x);
      ++count;
    }
  }
  P.wsum[g] = (float)total;
  P.cover[g] = count;
}

// ---------------------------------------------------------------------------
// One launch per stage
// ---------------------------------------------------------------------------
__global__ void plan_header_kernel(int64_t* hdr, HeaderArgs a, int* nitem_total,
                                   int* nclass_total) {
  stage_header(hdr, a, nitem_total, nclass_total);
}

__global__ void __launch_bounds__(256) plan_base_kernel(const float* __restrict__ E, PlanView P,
                                                       float thr) {
  extern __shared__ float s_rows[];
  stage_base(E, P, thr, blockIdx.x, s_rows);
}

__global__ void __launch_bounds__(1024) plan_windows_kernel(PlanView P) {
  stage_windows(P, blockIdx.x);
}

__global__ void __launch_bounds__(256) sort_init_kernel(const float* __restrict__ E, int b,
                                                       PlanView P, uint32_t* keys, int* vals) {
  stage_sort_init(E, b, P, keys, vals, blockIdx.x * blockDim.x);
}

__global__ void __launch_bounds__(256) sort_hist_kernel(const uint32_t* __restrict__ keys, int n,
                                                       int shift, uint32_t* hist, int ntile) {
  stage_sort_hist(keys, n, shift, hist, ntile, blockIdx.x);
}

__global__ void __launch_bounds__(1024) sort_scan_kernel(uint32_t* hist, int m) {
  stage_sort_scan(hist, m);
}

__global__ void __launch_bounds__(256) sort_scatter_kernel(const uint32_t* __restrict__ kin,
                                                          const int* __restrict__ vin,
                                                          uint32_t* kout, int* vout, int n,
                                                          int shift, const uint32_t* hist,
                                                          int ntile) {
  stage_sort_scatter(kin, vin, kout, vout, n, shift, hist, ntile, blockIdx.x);
}

__global__ void __launch_bounds__(1024) plan_global_kernel(PlanView P) {
  stage_global(P, blockIdx.x);
}

__global__ void __launch_bounds__(256) plan_wsum_kernel(PlanView P) {
  stage_wsum(P, blockIdx.x * (int64_t)blockDim.x);
}

// ---------------------------------------------------------------------------
// Detail map + planner in one cooperative launch.  Every block runs every
// stage over its share of the items; a grid barrier separates the stages.
// The barrier is a monotone arrival counter in the plan's scratch (zeroed by
// the launcher); each wait is bounded by kPlanWaitNs of %globaltimer, after
// which the block raises the abort word, records g_plan_error and returns,
// and every other block leaves at its next barrier.
// ---------------------------------------------------------------------------
constexpr int kFusedThreads = 256;
constexpr uint64_t kPlanWaitNs = 2000000000ull;

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ bool grid_sync(unsigned* bar, unsigned target, uint64_t wait_ns, int* s_ok) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();                           // this block's writes, then its arrival
    atomicAdd(bar, 1u);
    const uint64_t t0 = global_ns();
    int ok = 1;
    for (;;) {
      unsigned v, ab;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
      if (v >= target) break;
      asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(ab) : "l"(bar + 1) : "memory");
      if (ab != 0u || global_ns() - t0 > wait_ns) {
        ok = 0;
        atomicExch(bar + 1, 1u);
        atomicExch(&g_plan_error, 1);
        break;
      }
      __nanosleep(32);
    }
    __threadfence();
    *s_ok = ok;
  }
  __syncthreads();
  return *s_ok != 0;
}

struct FusedArgs {
  const void* src;       // detail source [B, N, C] (DWT stage), else null
  int C;
  float inv_c;           // fl32(1 / C)
  float* energy;         // [B, Hg/2, Wg/2]
  float thr;
  int64_t* hdr;
  uint32_t *ka, *kb, *hist;
  int *va, *vb;
  int nt;                // sort tiles
  unsigned* bar;         // [arrivals, abort]
  unsigned target_extra; // added to every barrier target (0; 1 only in the expiry test hook)
  uint64_t wait_ns;      // bound of each barrier wait
};

template <typename T, int MODE, bool VEC>
__global__ void __launch_bounds__(kFusedThreads, 2) plan_fused_kernel(PlanView P, FusedArgs A,
                                                                  HeaderArgs h) {
  extern __shared__ float s_rows[];
  __shared__ int s_ok;
  unsigned nbar = 0;
  auto sync = [&]() {
    return grid_sync(A.bar, ++nbar * gridDim.x + A.target_extra, A.wait_ns, &s_ok);
  };
  const int G = gridDim.x;
  const int n = P.N;
  // detail map
  if (A.src) {
    const int64_t ncell = (int64_t)P.B * (P.Hg / 2) * (P.Wg / 2);
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < ncell;
         g += (int64_t)G * blockDim.x)
      A.energy[g] = detail_cell<T, MODE, VEC>(static_cast<const T*>(A.src), A.C, g, P.Hg, P.Wg,
                                              A.inv_c);
    if (!sync()) return;
  }
  // header, split scores, sort keys of element 0
  {
    const int nbase = P.B * P.nb_cap, ninit = (n + blockDim.x - 1) / blockDim.x;
    if (blockIdx.x == 0) stage_header(A.hdr, h, P.nitem + P.B, P.nclass + P.B * 4);
    for (int it = blockIdx.x; it < nbase + ninit; it += G) {
      if (it < nbase) stage_base(A.energy, P, A.thr, it, s_rows);
      else stage_sort_init(A.energy, 0, P, A.ka, A.va, (it - nbase) * blockDim.x);
    }
    if (!sync()) return;
  }
  for (int b = 0; b < P.B; ++b) {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 8 * pass;
      const uint32_t* kin = (pass & 1) ? A.kb : A.ka;
      const int* vin = (pass & 1) ? A.vb : A.va;
      uint32_t* kout = (pass & 1) ? A.ka : A.kb;
      int* vout = (pass == 3) ? P.order + (int64_t)b * n : ((pass & 1) ? A.va : A.vb);
      // histogram (the first pass of element 0 also builds the windows)
      const int nwin_items = (b == 0 && pass == 0) ? P.B : 0;
      for (int it = blockIdx.x; it < nwin_items + A.nt; it += G) {
        if (it < nwin_items) stage_windows(P, it);
        else stage_sort_hist(kin, n, shift, A.hist, A.nt, it - nwin_items);
      }
      if (!sync()) return;
      for (int it = blockIdx.x; it < A.nt; it += G)
        stage_sort_scatter(kin, vin, kout, vout, n, shift, A.hist, A.nt, it, /*raw=*/true);
      if (!sync()) return;
    }
    if (b + 1 < P.B) {                         // keys of the next element
      for (int it = blockIdx.x; it < (n + (int)blockDim.x - 1) / (int)blockDim.x; it += G)
        stage_sort_init(A.energy, b + 1, P, A.ka, A.va, it * blockDim.x);
      if (!sync()) return;
    }
  }
  // global-KV lists and merge-weight sums
  {
    const int nglob = P.B * P.nw;
    const int nws = (int)(((int64_t)P.B * n + blockDim.x - 1) / blockDim.x);
    for (int it = blockIdx.x; it < nglob + nws; it += G) {
      if (it < nglob) stage_global(P, it);
      else stage_wsum(P, (int64_t)(it - nglob) * blockDim.x);
    }
  }
}

}  // namespace

namespace {
HeaderArgs header_args(const PlanLayout& L) {
  HeaderArgs h = {};
  h.v[0] = AREA_PLAN_MAGIC; h.v[1] = AREA_PLAN_VERSION;
  h.v[2] = L.B; h.v[3] = L.Hg; h.v[4] = L.Wg; h.v[5] = L.w; h.v[6] = L.halo; h.v[7] = L.G;
  h.v[8] = L.nb_cap; h.v[9] = L.nw;
  for (int i = 0; i < AREA_PLAN_NSEC; ++i) h.v[10 + i] = L.off[i];
  h.v[10 + AREA_PLAN_NSEC] = L.nitem_max;
  h.v[11 + AREA_PLAN_NSEC] = L.N;
  h.v[12 + AREA_PLAN_NSEC] = L.nb;
  h.v[13 + AREA_PLAN_NSEC] = L.sy;
  h.v[14 + AREA_PLAN_NSEC] = L.sx;
  return h;
}
}  // namespace

cudaError_t launch_window_plan(const float* energy, const area_plan_cfg* cfg,
                               const PlanLayout& L, void* plan, cudaStream_t s) {
  PlanView P = plan_view(L, plan);
  char* base = static_cast<char*>(plan);
  const HeaderArgs h = header_args(L);
  plan_header_kernel<<<1, 32, 0, s>>>(reinterpret_cast<int64_t*>(base), h, P.nitem + L.B,
                                      P.nclass + L.B * 4);
  const int smem = (int)(L.hy * sizeof(float));
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(plan_base_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  plan_base_kernel<<<(unsigned)(L.B * L.nb_cap), 256, smem, s>>>(energy, P, cfg->split_thr);
  plan_windows_kernel<<<(unsigned)L.B, 1024, 0, s>>>(P);
  uint32_t* ka = reinterpret_cast<uint32_t*>(base + L.scratch_keys_a);
  uint32_t* kb = reinterpret_cast<uint32_t*>(base + L.scratch_keys_b);
  int* va = reinterpret_cast<int*>(base + L.scratch_vals_a);
  int* vb = reinterpret_cast<int*>(base + L.scratch_vals_b);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + L.scratch_hist);
  const int n = (int)L.N, nt = (int)L.ntile_sort;
  for (int b = 0; b < L.B; ++b) {
    sort_init_kernel<<<(n + 255) / 256, 256, 0, s>>>(energy, b, P, ka, va);
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 8 * pass;
      const uint32_t* kin = (pass & 1) ? kb : ka;
      const int* vin = (pass & 1) ? vb : va;
      uint32_t* kout = (pass & 1) ? ka : kb;
      int* vout = (pass == 3) ? P.order + (int64_t)b * L.N : ((pass & 1) ? va : vb);
      sort_hist_kernel<<<nt, 256, 0, s>>>(kin, n, shift, hist, nt);
      sort_scan_kernel<<<1, 1024, 0, s>>>(hist, 256 * nt);
      sort_scatter_kernel<<<nt, 256, 0, s>>>(kin, vin, kout, vout, n, shift, hist, nt);
    }
  }
  plan_global_kernel<<<(unsigned)(L.B * L.nw), 1024, 0, s>>>(P);
  const int64_t ntok = L.B * L.N;
  plan_wsum_kernel<<<(unsigned)((ntok + 255) / 256), 256, 0, s>>>(P);
  return cudaGetLastError();
}

template <typename T, int MODE, bool VEC>
static cudaError_t launch_fused_typed(const PlanLayout& L, const PlanView& P, const FusedArgs& A,
                                     const HeaderArgs& h, cudaStream_t s) {
  auto fn = plan_fused_kernel<T, MODE, VEC>;
  const int smem = (int)(L.hy * sizeof(float)) > 16 ? (int)(L.hy * sizeof(float)) : 16;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kFusedThreads, smem)) !=
      cudaSuccess)
    return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int grid = sms * (per_sm < 2 ? per_sm : 2);  // every block resident at once
  if ((e = cudaMemsetAsync(A.bar, 0, 2 * sizeof(unsigned), s)) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, P, A, h);
}

cudaError_t launch_dwt_window_plan(const void* src, int src_dtype, int C, int mode, float* energy,
                                   const area_plan_cfg* cfg, const PlanLayout& L, void* plan,
                                   cudaStream_t s, unsigned target_extra, uint64_t wait_ns) {
  PlanView P = plan_view(L, plan);
  char* base = static_cast<char*>(plan);
  FusedArgs A = {};
  A.src = src;
  A.C = C;
  A.inv_c = 1.0f / (float)C;                   // host IEEE division: fl32(1 / C)
  A.energy = energy;
  A.thr = cfg->split_thr;
  A.hdr = reinterpret_cast<int64_t*>(base);
  A.ka = reinterpret_cast<uint32_t*>(base + L.scratch_keys_a);
  A.kb = reinterpret_cast<uint32_t*>(base + L.scratch_keys_b);
  A.va = reinterpret_cast<int*>(base + L.scratch_vals_a);
  A.vb = reinterpret_cast<int*>(base + L.scratch_vals_b);
  A.hist = reinterpret_cast<uint32_t*>(base + L.scratch_hist);
  A.nt = (int)L.ntile_sort;
  A.bar = reinterpret_cast<unsigned*>(base + L.scratch_bar);
  A.target_extra = target_extra;
  A.wait_ns = wait_ns ? wait_ns : kPlanWaitNs;
  const HeaderArgs h = header_args(L);
  const bool vec = C % (src_dtype == AREA_DTYPE_BF16 ? 8 : 4) == 0 &&
                   (reinterpret_cast<uintptr_t>(src) & 15) == 0;
#define AREA_FUSED(T, M, V) launch_fused_typed<T, M, V>(L, P, A, h, s)
  if (src_dtype == AREA_DTYPE_BF16) {
    if (mode == AREA_DETAIL_HH)
      return vec ? AREA_FUSED(__nv_bfloat16, AREA_DETAIL_HH, true)
                 : AREA_FUSED(__nv_bfloat16, AREA_DETAIL_HH, false);
    return vec ? AREA_FUSED(__nv_bfloat16, AREA_DETAIL_ALL3, true)
               : AREA_FUSED(__nv_bfloat16, AREA_DETAIL_ALL3, false);
  }
  if (mode == AREA_DETAIL_HH)
    return vec ? AREA_FUSED(float, AREA_DETAIL_HH, true) : AREA_FUSED(float, AREA_DETAIL_HH, false);
  return vec ? AREA_FUSED(float, AREA_DETAIL_ALL3, true) : AREA_FUSED(float, AREA_DETAIL_ALL3, false);
#undef AREA_FUSED
}

cudaError_t read_and_clear_plan_error(int* code) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(code, g_plan_error, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_plan_error, &zero, sizeof(int));
}

}  // namespace area
