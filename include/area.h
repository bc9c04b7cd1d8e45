/*
 * libarea -- C-ABI of the AReA attention hot path on B200 (sm_100a).
 *
 * AReA ("Adaptive Receptive-Field Attention for Efficient High-Resolution
 * Diffusion Transformers", arXiv 2610.17227) replaces full self-attention of a
 * diffusion transformer above its native resolution by
 *   Phase I  -- cross-scale coarse attention: full-resolution queries against
 *               keys/values pooled over f x f token blocks;
 *   Phase II -- adaptive windowed attention: shrinking windows, quadrant
 *               splits of smooth windows (Haar DWT detail map), a Halo ring of
 *               neighbouring keys, a global-KV bridge, and centre-weighted
 *               blending of overlapping window outputs.
 * Citations below name the summary pages the method is taken from:
 *   [ai]   ai.info paper summary, "Methodology in Plain English";
 *   [blog] gpt-diffusion.com blog, "Las dos fases de AReA" (Fase I/Fase II);
 *   [wiki] github.com/KooroshRH/AReA wiki (overview, canvas rules).
 *
 * Conventions (all functions):
 *   - Every buffer is owned by the caller and lives in device memory unless
 *     stated otherwise.  The library allocates no device memory and keeps no
 *     state between calls.
 *   - Tensors are dense and contiguous.  Q, K, V, O: [B, H, N, D] with the
 *     token index n = y * Wg + x over an Hg x Wg token grid (row-major).
 *     Q and K arrive already rotated (RoPE is the caller's business).
 *   - dtype: AREA_DTYPE_BF16 (storage bf16, tensor-core MMA with fp32
 *     accumulation, D = 128 or 64) or AREA_DTYPE_F32 (storage fp32, fp32
 *     CUDA-core arithmetic, D = 64 or 128).
 *   - Every kernel call is asynchronous on the given stream (0 = legacy
 *     default stream) and never synchronises the host.  No CTA waits on
 *     another, except in two calls, always with bounded waits:
 *     area_dwt_window_plan, a cooperative launch (every CTA resident) with
 *     grid barriers; and the window-attention calls on the tensor cores,
 *     where a CTA about to add a later parity class of windows into an
 *     overlapped token's accumulator row waits until every unit of the
 *     earlier classes of the same head has completed (a head's units are
 *     claimed in class order by running CTAs, so every unit waited on is
 *     held by a running CTA).  The return value
 *     reports argument validation and launch errors only; AREA_ECUDA carries
 *     the CUDA error, see area_status_string.  The schedule functions at the
 *     end are host arithmetic (no device memory, no stream).
 *   - Device pointers passed to the attention calls must be 16-byte aligned;
 *     their outputs (o) and the window workspace (ws) 32-byte aligned.
 */
#ifndef AREA_H_
#define AREA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define AREA_OK            0
#define AREA_EINVAL        1   /* null pointer, bad size, bad enum value       */
#define AREA_EUNSUPPORTED  2   /* dtype / head_dim / grid the library lacks    */
#define AREA_ENOSPACE      3   /* plan or workspace buffer too small           */
#define AREA_ECUDA         4   /* CUDA launch error (area_last_cuda_error())   */

/* ---- enums ------------------------------------------------------------- */
#define AREA_DTYPE_F32     0
#define AREA_DTYPE_BF16    1

#define AREA_POOL_MEAN     0   /* block average                                */
#define AREA_POOL_CENTER   1   /* token (py*f + f/2, px*f + f/2)               */

#define AREA_DETAIL_HH     0   /* e = HH^2                                     */
#define AREA_DETAIL_ALL3   1   /* e = (LH^2 + HL^2) + HH^2                     */

#define AREA_PHASE_COARSE  1   /* Phase I step: pool K/V by f, coarse attention */
#define AREA_PHASE_WINDOW  2   /* Phase II step: DWT, plan, window attention    */

/* Returns a static, human-readable string for a status code. */
const char* area_status_string(int status);
/* CUDA error code of the most recent AREA_ECUDA return on this thread. */
int area_last_cuda_error(void);
/* Library version, e.g. "libarea 0.1.0 sm_100a". */
const char* area_version(void);
#define AREA_KERR_TC_WAIT        1  /* a tensor-core kernel's mbarrier wait expired */
#define AREA_KERR_PLAN_BARRIER    2  /* a grid barrier of area_dwt_window_plan expired */
/*
 * area_kernel_error -- synchronises the current device, then reports in
 * *code whether a kernel gave up a bounded wait since the last call (0 =
 * none; else an OR of AREA_KERR_* bits; the output of that launch is
 * invalid), and clears the flags.  Meant for tests and health checks, not
 * the hot path.   Errors: AREA_EINVAL (null), AREA_ECUDA.
 */
int area_kernel_error(int* code);

/* ---- Phase I ----------------------------------------------------------- */

/*
 * area_pool_kv -- one representative key/value token per f x f block.
 * [blog] Fase I / [ai] Phase I: keys and values are pooled to one token per
 * f x f block, on a (Hg/f) x (Wg/f) grid.
 *
 *   k, v   : [B, H, Hg*Wg, D] input (dtype)
 *   kp, vp : [B, H, (Hg/f)*(Wg/f), D] output (dtype); pooled token index
 *            py*(Wg/f) + px.
 *   mode   : AREA_POOL_MEAN (fp32 sum over the block, rows then columns,
 *            divided by f*f, rounded to the output dtype) or AREA_POOL_CENTER.
 * Errors: AREA_EINVAL if a pointer is null, a size is < 1, f does not divide
 * Hg and Wg (the canvas rule of [wiki]: the two patch counts must share the
 * pooling factor), or mode/dtype is unknown.  D must be a multiple of 8.
 */
int area_pool_kv(const void* k, const void* v, void* kp, void* vp,
                 int B, int H, int Hg, int Wg, int D, int f, int mode,
                 int dtype, cudaStream_t stream);

/*
 * area_coarse_attn -- Phase I cross-scale coarse attention ([ai] Phase I):
 *   O = softmax(scale * Q Kp^T) Vp   per (b, h), text tokens absent.
 *   q  : [B, H, N, D]; kp, vp : [B, H, Nk, D]; o : [B, H, N, D] (dtype).
 * bf16 (D = 64 or 128) runs on the tcgen05 tensor-core kernel, fp32 on the
 * CUDA-core kernel.
 * Errors: AREA_EINVAL (null, N < 1, Nk < 1), AREA_EUNSUPPORTED (D not 64/128,
 * unknown dtype).
 */
int area_coarse_attn(const void* q, const void* kp, const void* vp, void* o,
                     int B, int H, int N, int Nk, int D, float scale,
                     int dtype, cudaStream_t stream);

/*
 * area_coarse_attn_text -- Phase I with text tokens ([ai] Phase I: text tokens
 * are never pooled, so each of the N queries attends to T + N/f^2 keys):
 *   O = softmax(scale * Q [Kp; Kt]^T) [Vp; Vt]   per (b, h).
 *   kt, vt : [B, H, T, D] text keys and values (dtype), T >= 0 (0 = none).
 * Outputs are the image queries' rows only; text queries are the caller's.
 * Errors: as area_coarse_attn, and AREA_EINVAL for T < 0 or null kt/vt with
 * T > 0.
 */
int area_coarse_attn_text(const void* q, const void* kp, const void* vp,
                          const void* kt, const void* vt, void* o,
                          int B, int H, int N, int Nk, int T, int D,
                          float scale, int dtype, cudaStream_t stream);

/*
 * area_full_attn -- full global attention over all N tokens, the operation
 * AReA replaces ([ai] "Main Findings": speedups are quoted against it).
 * Same kernels as area_coarse_attn with Nk = N.
 */
int area_full_attn(const void* q, const void* k, const void* v, void* o,
                   int B, int H, int N, int D, float scale,
                   int dtype, cudaStream_t stream);

/* ---- Phase II ---------------------------------------------------------- */

/*
 * area_dwt_detail -- Haar detail energy per 2x2 token cell ([ai] Phase II:
 * "a DWT map computed from the current hidden states measures fine detail").
 * For cell (cy, cx) and channel c, with a = x(2cy,2cx), b = x(2cy,2cx+1),
 * c' = x(2cy+1,2cx), d = x(2cy+1,2cx+1) widened to fp32:
 *   HH = ((a - b) - (c' - d)) * 0.5,  LH = ((a + b) - (c' + d)) * 0.5,
 *   HL = ((a - b) + (c' - d)) * 0.5,
 *   e_c = HH^2 (AREA_DETAIL_HH) or (LH^2 + HL^2) + HH^2 (AREA_DETAIL_ALL3),
 *   E = ((..((0 + e_0) + e_1)..) + e_{C-1}) * (1/C),
 * every operation in round-to-nearest fp32 without contraction, so the map
 * is bit-reproducible.
 *   src    : [B, Hg*Wg, C] channels-last, src_dtype (F32 or BF16)
 *   energy : [B, Hg/2, Wg/2] fp32 output
 * Errors: AREA_EINVAL (null, Hg or Wg odd or < 2, C < 1, bad mode/dtype).
 */
int area_dwt_detail(const void* src, int src_dtype, int C, float* energy,
                    int B, int Hg, int Wg, int mode, cudaStream_t stream);

/* Configuration of one Phase II step.  split_thr is the mean-energy bound
 * below which a window splits.  jitter_seed = 0 gives the fixed plan; any
 * other value turns on the seeded randomness of [ai] Phase II and [blog]
 * README notes (the seed sets border jitter and Halo widths):
 *   - border shift s in [0, w_e) per axis (SplitMix64 output number 2^32 and
 *     2^32 + 1 of the sequence seeded with jitter_seed, mod w_e): the base
 *     tiling is the even tiling of the extended axis [-s, L), clipped to
 *     [0, L);
 *   - Halo width per final window i of batch element b: output number
 *     2 * 2^32 + b * 2^20 + i of the same sequence, mod (halo + 1).
 * Pass a different seed per denoising step to move the seams. */
typedef struct area_plan_cfg {
  int B;            /* batch elements (one plan each)                        */
  int Hg, Wg;       /* token grid                                            */
  int w;            /* scheduled window side                                 */
  int halo;         /* Halo width h >= 0                                     */
  int G;            /* global-KV tokens per window, 0 <= G <= 4096           */
  float split_thr;  /* split when score < fl32(split_thr * hy * wx)          */
  unsigned long long jitter_seed;   /* 0: no jitter, fixed Halo             */
} area_plan_cfg;

/*
 * Plan buffer layout (device memory, written by area_window_plan).  The
 * first 256 bytes hold an int64 header; every section starts 256-byte
 * aligned at the byte offset stored in the header.  Windows are indexed per
 * batch element b in [0, B); "nb" = base-window capacity per element (room
 * for one extra window per axis under a border shift), "nw" = 4*nb.
 *   header[0]  = AREA_PLAN_MAGIC        header[1] = AREA_PLAN_VERSION
 *   header[2..8] = B, Hg, Wg, w, halo, G, nb
 *   header[9]  = nw
 *   header[10+s] = byte offset of section s (AREA_PLAN_SEC_*)
 *   header[26] = work-item capacity per element ("ni"), header[27] = N,
 *   header[28] = base windows of this plan (<= nb; fewer than the capacity
 *   when a border shift is drawn), header[29..30] = border shift (sy, sx)
 * Sections:
 *   BASE    int32 [B][nb][4]   base windows (y0, x0, hy, wx), row-major
 *   SCORE   f32   [B][nb]      sum of token energy over the base window
 *   SPLIT   u8    [B][nb]      1 = split into quadrants
 *   NWIN    int32 [B]          number of final windows
 *   WIN     int32 [B][nw][4]   final windows (y0, x0, hy, wx)
 *   PARENT  int32 [B][nw]      base window of each final window
 *   EXT     int32 [B][nw][4]   Halo rectangle (y0, x0, hy, wx), clipped
 *   GCOUNT  int32 [B][nw]      G_W = min(G, N - |ext|)
 *   GIDX    int32 [B][nw][G]   global-KV tokens in rank order, -1 padded
 *   WSUM    f32   [B][N]       sum of tent weights over final windows
 *   COVER   int32 [B][N]       number of final windows containing the token
 *   ORDER   int32 [B][N]       tokens by (energy desc, index asc)
 *   NITEM   int32 [B+1]        work items (window, query tile) per element,
 *                              last entry = total
 *   ITEMS   int32 [B][ni][2]   (window, block of 256 queries), grouped by
 *                              the parity class of the window's base window,
 *                              class = 2 * (row index & 1) + (column index & 1)
 *                              in the base tiling (windows of one class never
 *                              overlap); within a class, windows of unsplit
 *                              base windows first, then quadrants, each in
 *                              window order
 *   NCLASS  int32 [B+1][4]     work items per class; row B = totals
 *   SCRATCH                    sort and scan scratch (contents unspecified)
 */
#define AREA_PLAN_MAGIC    0x4145524150414c4eLL  /* "AREAPLAN" */
#define AREA_PLAN_VERSION  3
#define AREA_PLAN_SEC_BASE     0
#define AREA_PLAN_SEC_SCORE    1
#define AREA_PLAN_SEC_SPLIT    2
#define AREA_PLAN_SEC_NWIN     3
#define AREA_PLAN_SEC_WIN      4
#define AREA_PLAN_SEC_PARENT   5
#define AREA_PLAN_SEC_EXT      6
#define AREA_PLAN_SEC_GCOUNT   7
#define AREA_PLAN_SEC_GIDX     8
#define AREA_PLAN_SEC_WSUM     9
#define AREA_PLAN_SEC_ORDER    10
#define AREA_PLAN_SEC_NITEM    11
#define AREA_PLAN_SEC_ITEMS    12
#define AREA_PLAN_SEC_COVER    13
#define AREA_PLAN_SEC_NCLASS   14
#define AREA_PLAN_SEC_SCRATCH  15
#define AREA_PLAN_NSEC         16

/*
 * area_window_plan_bytes -- size of the plan buffer for cfg (host only).
 * Errors: AREA_EINVAL (null, bad sizes, G > 4096, B > 2048).
 */
int area_window_plan_bytes(const area_plan_cfg* cfg, size_t* plan_bytes);

/*
 * area_window_plan -- Phase II plan on the device ([ai] Phase II, steps in
 * the pages' order):
 *   1. base tiling: per axis of length L, w_e = min(w, L),
 *      n = ceil(L / w_e), start_i = floor(i (L - w_e) / (n - 1));
 *   2. split score S = sum of token energy (token (y,x) takes the energy of
 *      cell (y/2, x/2)), rows summed left to right then rows top to bottom,
 *      in fp32; split iff S < fl32(split_thr * hy * wx) and hy, wx >= 2;
 *   3. quadrants TL, TR, BL, BR, top/left halves floor(side/2);
 *   4. Halo rectangle: the window dilated by h, clipped to the grid;
 *   5. global-KV bridge: the first G_W = min(G, N - |ext|) tokens by
 *      (energy desc, token index asc) that lie outside the Halo rectangle;
 *   6. per-token sum of tent weights
 *      t = min(y-y0+1, y0+hy-y) * min(x-x0+1, x0+wx-x) over final windows,
 *      and the number of final windows containing the token;
 *   7. the list of (window, 256-query block) work items by parity class,
 *      costliest first within a class (see ITEMS).
 *   energy : [B, Hg/2, Wg/2] fp32 from area_dwt_detail
 *   plan   : device buffer of plan_bytes >= area_window_plan_bytes(cfg)
 * The plan never leaves the device.  Errors: AREA_EINVAL, AREA_ENOSPACE.
 */
int area_window_plan(const float* energy, const area_plan_cfg* cfg,
                     void* plan, size_t plan_bytes, cudaStream_t stream);

/*
 * area_dwt_window_plan -- area_dwt_detail followed by area_window_plan in ONE
 * cooperative kernel launch (plus a 8-byte memset of the plan's barrier
 * words): every block runs every stage -- detail map, split scores, windows,
 * the four radix-sort passes, global-KV lists, merge-weight sums -- over its
 * share of the work, with a grid barrier between stages.  Results are
 * bit-identical to the two separate calls.  The grid is at most two blocks of
 * 256 threads per SM, all resident at once (cooperative launch); each barrier
 * wait is bounded (2 s), after which the kernel stops and area_kernel_error
 * reports AREA_KERR_PLAN_BARRIER.
 *   src, src_dtype, C, mode : as area_dwt_detail (B, Hg, Wg from cfg);
 *   energy : fp32 [B, Hg/2, Wg/2] output, as area_dwt_detail;
 *   cfg, plan, plan_bytes   : as area_window_plan.
 * Errors: as area_dwt_detail and area_window_plan; AREA_ECUDA when the
 * device cannot co-schedule the grid.
 */
int area_dwt_window_plan(const void* src, int src_dtype, int C, int mode,
                         float* energy, const area_plan_cfg* cfg, void* plan,
                         size_t plan_bytes, cudaStream_t stream);

/*
 * area_window_attn_ws_bytes -- workspace for area_window_attn (host only):
 * a header of 1 + 4 * B * H uint32 counters (the unit counter and one
 * completion counter per batch element, head and parity class) rounded up
 * to 256 bytes, then one fp32 row of D values per (batch element, head,
 * token covered by more than one base window):
 *   hdr + B * H * n_ov * D * 4 bytes, hdr = ceil256(4 * (1 + 4 * B * H)),
 * n_ov = ny2 * Wg + (Hg - ny2) * nx2, where ny2 (nx2) counts the rows
 * (columns) of the grid that two base windows share along that axis under
 * the plan's border shift.  Windows that tile an axis exactly share nothing
 * (e.g. 64-token windows on a 384-token axis), and then the workspace is the
 * header alone.
 */
int area_window_attn_ws_bytes(const area_plan_cfg* cfg, int H, int D,
                              size_t* ws_bytes);

/*
 * area_window_attn_stage_bytes -- optional extra workspace (host only): when
 * the ws given to area_window_attn (or _text) holds at least
 * area_window_attn_ws_bytes() + stage_bytes, the bf16 tensor-core path first
 * copies each window's global-KV rows that fill whole 128-row tiles into it
 * (one launch on the stream), as [B][H][nw][G][D] K then V with nw the
 * plan's final-window capacity, and the attention kernel then loads them as
 * tiles instead of gathering them row by row in every work unit.  The result
 * is the same (the same keys in the same order).  stage_bytes =
 * 2 * B * H * nw * G * D * 2; 0 when G = 0.  The fp32 path and the bridged
 * calls do not use it.
 */
int area_window_attn_stage_bytes(const area_plan_cfg* cfg, int H, int D,
                                 size_t* stage_bytes);

/*
 * area_window_attn -- Phase II windowed attention and centre-weighted merge
 * ([ai] Phase II).  For every final window W of the plan:
 *   O_W(q) = softmax(scale * q K_S^T) V_S,  S = ext(W) followed by G_W,
 * then O(q) = sum_W t_W(q) O_W(q) / sum_W t_W(q).
 *   q, k, v, o : [B, H, Hg*Wg, D] (dtype)
 *   cfg, plan  : the configuration and buffer given to area_window_plan
 *   ws         : workspace of ws_bytes >= area_window_attn_ws_bytes(),
 *                32-byte aligned; contents on entry are ignored, on exit
 *                unspecified.  The call resets its counter header (a memset
 *                on the stream) before the kernel.  With ws_bytes >=
 *                area_window_attn_ws_bytes() + area_window_attn_stage_bytes()
 *                the global-KV rows are staged first (faster, same result).
 * Merge order: a token covered by several windows is summed over them in a
 * fixed order (by the parity class of the base window, see the plan's ITEMS;
 * the units of one head run class by class), so the output is bit-identical
 * from run to run and in CUDA-graph replays.
 * Errors: AREA_EINVAL, AREA_EUNSUPPORTED (D, dtype), AREA_ENOSPACE.
 */
int area_window_attn(const void* q, const void* k, const void* v,
                     const area_plan_cfg* cfg, const void* plan,
                     size_t plan_bytes, void* o, void* ws, size_t ws_bytes,
                     int H, int D, float scale, int dtype,
                     cudaStream_t stream);

/*
 * area_window_attn_text -- area_window_attn with text tokens: every window's
 * key set is ext(W), then G_W, then all T text keys [B, H, T, D] (kt, vt).
 * The pages state that text tokens are never pooled and every query attends
 * to them in Phase I; applying the same to Phase II windows is this
 * library's reading.  The merge is unchanged.
 * Errors: as area_window_attn, and AREA_EINVAL for T < 0 or null kt/vt with
 * T > 0.
 */
int area_window_attn_text(const void* q, const void* k, const void* v,
                          const void* kt, const void* vt, int T,
                          const area_plan_cfg* cfg, const void* plan,
                          size_t plan_bytes, void* o, void* ws, size_t ws_bytes,
                          int H, int D, float scale, int dtype,
                          cudaStream_t stream);

/*
 * area_bridge_select -- the global-KV bridge as the pages describe it ([ai]
 * Phase II: R = (rho w)^2 tokens from the rest of the grid, selected by
 * their deviation from the global mean key and spread spatially, rho = 0.5).
 * Per (b, h), with K widened to fp32 and every operation round-to-nearest:
 *   mean_d = (in-order sum over 1024-token chunks of the in-order chunk
 *            sums of K[t, d]) * fl32(1/N);
 *   dev(t) = (((0 + e_0) + e_1) + ...), e_d = (K[t, d] - mean_d)^2;
 * the grid is cut into ry x rx cells (cell (cy, cx) holds rows
 * floor(cy Hg/ry) .. floor((cy+1) Hg/ry) - 1 and likewise for columns); each
 * cell contributes its token of largest dev, the lowest index among equals.
 * Choose ry, rx = round(rho * window side) per axis for R = (rho w)^2.
 *   k    : [B, H, Hg*Wg, D] (dtype), 16-byte aligned
 *   cand : int32 [B, H, ry*rx] output, cells row-major
 *   ws   : device scratch of ws_bytes >= area_bridge_select_ws_bytes(),
 *          16-byte aligned, owned by the caller; it holds the mean keys and
 *          the 1024-token chunk sums and needs no initial value
 * K is read twice (chunk sums, then deviations); three kernels on `stream`.
 * Errors: AREA_EINVAL, AREA_EUNSUPPORTED (D, N above 232448*256/D tokens, or
 * rx above 16384), AREA_ENOSPACE (ws too small).
 */
/*
 * area_bridge_select_ws_bytes -- scratch size of area_bridge_select:
 * B*H*D*(1 + ceil(Hg*Wg/1024))*4 bytes.  Errors: AREA_EINVAL (null output,
 * a size below 1), AREA_EUNSUPPORTED (Hg*Wg above 2^31 - 1).
 */
int area_bridge_select_ws_bytes(int B, int H, int Hg, int Wg, int D,
                                size_t* ws_bytes);

int area_bridge_select(const void* k, int dtype, int B, int H, int Hg, int Wg,
                       int D, int ry, int rx, int* cand, void* ws,
                       size_t ws_bytes, cudaStream_t stream);

/*
 * area_window_attn_bridge -- area_window_attn with the pages' bridge: the
 * global part of window W's key set, for head h, is the candidates of
 * area_bridge_select for (b, h) that lie outside ext(W), instead of the
 * plan's energy-ranked list (the plan's G is ignored; build it with G = 0).
 *   cand : int32 [B, H, R] from area_bridge_select (R = ry*rx)
 *   ws   : as area_window_attn; with ws_bytes >= area_window_attn_ws_bytes()
 *          + area_window_attn_bridge_stage_bytes() the bf16 tensor-core path
 *          first copies each head's candidate rows that fill whole 128-row
 *          tiles into it (one launch), and loads those tiles as tiles; the
 *          result is the same.
 * Errors: as area_window_attn, and AREA_EINVAL for null cand or R < 1.
 */
int area_window_attn_bridge_stage_bytes(int B, int H, int R, int D,
                                        size_t* stage_bytes);   /* 2 * B * H * R * D * 2 */
int area_window_attn_bridge(const void* q, const void* k, const void* v,
                            const int* cand, int R, const area_plan_cfg* cfg,
                            const void* plan, size_t plan_bytes, void* o,
                            void* ws, size_t ws_bytes, int H, int D,
                            float scale, int dtype, cudaStream_t stream);

/*
 * area_window_attn_noalloc -- area_window_attn for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is a library
 * convenience, not part of the method.
 *
 * Some callers cannot call cudaMalloc (or any allocating routine) at the
 * point where they run attention: code hosted by a runtime that owns every
 * device allocation and hands out only fixed input/output buffers, or a
 * serving loop that must not allocate once it has started.  Such a caller
 * still passes the inputs, the plan and the output, but not the fp32 merge
 * workspace: it lives in a static device array of 32 MiB inside the library,
 * which every GPU that loads libarea holds until the process exits.
 *
 *   Arguments: as area_window_attn, without ws / ws_bytes.
 *   Limit: the workspace area_window_attn would need,
 *          area_window_attn_ws_bytes(cfg, H, D), must not exceed 32 MiB;
 *          larger sizes return AREA_ENOSPACE before anything is launched.
 *   Set-up: the first call in a CUDA context (per device; again after
 *          cudaDeviceReset or under another context) looks up the array's
 *          device address with cudaGetSymbolAddress, with that device
 *          current; make that first call outside any stream capture.  It
 *          allocates nothing and calls no cudaMalloc / cudaFree.
 *   Sharing: all calls on a device use the same array.  It keeps the last
 *          call's contents; each call resets the counters at its start, and
 *          every accumulator row is written before it is read.  Calls that
 *          overlap on the GPU (other streams, other threads) race on it and
 *          must be serialised by the caller.
 * Errors: AREA_EINVAL, AREA_EUNSUPPORTED, AREA_ENOSPACE, AREA_ECUDA.
 */
int area_window_attn_noalloc(const void* q, const void* k, const void* v,
                             const area_plan_cfg* cfg, const void* plan,
                             size_t plan_bytes, void* o, int H, int D,
                             float scale, int dtype, cudaStream_t stream);

/*
 * area_test_plan_barrier_expiry -- TEST HOOK, not part of the method (the
 * pages have no counterpart).  Runs the one-launch detail map + planner of
 * area_dwt_window_plan (AREA_DETAIL_HH) with every grid-barrier target set
 * one above the number of blocks and each barrier wait bounded by 1 ms, so
 * the first barrier cannot complete.  Every block gives up after about 1 ms
 * and returns; the launch ends and the context stays usable.  A following
 * area_kernel_error reports AREA_KERR_PLAN_BARRIER (and clears it).  The
 * energy and plan buffers are left partly written: their contents are
 * unspecified.  Exists so that tests can drive the bounded-wait path of the
 * cooperative planner to expiry without a fault or a hang.
 *   Arguments: as area_dwt_window_plan, without the detail mode.
 * Errors: AREA_EINVAL, AREA_ENOSPACE, AREA_ECUDA.
 */
int area_test_plan_barrier_expiry(const void* src, int src_dtype, int C,
                                  float* energy, const area_plan_cfg* cfg,
                                  void* plan, size_t plan_bytes,
                                  cudaStream_t stream);

/* ---- schedule (host functions: no device memory, no stream) ------------ */

/*
 * area_pool_ramp -- Phase I pooling factor per step ([ai] Phase I: the factor
 * starts at f0 and ramps down linearly to the floor f_min, each value snapped
 * to a valid grid divisor; [blog] Fase I prints [4,4,4,4,2,2,2,2] for f0 = 4
 * over 8 steps at a 256 x 256 grid).  Step t's linear value
 * f0 + (f_min - f0) * t / (steps - 1) (double precision) goes to the nearest
 * factor that divides both Hg and Wg, the larger one on a tie.
 *   ramp : host int[steps] output.   Errors: AREA_EINVAL.
 */
int area_pool_ramp(int f0, int f_min, int steps, int Hg, int Wg, int* ramp);

/*
 * area_window_sides -- Phase II window side per step ([ai] Phase II: windows
 * shrink geometrically from w_start to w_min): w_t = w0 * (w_min / w0)^(t /
 * (steps - 1)) in double precision, rounded to the nearest multiple of 8
 * (halves up), at least 8.
 *   sides : host int[steps] output.   Errors: AREA_EINVAL.
 */
int area_window_sides(int w0, int w_min, int steps, int* sides);

/*
 * area_bridge_lattice -- cells per axis of the global-KV bridge for window
 * side w ([ai] Phase II: R = (rho w)^2 tokens, rho = 0.5): round(0.5 * side)
 * per axis of the window clipped to the grid, at least 1, at most the grid
 * side.  Outputs are host ints.   Errors: AREA_EINVAL.
 */
int area_bridge_lattice(int w, int Hg, int Wg, int* ry, int* rx);

/*
 * area_phase_switch -- number of Phase I steps for a sampler's noise levels
 * ([ai] "Scheduling the switch": Phase I ends at a noise level sigma*, not at
 * a step count; [wiki] usage notes: sigma* between 0.86 and 0.96 for the
 * tuned models).  Phase I is the leading run of steps with
 * sigmas[t] >= sigma_star (fp32 comparison); every later step is Phase II.
 *   sigmas : host float[steps], the sampler's noise level at each step.
 * Errors: AREA_EINVAL.
 */
int area_phase_switch(const float* sigmas, int steps, float sigma_star,
                      int* n_phase1);

/*
 * area_schedule -- the whole AReA schedule of a sampling run: the phase
 * switch above, the pooling ramp f0 -> f_min over the Phase I steps and the
 * window sides w0 -> w_min over the Phase II steps.
 *   kind  : host int[steps] output, AREA_PHASE_COARSE or AREA_PHASE_WINDOW;
 *   param : host int[steps] output, the pooling factor f (Phase I) or the
 *           window side w (Phase II) of each step.
 * The step calls are then area_pool_kv + area_coarse_attn (Phase I) and
 * area_dwt_detail + area_window_plan + area_window_attn (Phase II), all
 * asynchronous on one stream, so a whole schedule can be captured in one
 * CUDA graph.   Errors: AREA_EINVAL.
 */
int area_schedule(const float* sigmas, int steps, float sigma_star, int f0,
                  int f_min, int w0, int w_min, int Hg, int Wg, int* kind,
                  int* param);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* AREA_H_ */
