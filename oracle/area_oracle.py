"""CPU oracle for the AReA attention hot path.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously correct
statement of what the hot path computes.  Only the test-suite, the smoke check
of ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it;
the library and its Python binding never do, and it shares no code with them.

Source of every definition: AReA, "Adaptive Receptive-Field Attention for
Efficient High-Resolution Diffusion Transformers" (arXiv 2610.17227), as
summarised on
  [blog]  gpt-diffusion.com, "AReA: atencion training-free ...", section
          "Las dos fases de AReA" (Fase I / Fase II) and the README notes in
          "Como entra en tu pipeline";
  [ai]    ai.info paper summary, section "Methodology in Plain English"
          (paragraphs "Phase I", "Phase II", "Scheduling the switch");
  [wiki]  github.com/KooroshRH/AReA/wiki (method overview, canvas rules).
The pages give no formulas.  Where they are silent the plainest reading is
taken; every such reading is listed in the design notes and repeated in the
docstring of the function that makes it.

Precision: attention and pooling in float64; the DWT detail map and the
window plan in float32 with a fixed operation order and no fused
multiply-add, so that index lists and split decisions are reproducible bit
for bit.

Pins: each public function is checked by ``tests/test_oracle_*.py`` against
closed forms, brute force, library routines or values the pages print.  No
function here is "parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

F32 = np.float32


# ----------------------------------------------------------------------------
# Phase I: K/V pooling over f x f token blocks
# ----------------------------------------------------------------------------

def pool_kv(x: np.ndarray, Hg: int, Wg: int, f: int, mode: str = "mean") -> np.ndarray:
    """One representative K (or V) token per f x f block of the token grid.

    [blog] Fase I and [ai] Phase I: keys and values keep one token per f x f
    block, placed on a (W/f) x (H/f) grid.  Representative: ``mean`` (block
    average) or ``center`` (token (py*f + f//2, px*f + f//2); the pages name
    the block centre as their default but give no rule for even f, the
    floor(f/2) offset is a reading).

    x: [B, H, Hg*Wg, D]; returns float64 [B, H, (Hg/f)*(Wg/f), D] with pooled
    token index py*(Wg/f) + px.
    """
    B, H, N, D = x.shape
    if N != Hg * Wg or Hg % f or Wg % f:
        raise ValueError("grid must divide into whole f x f blocks")
    xb = np.asarray(x, dtype=np.float64).reshape(B, H, Hg // f, f, Wg // f, f, D)
    if mode == "mean":
        out = xb.mean(axis=(3, 5))
    elif mode == "center":
        c = f // 2
        out = xb[:, :, :, c, :, c, :]
    else:
        raise ValueError(mode)
    return out.reshape(B, H, (Hg // f) * (Wg // f), D)


# ----------------------------------------------------------------------------
# Attention by its definition (coarse, full and per-window)
# ----------------------------------------------------------------------------

def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * q k^T) v over the last two axes, in float64.

    q: [..., Nq, D], k and v: [..., Nk, D].  The row maximum is subtracted
    before exp (an identity of softmax).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = scale * np.matmul(q, np.swapaxes(k, -1, -2))
    s -= s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=-1, keepdims=True)
    return np.matmul(p, v)


def coarse_attn(q, kp, vp, scale, rows: Optional[np.ndarray] = None,
                kt: Optional[np.ndarray] = None, vt: Optional[np.ndarray] = None) -> np.ndarray:
    """Phase I cross-scale coarse attention ([blog] Fase I, [ai] Phase I).

    Every full-resolution query attends to all pooled keys and, when given,
    to all T text keys, which are never pooled: T + N/f^2 keys per query.
    q: [B, H, N, D]; kp, vp: [B, H, Nk, D]; kt, vt: [B, H, T, D].  ``rows``
    (optional) restricts the computation to those query indices.
    """
    if rows is not None:
        q = np.asarray(q)[:, :, rows, :]
    B, H = q.shape[:2]
    out = np.empty(q.shape, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            kk, vv = kp[b, h], vp[b, h]
            if kt is not None:
                kk = np.concatenate([np.asarray(kk), np.asarray(kt[b, h])])
                vv = np.concatenate([np.asarray(vv), np.asarray(vt[b, h])])
            out[b, h] = attention(q[b, h], kk, vv, scale)
    return out


def full_attn(q, k, v, scale, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """Full global self-attention over all N tokens: the operation AReA replaces."""
    return coarse_attn(q, k, v, scale, rows)


def pool_ramp(f0: int, f_min: int, steps: int, Hg: int, Wg: int) -> List[int]:
    """Phase I pooling-factor ramp: linear f0 -> f_min, snapped to valid divisors.

    [ai] Phase I: the factor starts at f0 and ramps down linearly to f_min,
    each value snapped to a valid grid divisor.  Reading: the linear value
    f0 + (f_min - f0) * t / (steps - 1) is snapped to the nearest f that
    divides both Hg and Wg (ties to the larger f).
    """
    divs = [d for d in range(1, max(Hg, Wg) + 1) if Hg % d == 0 and Wg % d == 0]
    out = []
    for t in range(steps):
        lin = f0 + (f_min - f0) * (t / (steps - 1) if steps > 1 else 0.0)
        best = min(divs, key=lambda d: (abs(d - lin), -d))
        out.append(int(best))
    return out


def window_sides(w0: int, w_min: int, steps: int) -> List[int]:
    """Phase II window side per step ([ai] Phase II: windows shrink
    geometrically from w_start to w_min).  Reading: the geometric sequence
    w0 * (w_min / w0)^(t / (steps - 1)), each value rounded to the nearest
    multiple of 8 (halves up), at least 8."""
    out = []
    for t in range(steps):
        e = t / (steps - 1) if steps > 1 else 0.0
        w = w0 * (w_min / w0) ** e
        out.append(max(8, 8 * int(math.floor(w / 8 + 0.5))))
    return out


def phase_switch(sigmas: Sequence[float], sigma_star: float) -> int:
    """Number of Phase I steps ([ai] "Scheduling the switch": the transition
    is a noise level sigma*, not a step count).  Reading: Phase I is the
    leading run of steps whose noise level is at least sigma* (compared in
    float32); every later step is Phase II."""
    star = np.float32(sigma_star)
    n = 0
    for sg in sigmas:
        if np.float32(sg) >= star:
            n += 1
        else:
            break
    return n


def phase_schedule(sigmas: Sequence[float], sigma_star: float, f0: int, f_min: int,
                   w0: int, w_min: int, Hg: int, Wg: int) -> List[Tuple[str, int]]:
    """The schedule of a sampling run: ("coarse", f) for each Phase I step
    (the pooling ramp over those steps), then ("window", w) for each Phase II
    step (the shrinking window sides over those steps)."""
    n1 = phase_switch(sigmas, sigma_star)
    n2 = len(sigmas) - n1
    out = [("coarse", f) for f in (pool_ramp(f0, f_min, n1, Hg, Wg) if n1 else [])]
    out += [("window", w) for w in (window_sides(w0, w_min, n2) if n2 else [])]
    return out


# ----------------------------------------------------------------------------
# Phase II: Haar DWT detail map
# ----------------------------------------------------------------------------

def dwt_detail(src: np.ndarray, Hg: int, Wg: int, mode: str = "hh") -> np.ndarray:
    """Per-2x2-cell Haar detail energy of the hidden states ([ai] Phase II).

    The pages say only that a DWT map computed from the current hidden states
    measures fine detail.  Reading: one level of the 2-D Haar transform per
    channel on each 2x2 cell (a b / c d), in float32 with no fused
    multiply-add:
        HH = ((a - b) - (c - d)) * 0.5
        LH = ((a + b) - (c + d)) * 0.5,  HL = ((a - b) + (c - d)) * 0.5
    mode "hh":   e_c = HH^2
    mode "all3": e_c = (LH^2 + HL^2) + HH^2
    E = (((0 + e_0) + e_1) + ... + e_{C-1}) * (1/C), summed in channel order,
    with 1/C the correctly rounded float32 reciprocal.

    src: [B, Hg*Wg, C] (values widened exactly to float32).
    Returns float32 [B, Hg/2, Wg/2].
    """
    B, N, C = src.shape
    if N != Hg * Wg or Hg % 2 or Wg % 2:
        raise ValueError("grid sides must be even")
    x = np.asarray(src, dtype=F32).reshape(B, Hg // 2, 2, Wg // 2, 2, C)
    a = x[:, :, 0, :, 0, :]
    b = x[:, :, 0, :, 1, :]
    c = x[:, :, 1, :, 0, :]
    d = x[:, :, 1, :, 1, :]
    half = F32(0.5)
    hh = ((a - b) - (c - d)) * half
    if mode == "hh":
        e = hh * hh
    elif mode == "all3":
        lh = ((a + b) - (c + d)) * half
        hl = ((a - b) + (c - d)) * half
        e = (lh * lh + hl * hl) + hh * hh
    else:
        raise ValueError(mode)
    acc = np.zeros(e.shape[:-1], dtype=F32)
    for ch in range(C):
        acc = acc + e[..., ch]
    inv = F32(1) / F32(C)
    return (acc * inv).astype(F32)


def token_energy(E: np.ndarray) -> np.ndarray:
    """Per-token energy: each token takes the energy of its 2x2 cell.  [Hg, Wg]."""
    return np.repeat(np.repeat(np.asarray(E, dtype=F32), 2, axis=0), 2, axis=1)


# ----------------------------------------------------------------------------
# Phase II: window plan
# ----------------------------------------------------------------------------

def tile_starts(L: int, w: int) -> Tuple[List[int], int]:
    """Evenly spaced window starts along one axis of length L.

    [ai] Phase II: the grid is covered by a base tiling spaced evenly so the
    overlap is shared equally.  Reading: side w_e = min(w, L), count
    n = ceil(L / w_e), start_i = floor(i * (L - w_e) / (n - 1)) (0 when n = 1).
    """
    we = min(w, L)
    n = -(-L // we)
    if n == 1:
        return [0], we
    return [(i * (L - we)) // (n - 1) for i in range(n)], we


# ----------------------------------------------------------------------------
# Seeded randomness: border jitter and Halo widths
# ----------------------------------------------------------------------------

_GAMMA = 0x9E3779B97F4A7C15
_M64 = (1 << 64) - 1
STREAM_JITTER, STREAM_HALO = 1, 2


def splitmix64(state: int) -> int:
    """One SplitMix64 step (Steele, Lea and Flood, "Fast splittable pseudorandom
    number generators", OOPSLA 2014; finaliser constants of Vigna's reference
    version): advance the state by the golden-ratio increment, then mix."""
    z = (state + _GAMMA) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def counter_random(seed: int, stream: int, index: int) -> int:
    """Counter-based 64-bit draw: output number (stream * 2^32 + index) of the
    SplitMix64 sequence seeded with `seed` (stream 0, index 0 is its first
    output)."""
    return splitmix64((seed + _GAMMA * ((stream << 32) + index)) & _M64)


def jitter_shifts(seed: int, Hg: int, Wg: int, w: int) -> Tuple[int, int]:
    """Border shift (sy, sx) of one plan ([ai] Phase II: window boundaries are
    randomly shifted across steps so seams never form at fixed places).
    Reading: s in [0, w_e) per axis, drawn from the seed; 0 when the window
    spans the axis or the seed is 0."""
    if seed == 0:
        return 0, 0
    hy, wx = min(w, Hg), min(w, Wg)
    sy = counter_random(seed, STREAM_JITTER, 0) % hy if hy < Hg else 0
    sx = counter_random(seed, STREAM_JITTER, 1) % wx if wx < Wg else 0
    return sy, sx


def tile_windows(L: int, w: int, shift: int = 0) -> List[Tuple[int, int]]:
    """(start, size) of the base windows along one axis.

    Reading of the border shift: the even tiling (tile_starts) of the extended
    axis [-shift, L) with side w_e = min(w, L), clipped back to [0, L).
    shift = 0 gives tile_starts exactly."""
    we = min(w, L)
    starts, _ = tile_starts(L + shift, we)
    out = []
    for s0 in starts:
        a = s0 - shift
        lo, hi = max(0, a), min(L, a + we)
        out.append((lo, hi - lo))
    return out


def halo_width(seed: int, halo: int, b: int, i: int) -> int:
    """Halo width of final window i of batch element b: fixed `halo` when the
    seed is 0, else a draw in [0, halo] ([blog] README notes: the seed sets
    the Halo widths, up to delta_max)."""
    if seed == 0:
        return halo
    return counter_random(seed, STREAM_HALO, (b << 20) + i) % (halo + 1)


def window_score(Etok: np.ndarray, y0: int, x0: int, hy: int, wx: int) -> np.float32:
    """Sum of token energies over a window, in a fixed float32 order.

    Row sums r_y are accumulated left to right, then the r_y top to bottom.
    """
    sub = np.asarray(Etok[y0:y0 + hy, x0:x0 + wx], dtype=F32)
    r = np.zeros(hy, dtype=F32)
    for x in range(wx):
        r = r + sub[:, x]
    s = F32(0)
    for y in range(hy):
        s = F32(s + r[y])
    return s


def split_threshold(thr: float, hy: int, wx: int) -> np.float32:
    """Split bound fl32(fl32(thr) * area): windows scoring strictly below it split."""
    return F32(F32(thr) * F32(hy * wx))


def quadrants(y0: int, x0: int, hy: int, wx: int):
    """Four quadrants TL, TR, BL, BR; top/left halves take floor(side/2)."""
    ht, wl = hy // 2, wx // 2
    return [(y0, x0, ht, wl), (y0, x0 + wl, ht, wx - wl),
            (y0 + ht, x0, hy - ht, wl), (y0 + ht, x0 + wl, hy - ht, wx - wl)]


def halo_rect(y0, x0, hy, wx, h, Hg, Wg):
    """Halo-extended rectangle clipped to the grid: (ey0, ex0, ehy, ewx).

    [ai] Phase II / [blog] Fase II: each window's keys and values are
    extended by a ring of neighbouring tokens across its border (fixed
    width h here; the pages draw it at random up to 8).
    """
    ey0, ex0 = max(0, y0 - h), max(0, x0 - h)
    ey1, ex1 = min(Hg, y0 + hy + h), min(Wg, x0 + wx + h)
    return ey0, ex0, ey1 - ey0, ex1 - ex0


def tent_weight(y: int, x: int, y0: int, x0: int, hy: int, wx: int) -> int:
    """Centre-weighted blending weight of a token inside a window (integer tent).

    [ai] Phase II: overlapping window outputs are blended with centre-weighted
    averaging.  Reading: t = min(y-y0+1, y0+hy-y) * min(x-x0+1, x0+wx-x).
    """
    return min(y - y0 + 1, y0 + hy - y) * min(x - x0 + 1, x0 + wx - x)


def global_rank(Etok: np.ndarray) -> np.ndarray:
    """All token indices ordered by (energy descending, index ascending)."""
    e = np.asarray(Etok, dtype=F32).reshape(-1)
    idx = np.arange(e.size)
    return np.lexsort((idx, -e))


@dataclass
class Plan:
    """Window plan of one batch element."""
    Hg: int
    Wg: int
    w: int
    halo: int
    G: int
    base: np.ndarray        # int32 [n_base, 4]  (y0, x0, hy, wx)
    score: np.ndarray       # float32 [n_base]  split score (sum of token energy)
    split: np.ndarray       # uint8 [n_base]
    windows: np.ndarray     # int32 [n_win, 4]  final windows
    parent: np.ndarray      # int32 [n_win]     base window of each final window
    ext: np.ndarray         # int32 [n_win, 4]  (ey0, ex0, ehy, ewx)
    gcount: np.ndarray      # int32 [n_win]
    gidx: np.ndarray        # int32 [n_win, G], -1 padded
    wsum: np.ndarray        # float32 [Hg*Wg]   sum of tent weights per token


def window_plan(E: np.ndarray, Hg: int, Wg: int, w: int, halo: int, G: int,
                thr: float, seed: int = 0, b: int = 0) -> Plan:
    """Phase II plan of one batch element from its detail map E [Hg/2, Wg/2].

    Steps in the pages' order ([ai] Phase II, [blog] Fase II):
      1. base tiling (tile_windows per axis, shifted by jitter_shifts(seed);
         windows row-major, y then x);
      2. detail score per base window (window_score);
      3. windows over smooth regions (score < split_threshold) are split
         into four quadrants (one level; sides < 2 never split);
      4. Halo rectangle per final window (halo_rect; width halo_width(seed));
      5. global-KV bridge: the first G_W = min(G, N - |ext|) tokens of
         global_rank that lie outside the Halo rectangle, in rank order (the
         pages select by deviation from the global mean key; the rule used
         here, top-G by detail energy, is the configured reading);
      6. per-token sum of tent weights over the final windows.
    """
    Etok = token_energy(E)
    assert Etok.shape == (Hg, Wg)
    sy, sx = jitter_shifts(seed, Hg, Wg, w)
    ywin = tile_windows(Hg, w, sy)
    xwin = tile_windows(Wg, w, sx)
    base, score, split, wins, parent = [], [], [], [], []
    for (y0, hy) in ywin:
        for (x0, wx) in xwin:
            bi = len(base)
            base.append((y0, x0, hy, wx))
            s = window_score(Etok, y0, x0, hy, wx)
            score.append(s)
            do_split = hy >= 2 and wx >= 2 and s < split_threshold(thr, hy, wx)
            split.append(1 if do_split else 0)
            if do_split:
                for qd in quadrants(y0, x0, hy, wx):
                    wins.append(qd)
                    parent.append(bi)
            else:
                wins.append((y0, x0, hy, wx))
                parent.append(bi)
    N = Hg * Wg
    order = global_rank(Etok)
    oy, ox = order // Wg, order % Wg
    ext, gcount = [], []
    gidx = np.full((len(wins), G), -1, dtype=np.int32)
    wsum = np.zeros((Hg, Wg), dtype=F32)
    for i, (y0, x0, h_, w_) in enumerate(wins):
        e = halo_rect(y0, x0, h_, w_, halo_width(seed, halo, b, i), Hg, Wg)
        ext.append(e)
        ey0, ex0, ehy, ewx = e
        gw = min(G, N - ehy * ewx)
        outside = ~((oy >= ey0) & (oy < ey0 + ehy) & (ox >= ex0) & (ox < ex0 + ewx))
        sel = order[outside][:gw]
        gidx[i, :gw] = sel
        gcount.append(gw)
        yy = np.arange(y0, y0 + h_)[:, None]
        xx = np.arange(x0, x0 + w_)[None, :]
        t = np.minimum(yy - y0 + 1, y0 + h_ - yy) * np.minimum(xx - x0 + 1, x0 + w_ - xx)
        wsum[y0:y0 + h_, x0:x0 + w_] += t.astype(F32)
    return Plan(Hg=Hg, Wg=Wg, w=w, halo=halo, G=G,
                base=np.array(base, dtype=np.int32).reshape(-1, 4),
                score=np.array(score, dtype=F32),
                split=np.array(split, dtype=np.uint8),
                windows=np.array(wins, dtype=np.int32).reshape(-1, 4),
                parent=np.array(parent, dtype=np.int32),
                ext=np.array(ext, dtype=np.int32).reshape(-1, 4),
                gcount=np.array(gcount, dtype=np.int32),
                gidx=gidx,
                wsum=wsum.reshape(-1))


# ----------------------------------------------------------------------------
# The pages' global-KV bridge: distinctive keys by deviation, spread spatially
# ----------------------------------------------------------------------------

BRIDGE_CHUNK = 1024


def bridge_lattice(w: int, Hg: int, Wg: int, rho: float = 0.5) -> Tuple[int, int]:
    """Cells per axis of the bridge lattice: R = (rho * w)^2 tokens per window
    ([ai] Phase II, rho = 0.5).  Reading: r = round(rho * side) per axis of
    the (clipped) window, at least 1 and at most the grid side."""
    hy, wx = min(w, Hg), min(w, Wg)
    ry = min(Hg, max(1, int(math.floor(rho * hy + 0.5))))
    rx = min(Wg, max(1, int(math.floor(rho * wx + 0.5))))
    return ry, rx


def key_deviation(k: np.ndarray) -> np.ndarray:
    """Squared deviation of every key from the mean key of its head, float32.

    k: [N, D] (storage values).  Mean: per dimension, tokens summed in order
    within chunks of 1024, the chunk sums added in order, times the float32
    reciprocal of N.  dev(t) = (((0 + e_0) + e_1) + ...) over dimensions with
    e_d = (k[t, d] - mean_d)^2; float32, no fused multiply-add."""
    k = np.asarray(k, dtype=F32)
    N, D = k.shape
    total = np.zeros(D, dtype=F32)
    for c0 in range(0, N, BRIDGE_CHUNK):
        part = np.zeros(D, dtype=F32)
        for t in range(c0, min(N, c0 + BRIDGE_CHUNK)):
            part = part + k[t]
        total = total + part
    mean = total * (F32(1) / F32(N))
    dev = np.zeros(N, dtype=F32)
    for d in range(D):
        e = k[:, d] - mean[d]
        dev = dev + e * e
    return dev


def bridge_candidates(k: np.ndarray, Hg: int, Wg: int, ry: int, rx: int) -> np.ndarray:
    """Distinctive tokens of one head ([ai] Phase II: drawn from the rest of
    the grid, selected by their deviation from the global mean key and spread
    spatially).  Reading: the grid is cut into ry x rx cells (cell (cy, cx)
    holds rows floor(cy*Hg/ry) .. floor((cy+1)*Hg/ry) - 1 and likewise for
    columns); each cell gives its token of largest key_deviation, the lowest
    token index among equals.  Returns int32 [ry * rx], cells row-major."""
    dev = key_deviation(k).reshape(Hg, Wg)
    out = np.empty(ry * rx, dtype=np.int32)
    for cy in range(ry):
        y0, y1 = (cy * Hg) // ry, ((cy + 1) * Hg) // ry
        for cx in range(rx):
            x0, x1 = (cx * Wg) // rx, ((cx + 1) * Wg) // rx
            best, bt = None, -1
            for y in range(y0, y1):
                for x in range(x0, x1):
                    v = dev[y, x]
                    if best is None or v > best:
                        best, bt = v, y * Wg + x
            out[cy * rx + cx] = bt
    return out


def bridge_window_tokens(cand: np.ndarray, ext_rect, Wg: int) -> np.ndarray:
    """The bridge keys of one window: the candidates outside its Halo rectangle."""
    ey0, ex0, ehy, ewx = (int(v) for v in ext_rect)
    cy, cx = cand // Wg, cand % Wg
    inside = (cy >= ey0) & (cy < ey0 + ehy) & (cx >= ex0) & (cx < ex0 + ewx)
    return cand[~inside].astype(np.int64)


def window_tokens(rect, Wg: int) -> np.ndarray:
    """Token indices of a rectangle (y0, x0, hy, wx), row-major."""
    y0, x0, hy, wx = (int(v) for v in rect)
    yy = np.arange(y0, y0 + hy)[:, None]
    xx = np.arange(x0, x0 + wx)[None, :]
    return (yy * Wg + xx).reshape(-1)


def window_kv_tokens(plan: Plan, i: int) -> np.ndarray:
    """Key/value token set of final window i: Halo rectangle then global list."""
    ext = window_tokens(plan.ext[i], plan.Wg)
    g = plan.gidx[i, : plan.gcount[i]]
    return np.concatenate([ext, g.astype(np.int64)])


def window_attn(q, k, v, plans: Sequence[Plan], scale: float,
                rows: Optional[np.ndarray] = None, heads: Optional[Sequence[int]] = None,
                kt: Optional[np.ndarray] = None, vt: Optional[np.ndarray] = None,
                bridge: Optional[np.ndarray] = None) -> np.ndarray:
    """Phase II windowed attention with centre-weighted merge ([ai] Phase II).

    For each final window W: O_W(q) = softmax(scale * q K_S^T) V_S over
    S = ext(W) u G_W (u the T text keys when kt, vt [B, H, T, D] are given:
    the pages keep text keys unpooled and visible to every query in Phase I;
    keeping them in every window is the reading taken for Phase II); then
    O(q) = sum_W t_W(q) O_W(q) / sum_W t_W(q), over the windows that contain
    q.  q, k, v: [B, H, N, D]; plans: one per batch element.  ``rows``
    restricts the output to those token indices and ``heads`` to those heads;
    the result is [B, len(heads), len(rows), D].
    """
    B, H, N, D = q.shape
    heads = list(range(H)) if heads is None else list(heads)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    pos = np.full(N, -1, dtype=np.int64)
    pos[rows] = np.arange(rows.size)
    out = np.zeros((B, len(heads), rows.size, D), dtype=np.float64)
    for b in range(B):
        plan = plans[b]
        for i in range(plan.windows.shape[0]):
            y0, x0, hy, wx = (int(t) for t in plan.windows[i])
            toks = window_tokens(plan.windows[i], plan.Wg)
            keep = pos[toks] >= 0
            if not keep.any():
                continue
            toks = toks[keep]
            ty, tx = toks // plan.Wg, toks % plan.Wg
            t = (np.minimum(ty - y0 + 1, y0 + hy - ty) *
                 np.minimum(tx - x0 + 1, x0 + wx - tx)).astype(np.float64)
            kv = window_kv_tokens(plan, i)
            for hi, h in enumerate(heads):
                if bridge is not None:
                    kv = np.concatenate([window_tokens(plan.ext[i], plan.Wg),
                                         bridge_window_tokens(bridge[b, h], plan.ext[i], plan.Wg)])
                kk, vv = k[b, h][kv], v[b, h][kv]
                if kt is not None:
                    kk = np.concatenate([kk, np.asarray(kt[b, h])])
                    vv = np.concatenate([vv, np.asarray(vt[b, h])])
                o = attention(q[b, h][toks], kk, vv, scale)
                out[b, hi, pos[toks]] += t[:, None] * o
        ws = plan.wsum.astype(np.float64)[rows]
        out[b] /= ws[None, :, None]
    return out
