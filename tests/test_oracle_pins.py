"""Pins of the CPU oracle against things other than itself.

Each test checks one oracle function against a closed form, a brute-force
restatement on a tiny input, a library routine, or a value the AReA pages
print.  The cases are chosen so that a plausible slip (a dropped term, a sign,
a transposed operand, a wrong block index, a wrong tie-break) fails one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import area_oracle as ora
from workloads import CONFIGS, flow_sigmas, make_detail_source, texture_mask

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


# --------------------------------------------------------------------------
# pooling
# --------------------------------------------------------------------------

@pytest.mark.parametrize("f", [1, 2, 3, 4])
def test_pool_mean_matches_avg_pool2d(f):
    rng = np.random.default_rng(11)
    Hg, Wg, D = 12, 24, 5
    x = rng.standard_normal((2, 3, Hg * Wg, D))
    got = ora.pool_kv(x, Hg, Wg, f, "mean")
    t = torch.from_numpy(x).reshape(2 * 3, Hg, Wg, D).permute(0, 3, 1, 2)
    ref = torch.nn.functional.avg_pool2d(t, f).permute(0, 2, 3, 1).reshape(2, 3, -1, D)
    np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-13)


def test_pool_identity_at_f1():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 2, 6 * 8, 4))
    assert np.array_equal(ora.pool_kv(x, 6, 8, 1, "mean"), x)
    assert np.array_equal(ora.pool_kv(x, 6, 8, 1, "center"), x)


def test_pool_mean_of_linear_field_is_block_centroid():
    # value = 3*y + 5*x  ->  block mean = value at the block centroid
    Hg, Wg, f = 12, 18, 3
    yy, xx = np.meshgrid(np.arange(Hg), np.arange(Wg), indexing="ij")
    x = (3.0 * yy + 5.0 * xx).reshape(1, 1, -1, 1)
    got = ora.pool_kv(x, Hg, Wg, f).reshape(Hg // f, Wg // f)
    cy = np.arange(Hg // f) * f + (f - 1) / 2
    cx = np.arange(Wg // f) * f + (f - 1) / 2
    np.testing.assert_allclose(got, 3.0 * cy[:, None] + 5.0 * cx[None, :], atol=1e-12)


def test_pool_center_picks_floor_half_offset():
    Hg, Wg, f = 8, 12, 4
    x = np.arange(Hg * Wg, dtype=np.float64).reshape(1, 1, -1, 1)
    got = ora.pool_kv(x, Hg, Wg, f, "center").reshape(-1)
    want = [(py * f + 2) * Wg + (px * f + 2) for py in range(Hg // f) for px in range(Wg // f)]
    assert got.tolist() == want


def test_pool_rejects_non_dividing_factor():
    with pytest.raises(ValueError):
        ora.pool_kv(np.zeros((1, 1, 30, 2)), 5, 6, 2)


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def test_attention_matches_sdpa_float64():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 3, 17, 8))
    k = rng.standard_normal((2, 3, 29, 8))
    v = rng.standard_normal((2, 3, 29, 8))
    got = ora.attention(q, k, v, 0.37)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), scale=0.37)
    np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


def test_attention_brute_force_loops():
    rng = np.random.default_rng(4)
    nq, nk, d, s = 3, 5, 4, 0.5
    q = rng.standard_normal((nq, d))
    k = rng.standard_normal((nk, d))
    v = rng.standard_normal((nk, 2))
    got = ora.attention(q, k, v, s)
    for i in range(nq):
        logits = [s * sum(q[i, c] * k[j, c] for c in range(d)) for j in range(nk)]
        z = sum(math.exp(t) for t in logits)
        for c in range(2):
            want = sum(math.exp(logits[j]) / z * v[j, c] for j in range(nk))
            assert abs(got[i, c] - want) < 1e-12


def test_attention_identical_keys_average_values():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((4, 6))
    k = np.tile(rng.standard_normal((1, 6)), (7, 1))
    v = rng.standard_normal((7, 3))
    np.testing.assert_allclose(ora.attention(q, k, v, 1.0), np.tile(v.mean(0), (4, 1)), atol=1e-13)


def test_coarse_equals_full_for_block_constant_kv():
    # Pages: each query sees the whole image at 1/f^2 of the cost.  When K/V are
    # constant inside every f x f block the pooled keys carry each value with
    # multiplicity f^2, which cancels in the softmax: pooled == full attention.
    rng = np.random.default_rng(6)
    Hg, Wg, f, D = 8, 12, 2, 6
    kc = rng.standard_normal((1, 2, Hg // f, Wg // f, D))
    vc = rng.standard_normal((1, 2, Hg // f, Wg // f, D))
    up = lambda a: np.repeat(np.repeat(a, f, axis=2), f, axis=3).reshape(1, 2, Hg * Wg, D)
    k, v = up(kc), up(vc)
    q = rng.standard_normal((1, 2, Hg * Wg, D))
    kp, vp = ora.pool_kv(k, Hg, Wg, f), ora.pool_kv(v, Hg, Wg, f)
    assert kp.shape[2] == Hg * Wg // (f * f)       # N / f^2 keys
    np.testing.assert_allclose(ora.coarse_attn(q, kp, vp, 0.4), ora.full_attn(q, k, v, 0.4),
                               atol=1e-12)


def test_coarse_with_f1_is_full_attention():
    rng = np.random.default_rng(7)
    q, k, v = (rng.standard_normal((1, 1, 36, 4)) for _ in range(3))
    kp, vp = ora.pool_kv(k, 6, 6, 1), ora.pool_kv(v, 6, 6, 1)
    np.testing.assert_allclose(ora.coarse_attn(q, kp, vp, 0.5), ora.full_attn(q, k, v, 0.5), atol=0)


def test_coarse_rows_subset():
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((1, 2, 20, 4)) for _ in range(3))
    rows = np.array([0, 7, 19])
    full = ora.coarse_attn(q, k, v, 0.3)
    np.testing.assert_allclose(ora.coarse_attn(q, k, v, 0.3, rows=rows), full[:, :, rows], atol=0)


def test_pool_ramp_reproduces_printed_example():
    g = _golden("ramp_flux4096.json")
    assert ora.pool_ramp(g["f0"], g["f_min"], g["steps"], g["Hg"], g["Wg"]) == g["ramp"]
    assert [g["Hg"] // g["f0"], g["Wg"] // g["f0"]] == g["pooled_grid_at_f0"]


def test_phase_switch_reproduces_the_flux_split():
    # a sampler whose noise level crosses the pages' sigma* range between
    # steps 8 and 9 gives the 8 Phase I steps the pages state for FLUX.1
    g = _golden("phase_switch_flux.json")
    sig = flow_sigmas(g["steps"], 3.0)
    lo, hi = g["sigma_star_range"]
    n = g["phase1_steps"]
    assert lo <= sig[n] < sig[n - 1] <= hi
    for star in (float(sig[n]) + 1e-4, 0.5 * float(sig[n] + sig[n - 1]), float(sig[n - 1])):
        assert ora.phase_switch(sig, star) == n
    assert ora.phase_switch(sig, 1.5) == 0 and ora.phase_switch(sig, 0.0) == g["steps"]


def test_phase_switch_is_the_leading_run():
    # invariant on arbitrary (also non-monotone) lists: every step before the
    # switch is at or above sigma*, the step at the switch is below it
    rng = np.random.default_rng(7)
    for _ in range(200):
        sig = rng.random(rng.integers(1, 12)).astype(np.float32)
        star = float(rng.random())
        n = ora.phase_switch(sig, star)
        assert all(sig[:n] >= np.float32(star))
        assert n == len(sig) or sig[n] < np.float32(star)
    # a later step above sigma* does not re-enter Phase I
    assert ora.phase_switch([0.99, 0.5, 0.99], 0.9) == 1


def test_window_sides_reproduce_the_config_tables():
    # the configs' 8-step tables (integers) follow the geometric shrink
    assert ora.window_sides(64, 32, 8) == list(CONFIGS["flux2048"].schedule)
    assert ora.window_sides(256, 64, 8) == list(CONFIGS["flux4096"].schedule)
    assert ora.window_sides(192, 64, 8) == list(CONFIGS["flux6144"].schedule)
    assert ora.window_sides(272, 64, 8) == list(CONFIGS["qwen6144x2048"].schedule)


def test_window_sides_are_geometric_up_to_rounding():
    for w0, wm, n in [(192, 64, 20), (256, 64, 20), (272, 64, 40), (96, 96, 5), (64, 32, 1)]:
        ws = ora.window_sides(w0, wm, n)
        assert len(ws) == n and ws[0] == w0 and (n == 1 or ws[-1] == wm)
        assert all(a >= b for a, b in zip(ws, ws[1:]))
        assert all(w % 8 == 0 for w in ws)
        for t, w in enumerate(ws):
            exact = w0 * (wm / w0) ** (t / (n - 1) if n > 1 else 0.0)
            assert abs(w - exact) <= 4.0


def test_phase_schedule_concatenates_ramp_and_windows():
    g = _golden("ramp_flux4096.json")
    sig = flow_sigmas(28, 3.0)
    sched = ora.phase_schedule(sig, 0.89, g["f0"], g["f_min"], 256, 64, g["Hg"], g["Wg"])
    assert [p for k, p in sched if k == "coarse"] == g["ramp"]           # printed ramp
    wins = [p for k, p in sched if k == "window"]
    assert len(wins) == 20 and wins[0] == 256 and wins[-1] == 64
    assert [k for k, _ in sched] == ["coarse"] * 8 + ["window"] * 20


# --------------------------------------------------------------------------
# DWT detail map
# --------------------------------------------------------------------------

def _haar2x2(cell):
    # 2-D Haar of one 2x2 cell via the Kronecker product of 1-D Haar matrices
    h = np.array([[1.0, 1.0], [1.0, -1.0]]) / math.sqrt(2.0)
    c = h @ np.asarray(cell, dtype=np.float64) @ h.T     # [[LL, HL], [LH, HH]]
    return c[1, 0], c[0, 1], c[1, 1]                      # LH, HL, HH


def test_dwt_golden_cells():
    for case in _golden("haar_cell.json")["cases"]:
        cell = np.asarray(case["cell"], dtype=np.float32)
        src = cell.reshape(1, 4, 1)
        lh, hl, hh = _haar2x2(cell)
        assert abs(hh - case["HH"]) < 1e-12 and abs(lh - case["LH"]) < 1e-12
        assert abs(hl - case["HL"]) < 1e-12
        e = ora.dwt_detail(src, 2, 2, "hh")
        assert e.shape == (1, 1, 1) and float(e[0, 0, 0]) == case["HH"] ** 2
        e3 = ora.dwt_detail(src, 2, 2, "all3")
        assert float(e3[0, 0, 0]) == case["HH"] ** 2 + case["LH"] ** 2 + case["HL"] ** 2


def test_dwt_constant_is_exactly_zero():
    src = np.full((2, 16 * 10, 4), 1.7, dtype=np.float32)
    assert not ora.dwt_detail(src, 16, 10, "hh").any()
    assert not ora.dwt_detail(src, 16, 10, "all3").any()


def test_dwt_checkerboard_and_stripes():
    Hg, Wg = 8, 6
    yy, xx = np.meshgrid(np.arange(Hg), np.arange(Wg), indexing="ij")
    board = ((-1.0) ** (yy + xx)).astype(np.float32).reshape(1, -1, 1)
    rows = ((-1.0) ** yy).astype(np.float32).reshape(1, -1, 1)
    cols = ((-1.0) ** xx).astype(np.float32).reshape(1, -1, 1)
    assert np.all(ora.dwt_detail(board, Hg, Wg, "hh") == 4.0)
    assert not ora.dwt_detail(rows, Hg, Wg, "hh").any()
    assert not ora.dwt_detail(cols, Hg, Wg, "hh").any()
    assert np.all(ora.dwt_detail(rows, Hg, Wg, "all3") == 4.0)
    assert np.all(ora.dwt_detail(cols, Hg, Wg, "all3") == 4.0)


def test_dwt_channel_mean_and_cell_placement():
    rng = np.random.default_rng(9)
    Hg, Wg, C = 6, 10, 16
    src = rng.standard_normal((1, Hg * Wg, C)).astype(np.float32)
    got = ora.dwt_detail(src, Hg, Wg, "hh")
    x = src.astype(np.float64).reshape(Hg, Wg, C)
    for cy in range(Hg // 2):
        for cx in range(Wg // 2):
            hh = [_haar2x2(x[2 * cy:2 * cy + 2, 2 * cx:2 * cx + 2, c])[2] for c in range(C)]
            want = float(np.mean(np.square(hh)))
            assert abs(float(got[0, cy, cx]) - want) <= 2e-6 * max(1.0, want)


def test_token_energy_repeats_cells():
    E = np.arange(6, dtype=np.float32).reshape(2, 3)
    t = ora.token_energy(E)
    assert t.shape == (4, 6)
    for y in range(4):
        for x in range(6):
            assert t[y, x] == E[y // 2, x // 2]


# --------------------------------------------------------------------------
# tiling, scores, splits, halo, global KV, merge weights
# --------------------------------------------------------------------------

def test_tile_starts_golden_and_invariants():
    for case in _golden("tilings.json")["cases"]:
        starts, we = ora.tile_starts(case["L"], case["w"])
        assert (starts, we) == (case["starts"], case["we"])
    for L in range(1, 70):
        for w in range(1, 80):
            starts, we = ora.tile_starts(L, w)
            cover = np.zeros(L, dtype=int)
            for s in starts:
                assert 0 <= s and s + we <= L
                cover[s:s + we] += 1
            assert cover.min() >= 1 and starts[0] == 0 and starts[-1] == L - we
            gaps = np.diff(starts)
            if gaps.size:
                assert gaps.max() - gaps.min() <= 1          # evenly spaced
            assert len(starts) == -(-L // we)                 # fewest windows


def test_window_score_exact_on_dyadic_values():
    rng = np.random.default_rng(10)
    Et = (rng.integers(0, 64, size=(20, 24)) / 64.0).astype(np.float32)
    s = ora.window_score(Et, 3, 5, 9, 11)
    assert float(s) == float(Et[3:12, 5:16].astype(np.float64).sum())


def test_window_score_order_is_rows_then_columns():
    # 1 + 2^-24 + 2^-24 ... : sequential float32 order matters and is fixed
    Et = np.full((2, 3), np.float32(2.0 ** -24))
    Et[0, 0] = 1.0
    s = ora.window_score(Et, 0, 0, 2, 3)
    r0 = np.float32(np.float32(np.float32(1.0) + np.float32(2 ** -24)) + np.float32(2 ** -24))
    r1 = np.float32(np.float32(2 ** -24) * 3)
    assert s == np.float32(np.float32(0) + r0) + r1


def test_quadrants_partition_parent():
    for hy, wx in [(8, 8), (7, 9), (2, 3), (136, 64)]:
        cover = np.zeros((hy + 5, wx + 7), dtype=int)
        for (y0, x0, h, w) in ora.quadrants(2, 3, hy, wx):
            cover[y0:y0 + h, x0:x0 + w] += 1
        assert cover[2:2 + hy, 3:3 + wx].min() == 1 and cover.sum() == hy * wx


def test_tent_weight_closed_form():
    assert [ora.tent_weight(y, 0, 0, 0, 4, 1) for y in range(4)] == [1, 2, 2, 1]
    assert [ora.tent_weight(0, x, 0, 0, 1, 5) for x in range(5)] == [1, 2, 3, 2, 1]
    assert ora.tent_weight(5, 7, 2, 3, 8, 8) == 4 * 4


def _brute_plan_checks(plan, E, thr, seed=0):
    Hg, Wg, G = plan.Hg, plan.Wg, plan.G
    N = Hg * Wg
    Etok = ora.token_energy(E)
    rank_key = lambda t: (-float(Etok[t // Wg, t % Wg]), t)
    # base tiling covers every token; quadrants partition their split parents
    cover = np.zeros((Hg, Wg), dtype=int)
    for bi, (y0, x0, hy, wx) in enumerate(plan.base):
        cover[y0:y0 + hy, x0:x0 + wx] += 1
        kids = plan.windows[plan.parent == bi]
        if plan.split[bi]:
            assert len(kids) == 4
            c2 = np.zeros((Hg, Wg), dtype=int)
            for (a, b, c, d) in kids:
                c2[a:a + c, b:b + d] += 1
            assert c2[y0:y0 + hy, x0:x0 + wx].min() == 1 and c2.sum() == hy * wx
            assert float(plan.score[bi]) < float(np.float32(np.float32(thr) * np.float32(hy * wx)))
        else:
            assert len(kids) == 1 and tuple(kids[0]) == (y0, x0, hy, wx)
            assert not float(plan.score[bi]) < float(np.float32(np.float32(thr) * np.float32(hy * wx)))
    assert cover.min() >= 1
    wsum = np.zeros(N)
    for i, (y0, x0, hy, wx) in enumerate(plan.windows):
        h = ora.halo_width(seed, plan.halo, 0, i)
        assert 0 <= h <= plan.halo
        ext = set()
        for t in range(N):
            y, x = divmod(t, Wg)
            if y0 - h <= y < y0 + hy + h and x0 - h <= x < x0 + wx + h:
                ext.add(t)
        ey0, ex0, ehy, ewx = plan.ext[i]
        assert set(ora.window_tokens(plan.ext[i], Wg).tolist()) == ext
        gw = int(plan.gcount[i])
        sel = plan.gidx[i, :gw].tolist()
        assert gw == min(G, N - len(ext)) and np.all(plan.gidx[i, gw:] == -1)
        assert len(set(sel)) == gw and not (set(sel) & ext)
        outside = sorted((t for t in range(N) if t not in ext), key=rank_key)
        assert sel == outside[:gw]                       # rank order, ties by index
        for y in range(y0, y0 + hy):
            for x in range(x0, x0 + wx):
                wsum[y * Wg + x] += min(y - y0 + 1, y0 + hy - y) * min(x - x0 + 1, x0 + wx - x)
    assert np.array_equal(wsum.astype(np.float32), plan.wsum)


def test_plan_brute_force_invariants_random():
    rng = np.random.default_rng(12)
    thr = 0.2
    for (Hg, Wg, w, h, G) in [(16, 16, 8, 1, 5), (12, 10, 6, 2, 7), (10, 14, 20, 0, 3),
                              (20, 12, 7, 3, 9), (16, 16, 5, 1, 4)]:
        E = rng.random((Hg // 2, Wg // 2)).astype(np.float32)
        half = E.shape[1] // 2
        E[:, :half] += 0.5                              # detailed left half
        E[:, half:] *= 0.01                             # smooth right half
        tie = rng.random(E.shape) < 0.3                 # force energy ties
        E[:, :half][tie[:, :half]] = 0.75
        E[:, half:][tie[:, half:]] = 0.003
        plan = ora.window_plan(E, Hg, Wg, w, h, G, thr)
        if w < max(Hg, Wg):
            assert plan.split.any() and not plan.split.all()
        _brute_plan_checks(plan, E, thr)


def test_plan_constant_source_splits_everything_and_picks_lowest_indices():
    Hg, Wg = 16, 16
    src = np.full((1, Hg * Wg, 4), 0.3, dtype=np.float32)
    E = ora.dwt_detail(src, Hg, Wg)[0]
    plan = ora.window_plan(E, Hg, Wg, 8, 1, 6, 0.05)
    assert plan.split.all() and plan.windows.shape[0] == 4 * plan.base.shape[0]
    for i in range(plan.windows.shape[0]):
        ext = set(ora.window_tokens(plan.ext[i], Wg).tolist())
        want = [t for t in range(Hg * Wg) if t not in ext][:6]
        assert plan.gidx[i, :6].tolist() == want
    _brute_plan_checks(plan, E, 0.05)


def test_tiny_config_split_pattern():
    # Detail source: texture (noise) on the left half, smooth field on the right.
    # Windows over the textured half keep their size, the smooth ones split.
    cfg = CONFIGS["tiny"]
    src = make_detail_source(cfg)
    E = ora.dwt_detail(src, cfg.Hg, cfg.Wg)[0]
    plan = ora.window_plan(E, cfg.Hg, cfg.Wg, cfg.schedule[0], cfg.halo, cfg.G, cfg.split_thr)
    mask = texture_mask(cfg)
    for bi, (y0, x0, hy, wx) in enumerate(plan.base):
        textured = mask[y0:y0 + hy, x0:x0 + wx].mean() > 0.5
        assert plan.split[bi] == (0 if textured else 1)
    _brute_plan_checks(plan, E, cfg.split_thr)


# --------------------------------------------------------------------------
# windowed attention
# --------------------------------------------------------------------------

def test_window_single_window_no_halo_is_full_attention():
    rng = np.random.default_rng(13)
    Hg, Wg = 6, 8
    q, k, v = (rng.standard_normal((1, 2, Hg * Wg, 4)) for _ in range(3))
    E = rng.random((Hg // 2, Wg // 2)).astype(np.float32)
    plan = ora.window_plan(E, Hg, Wg, 64, 0, 5, 0.0)
    assert plan.windows.shape[0] == 1 and plan.gcount[0] == 0
    np.testing.assert_allclose(ora.window_attn(q, k, v, [plan], 0.6),
                               ora.full_attn(q, k, v, 0.6), atol=1e-12)


def _masked_reference(q, k, v, plan, scale):
    """Brute force: per window, full attention under a boolean key mask; then merge."""
    B, H, N, D = q.shape
    Wg = plan.Wg
    num = np.zeros((H, N, D))
    den = np.zeros(N)
    for i, (y0, x0, hy, wx) in enumerate(plan.windows):
        allowed = np.zeros(N, dtype=bool)
        ey0, ex0, ehy, ewx = plan.ext[i]
        for t in range(N):
            y, x = divmod(t, Wg)
            if ey0 <= y < ey0 + ehy and ex0 <= x < ex0 + ewx:
                allowed[t] = True
        allowed[plan.gidx[i, : plan.gcount[i]]] = True
        for y in range(y0, y0 + hy):
            for x in range(x0, x0 + wx):
                t = y * Wg + x
                wgt = min(y - y0 + 1, y0 + hy - y) * min(x - x0 + 1, x0 + wx - x)
                den[t] += wgt
                for hh in range(H):
                    s = scale * k[0, hh] @ q[0, hh, t]
                    s = np.where(allowed, s, -np.inf)
                    p = np.exp(s - s.max())
                    num[hh, t] += wgt * (p / p.sum()) @ v[0, hh]
    return (num / den[None, :, None])[None]


@pytest.mark.parametrize("Hg,Wg,w,h,G,thr", [(8, 8, 4, 1, 3, 0.7), (12, 10, 6, 1, 4, 0.9),
                                              (10, 12, 5, 2, 6, 1.0)])
def test_window_attention_equals_masked_full_attention(Hg, Wg, w, h, G, thr):
    rng = np.random.default_rng(14 + Hg)
    q, k, v = (rng.standard_normal((1, 2, Hg * Wg, 5)) for _ in range(3))
    E = (rng.random((Hg // 2, Wg // 2)) ** 2).astype(np.float32)
    plan = ora.window_plan(E, Hg, Wg, w, h, G, thr)
    np.testing.assert_allclose(ora.window_attn(q, k, v, [plan], 0.45),
                               _masked_reference(q, k, v, plan, 0.45), atol=1e-12)


def test_window_attention_non_overlapping_merge_is_identity():
    rng = np.random.default_rng(15)
    Hg = Wg = 16
    q, k, v = (rng.standard_normal((1, 1, Hg * Wg, 4)) for _ in range(3))
    E = np.ones((Hg // 2, Wg // 2), dtype=np.float32)
    plan = ora.window_plan(E, Hg, Wg, 4, 1, 2, 0.0)      # starts 0,4,8,12: no overlap
    got = ora.window_attn(q, k, v, [plan], 0.5)
    for i, rect in enumerate(plan.windows):
        toks = ora.window_tokens(rect, Wg)
        kv = ora.window_kv_tokens(plan, i)
        want = ora.attention(q[0, 0][toks], k[0, 0][kv], v[0, 0][kv], 0.5)
        np.testing.assert_allclose(got[0, 0, toks], want, atol=1e-13)


def test_window_attention_rows_and_heads_subset():
    rng = np.random.default_rng(16)
    Hg, Wg = 8, 8
    q, k, v = (rng.standard_normal((1, 3, Hg * Wg, 4)) for _ in range(3))
    E = rng.random((4, 4)).astype(np.float32)
    plan = ora.window_plan(E, Hg, Wg, 5, 1, 4, 0.5)
    full = ora.window_attn(q, k, v, [plan], 0.5)
    rows = np.array([0, 9, 33, 63])
    sub = ora.window_attn(q, k, v, [plan], 0.5, rows=rows, heads=[2])
    np.testing.assert_allclose(sub[0, 0], full[0, 2, rows], atol=1e-14)


# --------------------------------------------------------------------------
# text tokens (never pooled; every query attends to them)
# --------------------------------------------------------------------------

def test_coarse_with_text_matches_sdpa_over_concatenated_keys():
    rng = np.random.default_rng(21)
    Hg, Wg, f, D, T = 8, 6, 2, 4, 5
    q, k, v = (rng.standard_normal((1, 2, Hg * Wg, D)) for _ in range(3))
    kt, vt = (rng.standard_normal((1, 2, T, D)) for _ in range(2))
    kp, vp = ora.pool_kv(k, Hg, Wg, f), ora.pool_kv(v, Hg, Wg, f)
    got = ora.coarse_attn(q, kp, vp, 0.3, kt=kt, vt=vt)
    kk = torch.cat([torch.from_numpy(kp), torch.from_numpy(kt)], dim=2)
    vv = torch.cat([torch.from_numpy(vp), torch.from_numpy(vt)], dim=2)
    assert kk.shape[2] == T + Hg * Wg // (f * f)          # T + N/f^2 keys per query
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q), kk, vv, scale=0.3)
    np.testing.assert_allclose(got, ref.numpy(), atol=1e-12)
    np.testing.assert_allclose(ora.coarse_attn(q, kp, vp, 0.3, kt=kt[:, :, :0], vt=vt[:, :, :0]),
                               ora.coarse_attn(q, kp, vp, 0.3), atol=0)


def test_window_with_text_equals_masked_attention_plus_text():
    rng = np.random.default_rng(22)
    Hg, Wg, T = 10, 12, 3
    q, k, v = (rng.standard_normal((1, 2, Hg * Wg, 4)) for _ in range(3))
    kt, vt = (rng.standard_normal((1, 2, T, 4)) for _ in range(2))
    E = (rng.random((Hg // 2, Wg // 2)) ** 2).astype(np.float32)
    plan = ora.window_plan(E, Hg, Wg, 5, 1, 4, 0.2)
    got = ora.window_attn(q, k, v, [plan], 0.5, kt=kt, vt=vt)
    # brute force: per window, keys = allowed image tokens (boolean mask) + all text keys
    N = Hg * Wg
    num = np.zeros((2, N, 4))
    den = np.zeros(N)
    for i, (y0, x0, hy, wx) in enumerate(plan.windows):
        allowed = np.zeros(N, dtype=bool)
        allowed[ora.window_kv_tokens(plan, i)] = True
        for y in range(y0, y0 + hy):
            for x in range(x0, x0 + wx):
                t = y * Wg + x
                w = min(y - y0 + 1, y0 + hy - y) * min(x - x0 + 1, x0 + wx - x)
                den[t] += w
                for h in range(2):
                    s_img = np.where(allowed, 0.5 * k[0, h] @ q[0, h, t], -np.inf)
                    s_all = np.concatenate([s_img, 0.5 * kt[0, h] @ q[0, h, t]])
                    p = np.exp(s_all - s_all.max())
                    num[h, t] += w * (p / p.sum()) @ np.concatenate([v[0, h], vt[0, h]])
    np.testing.assert_allclose(got[0], num / den[None, :, None], atol=1e-12)


# --------------------------------------------------------------------------
# seeded border jitter and Halo widths
# --------------------------------------------------------------------------

def test_splitmix64_reference_sequence():
    g = _golden("splitmix64.json")
    got = [ora.counter_random(g["seed"], 0, i) for i in range(3)]
    assert got == [int(x, 16) for x in g["outputs_hex"]]
    # counter_random(seed, stream, i) is output number stream*2^32 + i
    assert ora.counter_random(7, 1, 5) == ora.counter_random(7, 0, (1 << 32) + 5)


def test_tile_windows_shift_zero_is_the_base_tiling():
    for L in range(2, 60):
        for w in range(1, 70):
            starts, we = ora.tile_starts(L, w)
            assert ora.tile_windows(L, w, 0) == [(s0, we) for s0 in starts]


def test_tile_windows_shifted_cover_the_axis_and_move_the_seams():
    for L in range(3, 50):
        for w in range(2, 40):
            we = min(w, L)
            for shift in range(0, we):
                wins = ora.tile_windows(L, w, shift)
                cover = np.zeros(L, dtype=int)
                for a, n in wins:
                    assert n >= 1 and 0 <= a and a + n <= L and n <= we
                    cover[a:a + n] += 1
                assert cover.min() >= 1
                if shift and we < L:
                    # the first window is clipped by exactly the shift
                    assert wins[0] == (0, we - shift)


def test_tile_windows_shifted_hand_worked():
    g = _golden("tilings.json")
    for c in g["shifted_cases"]:
        assert ora.tile_windows(c["L"], c["w"], c["shift"]) == [tuple(x) for x in c["windows"]], c


def test_seeded_draws_hand_worked_from_published_outputs():
    # seeds chosen so each stream's draws are the published SplitMix64
    # outputs of state 0; the shifts and widths are those outputs reduced by
    # hand (tests/golden/make_seeded_draws.py states the derivation)
    g = _golden("seeded_draws.json")
    for c in g["jitter"]:
        assert ora.jitter_shifts(int(c["seed_hex"], 16), c["Hg"], c["Wg"], c["w"]) == \
            (c["sy"], c["sx"]), c
    for c in g["halo"]:
        seed = int(c["seed_hex"], 16)
        got = [ora.halo_width(seed, c["halo"], c["b"], i) for i in c["windows"]]
        assert got == c["widths"], c
    # the jitter seed lands on the published outputs only through stream 1
    # and the Halo seeds only through stream 2 at index b * 2^20 + i
    pub = [int(h, 16) for h in _golden("splitmix64.json")["outputs_hex"]]
    sj = int(g["jitter"][0]["seed_hex"], 16)
    assert [ora.counter_random(sj, 1, i) for i in range(2)] == pub[:2]
    for c in g["halo"]:
        seed = int(c["seed_hex"], 16)
        assert [ora.counter_random(seed, 2, (c["b"] << 20) + i) for i in range(3)] == pub


def test_jitter_and_halo_draws():
    assert ora.jitter_shifts(0, 384, 384, 64) == (0, 0)
    assert ora.jitter_shifts(99, 256, 256, 256) == (0, 0)      # window spans the grid
    seen = set()
    for seed in range(1, 200):
        sy, sx = ora.jitter_shifts(seed, 384, 128, 96)
        assert 0 <= sy < 96 and 0 <= sx < 96
        seen.add(sy)
        h = ora.halo_width(seed, 8, 0, seed % 7)
        assert 0 <= h <= 8
    assert len(seen) > 50                                       # the shift really varies
    assert ora.halo_width(0, 4, 0, 3) == 4


def test_plan_with_seed_brute_force_invariants():
    rng = np.random.default_rng(31)
    for (Hg, Wg, w, h, G, seed) in [(16, 16, 6, 2, 5, 11), (20, 12, 7, 3, 9, 12345),
                                    (12, 18, 5, 1, 4, 2 ** 40 + 3)]:
        E = rng.random((Hg // 2, Wg // 2)).astype(np.float32)
        E[:, : E.shape[1] // 2] += 0.5
        plan = ora.window_plan(E, Hg, Wg, w, h, G, 0.2, seed=seed)
        sy, sx = ora.jitter_shifts(seed, Hg, Wg, w)
        assert (sy, sx) != (0, 0)
        ys = [(a, n) for a, n in ora.tile_windows(Hg, w, sy)]
        xs = [(a, n) for a, n in ora.tile_windows(Wg, w, sx)]
        assert [tuple(r) for r in plan.base] == [(a, c, n, m) for a, n in ys for c, m in xs]
        _brute_plan_checks(plan, E, 0.2, seed=seed)


# --------------------------------------------------------------------------
# the pages' global-KV bridge (deviation from the mean key, spread spatially)
# --------------------------------------------------------------------------

def test_bridge_lattice_is_rho_w_squared():
    # [ai] Phase II: R = (rho * w)^2 with rho = 0.5
    assert ora.bridge_lattice(64, 384, 384) == (32, 32)
    assert ora.bridge_lattice(72, 384, 384) == (36, 36)
    assert ora.bridge_lattice(272, 384, 128) == (136, 64)      # window clipped to 128 columns
    ry, rx = ora.bridge_lattice(8, 32, 32)
    assert ry * rx == 16


def test_key_deviation_matches_float64_definition():
    rng = np.random.default_rng(40)
    k = rng.standard_normal((3000, 16)).astype(np.float32)
    got = ora.key_deviation(k).astype(np.float64)
    mu = k.astype(np.float64).mean(0)
    want = ((k.astype(np.float64) - mu) ** 2).sum(1)
    np.testing.assert_allclose(got, want, rtol=2e-5, atol=2e-5)
    assert not ora.key_deviation(np.full((50, 4), 0.75, dtype=np.float32)).any()


def test_bridge_picks_planted_outliers_and_lowest_index_on_ties():
    Hg, Wg, D, ry, rx = 12, 16, 8, 3, 4
    rng = np.random.default_rng(41)
    k = np.zeros((Hg * Wg, D), dtype=np.float32)
    planted = []
    for cy in range(ry):
        for cx in range(rx):
            y = (cy * Hg) // ry + rng.integers(0, Hg // ry)
            x = (cx * Wg) // rx + rng.integers(0, Wg // rx)
            k[y * Wg + x] = 5.0 + cy + cx                  # far from the mean
            planted.append(y * Wg + x)
    assert ora.bridge_candidates(k, Hg, Wg, ry, rx).tolist() == planted
    # constant keys: every deviation is 0, so each cell gives its first token
    firsts = [((cy * Hg) // ry) * Wg + (cx * Wg) // rx for cy in range(ry) for cx in range(rx)]
    const = np.ones((Hg * Wg, D), dtype=np.float32)
    assert ora.bridge_candidates(const, Hg, Wg, ry, rx).tolist() == firsts


def test_window_attention_with_bridge_equals_masked_attention():
    rng = np.random.default_rng(42)
    Hg, Wg = 12, 10
    q, k, v = (rng.standard_normal((1, 2, Hg * Wg, 4)) for _ in range(3))
    E = (rng.random((Hg // 2, Wg // 2)) ** 2).astype(np.float32)
    plan = ora.window_plan(E, Hg, Wg, 6, 1, 0, 0.2)
    ry, rx = ora.bridge_lattice(6, Hg, Wg)
    cand = np.stack([ora.bridge_candidates(k[0, h].astype(np.float32), Hg, Wg, ry, rx)
                     for h in range(2)])[None]
    got = ora.window_attn(q, k, v, [plan], 0.5, bridge=cand)
    N = Hg * Wg
    num = np.zeros((2, N, 4))
    den = np.zeros(N)
    for i, (y0, x0, hy, wx) in enumerate(plan.windows):
        ey0, ex0, ehy, ewx = plan.ext[i]
        for h in range(2):
            allowed = np.zeros(N, dtype=bool)
            allowed[cand[0, h]] = True                          # all candidates ...
            for t in range(N):
                y, x = divmod(t, Wg)
                if ey0 <= y < ey0 + ehy and ex0 <= x < ex0 + ewx:
                    allowed[t] = True                           # ... and the Halo rectangle
            for y in range(y0, y0 + hy):
                for x in range(x0, x0 + wx):
                    t = y * Wg + x
                    w = min(y - y0 + 1, y0 + hy - y) * min(x - x0 + 1, x0 + wx - x)
                    if h == 0:
                        den[t] += w
                    sc = np.where(allowed, 0.5 * k[0, h] @ q[0, h, t], -np.inf)
                    p = np.exp(sc - sc.max())
                    num[h, t] += w * (p / p.sum()) @ v[0, h]
    np.testing.assert_allclose(got[0], num / den[None, :, None], atol=1e-12)
