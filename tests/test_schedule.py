"""Host schedules of the package against the oracle and the printed example."""
import json

import numpy as np
import os

from oracle import area_oracle as ora
import step_adaptive_sparse_b200 as area
from workloads import CONFIGS, flow_sigmas

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_pool_ramp_printed_example():
    g = json.load(open(os.path.join(GOLDEN, "ramp_flux4096.json")))
    assert area.area_pool_ramp(g["f0"], g["f_min"], g["steps"], g["Hg"], g["Wg"]) == g["ramp"]


def test_pool_ramp_matches_oracle_on_every_config_grid():
    for cfg in CONFIGS.values():
        for f0 in (2, 3, 4, 6, 8):
            for steps in (1, 4, 8, 20):
                assert (area.area_pool_ramp(f0, 2, steps, cfg.Hg, cfg.Wg) ==
                        ora.pool_ramp(f0, 2, steps, cfg.Hg, cfg.Wg))


def test_config_schedules_follow_the_geometric_formula():
    # the configs store explicit tables; they must equal the stated formula
    assert list(CONFIGS["flux2048"].schedule) == area.area_window_sides(64, 32, 8)
    assert list(CONFIGS["flux4096"].schedule) == area.area_window_sides(256, 64, 8)
    assert list(CONFIGS["flux6144"].schedule) == area.area_window_sides(192, 64, 8)
    assert list(CONFIGS["qwen6144x2048"].schedule) == area.area_window_sides(272, 64, 8)


def test_bridge_lattice_matches_oracle():
    for cfg in CONFIGS.values():
        for w in list(cfg.schedule) + [2, 5, 1000]:
            assert area.area_bridge_lattice(w, cfg.Hg, cfg.Wg) == ora.bridge_lattice(w, cfg.Hg, cfg.Wg)


def test_window_sides_match_oracle():
    for w0 in (64, 96, 192, 256, 272):
        for wm in (32, 64, 96):
            for n in (1, 2, 8, 20, 33):
                assert area.area_window_sides(w0, wm, n) == ora.window_sides(w0, wm, n)


def test_phase_switch_matches_oracle():
    rng = np.random.default_rng(3)
    lists = [flow_sigmas(28, 3.0), flow_sigmas(50, 4.0), np.array([0.99, 0.5, 0.99], np.float32)]
    lists += [rng.random(rng.integers(1, 30)).astype(np.float32) for _ in range(50)]
    for sig in lists:
        for star in (0.0, 0.3, 0.86, 0.89, 0.9, 0.96, 1.0, float(sig[0])):
            assert area.area_phase_switch(sig, star) == ora.phase_switch(sig, star)


def test_schedule_matches_oracle():
    names = {area.AREA_PHASE_COARSE: "coarse", area.AREA_PHASE_WINDOW: "window"}
    for cfg in CONFIGS.values():
        for steps, shift, star in [(28, 3.0, 0.89), (28, 3.0, 0.96), (50, 3.0, 0.9), (8, 1.0, 0.5)]:
            sig = flow_sigmas(steps, shift)
            w0, wm = cfg.schedule[0], cfg.schedule[-1]
            got = area.area_schedule(sig, star, cfg.f, 2, w0, wm, cfg.Hg, cfg.Wg)
            want = ora.phase_schedule(sig, star, cfg.f, 2, w0, wm, cfg.Hg, cfg.Wg)
            assert [(names[k], p) for k, p in got] == want
