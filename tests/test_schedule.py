"""Host schedules of the package against the oracle and the printed example."""
import json
import os

from oracle import area_oracle as ora
from step_adaptive_sparse_b200 import schedule
from workloads import CONFIGS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_pool_ramp_printed_example():
    g = json.load(open(os.path.join(GOLDEN, "ramp_flux4096.json")))
    assert schedule.pool_ramp(g["f0"], g["f_min"], g["steps"], g["Hg"], g["Wg"]) == g["ramp"]


def test_pool_ramp_matches_oracle_on_every_config_grid():
    for cfg in CONFIGS.values():
        for f0 in (2, 3, 4, 6, 8):
            for steps in (1, 4, 8, 20):
                assert (schedule.pool_ramp(f0, 2, steps, cfg.Hg, cfg.Wg) ==
                        ora.pool_ramp(f0, 2, steps, cfg.Hg, cfg.Wg))


def test_config_schedules_follow_the_geometric_formula():
    # the configs store explicit tables; they must equal the stated formula
    assert list(CONFIGS["flux2048"].schedule) == schedule.window_schedule(64, 32)
    assert list(CONFIGS["flux4096"].schedule) == schedule.window_schedule(256, 64)
    assert list(CONFIGS["flux6144"].schedule) == schedule.window_schedule(192, 64)
    assert list(CONFIGS["qwen6144x2048"].schedule) == schedule.window_schedule(272, 64)


def test_bridge_lattice_matches_oracle():
    for cfg in CONFIGS.values():
        for w in list(cfg.schedule) + [2, 5, 1000]:
            assert schedule.bridge_lattice(w, cfg.Hg, cfg.Wg) == ora.bridge_lattice(w, cfg.Hg, cfg.Wg)
