"""The C-ABI library loads, exports every declared symbol, and validates its
arguments on the host (no kernel is launched by any test in this file)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "area.h")


@pytest.fixture(scope="module")
def area():
    import step_adaptive_sparse_b200 as area
    from step_adaptive_sparse_b200 import binding
    if not os.path.exists(binding.LIB_PATH):
        from step_adaptive_sparse_b200.build import build
        build()
    area.library()
    return area


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(area_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary_calls():
    names = declared_functions()
    for want in ["area_pool_kv", "area_coarse_attn", "area_full_attn", "area_dwt_detail",
                 "area_window_plan", "area_window_plan_bytes", "area_window_attn",
                 "area_status_string", "area_version"]:
        assert want in names


def test_library_exports_every_declared_symbol(area):
    lib = area.library()
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in area.h but not exported"
    from step_adaptive_sparse_b200 import binding
    assert set(binding.EXPORTED) <= set(declared_functions())


def test_version_and_status_strings(area):
    assert "sm_100a" in area.area_version()
    for st in range(5):
        assert area.status_string(st).startswith("AREA_")
    assert "unknown" in area.status_string(99)


def test_null_and_bad_arguments_rejected_on_host(area):
    with pytest.raises(area.AreaError) as e:
        area.area_pool_kv(None, None, None, None, 1, 1, 4, 4, 8, 2, 0, 1)
    assert e.value.status == area.AREA_EINVAL
    fake = 1 << 20   # never dereferenced: validation fails first
    cases = [
        (lambda: area.area_pool_kv(fake, fake, fake, fake, 1, 1, 6, 4, 8, 4, 0, 1), area.AREA_EINVAL),
        (lambda: area.area_pool_kv(fake, fake, fake, fake, 1, 1, 4, 4, 8, 2, 7, 1), area.AREA_EINVAL),
        (lambda: area.area_pool_kv(fake, fake, fake, fake, 1, 1, 4, 4, 8, 2, 0, 5), area.AREA_EINVAL),
        (lambda: area.area_pool_kv(fake, fake, fake, fake, 1, 1, 4, 4, 6, 2, 0, 1), area.AREA_EUNSUPPORTED),
        (lambda: area.area_pool_kv(fake + 2, fake, fake, fake, 1, 1, 4, 4, 8, 2, 0, 1), area.AREA_EINVAL),
        (lambda: area.area_coarse_attn(fake, fake, fake, fake, 1, 1, 16, 0, 128, 1.0, 1), area.AREA_EINVAL),
        (lambda: area.area_coarse_attn(fake, fake, fake, fake, 1, 1, 16, 4, 96, 1.0, 1), area.AREA_EUNSUPPORTED),
        (lambda: area.area_coarse_attn(fake, fake, fake, fake, 1, 1, 16, 4, 128, 1.0, 3), area.AREA_EUNSUPPORTED),
        (lambda: area.area_full_attn(None, fake, fake, fake, 1, 1, 16, 128, 1.0, 1), area.AREA_EINVAL),
        (lambda: area.area_coarse_attn_text(fake, fake, fake, None, None, fake, 1, 1, 16, 4, 3, 128, 1.0, 1), area.AREA_EINVAL),
        (lambda: area.area_coarse_attn_text(fake, fake, fake, fake, fake, fake, 1, 1, 16, 4, -1, 128, 1.0, 1), area.AREA_EINVAL),
        (lambda: area.area_dwt_detail(fake, 1, 16, fake, 1, 7, 8), area.AREA_EINVAL),
        (lambda: area.area_bridge_select(fake, 1, 1, 2, 8, 8, 128, 9, 2, fake, fake, 1024), area.AREA_EINVAL),
        (lambda: area.area_bridge_select(fake, 1, 1, 2, 8, 8, 128, 4, 4, fake, fake, 2047), area.AREA_ENOSPACE),
        (lambda: area.area_bridge_select_ws_bytes(1, 0, 8, 8, 128), area.AREA_EINVAL),
        (lambda: area.area_pool_ramp(4, 2, 0, 8, 8), area.AREA_EINVAL),
        (lambda: area.area_dwt_window_plan(None, 1, 16, 0, fake, area.make_cfg(1, 16, 16, 8, 1, 4, 0.1), fake, 1 << 20), area.AREA_EINVAL),
        (lambda: area.area_dwt_window_plan(fake, 1, 16, 7, fake, area.make_cfg(1, 16, 16, 8, 1, 4, 0.1), fake, 1 << 20), area.AREA_EINVAL),
        (lambda: area.area_dwt_window_plan(fake, 1, 16, 0, fake, area.make_cfg(1, 16, 16, 8, 1, 4, 0.1), fake, 256), area.AREA_ENOSPACE),
        (lambda: area.area_dwt_window_plan(fake, 1, 16, 0, fake, area.make_cfg(1, 15, 16, 8, 1, 4, 0.1), fake, 1 << 20), area.AREA_EINVAL),
        (lambda: area.area_window_sides(0, 64, 8), area.AREA_EINVAL),
        (lambda: area.area_bridge_lattice(0, 8, 8), area.AREA_EINVAL),
        (lambda: area.area_schedule([], 0.9, 4, 2, 64, 32, 8, 8), area.AREA_EINVAL),
        (lambda: area.area_bridge_select(fake, 1, 1, 2, 8, 8, 96, 4, 4, fake, fake, 4096), area.AREA_EUNSUPPORTED),
        (lambda: area.area_dwt_detail(fake, 1, 0, fake, 1, 8, 8), area.AREA_EINVAL),
        (lambda: area.area_dwt_detail(fake, 1, 4, fake, 1, 8, 8, 9), area.AREA_EINVAL),
    ]
    for fn, status in cases:
        with pytest.raises(area.AreaError) as e:
            fn()
        assert e.value.status == status


def test_bridge_ws_bytes(area):
    # mean keys [B*H][D] plus one row of D chunk sums per 1024 tokens, fp32
    assert area.area_bridge_select_ws_bytes(1, 2, 8, 8, 128) == 2 * 128 * 2 * 4
    assert area.area_bridge_select_ws_bytes(1, 24, 384, 384, 128) == 24 * 128 * (1 + 144) * 4
    assert area.area_bridge_select_ws_bytes(2, 1, 33, 31, 64) == 2 * 64 * (1 + 1) * 4
    assert area.area_bridge_select_ws_bytes(1, 1, 32, 33, 64) == 64 * (1 + 2) * 4


def test_plan_config_validation_and_sizes(area):
    good = area.make_cfg(1, 256, 256, 64, 4, 512, 0.4)
    n = area.area_window_plan_bytes(good)
    assert n > 0 and n % 256 == 0
    # plan size grows with G and with the number of windows
    assert area.area_window_plan_bytes(area.make_cfg(1, 256, 256, 64, 4, 1024, 0.4)) > n
    assert area.area_window_plan_bytes(area.make_cfg(1, 256, 256, 32, 4, 512, 0.4)) > n
    assert area.area_window_plan_bytes(area.make_cfg(2, 256, 256, 64, 4, 512, 0.4)) > n
    # 64-token windows tile 256 exactly: no overlap, only the counter header
    # (1 + 4 * B * H uint32 counters, rounded up to 256 bytes)
    assert area.area_window_attn_ws_bytes(good, 24, 128) == 512
    assert area.area_window_attn_ws_bytes(good, 1, 128) == 256
    for bad in [area.make_cfg(0, 256, 256, 64, 4, 512, 0.4),
                area.make_cfg(1, 255, 256, 64, 4, 512, 0.4),
                area.make_cfg(1, 256, 256, 0, 4, 512, 0.4),
                area.make_cfg(1, 256, 256, 64, -1, 512, 0.4),
                area.make_cfg(1, 256, 256, 64, 4, 5000, 0.4),
                area.make_cfg(4096, 256, 256, 64, 4, 512, 0.4)]:
        with pytest.raises(area.AreaError) as e:
            area.area_window_plan_bytes(bad)
        assert e.value.status == area.AREA_EINVAL


def test_stage_bytes(area):
    # K and V rows of every window slot: 2 * B * H * nw * G * D * 2 bytes with
    # nw = 4 quadrants per base-window slot (16 slots at w = 64 on 256; 25
    # when a seed may shift the tiling by up to one window per axis)
    unit = 2 * 24 * 512 * 128 * 2
    assert area.area_window_attn_stage_bytes(area.make_cfg(1, 256, 256, 64, 4, 512, 0.4), 24,
                                             128) == 64 * unit
    assert area.area_window_attn_stage_bytes(area.make_cfg(1, 256, 256, 64, 4, 512, 0.4, 99), 24,
                                             128) == 100 * unit
    assert area.area_window_attn_stage_bytes(area.make_cfg(2, 256, 256, 64, 4, 512, 0.4), 12,
                                             64) == 64 * unit // 2
    assert area.area_window_attn_stage_bytes(area.make_cfg(1, 256, 256, 64, 4, 0, 0.4), 24,
                                             128) == 0


def test_bridge_stage_bytes(area):
    # K and V rows of every head's candidates: 2 * B * H * R * D * 2 bytes
    assert area.area_window_attn_bridge_stage_bytes(1, 24, 1024, 128) == 2 * 24 * 1024 * 128 * 2
    assert area.area_window_attn_bridge_stage_bytes(2, 3, 240, 64) == 2 * 2 * 3 * 240 * 64 * 2
    with pytest.raises(area.AreaError):
        area.area_window_attn_bridge_stage_bytes(1, 24, 0, 128)


def test_plan_size_with_seed_covers_every_shift(area):
    # a seeded plan may hold one more base window per axis
    base = area.area_window_plan_bytes(area.make_cfg(1, 384, 384, 72, 4, 512, 0.4))
    seeded = area.area_window_plan_bytes(area.make_cfg(1, 384, 384, 72, 4, 512, 0.4, 99))
    assert seeded >= base


def test_window_calls_reject_small_buffers_on_host(area):
    cfg = area.make_cfg(1, 32, 32, 8, 1, 16, 0.05)
    need = area.area_window_plan_bytes(cfg)
    fake = 1 << 20
    with pytest.raises(area.AreaError) as e:
        area.area_window_plan(fake, cfg, fake, need - 256)
    assert e.value.status == area.AREA_ENOSPACE
    ws = area.area_window_attn_ws_bytes(cfg, 2, 64)
    with pytest.raises(area.AreaError) as e:
        area.area_window_attn(fake, fake, fake, cfg, fake, need, fake, fake, ws - 4, 2, 64, 0.125, 0)
    assert e.value.status == area.AREA_ENOSPACE
    with pytest.raises(area.AreaError) as e:
        area.area_window_attn(fake, fake, fake, cfg, fake, need - 1, fake, fake, ws, 2, 64, 0.125, 0)
    assert e.value.status == area.AREA_ENOSPACE
    with pytest.raises(area.AreaError) as e:
        area.area_window_attn(fake, fake, fake, cfg, fake + 16, need, fake, fake, ws, 2, 64, 0.125, 0)
    assert e.value.status == area.AREA_EINVAL
    # outputs and the workspace are written 32 bytes per thread: 16-byte
    # aligned ones are refused
    for o, w in ((fake + 16, fake), (fake, fake + 16)):
        with pytest.raises(area.AreaError) as e:
            area.area_window_attn(fake, fake, fake, cfg, fake, need, o, w, ws, 2, 64, 0.125, 1)
        assert e.value.status == area.AREA_EINVAL
    with pytest.raises(area.AreaError) as e:
        area.area_coarse_attn(fake, fake, fake, fake + 16, 1, 1, 16, 4, 128, 1.0, 1)
    assert e.value.status == area.AREA_EINVAL


def test_binding_has_no_oracle_dependency():
    # The product path never reaches the oracle: no module of the package
    # imports it, and the binding fails loudly without the shared library.
    pkg = os.path.join(ROOT, "step_adaptive_sparse_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", text, flags=re.M), fn
                assert "area_oracle" not in text, fn


def test_plain_c_consumer(tmp_path):
    # the header and the shared library are usable from C alone: compile a C
    # program against include/area.h, link libarea.so and run its host checks
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    cuda_inc = next((p for p in ("/usr/local/cuda/include",) if os.path.isdir(p)), None)
    if gcc is None or cuda_inc is None:
        pytest.skip("gcc or the CUDA headers are not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.join(root, "step_adaptive_sparse_b200", "lib")
    exe = str(tmp_path / "c_abi_check")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                    "-I", cuda_inc, os.path.join(root, "tests", "c_abi_check.c"),
                    "-L", libdir, "-larea", f"-Wl,-rpath,{libdir}", "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert "C-ABI host checks passed" in r.stdout


def test_merge_geometry_host_check(tmp_path):
    # The window kernels' merge geometry (which windows share a token, which
    # of them stores first and which normalises last, the token's accumulator
    # row) is plain integer arithmetic in area_internal.cuh.  Compile it on
    # the host and check every token of many tilings, with border shifts.
    import shutil
    import subprocess
    from step_adaptive_sparse_b200 import build as b
    nvcc = b.nvcc()
    if shutil.which(nvcc) is None and not os.path.exists(nvcc):
        pytest.skip("nvcc is not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    exe = str(tmp_path / "merge_geometry_check")
    subprocess.run([nvcc, "-O2", "-std=c++17", "-Wno-deprecated-gpu-targets", "-I",
                    os.path.join(root, "include"), "-I", b.CSRC,
                    os.path.join(root, "tests", "merge_geometry_check.cu"), "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert "tilings checked" in r.stdout


def test_rect_tiling_host_check(tmp_path):
    # The tensor-core window kernel loads a Halo rectangle as full 16 x 8
    # patches plus 4 x 4 cells of its right and bottom strips, and a window's
    # queries in 4 x 4 cells: integer arithmetic in area_internal.cuh.  Check
    # on the host that every key of every rectangle up to 72 x 72 (and some
    # large ones) lands in exactly one tile row and that the query positions
    # enumerate each window's tokens once.
    import shutil
    import subprocess
    from step_adaptive_sparse_b200 import build as b
    nvcc = b.nvcc()
    if shutil.which(nvcc) is None and not os.path.exists(nvcc):
        pytest.skip("nvcc is not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    exe = str(tmp_path / "rect_tiling_check")
    subprocess.run([nvcc, "-O2", "-std=c++17", "-Wno-deprecated-gpu-targets", "-I",
                    os.path.join(root, "include"), "-I", b.CSRC,
                    os.path.join(root, "tests", "rect_tiling_check.cu"), "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert "rectangles and" in r.stdout


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    # no fallback: without the built library every call raises
    from step_adaptive_sparse_b200 import binding
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "libarea.so"))
    monkeypatch.setattr(binding, "_LIB", None)
    with pytest.raises(ImportError):
        binding.area_version()
    with pytest.raises(ImportError):
        binding.area_pool_ramp(4, 2, 8, 256, 256)


def test_noalloc_rejects_bad_input_with_the_status_of_area_window_attn(area):
    # Both calls validate on the host before any CUDA call; for the same bad
    # input they must give the same status.
    fake = 1 << 20
    cfg = area.make_cfg(1, 16, 16, 8, 1, 4, 0.1)
    nb = area.area_window_plan_bytes(cfg)
    ws_big = 1 << 40
    cases = [
        dict(q=None),                           # null input
        dict(plan=None),                        # null plan
        dict(H=0),                              # no heads
        dict(D=96),                             # unsupported head_dim
        dict(dtype=5),                          # unknown dtype
        dict(cfg=area.make_cfg(1, 15, 16, 8, 1, 4, 0.1)),   # odd grid side
        dict(cfg=area.make_cfg(1, 16, 16, 0, 1, 4, 0.1)),   # zero window side
    ]
    for c in cases:
        a = dict(q=fake, k=fake, v=fake, cfg=cfg, plan=fake, o=fake, H=2, D=128, dtype=1)
        a.update(c)
        with pytest.raises(area.AreaError) as e1:
            area.area_window_attn(a["q"], a["k"], a["v"], a["cfg"], a["plan"], nb, a["o"], fake,
                                  ws_big, a["H"], a["D"], 1.0, a["dtype"])
        with pytest.raises(area.AreaError) as e2:
            area.area_window_attn_noalloc(a["q"], a["k"], a["v"], a["cfg"], a["plan"], nb,
                                          a["o"], a["H"], a["D"], 1.0, a["dtype"])
        assert e1.value.status == e2.value.status, c
    # beyond the static workspace: refused before any launch
    big = area.make_cfg(1, 256, 256, 80, 4, 16, 0.1)
    with pytest.raises(area.AreaError) as e:
        area.area_window_attn_noalloc(fake, fake, fake, big, fake, area.area_window_plan_bytes(big),
                                      fake, 24, 128, 1.0, 1)
    assert e.value.status == area.AREA_ENOSPACE


def test_window_ws_bytes_count_the_overlapped_tokens(area):
    # Workspace = counter header (1 + 4 * B * H uint32, rounded up to 256
    # bytes) + one fp32 row of D per (element, head, token covered by more
    # than one base window).  The overlapped
    # tokens are counted here by brute force over the oracle's base tiling
    # (with the border shift the seed draws).
    from oracle import area_oracle as ora
    import numpy as np
    for (B, Hg, Wg, w, seed) in [(1, 256, 256, 80, 0), (2, 384, 128, 96, 0), (1, 32, 32, 10, 0),
                                 (1, 384, 384, 168, 0), (1, 384, 384, 192, 0), (1, 40, 28, 12, 777),
                                 (3, 64, 48, 24, 5), (1, 20, 12, 6, 2 ** 40 + 3)]:
        sy, sx = ora.jitter_shifts(seed, Hg, Wg, w)
        cy = np.zeros(Hg, dtype=int)
        cx = np.zeros(Wg, dtype=int)
        for a, n in ora.tile_windows(Hg, w, sy):
            cy[a:a + n] += 1
        for a, n in ora.tile_windows(Wg, w, sx):
            cx[a:a + n] += 1
        assert cy.max() <= 2 and cx.max() <= 2       # only neighbours overlap
        n_ov = int(((cy[:, None] * cx[None, :]) > 1).sum())
        for H, D in [(1, 64), (24, 128)]:
            cfg = area.make_cfg(B, Hg, Wg, w, 4, 16, 0.1, seed)
            hdr = (4 * (1 + 4 * B * H) + 255) // 256 * 256
            assert area.area_window_attn_ws_bytes(cfg, H, D) == hdr + B * H * n_ov * D * 4
