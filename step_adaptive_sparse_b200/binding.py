"""ctypes binding of libarea: argument marshalling only.

Each function has the name and argument order of its C counterpart in
include/area.h.  Pointer arguments accept a torch tensor (its data_ptr is
passed), an int address, or None (NULL).  The stream argument accepts a
torch.cuda.Stream, an int handle, or None (the legacy default stream).
A non-zero status raises AreaError.  There is no fallback: when the shared
library is missing the first call raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libarea.so")

AREA_OK, AREA_EINVAL, AREA_EUNSUPPORTED, AREA_ENOSPACE, AREA_ECUDA = 0, 1, 2, 3, 4
AREA_DTYPE_F32, AREA_DTYPE_BF16 = 0, 1
AREA_POOL_MEAN, AREA_POOL_CENTER = 0, 1
AREA_DETAIL_HH, AREA_DETAIL_ALL3 = 0, 1
AREA_PHASE_COARSE, AREA_PHASE_WINDOW = 1, 2
AREA_KERR_TC_WAIT, AREA_KERR_PLAN_BARRIER = 1, 2
AREA_PLAN_MAGIC = 0x4145524150414C4E
SECTIONS = ("BASE", "SCORE", "SPLIT", "NWIN", "WIN", "PARENT", "EXT", "GCOUNT", "GIDX",
            "WSUM", "ORDER", "NITEM", "ITEMS", "COVER", "NCLASS", "SCRATCH")

EXPORTED = ("area_status_string", "area_last_cuda_error", "area_version", "area_kernel_error",
            "area_pool_kv", "area_coarse_attn_text", "area_window_attn_text",
            "area_bridge_select_ws_bytes", "area_bridge_select", "area_window_attn_bridge",
            "area_dwt_window_plan", "area_pool_ramp", "area_window_sides", "area_bridge_lattice", "area_phase_switch",
            "area_schedule",
            "area_coarse_attn", "area_full_attn", "area_dwt_detail", "area_window_plan_bytes",
            "area_window_plan", "area_window_attn_ws_bytes", "area_window_attn_stage_bytes",
            "area_window_attn_bridge_stage_bytes",
            "area_window_attn",
            "area_window_attn_noalloc", "area_test_plan_barrier_expiry")


class AreaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)}"
        if status == AREA_ECUDA:
            msg += f" (cudaError {_lib().area_last_cuda_error()})"
        super().__init__(msg)


class area_plan_cfg(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hg", ctypes.c_int), ("Wg", ctypes.c_int),
                ("w", ctypes.c_int), ("halo", ctypes.c_int), ("G", ctypes.c_int),
                ("split_thr", ctypes.c_float), ("jitter_seed", ctypes.c_ulonglong)]


_LIB: Optional[ctypes.CDLL] = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_SIGS = {
    "area_status_string": (ctypes.c_char_p, [_I]),
    "area_last_cuda_error": (_I, []),
    "area_version": (ctypes.c_char_p, []),
    "area_kernel_error": (_I, [ctypes.POINTER(_I)]),
    "area_pool_kv": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P]),
    "area_coarse_attn": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P]),
    "area_full_attn": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "area_coarse_attn_text": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "area_window_attn_text": (_I, [_P, _P, _P, _P, _P, _I, ctypes.POINTER(area_plan_cfg), _P, _SZ,
                                   _P, _P, _SZ, _I, _I, _F, _I, _P]),
    "area_dwt_detail": (_I, [_P, _I, _I, _P, _I, _I, _I, _I, _P]),
    "area_window_plan_bytes": (_I, [ctypes.POINTER(area_plan_cfg), ctypes.POINTER(_SZ)]),
    "area_window_plan": (_I, [_P, ctypes.POINTER(area_plan_cfg), _P, _SZ, _P]),
    "area_window_attn_ws_bytes": (_I, [ctypes.POINTER(area_plan_cfg), _I, _I, ctypes.POINTER(_SZ)]),
    "area_window_attn_stage_bytes": (_I, [ctypes.POINTER(area_plan_cfg), _I, _I,
                                          ctypes.POINTER(_SZ)]),
    "area_window_attn_bridge_stage_bytes": (_I, [_I, _I, _I, _I, ctypes.POINTER(_SZ)]),
    "area_window_attn": (_I, [_P, _P, _P, ctypes.POINTER(area_plan_cfg), _P, _SZ, _P, _P, _SZ,
                              _I, _I, _F, _I, _P]),
    "area_window_attn_noalloc": (_I, [_P, _P, _P, ctypes.POINTER(area_plan_cfg), _P, _SZ, _P,
                                      _I, _I, _F, _I, _P]),
    "area_dwt_window_plan": (_I, [_P, _I, _I, _I, _P, ctypes.POINTER(area_plan_cfg), _P, _SZ,
                                  _P]),
    "area_test_plan_barrier_expiry": (_I, [_P, _I, _I, _P, ctypes.POINTER(area_plan_cfg), _P,
                                           _SZ, _P]),
    "area_pool_ramp": (_I, [_I, _I, _I, _I, _I, _P]),
    "area_window_sides": (_I, [_I, _I, _I, _P]),
    "area_bridge_lattice": (_I, [_I, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "area_phase_switch": (_I, [_P, _I, _F, ctypes.POINTER(_I)]),
    "area_schedule": (_I, [_P, _I, _F, _I, _I, _I, _I, _I, _I, _P, _P]),
    "area_bridge_select_ws_bytes": (_I, [_I, _I, _I, _I, _I, ctypes.POINTER(_SZ)]),
    "area_bridge_select": (_I, [_P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P]),
    "area_window_attn_bridge": (_I, [_P, _P, _P, _P, _I, ctypes.POINTER(area_plan_cfg), _P, _SZ,
                                     _P, _P, _SZ, _I, _I, _F, _I, _P]),
}


def _lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libarea is not built ({LIB_PATH} missing); run "
                              "`python -m step_adaptive_sparse_b200.build` first")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def library() -> ctypes.CDLL:
    """The loaded shared library (loads it on first use)."""
    return _lib()


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, where: str) -> None:
    if status != AREA_OK:
        raise AreaError(status, where)


def make_cfg(B: int, Hg: int, Wg: int, w: int, halo: int, G: int, split_thr: float,
             jitter_seed: int = 0) -> area_plan_cfg:
    return area_plan_cfg(B, Hg, Wg, w, halo, G, split_thr, jitter_seed)


def status_string(status: int) -> str:
    return _lib().area_status_string(status).decode()


def area_version() -> str:
    return _lib().area_version().decode()


def area_kernel_error() -> int:
    """Synchronise; return and clear the bounded-wait expiry flag (0 = none)."""
    out = _I(0)
    _check(_lib().area_kernel_error(ctypes.byref(out)), "area_kernel_error")
    return int(out.value)


def area_pool_kv(k, v, kp, vp, B, H, Hg, Wg, D, f, mode, dtype, stream=None) -> None:
    _check(_lib().area_pool_kv(_ptr(k), _ptr(v), _ptr(kp), _ptr(vp), B, H, Hg, Wg, D, f, mode,
                               dtype, _stream(stream)), "area_pool_kv")


def area_coarse_attn(q, kp, vp, o, B, H, N, Nk, D, scale, dtype, stream=None) -> None:
    _check(_lib().area_coarse_attn(_ptr(q), _ptr(kp), _ptr(vp), _ptr(o), B, H, N, Nk, D, scale,
                                   dtype, _stream(stream)), "area_coarse_attn")


def area_coarse_attn_text(q, kp, vp, kt, vt, o, B, H, N, Nk, T, D, scale, dtype,
                          stream=None) -> None:
    _check(_lib().area_coarse_attn_text(_ptr(q), _ptr(kp), _ptr(vp), _ptr(kt), _ptr(vt), _ptr(o),
                                        B, H, N, Nk, T, D, scale, dtype, _stream(stream)),
           "area_coarse_attn_text")


def area_window_attn_text(q, k, v, kt, vt, T, cfg: area_plan_cfg, plan, plan_bytes, o, ws,
                          ws_bytes, H, D, scale, dtype, stream=None) -> None:
    _check(_lib().area_window_attn_text(_ptr(q), _ptr(k), _ptr(v), _ptr(kt), _ptr(vt), T,
                                        ctypes.byref(cfg), _ptr(plan), plan_bytes, _ptr(o),
                                        _ptr(ws), ws_bytes, H, D, scale, dtype, _stream(stream)),
           "area_window_attn_text")


def area_full_attn(q, k, v, o, B, H, N, D, scale, dtype, stream=None) -> None:
    _check(_lib().area_full_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, D, scale, dtype,
                                 _stream(stream)), "area_full_attn")


def area_dwt_detail(src, src_dtype, C, energy, B, Hg, Wg, mode=AREA_DETAIL_HH, stream=None) -> None:
    _check(_lib().area_dwt_detail(_ptr(src), src_dtype, C, _ptr(energy), B, Hg, Wg, mode,
                                  _stream(stream)), "area_dwt_detail")


def area_window_plan_bytes(cfg: area_plan_cfg) -> int:
    out = _SZ(0)
    _check(_lib().area_window_plan_bytes(ctypes.byref(cfg), ctypes.byref(out)),
           "area_window_plan_bytes")
    return int(out.value)


def area_window_plan(energy, cfg: area_plan_cfg, plan, plan_bytes: int, stream=None) -> None:
    _check(_lib().area_window_plan(_ptr(energy), ctypes.byref(cfg), _ptr(plan), plan_bytes,
                                   _stream(stream)), "area_window_plan")


def area_dwt_window_plan(src, src_dtype, C, mode, energy, cfg: area_plan_cfg, plan, plan_bytes,
                         stream=None) -> None:
    _check(_lib().area_dwt_window_plan(_ptr(src), src_dtype, C, mode, _ptr(energy),
                                       ctypes.byref(cfg), _ptr(plan), plan_bytes,
                                       _stream(stream)), "area_dwt_window_plan")


def area_test_plan_barrier_expiry(src, src_dtype, C, energy, cfg: area_plan_cfg, plan,
                                  plan_bytes, stream=None) -> None:
    """Test hook: the one-launch planner with barriers that cannot complete
    and 1 ms wait bounds (see include/area.h)."""
    _check(_lib().area_test_plan_barrier_expiry(_ptr(src), src_dtype, C, _ptr(energy),
                                                ctypes.byref(cfg), _ptr(plan), plan_bytes,
                                                _stream(stream)),
           "area_test_plan_barrier_expiry")


def area_window_attn_ws_bytes(cfg: area_plan_cfg, H: int, D: int) -> int:
    out = _SZ(0)
    _check(_lib().area_window_attn_ws_bytes(ctypes.byref(cfg), H, D, ctypes.byref(out)),
           "area_window_attn_ws_bytes")
    return int(out.value)


def area_window_attn_stage_bytes(cfg: area_plan_cfg, H: int, D: int) -> int:
    out = _SZ(0)
    _check(_lib().area_window_attn_stage_bytes(ctypes.byref(cfg), H, D, ctypes.byref(out)),
           "area_window_attn_stage_bytes")
    return int(out.value)


def area_window_attn_bridge_stage_bytes(B: int, H: int, R: int, D: int) -> int:
    out = _SZ(0)
    _check(_lib().area_window_attn_bridge_stage_bytes(B, H, R, D, ctypes.byref(out)),
           "area_window_attn_bridge_stage_bytes")
    return int(out.value)


def area_window_attn(q, k, v, cfg: area_plan_cfg, plan, plan_bytes, o, ws, ws_bytes, H, D,
                     scale, dtype, stream=None) -> None:
    _check(_lib().area_window_attn(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(cfg), _ptr(plan),
                                   plan_bytes, _ptr(o), _ptr(ws), ws_bytes, H, D, scale, dtype,
                                   _stream(stream)), "area_window_attn")


def area_window_attn_noalloc(q, k, v, cfg: area_plan_cfg, plan, plan_bytes, o, H, D, scale,
                             dtype, stream=None) -> None:
    """area_window_attn without a workspace argument, for callers that cannot
    allocate device memory; the workspace is a 32 MiB static array of the
    library (see include/area.h for the limit and the sharing rules)."""
    _check(_lib().area_window_attn_noalloc(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(cfg),
                                           _ptr(plan), plan_bytes, _ptr(o), H, D, scale, dtype,
                                           _stream(stream)), "area_window_attn_noalloc")


def _ints(n: int):
    return (ctypes.c_int * n)()


def _floats(values):
    arr = (ctypes.c_float * len(values))(*[float(x) for x in values])
    return arr


def area_pool_ramp(f0: int, f_min: int, steps: int, Hg: int, Wg: int) -> list:
    out = _ints(max(steps, 1))
    _check(_lib().area_pool_ramp(f0, f_min, steps, Hg, Wg, out), "area_pool_ramp")
    return list(out)[:steps]


def area_window_sides(w0: int, w_min: int, steps: int) -> list:
    out = _ints(max(steps, 1))
    _check(_lib().area_window_sides(w0, w_min, steps, out), "area_window_sides")
    return list(out)[:steps]


def area_bridge_lattice(w: int, Hg: int, Wg: int):
    ry, rx = _I(0), _I(0)
    _check(_lib().area_bridge_lattice(w, Hg, Wg, ctypes.byref(ry), ctypes.byref(rx)),
           "area_bridge_lattice")
    return ry.value, rx.value


def area_phase_switch(sigmas, sigma_star: float) -> int:
    arr = _floats(sigmas)
    n = _I(0)
    _check(_lib().area_phase_switch(arr, len(arr), sigma_star, ctypes.byref(n)),
           "area_phase_switch")
    return n.value


def area_schedule(sigmas, sigma_star: float, f0: int, f_min: int, w0: int, w_min: int,
                  Hg: int, Wg: int):
    """Per step (kind, param): (AREA_PHASE_COARSE, f) or (AREA_PHASE_WINDOW, w)."""
    arr = _floats(sigmas)
    n = len(arr)
    kind, param = _ints(max(n, 1)), _ints(max(n, 1))
    _check(_lib().area_schedule(arr, n, sigma_star, f0, f_min, w0, w_min, Hg, Wg, kind, param),
           "area_schedule")
    return [(kind[t], param[t]) for t in range(n)]


def area_bridge_select_ws_bytes(B: int, H: int, Hg: int, Wg: int, D: int) -> int:
    out = _SZ(0)
    _check(_lib().area_bridge_select_ws_bytes(B, H, Hg, Wg, D, ctypes.byref(out)),
           "area_bridge_select_ws_bytes")
    return out.value


def area_bridge_select(k, dtype, B, H, Hg, Wg, D, ry, rx, cand, ws, ws_bytes, stream=None) -> None:
    _check(_lib().area_bridge_select(_ptr(k), dtype, B, H, Hg, Wg, D, ry, rx, _ptr(cand), _ptr(ws),
                                     ws_bytes, _stream(stream)), "area_bridge_select")


def area_window_attn_bridge(q, k, v, cand, R, cfg: area_plan_cfg, plan, plan_bytes, o, ws,
                            ws_bytes, H, D, scale, dtype, stream=None) -> None:
    _check(_lib().area_window_attn_bridge(_ptr(q), _ptr(k), _ptr(v), _ptr(cand), R,
                                          ctypes.byref(cfg), _ptr(plan), plan_bytes, _ptr(o),
                                          _ptr(ws), ws_bytes, H, D, scale, dtype,
                                          _stream(stream)), "area_window_attn_bridge")


def parse_plan(buf: np.ndarray) -> dict:
    """Decode a plan buffer copied to the host (uint8 array) into numpy arrays.

    Follows the documented layout of include/area.h: an int64 header with
    the sizes and the byte offset of each section.
    """
    buf = np.ascontiguousarray(buf, dtype=np.uint8)
    hdr = buf[:256].view(np.int64)
    if int(hdr[0]) != AREA_PLAN_MAGIC:
        raise ValueError("not a libarea plan buffer (bad magic)")
    B, Hg, Wg, w, halo, G, nb, nw = (int(x) for x in hdr[2:10])
    N = Hg * Wg
    off = {name: int(hdr[10 + i]) for i, name in enumerate(SECTIONS)}

    def sec(name, dtype, count):
        o = off[name]
        return np.frombuffer(buf[o:o + count * np.dtype(dtype).itemsize].tobytes(), dtype=dtype)

    nitem = sec("NITEM", np.int32, B + 1)
    nitem_max = int(hdr[10 + len(SECTIONS)])
    nb_act = int(hdr[12 + len(SECTIONS)])          # base windows of this plan
    sy, sx = int(hdr[13 + len(SECTIONS)]), int(hdr[14 + len(SECTIONS)])
    out = {"B": B, "Hg": Hg, "Wg": Wg, "w": w, "halo": halo, "G": G, "nb": nb_act,
           "nb_cap": nb, "nw": nw, "shift": (sy, sx),
           "base": sec("BASE", np.int32, B * nb * 4).reshape(B, nb, 4)[:, :nb_act],
           "score": sec("SCORE", np.float32, B * nb).reshape(B, nb)[:, :nb_act],
           "split": sec("SPLIT", np.uint8, B * nb).reshape(B, nb)[:, :nb_act],
           "nwin": sec("NWIN", np.int32, B),
           "win": sec("WIN", np.int32, B * nw * 4).reshape(B, nw, 4),
           "parent": sec("PARENT", np.int32, B * nw).reshape(B, nw),
           "ext": sec("EXT", np.int32, B * nw * 4).reshape(B, nw, 4),
           "gcount": sec("GCOUNT", np.int32, B * nw).reshape(B, nw),
           "gidx": sec("GIDX", np.int32, B * nw * G).reshape(B, nw, G),
           "wsum": sec("WSUM", np.float32, B * N).reshape(B, N),
           "cover": sec("COVER", np.int32, B * N).reshape(B, N),
           "order": sec("ORDER", np.int32, B * N).reshape(B, N),
           "nitem": nitem,
           "items": sec("ITEMS", np.int32, B * nitem_max * 2).reshape(B, nitem_max, 2),
           "nclass": sec("NCLASS", np.int32, (B + 1) * 4).reshape(B + 1, 4)}
    return out
