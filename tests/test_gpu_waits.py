"""Bounded device waits driven to expiry on the GPU, without a fault or a hang.

The one-launch planner (area_dwt_window_plan) is a cooperative launch whose
blocks meet at grid barriers; every barrier wait is bounded, and on expiry the
block raises an abort word and returns, so the launch ends and the context
stays usable.  The test hook area_test_plan_barrier_expiry sets every barrier
target one above the number of blocks (no barrier can complete) and bounds
each wait by 1 ms.  The test checks that the call returns, that
area_kernel_error reports the planner's bit, and that a normal call right after
it is still bit-exact.

The tensor-core attention kernel's mbarrier waits are bounded the same way,
but they guard TMA copies and tensor-core work in flight; forcing one of them
to expire would abandon that work mid-way, so that path is not driven on a GPU.
"""
import time

import numpy as np
import pytest
import torch

from oracle import area_oracle as ora
import gpu_runner as gr

pytestmark = pytest.mark.gpu


def _inputs(seed=7, B=1, Hg=64, Wg=48, C=16):
    rng = np.random.default_rng(seed)
    src = rng.standard_normal((B, Hg * Wg, C)).astype(np.float32)
    src[:, : Hg * Wg // 3] *= 0.05
    dsrc = gr.to_dev(src, "bf16")
    return gr.to_host(dsrc).astype(np.float32), dsrc


def test_plan_barrier_expiry_reports_and_recovers():
    B, Hg, Wg, C, w, h, G, thr = 1, 64, 48, 16, 24, 4, 130, 0.3
    src, dsrc = _inputs(B=B, Hg=Hg, Wg=Wg, C=C)
    pcfg = gr.area.make_cfg(B, Hg, Wg, w, h, G, thr)
    nb = gr.area.area_window_plan_bytes(pcfg)
    plan = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    energy = torch.zeros((B, Hg // 2, Wg // 2), dtype=torch.float32, device="cuda")
    assert gr.area.area_kernel_error() == 0
    t0 = time.perf_counter()
    gr.area.area_test_plan_barrier_expiry(dsrc, gr.area.AREA_DTYPE_BF16, C, energy, pcfg, plan,
                                          nb)
    torch.cuda.synchronize()
    took = time.perf_counter() - t0
    assert took < 5.0, f"the expired launch took {took:.2f} s"
    assert gr.area.area_kernel_error() == gr.area.AREA_KERR_PLAN_BARRIER
    assert gr.area.area_kernel_error() == 0            # read and cleared
    # the same buffers, a normal call: bit-exact against the oracle
    gr.area.area_dwt_window_plan(dsrc, gr.area.AREA_DTYPE_BF16, C, gr.area.AREA_DETAIL_HH,
                                 energy, pcfg, plan, nb)
    torch.cuda.synchronize()
    assert gr.area.area_kernel_error() == 0
    E = ora.dwt_detail(src, Hg, Wg)
    assert np.array_equal(energy.cpu().numpy().view(np.uint32), E.view(np.uint32))
    want = ora.window_plan(E[0], Hg, Wg, w, h, G, thr)
    gr.compare_plan(gr.parse(plan), want)


def test_plan_barrier_expiry_twice_in_a_row():
    # the abort word and the arrival counter are reset by every launch
    B, Hg, Wg, C = 2, 40, 28, 16
    _, dsrc = _inputs(seed=3, B=B, Hg=Hg, Wg=Wg, C=C)
    pcfg = gr.area.make_cfg(B, Hg, Wg, 12, 6, 9, 0.2, 99)
    nb = gr.area.area_window_plan_bytes(pcfg)
    plan = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    energy = torch.zeros((B, Hg // 2, Wg // 2), dtype=torch.float32, device="cuda")
    for _ in range(2):
        gr.area.area_test_plan_barrier_expiry(dsrc, gr.area.AREA_DTYPE_BF16, C, energy, pcfg,
                                              plan, nb)
        torch.cuda.synchronize()
        assert gr.area.area_kernel_error() == gr.area.AREA_KERR_PLAN_BARRIER
    ref = torch.zeros_like(plan)
    e_ref = torch.zeros_like(energy)
    gr.area.area_dwt_detail(dsrc, gr.area.AREA_DTYPE_BF16, C, e_ref, B, Hg, Wg,
                            gr.area.AREA_DETAIL_HH)
    gr.area.area_window_plan(e_ref, pcfg, ref, nb)
    gr.area.area_dwt_window_plan(dsrc, gr.area.AREA_DTYPE_BF16, C, gr.area.AREA_DETAIL_HH,
                                 energy, pcfg, plan, nb)
    torch.cuda.synchronize()
    assert gr.area.area_kernel_error() == 0
    hdr = ref[:256].cpu().numpy().view(np.int64)
    end = int(hdr[10 + gr.area.SECTIONS.index("SCRATCH")])
    assert torch.equal(plan[:end], ref[:end])
    assert torch.equal(energy.view(torch.int32), e_ref.view(torch.int32))
