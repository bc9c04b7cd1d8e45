"""The build's check of ptxas -v output for the attention kernels: the window
instantiations must enter with the register count their setmaxnreg split
assumes, and no attention kernel may spill (CPU only)."""
import pytest

from step_adaptive_sparse_b200 import build as b


def _log(entries):
    lines = []
    for name, regs, stores, loads in entries:
        lines += [
            f"ptxas info    : Compiling entry function '{name}' for 'sm_100a'",
            f"ptxas info    : Function properties for {name}",
            f"    0 bytes stack frame, {stores} bytes spill stores, {loads} bytes spill loads",
            f"ptxas info    : Used {regs} registers, used 1 barriers, 400 bytes smem",
        ]
    return "\n".join(lines)


WIN = "_ZN4area12_GLOBAL__N_114attn_tc_kernelILb1ELb0ELi128EEEvNS0_6TcMapsENS0_8TcParamsE"
DENSE = "_ZN4area12_GLOBAL__N_114attn_tc_kernelILb0ELb0ELi128EEEvNS0_6TcMapsENS0_8TcParamsE"
OTHER = "_ZN4area12_GLOBAL__N_116stage_list_kernelILi128EEEvPK13__nv_bfloat16"


def test_good_log_passes():
    assert b.check_attn_resources(_log([(WIN, 168, 0, 0), (DENSE, 165, 0, 0), (OTHER, 40, 8, 8)])) == []


@pytest.mark.parametrize("regs", [160, 176])
def test_window_register_count_is_checked(regs):
    probs = b.check_attn_resources(_log([(WIN, regs, 0, 0), (DENSE, 165, 0, 0)]))
    assert len(probs) == 1 and f"{regs} registers" in probs[0]


def test_dense_register_count_is_free():
    assert b.check_attn_resources(_log([(DENSE, 150, 0, 0)])) == []


@pytest.mark.parametrize("stores,loads", [(4, 0), (0, 8), (60, 104)])
def test_spills_are_reported(stores, loads):
    probs = b.check_attn_resources(_log([(DENSE, 165, stores, loads)]))
    assert len(probs) == 1 and f"{stores} bytes spill stores, {loads} bytes spill loads" in probs[0]


def test_missing_kernel_is_reported():
    assert b.check_attn_resources(_log([(OTHER, 40, 0, 0)]))
