"""The build's register guard: a prefill kernel whose compiled register count
differs from the launch allocation its register split assumes fails build()."""

import re

import pytest

from paged_kv_cache_exact_b200 import build


def _want():
    src = open(build.os.path.join(build.CSRC, "prefill_sm100.cu")).read()
    return int(re.search(r"constexpr\s+int\s+kLaunchRegs\s*=\s*(\d+)\s*;", src).group(1))


def _log(n):
    return ("ptxas info    : Compiling entry function '_ZN3pkv14prefill_kernelILb0ELb0EEEv' "
            "for 'sm_100a'\n"
            f"ptxas info    : Used {n} registers, used 1 barriers\n"
            "ptxas info    : Compiling entry function '_ZN3pkv13combine_kernelEv' for 'sm_100a'\n"
            "ptxas info    : Used 40 registers\n")


def test_register_guard_accepts_the_declared_count():
    build.check_launch_registers("prefill_sm100.cu", _log(_want()))


@pytest.mark.parametrize("delta", [-8, 8])
def test_register_guard_rejects_another_count(delta):
    with pytest.raises(RuntimeError, match="registers"):
        build.check_launch_registers("prefill_sm100.cu", _log(_want() + delta))


def test_register_guard_rejects_a_log_without_the_kernel():
    with pytest.raises(RuntimeError, match="no 'prefill_kernel'"):
        build.check_launch_registers("prefill_sm100.cu", "ptxas info    : Used 40 registers\n")
