"""The bounded waits' timeout path on the GPU, with no fault and no hang.

Every wait of the pipelined kernels gives up after a bounded number of SM
cycles, sets a sticky flag and lets the kernel return. Here a diagnostic
kernel of each family waits, with that same wait function and a short limit,
on a shared-memory barrier nothing completes (a flag that nothing sets): the
wait must give up, the flag must read 1 through qknr_pipeline_error and clear
on reset, and the context must stay usable for an ordinary call afterwards.
"""
import time

import pytest
import torch

import parity
import workloads
import qk_rmsnorm_rope_norm_b200 as qknr
from qk_rmsnorm_rope_norm_b200 import build as qbuild

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    qbuild.build()
    qknr.load_library()
    return torch.device("cuda")


@pytest.mark.parametrize("family", [0, 1], ids=["per-head", "layerwise"])
def test_wait_gives_up_and_reports(cuda, family):
    qknr.pipeline_error(reset=True)
    assert qknr.pipeline_error() == 0
    try:
        t0 = time.perf_counter()
        qknr.wait_selftest(family, limit_cycles=100_000)
        torch.cuda.synchronize()
        waited = time.perf_counter() - t0
        assert waited < 5.0, f"the bounded wait took {waited:.2f} s"
        assert qknr.pipeline_error() == 1          # bit 0: a wait gave up
        assert qknr.pipeline_error(reset=True) == 1
        assert qknr.pipeline_error() == 0          # cleared
    finally:
        qknr.pipeline_error(reset=True)
    # the context is still usable: an ordinary call checks out
    inp = workloads.make_inputs("tiny")
    parity.check(inp, parity.gpu_run(inp))
    assert qknr.pipeline_error() == 0


def test_selftest_rejects_bad_arguments(cuda):
    for fam, lim in ((2, 1000), (-1, 1000), (0, 0), (1, 1 << 40)):
        with pytest.raises(qknr.QKNRError):
            qknr.wait_selftest(fam, lim)
