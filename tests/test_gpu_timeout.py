"""The failure path of the kernels' bounded waits, reached without a GPU fault.

The one-launch expert kernel is told, through the test hook
moe_testing_set_expert_wait, that each layer-2 tile needs one more layer-1
release than will ever come, with a 1 ms limit on its waits.  The forward
must then return, report MOE_DEV_TIMEOUT in moe_stats.status, and leave the
context usable: the next forward on the same buffers (tensor memory freed, no
barrier left armed) matches the float64 oracle."""
import numpy as np
import pytest
import torch

import moe_workloads as mw
import mixture_experts_layer_logit_b200 as moe
from tests.gpu_harness import DeviceLayer
from tests.test_gpu_layer import run_and_check

pytestmark = pytest.mark.gpu

# bf16, k <= 2, T*k < 512*E: the forward runs both expert layers and the
# combine as the one-launch kernel the hook acts on
LAYER = mw.Workload("timeout_relu", T=1000, d=128, E=8, F=256, k=2, act=mw.RELU, dtype=mw.BF16,
                    capacity_factor=1.25, seed=41)


def test_unreachable_dependency_times_out_and_the_next_forward_is_clean():
    L = DeviceLayer(LAYER)
    assert L.T * LAYER.k < 512 * LAYER.E
    moe.moe_testing_set_expert_wait(1_000_000, 1)   # 1 ms; one release too many
    try:
        res = L.forward()
    finally:
        moe.moe_testing_set_expert_wait(0, 0)        # back to the defaults
    st = res["stats"]
    assert st["status"] & moe.MOE_DEV_TIMEOUT, st
    assert not st["status"] & moe.MOE_DEV_BOUNDS, st
    # routing and permutation ran before the expert kernel and are intact
    assert st["rows_kept"] == int(res["offsets"][-1]) > 0
    # the same buffers again, with the default limits: a clean forward
    _, rel, _ = run_and_check(L)
    assert rel <= 2e-2


def test_hook_rejects_bad_values():
    with pytest.raises(moe.MoeError):
        moe.moe_testing_set_expert_wait(61 * 10**9, 0)
    with pytest.raises(moe.MoeError):
        moe.moe_testing_set_expert_wait(0, -1)
    moe.moe_testing_set_expert_wait(0, 0)
