"""Failure detection without a GPU fault: the prefill kernel's bounded waits.

`wall_debug_set_fault(1, ms)` makes the producer skip the first key tile, so
the consumers' waits run out after `ms` milliseconds.  The kernel must then
wind down on its own (drain its copies, free tensor memory), report
WALL_ERR_DEVICE_TIMEOUT through the device error word, and leave the context
usable: the next normal call must succeed and match the oracle.  Nothing here
traps, faults or hangs the GPU.
"""
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_util import assert_close

pytestmark = pytest.mark.gpu

WALL_ERR_DEVICE_TIMEOUT = 4


def test_starved_consumers_time_out_and_recover():
    import decayed_softmax_attention_b200 as wall
    spec = W.PrefillSpec("fault", B=1, T=256, HQ=2, H=1, K=128, V=128, dtype="bf16",
                         g_scalar=True, seed=3)
    d = W.gen_prefill(spec, device="cuda")
    assert wall.wall_device_error() == 0
    wall.wall_debug_set_fault(1, 100)
    try:
        wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], scale=d["scale"])
        status = wall.wall_device_error()
    finally:
        wall.wall_debug_set_fault(0, 0)
    assert status == WALL_ERR_DEVICE_TIMEOUT
    # the error word is cleared by the read and the context still works
    o = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], scale=d["scale"])
    assert wall.wall_device_error() == 0
    ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], scale=d["scale"])
    assert_close(o, ro, torch.bfloat16, "after recovery")
