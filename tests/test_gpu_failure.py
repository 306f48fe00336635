"""Device-side failure detection without a GPU fault: a pipeline wait that runs out.

The library's test hook withholds one arrival in the first CTA of the gate_up kernel.
That CTA's bounded wait expires (about 2 s), it drains its copies, frees its tensor
memory and exits; the status word then reads MOE_ERR_TIMEOUT, and the next call on
the same context is correct again.
"""
import numpy as np
import pytest

import mxfp4_expert_gemm_b200 as moe
from _gpu_case import assert_parity, bf16_host, case, oracle_rows, parity_stats
from test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("path", ["gemv", "gemm"])
def test_timed_out_wait_is_reported_and_context_survives(path):
    c = case(SMALL["tiny"])
    cfg = c["cfg"]
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, path=path)
    ws = moe.new_workspace(dims, cfg.T)
    moe.moe_debug_inject_timeout(True)
    moe.moe_forward(dims, c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"], ws)
    assert moe.moe_device_status(ws) == moe.MOE_ERR_TIMEOUT
    # the hook cleared itself; the context still works
    y = moe.moe_forward(dims, c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"], ws)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    assert_parity(parity_stats(bf16_host(y), oracle_rows(c)["y"], c["x"]), path)
