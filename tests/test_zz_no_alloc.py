"""The forward entry point that allocates nothing (moe_forward_no_alloc).

Some callers cannot allocate device memory while they run: an allocator or memory-pool
callback, a plugin host that only lends out its own tensors, or a serving loop that
forbids cudaMalloc (and the synchronization it implies) once it is up.  For them the
library keeps a fixed 16 MiB scratch array in its own device memory instead of taking a
workspace.  This test calls that entry point through the C ABI twice in a row and checks
each result against the ordinary workspace-taking moe_forward, within the parity tests'
tolerance; it also checks that a batch too large for the scratch is refused.

It lives in its own file, named so that pytest collects it last, and passes both alone
in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import mxfp4_expert_gemm_b200 as moe
import synth
from _gpu_case import assert_parity, bf16_host, case, parity_stats

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,path", [("decode_20b", "auto"), ("tiny", "gemm")])
def test_no_alloc_forward_matches_workspace_forward_on_two_calls(name, path):
    cfg = synth.CONFIGS[name]
    c = case(cfg)
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, cfg.rms_eps, cfg.swiglu_limit, path=path)
    args = (c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"])
    ws = moe.new_workspace(dims, cfg.T)
    y_ref = moe.moe_forward(dims, *args, ws)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    ref = bf16_host(y_ref)

    # the caller owns the output and the status word; the entry point allocates nothing
    y = torch.empty_like(c["x_dev"])
    status = torch.empty(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        y.fill_(0)
        status.fill_(-1)
        moe.moe_forward_no_alloc(dims, *args, y=y, status_out=status)
        torch.cuda.synchronize()
        assert int(status.item()) == moe.MOE_OK, f"call {call}"
        got = bf16_host(y)
        assert_parity(parity_stats(got, ref, c["x"]), f"no-alloc call {call}")
        assert np.array_equal(got, ref), f"call {call}: the same kernels on the same inputs differ"


def test_no_alloc_forward_rejects_batches_beyond_its_scratch():
    cfg = synth.CONFIGS["decode_20b"]
    c = case(cfg)
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k)
    T = 1
    while moe.moe_workspace_bytes(dims, T + 1) <= (16 << 20):
        T += 1
    x_big = torch.zeros((T + 1, cfg.d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as err:
        moe.moe_forward_no_alloc(dims, x_big, c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"])
    assert err.value.status == moe.MOE_ERR_WORKSPACE
