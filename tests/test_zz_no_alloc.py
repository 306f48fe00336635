"""The forward entry point that allocates nothing (moe_forward_no_alloc).

Some callers cannot allocate device memory while they run: an allocator or memory-pool
callback, a plugin host that only lends out its own tensors, or a serving loop that
forbids cudaMalloc (and the synchronization it implies) once it is up.  For them the
library keeps a fixed 16 MiB scratch array in its own device memory instead of taking a
workspace.  This test calls that entry point through the C ABI twice in a row, on
different inputs (the second call has other tokens and fewer of them, so anything the
first call left in the shared array would show), and checks each result against the CPU
oracle and against the ordinary workspace-taking moe_forward, within the parity tests'
tolerance.  It also checks that a batch too large for the scratch is refused and that an
empty batch reports a clean status.

It lives in its own file, named so that pytest collects it last, and passes both alone
in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import mxfp4_expert_gemm_b200 as moe
import synth
from _gpu_case import assert_parity, bf16_dev, bf16_host, case, oracle_rows, parity_stats

pytestmark = pytest.mark.gpu


def _token_sets(T: int):
    """Two different batches of one workload: every token, then a smaller batch of other
    tokens in another order."""
    first = np.arange(T, dtype=np.int32)
    second = np.arange(T - 1, 0, -3, dtype=np.int32)
    return first, second


@pytest.mark.parametrize("name,path", [("decode_20b", "auto"), ("tiny", "gemm"), ("tiny", "gemv")])
def test_no_alloc_forward_two_calls_match_oracle_and_workspace_forward(name, path):
    cfg = synth.CONFIGS[name]
    c = case(cfg)
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, cfg.rms_eps, cfg.swiglu_limit, path=path)
    weights = (c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"])
    status = torch.empty(1, dtype=torch.int32, device="cuda")
    for call, toks in enumerate(_token_sets(cfg.T)):
        x = bf16_dev(c["x"][toks])
        # the caller owns the output and the status word; the entry point allocates nothing
        y = torch.full_like(x, float("nan"))
        status.fill_(-1)
        moe.moe_forward_no_alloc(dims, x, *weights, y=y, status_out=status)
        torch.cuda.synchronize()
        assert int(status.item()) == moe.MOE_OK, f"call {call}"
        got = bf16_host(y)
        ref = oracle_rows(c, tokens=toks)
        assert_parity(parity_stats(got, ref["y"], c["x"][toks]), f"no-alloc call {call} vs oracle")
        ws = moe.new_workspace(dims, len(toks))
        y_ws = moe.moe_forward(dims, x, *weights, ws)
        assert moe.moe_device_status(ws) == moe.MOE_OK
        assert_parity(parity_stats(got, bf16_host(y_ws), c["x"][toks]), f"no-alloc call {call} vs moe_forward")


def test_no_alloc_forward_rejects_batches_beyond_its_scratch_and_bad_arguments():
    cfg = synth.CONFIGS["decode_20b"]
    c = case(cfg)
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k)
    weights = (c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"])
    T = 1
    while moe.moe_workspace_bytes(dims, T + 1) <= (16 << 20):
        T += 1
    x_big = torch.zeros((T + 1, cfg.d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as err:
        moe.moe_forward_no_alloc(dims, x_big, *weights)
    assert err.value.status == moe.MOE_ERR_WORKSPACE
    # argument errors carry moe_forward's codes
    with pytest.raises(moe.MoeError) as err:
        moe.moe_forward_no_alloc(moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, path=9), c["x_dev"], *weights)
    assert err.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError) as err:
        moe.moe_forward_no_alloc(moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, block=16), c["x_dev"], *weights)
    assert err.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE
    # an empty batch computes nothing and reports a clean status
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    moe.moe_forward_no_alloc(dims, c["x_dev"][:0], *weights, y=torch.empty_like(c["x_dev"][:0]), status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == moe.MOE_OK
