"""The device-side timeout path on a B200, without faulting or hanging it.

Every wait in the kernels is bounded.  Here one wait is made to run out on
purpose: the handle is created with MOE_FLAG_TEST_HOLD_PANEL, so its first
forward withholds the publication of one routed up-projection panel, and the
producers of the down-projection stages that need it poll a flag that
nothing sets until a short wait limit runs out.  The test then checks that
  * the forward returns control (its kernels end) and the status word says
    MOE_ERR_DEVICE_TIMEOUT;
  * the CUDA context still works;
  * the next forward of the same handle (limit back to the default) matches
    the fp64 oracle and reports MOE_OK.
"""
import pytest
import torch

from moe_decode_block_b200 import MOE_ERR_DEVICE_TIMEOUT, MOE_FLAG_TEST_HOLD_PANEL, MOE_OK, synth
from gpu_helpers import Run, margin_x, oracle_check

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_reports_a_timeout_and_the_handle_recovers():
    s = synth.TINY
    wts = synth.make_weights(s, seed=0, device="cuda")
    run = Run(s, wts, max_batch=8, extra_flags=MOE_FLAG_TEST_HOLD_PANEL)
    try:
        run.blk.set_wait_limit(1 << 12)
        x = margin_x(4, s.hidden, wts, s.top_k, seed=4)
        run.forward(x)  # synchronises: the kernels ended
        assert run.blk.status() == MOE_ERR_DEVICE_TIMEOUT
        t = torch.arange(1024, device="cuda", dtype=torch.float32)
        assert float(t.sum()) == 1023 * 1024 / 2
        run.blk.set_wait_limit(0)
        for seed in (5, 6):
            x = margin_x(4, s.hidden, wts, s.top_k, seed=seed)
            out, ids, w = run.forward(x)
            oracle_check(wts, s.top_k, x, out, ids, w)
            assert run.blk.status() == MOE_OK
    finally:
        run.blk.close()
