"""The device-side failure path, exercised without a fault: every mbarrier
wait in the tensor-core kernels is bounded, and ttt_set_wait_limit shortens
the bound so far that waits run out on an ordinary call.  A wait that runs
out records TTT_EDEVICE in the workspace status word, stops every role of
its kernel, lets the copies and MMAs in flight finish, releases the tensor
memory and returns.  The test checks that the status is reported and that
the next call on the same workspace, with the default bound, succeeds and
matches the oracle: the context stays usable.  No kernel traps, faults or
hangs here; the shortened waits give up within microseconds."""
import pytest
import torch

from test_layer_reconstruction_b200 import inputs as tin
from test_layer_reconstruction_b200 import ttt
from ttt_testlib import TOL_O, TOL_THETA, bf16_inputs, compare_O, compare_theta, oracle_layer, to_device

pytestmark = pytest.mark.gpu

SHORT = 32   # SM clocks: far below a TMA load or an MMA group


def _until_device_fault(call, ws, attempts=6):
    """Run `call` with the short bound until the status word reports a fault."""
    ttt.set_wait_limit(SHORT)
    try:
        for _ in range(attempts):
            call()
            rc = ttt.check_status(ws)
            if rc == -6:
                return True
            assert rc == 0, rc
        return False
    finally:
        ttt.set_wait_limit(0)


# The wide case uses the 2000-view workload's head (d = 1024, h = 2048) on 4
# views, so a GEMM tile's accumulation takes microseconds and its waits run out.
@pytest.mark.parametrize("cfg", [tin.LayerConfig("abort_fused", 6, 37, 37, 5, 4, 64, 256, 2, 0.1, 41),
                                 tin.CONFIGS["views2000_37x37p5_h1_d1024_h2048"].with_views(4)],
                         ids=["fused", "wide"])
def test_wait_runs_out_then_the_next_call_succeeds(cfg):
    inp = bf16_inputs(tin.make_inputs(cfg))
    dev = to_device(inp)
    ws = ttt.make_workspace(cfg, ttt.OP_LAYER)

    def call():
        return ttt.layer(dev["Q"], dev["K"], dev["V"], dev["conv_w"], dev["theta"], cfg.lr, cfg.steps, cfg,
                         workspace=ws)

    assert _until_device_fault(call, ws)
    theta, O = call()
    assert ttt.check_status(ws) == 0
    ref = oracle_layer(cfg, inp, heads=[0, cfg.heads - 1])
    t_err, _ = compare_theta(cfg, inp, theta, ref, heads=[0, cfg.heads - 1])
    assert t_err <= TOL_THETA
    assert compare_O(O, ref, heads=[0, cfg.heads - 1]) <= TOL_O


def test_negative_limit_is_refused():
    with pytest.raises(ttt.TTTError) as e:
        ttt.set_wait_limit(-1)
    assert e.value.status == -1
