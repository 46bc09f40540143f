"""Failure detection on the GPU without a fault: the bounded barrier waits
that the decode kernels use give up at their time limit, report it through
the device error word, and leave the context usable; a wait called off by
another warp, or completed by it, returns at once."""
import pytest
import torch

import decode_attention_zipfusion_b200 as zf
import zfsynth
from gpu_util import DeviceCase, host_u16

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000_000


def fresh_ws():
    return zf.decode_workspace(1, 8, 1, 16, "cuda")


@pytest.mark.parametrize("mode", [zf.WAITCHECK_TIMEOUT, zf.WAITCHECK_PLAIN_TIMEOUT])
def test_wait_that_nothing_completes_gives_up(mode):
    ws = fresh_ws()
    outcome, ns = zf.check_bounded_wait(mode, ws)
    assert outcome == -1
    assert LIMIT_NS <= ns < LIMIT_NS + 500_000_000
    assert zf.get_device_error(ws) == zf.DEVERR_TIMEOUT
    # the context is still usable: a decode call afterwards is correct
    case = zfsynth.config(0)
    d = DeviceCase(case)
    out_c, lse_c = d.run()
    out_r, lse_r = d.run(compressed=False)
    torch.cuda.synchronize()
    assert zf.get_device_error(d.ws) == 0
    assert (host_u16(out_c) == host_u16(out_r)).all() and torch.equal(lse_c, lse_r)


def test_wait_called_off_by_another_warp():
    ws = fresh_ws()
    outcome, ns = zf.check_bounded_wait(zf.WAITCHECK_ABORT, ws)
    assert outcome == 0
    assert 900_000 <= ns < 100_000_000     # the other warp acts after 1 ms
    assert zf.get_device_error(ws) == 0


def test_wait_completed_by_another_warp():
    ws = fresh_ws()
    outcome, ns = zf.check_bounded_wait(zf.WAITCHECK_COMPLETE, ws)
    assert outcome == 1
    assert 900_000 <= ns < 100_000_000     # the other warp acts after 1 ms
    assert zf.get_device_error(ws) == 0
