"""Failure detection on the GPU without a fault: the bounded barrier waits
that the decode kernels use give up at their time limit, report it through
the device error word, and leave the context usable; a wait called off by
another warp, or completed by it, returns at once."""
import numpy as np
import pytest
import torch

import decode_attention_zipfusion_b200 as zf
import oracle
import zfsynth
from gpu_util import DeviceCase, dev_bf16, host_u16, host_u32

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


def test_compress_lookback_that_nothing_completes_gives_up():
    """The compress kernel's look-back, waiting on a predecessor tile that
    never publishes, gives up at the limit and reports it; a compress
    afterwards is still bit-exact to the oracle."""
    ws = fresh_ws()
    outcome, ns = zf.check_bounded_wait(zf.WAITCHECK_LOOKBACK_TIMEOUT, ws)
    assert outcome == -1
    assert LIMIT_NS <= ns < LIMIT_NS + 500_000_000
    assert zf.get_device_error(ws) == zf.DEVERR_TIMEOUT
    vals = zfsynth.config(1, scale_ctx=1 / 16).k_pool.reshape(-1)
    ref = oracle.compress(vals)
    z = zf.compress(dev_bf16(vals))
    torch.cuda.synchronize()
    assert z.units() == ref.units
    assert np.array_equal(host_u32(z.offs), ref.offs)
    assert np.array_equal(z.payload[: ref.units * 16].cpu().numpy(), ref.payload)


def test_compress_lookback_completed_by_another_warp():
    """The same look-back, when the missing predecessor publishes its
    aggregate after 1 ms, ends with the right prefix (10 + 7 + 7 + 5 + 3)."""
    ws = fresh_ws()
    outcome, ns = zf.check_bounded_wait(zf.WAITCHECK_LOOKBACK_COMPLETE, ws)
    assert outcome == 1
    assert 900_000 <= ns < 100_000_000
    assert zf.get_device_error(ws) == 0


def test_compress_kernel_with_a_withheld_stage_gives_up():
    """The compress kernel itself, with one CTA's first stage fill withheld:
    its compute warps' stage wait gives up at the limit and stops that CTA
    (its loader and look-back warp follow, the loader after a bounded wait
    for its fills), the other CTAs' look-backs give up on the tile that never
    publishes, and the launch ends with ZF_DEVERR_TIMEOUT; a compress
    afterwards is still bit-exact to the oracle."""
    ws = fresh_ws()
    outcome, ns = zf.check_bounded_wait(zf.WAITCHECK_COMPRESS_STALL, ws)
    assert outcome == -1
    assert LIMIT_NS <= ns < 4 * LIMIT_NS
    assert zf.get_device_error(ws) == zf.DEVERR_TIMEOUT
    vals = zfsynth.config(1, scale_ctx=1 / 16).k_pool.reshape(-1)
    ref = oracle.compress(vals)
    z = zf.compress(dev_bf16(vals))
    torch.cuda.synchronize()
    assert z.units() == ref.units
    assert np.array_equal(host_u32(z.offs), ref.offs)
    assert np.array_equal(z.payload[: ref.units * 16].cpu().numpy(), ref.payload)
