"""Failure paths on the GPU, exercised without faulting or hanging it.

* A bounded in-kernel wait that runs out: a test hook adds one to the decode
  split barrier's arrival target, so no CTA can ever see it reached, and
  shortens the wait limit to 2 ms.  Every CTA gives up, the kernel returns,
  sdpa_check_device_error reports SDPA_ERR_TIMEOUT with the barrier's code,
  and the next call on the same stream is correct again.
* A split-K workspace that cannot be allocated: a test hook makes the
  allocation fail; the call returns SDPA_ERR_NO_MEMORY with nothing launched,
  and the next call on the stream succeeds.
"""
import numpy as np
import pytest
import torch

import scaled_dot_product_14_b200 as S
from scaled_dot_product_14_b200 import inputs as I

from gpu_util import GpuCase, compare

pytestmark = pytest.mark.gpu

KERR_WAIT_SPLITS = 5   # device error code of the decode split barrier


@pytest.fixture(scope="module", autouse=True)
def built():
    from scaled_dot_product_14_b200 import build
    import oracle
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


@pytest.fixture
def hooks_reset():
    yield
    for knob in (S.SDPA_DEBUG_WAIT_LIMIT_NS, S.SDPA_DEBUG_DECODE_BARRIER_EXTRA, S.SDPA_DEBUG_FAIL_ALLOCS):
        S.sdpa_debug_set(knob, 0)


def _decode_case(seed=2001):
    return I.make_case(seed, 1, 32, 8, 1, 4096, 256, dtype=I.BF16, mask="decode_additive")


def test_decode_barrier_wait_runs_out_and_the_stream_recovers(hooks_reset):
    c = _decode_case()
    stream = torch.cuda.Stream()
    sp = stream.cuda_stream
    with torch.cuda.stream(stream):
        warm = GpuCase(c)
        assert warm.run(sp) == 0                 # allocates the stream's workspace
        stream.synchronize()
        assert S.sdpa_check_device_error(sp) == (0, 0)
        assert S.sdpa_debug_set(S.SDPA_DEBUG_WAIT_LIMIT_NS, 2_000_000) == 0
        assert S.sdpa_debug_set(S.SDPA_DEBUG_DECODE_BARRIER_EXTRA, 1) == 0
        bad = GpuCase(c)
        assert bad.run(sp) == 0                  # launched; the failure is on the device
        st, code = S.sdpa_check_device_error(sp)
        assert st == 7 and code == KERR_WAIT_SPLITS, (st, code)
        # the output of the timed-out call was not written (guard value NaN everywhere)
        assert np.isnan(bad.out_buf.float().cpu().numpy()).all()
        S.sdpa_debug_set(S.SDPA_DEBUG_DECODE_BARRIER_EXTRA, 0)
        S.sdpa_debug_set(S.SDPA_DEBUG_WAIT_LIMIT_NS, 0)
        assert S.sdpa_check_device_error(sp) == (0, 0)   # the flag was cleared
        for _ in range(2):                       # the same stream and workspace are correct again
            good = GpuCase(c)
            assert good.run(sp) == 0
            compare(c, good.output(), label="after timeout")
        assert S.sdpa_check_device_error(sp) == (0, 0)


def test_forced_workspace_allocation_failure_launches_nothing(hooks_reset):
    c = _decode_case(2002)
    stream = torch.cuda.Stream()                 # no workspace exists for it yet
    sp = stream.cuda_stream
    g = GpuCase(c)
    torch.cuda.synchronize()
    before = S.sdpa_get_counters()
    assert S.sdpa_debug_set(S.SDPA_DEBUG_FAIL_ALLOCS, 1) == 0
    assert g.run(sp) == 8                        # SDPA_ERR_NO_MEMORY
    assert S.sdpa_last_launch_count() == 0
    after = S.sdpa_get_counters()
    assert after["decode_mma_launches"] == before["decode_mma_launches"]
    assert after["rejected_calls"] == before["rejected_calls"] + 1
    stream.synchronize()
    assert np.isnan(g.out_buf.float().cpu().numpy()).all()
    # the hook was one-shot: the next call allocates and is correct
    assert g.run(sp) == 0
    compare(c, g.output(), label="after forced allocation failure")
