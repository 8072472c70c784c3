"""Failure detection without a GPU fault: a bounded device-side wait that
runs out reports SSD_ERR_TIMEOUT through the status word, the context stays
usable, and the host-side checks reject bad calls before any launch."""

import pytest

from parity import TOL, gpu_fwd, oracle_fwd, rel_err
from ssd_chunked_scan_02_b200 import build as ssd_build
from ssd_chunked_scan_02_b200 import inputs, ssd


@pytest.fixture(scope="module")
def lib():
    ssd_build.build()
    return ssd.load()


def test_expire_wait_rejects_bad_poll_counts(lib):
    assert lib.ssd_debug_expire_wait(0, None) == ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_debug_expire_wait((1 << 20) + 1, None) == ssd.SSD_ERR_INVALID_ARG


@pytest.mark.gpu
def test_bounded_wait_times_out_and_context_survives(lib):
    ssd.ssd_poll_device_status()                      # clear anything left over
    ssd.ssd_debug_expire_wait(4096)                   # a wait nothing will satisfy
    with pytest.raises(ssd.SSDError) as e:
        ssd.ssd_poll_device_status()
    assert e.value.status == ssd.SSD_ERR_TIMEOUT
    ssd.ssd_poll_device_status()                      # cleared by the read: no error now
    # the context is intact: a tensor-core forward still matches the oracle
    w = inputs.Workload("after_timeout", 1, 300, 4, 64, 128, 1, 256, "bf16", with_init=True,
                        want_final=True, seed=61)
    inp = inputs.make_inputs(w)
    y, f = gpu_fwd(inp, 256)
    y_ref, f_ref = oracle_fwd(inp)
    assert rel_err(y, y_ref) <= TOL["bf16"] and rel_err(f, f_ref) <= TOL["bf16"]
    ssd.ssd_poll_device_status()                      # and no wait gave up during it
