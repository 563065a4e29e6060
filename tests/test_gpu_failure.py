"""Failure detection on the GPU without a fault: a bounded device-side wait that runs out.

The diagnostic kernel waits on an mbarrier that nothing completes (no copy or MMA is ever in
flight) with the same bounded wait as the prefill kernels, the limit shortened to 1 ms.  The
kernel must return by itself, the status word must read GDN_ERR_DEVICE_TIMEOUT once and then
GDN_OK, and an ordinary prefill right after it must still match the oracle: the context
stays usable."""
import numpy as np
import pytest
import torch

from gated_deltanet_token_b200 import gdn
from gated_deltanet_token_b200.inputs import make_inputs
from tests._helpers import check_bf16, run_prefill

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_the_context_stays_usable(oracle_mod):
    assert gdn.gdn_read_device_status() in (gdn.GDN_OK, gdn.GDN_ERR_DEVICE_TIMEOUT)  # clear it
    gdn.gdn_set_wait_limit_ns(1_000_000)
    try:
        gdn.gdn_selftest_wait_timeout()
        assert gdn.gdn_read_device_status() == gdn.GDN_ERR_DEVICE_TIMEOUT
        assert gdn.gdn_read_device_status() == gdn.GDN_OK  # read and cleared
    finally:
        gdn.gdn_set_wait_limit_ns(2_000_000_000)
    inp = make_inputs("varlen8_prefill_bf16", lengths=[70, 5, 130], h_qk=2, h_v=4)
    ref = oracle_mod.prefill(inp)
    y, S = run_prefill(inp, torch.float32)
    check_bf16(y, ref["y"], S, ref["final_state"])
    assert gdn.gdn_read_device_status() == gdn.GDN_OK
    assert np.isfinite(y).all()


def test_wait_limit_rejects_zero():
    with pytest.raises(gdn.GdnError):
        gdn.gdn_set_wait_limit_ns(0)
