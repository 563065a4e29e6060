"""The tcgen05 operand layouts of the bf16 tensor-core path, checked on fixed synthetic tiles
against the same three-term bf16 products on CUDA cores (gdn_selftest_tc)."""
import pytest

from gated_deltanet_token_b200 import gdn

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", [0, 1, 2, 3, 4, 5])
def test_tc_layout_case(case):
    err, mag = gdn.gdn_selftest_tc(case)
    assert mag > 0.1
    assert err <= 1e-5 * mag, f"case {case}: max |tc - ref| = {err:.3e} (max |ref| = {mag:.3e})"
