"""A bounded wait that runs out, on the GPU, without stopping a pipeline.

mla_debug_wait_probe lowers the kernels' wait limit to 1 ms and runs one
thread that waits, with the kernels' own wait routine, on a barrier that
nothing arrives on: the wait gives up, the device error word says
MLA_ERR_DEVICE_TIMEOUT, mla_get_last_error reports and clears it, and the
context stays usable (a decode step afterwards matches the oracle).  No copy
or MMA is in flight when the wait gives up.  The file is named to be
collected last.
"""
import pytest

torch = pytest.importorskip("torch")

from head_latent_attention_03_b200 import inputs as I
from head_latent_attention_03_b200 import mla
from tests.test_gpu_parity import check_decode

pytestmark = pytest.mark.gpu

MLA_ERR_DEVICE_TIMEOUT = 5


def test_a_wait_that_runs_out_reports_a_timeout_and_the_context_stays_usable():
    assert mla.get_last_error() == 0
    assert mla.debug_wait_probe(1_000_000) == 0
    assert mla.get_last_error() == MLA_ERR_DEVICE_TIMEOUT
    assert mla.get_last_error() == 0  # read once, then cleared
    # the previous limit is back and the context works: a whole decode step
    # against the oracle, with no error recorded
    check_decode(I.WORKLOADS["tiny"])
    assert mla.get_last_error() == 0
