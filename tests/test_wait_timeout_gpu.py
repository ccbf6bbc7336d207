"""Failure detection: a device-side bounded wait that runs out is reported.

Every mbarrier wait in the kernels gives up after a time limit, records a
status bit and lets its role wind down, so a lost arrive never hangs the GPU;
feql_device_status reports FEQL_ERR_TIMEOUT.  Here a test build of the
library (20 ms limit, one accumulator-release arrive of the forward kernel
left out: libfeql_waittest.so) runs a forward whose CTAs each need to reuse
that accumulator buffer, so the MMA thread's wait for it runs out.  Then the
regular library, in the same process, must still give oracle-exact results:
the context survives.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import group_dft_structured_b200 as F
from group_dft_structured_b200 import build
from group_dft_structured_b200 import layer as Lyr
from group_dft_structured_b200.workloads import make_inputs
from oracle import feql_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    build.build_waittest()
    yield
    F._lib = None
    F.load()


def test_expired_wait_is_reported_and_the_context_stays_usable():
    mode = F.FEQL_FP16
    # 16 -> 16 channels: one 16-column output tile, accumulators double-buffered,
    # each of the SMs' CTAs takes four 128-token tiles, so buffer 0 is reused
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    N, C, D = 128 * sms * 4, 16, 16
    inp = make_inputs(16, N, C, D, "fp16")
    x, W, b = (torch.from_numpy(inp[k]).cuda() for k in ("x", "W", "b"))
    try:
        F._lib = None
        F.load(build.TIMEOUT_LIB)
        What = Lyr.weight_fft(W, mode)
        Lyr.forward(x, What, b, D, mode)
        assert F.feql_device_status() == F.FEQL_ERR_TIMEOUT
        assert F.feql_device_status() == F.FEQL_OK  # the status word was cleared
    finally:
        F._lib = None
        F.load()
    # the regular library on the same context
    What = Lyr.weight_fft(W, mode)
    y = Lyr.forward(x, What, b, D, mode)
    assert F.feql_device_status() == F.FEQL_OK
    r = {k: v.astype(np.float64) for k, v in inp.items()}
    assert O.rel_err(y.double().cpu().numpy(), O.forward(r["x"], r["W"], r["b"])) <= 5e-3
