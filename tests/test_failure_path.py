"""GPU check of the failure path the kernels share: a bounded wait that nothing completes gives
up after the limit, reports FA_ERR_TIMEOUT through the device error flag, and leaves the
context usable.  No fault, trap or endless loop is involved."""
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import assert_fwd_close, to_np

pytestmark = pytest.mark.gpu

DEFAULT_TIMEOUT_NS = 4_000_000_000  # the library's initial wait limit


def test_bounded_wait_times_out_and_the_context_stays_usable():
    import io_aware_exact_16_b200 as fa
    assert fa.check_device_error() == 0
    fa.set_wait_timeout_ns(2_000_000)  # 2 ms
    try:
        fa.selftest_wait_timeout()
        assert fa.check_device_error() == fa.FA_ERR_TIMEOUT
        assert fa.check_device_error() == 0  # read and cleared
    finally:
        fa.set_wait_timeout_ns(DEFAULT_TIMEOUT_NS)
    # the same context keeps computing correct results
    w = workloads.custom(1, 2, 300, 128, True, seed=9900)
    inp = workloads.make_inputs(w, with_grad=False)
    dev = torch.device("cuda", 0)
    O, lse = fa.forward(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), causal=True, scale=w.scale)
    assert fa.check_device_error() == 0
    O_ref, lse_ref = oracle.attention_fwd(inp.q, inp.k, inp.v, w.scale, True)
    assert_fwd_close(to_np(O), to_np(lse), O_ref, lse_ref, "after a timed-out wait")
