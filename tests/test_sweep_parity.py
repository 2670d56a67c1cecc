"""GPU parity of the throughput sweep (16384 tokens per batch, B = 16384 / N) against the fp64
oracle: every point N in {512, ..., 16384} x (H16, d128) and (H32, d64) x causal and not.

N <= 2048: forward and backward of every head checked in full.  N >= 4096: two seeded heads
checked in full (the oracle needs N^2 d work per head; the whole batch would take hours on the
host).  At N = 16384 each dQ row sums 128 key blocks, the longest fixed-point sum of the suite.
"""
import pytest

import oracle
import workloads
from tests.gpu_helpers import assert_fwd_close, assert_grad_close
from tests.test_bwd_parity import check_against_oracle, run_fwd_bwd

pytestmark = pytest.mark.gpu

FULL = [workloads.sweep(N, H, d, c) for N in (512, 1024, 2048)
        for (H, d) in workloads.SWEEP_HD for c in (False, True)]
SAMPLED = [workloads.sweep(N, H, d, c) for N in (4096, 8192, 16384)
           for (H, d) in workloads.SWEEP_HD for c in (False, True)]


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name.replace(" ", "-"))
def test_sweep_point_every_head(w):
    inp, got = run_fwd_bwd(w)
    check_against_oracle(w, inp, got)


@pytest.mark.parametrize("w", SAMPLED, ids=lambda w: w.name.replace(" ", "-"))
def test_sweep_point_two_seeded_heads(w):
    inp, got = run_fwd_bwd(w)
    for flat in workloads.seeded_sample(w.seed, w.B * w.H, 2):
        b, h = divmod(flat, w.H)
        ref = oracle.head_bwd(inp.q[b, h], inp.k[b, h], inp.v[b, h], inp.do[b, h], w.scale,
                              w.causal)
        what = f"{w.name} b{b} h{h}"
        assert_fwd_close(got["o"][b, h], got["lse"][b, h], ref["o"], ref["lse"], what)
        for name in ("dq", "dk", "dv"):
            assert_grad_close(got[name][b, h], ref[name], name, what)
