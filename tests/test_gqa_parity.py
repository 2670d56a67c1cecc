"""GPU parity of grouped-query / multi-query attention (fa_fwd_gqa, fa_bwd_gqa) against the
oracle's grouped-query definition on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import assert_fwd_close, assert_grad_close, to_np

pytestmark = pytest.mark.gpu


def run(w: workloads.Workload, inp=None):
    import io_aware_exact_16_b200 as fa
    inp = inp or workloads.make_inputs(w)
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    sl = inp.seqlens.to(dev) if inp.seqlens is not None else None
    O, lse = fa.forward(q, k, v, causal=w.causal, seqlens=sl, scale=w.scale)
    dq, dk, dv = fa.backward(q, k, v, O, do, lse, causal=w.causal, seqlens=sl, scale=w.scale)
    assert fa.check_device_error() == 0
    assert dk.shape == k.shape and dv.shape == v.shape
    return inp, {"o": to_np(O), "lse": to_np(lse), "dq": to_np(dq), "dk": to_np(dk),
                 "dv": to_np(dv)}


SHAPES = [
    # (B, H, H_kv, N, d, causal, pad_range)
    (2, 8, 2, 300, 128, True, None),
    (1, 6, 1, 257, 64, False, None),        # multi-query attention
    (3, 4, 2, 384, 128, False, (1, 384)),
    (2, 4, 1, 200, 64, True, (50, 200)),
    (2, 12, 4, 1024, 64, True, None),       # GPT-2-small shape with 4 key/value heads
    # causal launches walk groups of 16 heads: B*H_kv = 21 is one full group and a partial one
    (3, 14, 7, 300, 128, True, None),
    (3, 14, 7, 300, 64, True, None),
    # more units than SMs, non-causal, 16 query steps per key block: the persistent forward
    # and backward kernels with two query heads per key/value head
    (4, 32, 16, 1024, 128, False, None),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}H{}kv{}N{}d{}{}{}".format(
    s[0], s[1], s[2], s[3], s[4], "c" if s[5] else "", "pad" if s[6] else ""))
def test_gqa_matches_oracle(shape):
    B, H, H_kv, N, d, causal, pad = shape
    w = workloads.custom(B, H, N, d, causal, seed=6000 + N + H_kv, pad_range=pad, H_kv=H_kv)
    inp, got = run(w)
    ref = oracle.attention_bwd_gqa(inp.q, inp.k, inp.v, inp.do, w.scale, causal, inp.seqlens)
    assert_fwd_close(got["o"], got["lse"], ref["o"], ref["lse"], str(shape))
    for name in ("dq", "dk", "dv"):
        assert_grad_close(got[name], ref[name], name, str(shape))


def test_gqa_backward_is_bitwise_deterministic():
    w = workloads.custom(2, 8, 700, 128, False, seed=6100, H_kv=2)
    inp = workloads.make_inputs(w)
    _, a = run(w, inp)
    _, b = run(w, inp)
    for name in ("dq", "dk", "dv"):
        np.testing.assert_array_equal(a[name], b[name], err_msg=name)
