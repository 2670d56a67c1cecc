"""GPU parity of ``fa_bwd`` (dQ, dK, dV) against the fp64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import assert_fwd_close, assert_grad_close, to_np

pytestmark = pytest.mark.gpu


def _fa():
    import io_aware_exact_16_b200 as fa
    return fa


def run_fwd_bwd(w: workloads.Workload, inp=None):
    fa = _fa()
    inp = inp or workloads.make_inputs(w)
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    sl = inp.seqlens.to(dev) if inp.seqlens is not None else None
    O, lse = fa.forward(q, k, v, causal=w.causal, seqlens=sl, scale=w.scale)
    dq, dk, dv = fa.backward(q, k, v, O, do, lse, causal=w.causal, seqlens=sl, scale=w.scale)
    assert fa.check_device_error() == 0
    return inp, {"o": to_np(O), "lse": to_np(lse), "dq": to_np(dq), "dk": to_np(dk),
                 "dv": to_np(dv)}


def check_against_oracle(w, inp, got):
    ref = oracle.attention_bwd(inp.q, inp.k, inp.v, inp.do, w.scale, w.causal, inp.seqlens)
    assert_fwd_close(got["o"], got["lse"], ref["o"], ref["lse"], w.name)
    for name in ("dq", "dk", "dv"):
        assert_grad_close(got[name], ref[name], name, w.name)


SMALL = [
    (1, 1, 1, 64, False, None),
    (1, 1, 1, 128, True, None),
    (1, 2, 100, 64, False, None),
    (1, 2, 100, 128, True, None),
    (2, 1, 257, 64, True, None),
    (2, 2, 300, 128, False, None),
    (1, 2, 640, 64, True, None),
    (1, 2, 640, 128, True, None),
    (3, 2, 384, 128, False, (1, 384)),
    (4, 2, 333, 64, True, (1, 333)),
    (2, 2, 512, 64, False, (128, 512)),
    (2, 1, 520, 128, True, (100, 520)),
    # causal launches walk groups of 16 heads: B*H = 21 is one full group and a partial one
    (3, 7, 300, 128, True, None),
    (3, 7, 300, 64, True, None),
    (3, 7, 300, 64, True, (70, 300)),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "B{}H{}N{}d{}{}{}".format(
    s[0], s[1], s[2], s[3], "c" if s[4] else "", "pad" if s[5] else ""))
def test_small_shapes_match_oracle(shape):
    B, H, N, d, causal, pad = shape
    w = workloads.custom(B, H, N, d, causal, seed=3000 + N + d, pad_range=pad)
    inp, got = run_fwd_bwd(w)
    check_against_oracle(w, inp, got)


@pytest.mark.parametrize("w", [workloads.tiny(), workloads.gpt2_small(),
                               workloads.bert_large_padded()], ids=lambda w: w.name)
def test_full_configs(w):
    inp, got = run_fwd_bwd(w)
    check_against_oracle(w, inp, got)


def test_backward_is_bitwise_deterministic():
    w = workloads.custom(2, 3, 1000, 128, False, seed=3100)
    inp = workloads.make_inputs(w)
    _, a = run_fwd_bwd(w, inp)
    _, b = run_fwd_bwd(w, inp)
    for name in ("dq", "dk", "dv"):
        np.testing.assert_array_equal(a[name], b[name], err_msg=name)


def test_padded_keys_get_zero_gradient_and_garbage_changes_nothing():
    w = workloads.custom(2, 2, 300, 64, True, seed=3200, pad_range=(30, 200))
    inp = workloads.make_inputs(w)
    _, a = run_fwd_bwd(w, inp)
    k2, v2 = inp.k.clone(), inp.v.clone()
    for bi, L in enumerate(inp.seqlens.tolist()):
        k2[bi, :, L:] = 2.0e4
        v2[bi, :, L:] = -2.0e4
        assert np.all(a["dk"][bi, :, L:] == 0) and np.all(a["dv"][bi, :, L:] == 0)
    _, b = run_fwd_bwd(w, workloads.Inputs(inp.q, k2, v2, inp.do, inp.seqlens))
    for name in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_array_equal(a[name], b[name], err_msg=name)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_persistent_and_per_unit_launches_are_bitwise_identical(d, causal):
    """Head-major launches without key lengths and with more units than SMs run the
    persistent forward (causal or not) and, without the causal mask, the persistent backward;
    passing key lengths that are all N selects the one-CTA-per-unit kernels for the same
    computation.  Both run the same arithmetic in the same order, so every output must match
    bit for bit (and the oracle, on two heads)."""
    w = workloads.custom(4, 16, 1000, d, causal, seed=3300 + d + (7 if causal else 0))
    inp = workloads.make_inputs(w)
    _, a = run_fwd_bwd(w, inp)  # persistent (B*H*ceil(N/256) > SMs)
    full = torch.full((w.B,), w.N, dtype=torch.int32)
    _, b = run_fwd_bwd(w, workloads.Inputs(inp.q, inp.k, inp.v, inp.do, full))
    for name in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_array_equal(a[name], b[name], err_msg=name)
    for flat in workloads.seeded_sample(w.seed, w.B * w.H, 2):
        bi, h = divmod(flat, w.H)
        ref = oracle.head_bwd(inp.q[bi, h], inp.k[bi, h], inp.v[bi, h], inp.do[bi, h], w.scale,
                              causal)
        assert_fwd_close(a["o"][bi, h], a["lse"][bi, h], ref["o"], ref["lse"], f"b{bi} h{h}")
        for name in ("dq", "dk", "dv"):
            assert_grad_close(a[name][bi, h], ref[name], name, f"b{bi} h{h}")
