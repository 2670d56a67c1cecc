"""GPU parity of the head-dimension-256 kernels (``fa_fwd`` / ``fa_fwd_gqa`` / ``fa_fwd_varlen``
and ``fa_bwd`` / ``fa_bwd_gqa`` with d = 256) against the fp64 oracle on the same seeded bf16
inputs."""
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


def run_fwd(w: workloads.Workload, inp=None):
    fa = _fa()
    inp = inp or workloads.make_inputs(w, with_grad=False)
    dev = torch.device("cuda", 0)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    sl = inp.seqlens.to(dev) if inp.seqlens is not None else None
    O, lse = fa.forward(q, k, v, causal=w.causal, seqlens=sl, scale=w.scale)
    assert fa.check_device_error() == 0
    return inp, to_np(O), to_np(lse)


SMALL = [
    # (B, H, H_kv, N, causal, pad_range): one tile, several tiles with ragged tails, N = 1,
    # padding, grouped-query heads
    (1, 1, 1, 1, False, None),
    (1, 2, 2, 128, True, None),
    (1, 2, 2, 100, False, None),
    (2, 2, 2, 300, True, None),
    (2, 3, 3, 257, False, None),
    (1, 2, 2, 640, True, None),
    (3, 2, 2, 384, False, (1, 384)),
    (2, 2, 2, 520, True, (100, 520)),
    (2, 4, 2, 384, True, None),
    (1, 6, 1, 300, False, None),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "B{}H{}kv{}N{}{}{}".format(
    s[0], s[1], s[2], s[3], "c" if s[4] else "", "pad" if s[5] else ""))
def test_d256_matches_oracle(shape):
    B, H, H_kv, N, causal, pad = shape
    w = workloads.custom(B, H, N, 256, causal, seed=8000 + N + H, pad_range=pad, H_kv=H_kv)
    inp, O, lse = run_fwd(w)
    O_ref, lse_ref = oracle.attention_fwd_gqa(inp.q, inp.k, inp.v, w.scale, causal, inp.seqlens)
    assert_fwd_close(O, lse, O_ref, lse_ref, str(shape))


@pytest.mark.parametrize("causal", [False, True])
def test_d256_long_sequence_sampled_rows(causal):
    """B1 H4 N4096 d256: 2 heads' sampled rows (first, tile edges, last) against the oracle."""
    w = workloads.custom(1, 4, 4096, 256, causal, seed=8100 + int(causal), std=0.5)
    inp, O, lse = run_fwd(w)
    rows = sorted(set([0, 1, 127, 128, 255, 256, 2047, 2048, 4094, 4095] +
                      workloads.seeded_sample(8101, 4096, 54)))
    for h in workloads.seeded_sample(8102, 4, 2):
        O_ref, lse_ref = oracle.head_fwd_rows(inp.q[0, h], inp.k[0, h], inp.v[0, h], rows,
                                              w.scale, causal)
        assert_fwd_close(O[0, h, rows], lse[0, h, rows], O_ref, lse_ref, f"head {h}")


def test_d256_packed_sequences():
    fa = _fa()
    w = workloads.PackedWorkload("d256 packed", 6, 4, 2, 256, True, seed=8200,
                                 lengths=(1, 0, 129, 300, 128, 77))
    inp = workloads.make_packed_inputs(w)
    dev = torch.device("cuda", 0)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    O, lse = fa.forward_varlen(q, k, v, inp.cu_seqlens.to(dev), inp.max_seqlen, causal=True,
                               scale=w.scale)
    assert fa.check_device_error() == 0
    O_ref, lse_ref = oracle.attention_fwd_varlen(inp.q, inp.k, inp.v, inp.cu_seqlens, w.scale,
                                                 True)
    assert_fwd_close(to_np(O), to_np(lse), O_ref, lse_ref, "packed d256")


def test_d256_forward_is_deterministic():
    w = workloads.custom(2, 2, 700, 256, False, seed=8300)
    inp, O1, l1 = run_fwd(w)
    _, O2, l2 = run_fwd(w, inp)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(l1, l2)


def run_fwd_bwd(w: workloads.Workload, inp=None):
    fa = _fa()
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


BWD = [
    # (B, H, H_kv, N, causal, pad_range): one step, ragged tails across 64-query steps and
    # 128-key blocks, N = 1, padding, grouped-query and multi-query heads
    (1, 1, 1, 1, False, None),
    (1, 2, 2, 128, True, None),
    (1, 2, 2, 100, False, None),
    (2, 2, 2, 300, True, None),
    (2, 3, 3, 257, False, None),
    (3, 2, 2, 384, False, (1, 384)),
    (2, 2, 2, 520, True, (100, 520)),
    (2, 4, 2, 384, True, None),
    (1, 6, 1, 300, False, None),
    (1, 2, 2, 1000, True, None),
]


@pytest.mark.parametrize("shape", BWD, ids=lambda s: "B{}H{}kv{}N{}{}{}".format(
    s[0], s[1], s[2], s[3], "c" if s[4] else "", "pad" if s[5] else ""))
def test_d256_backward_matches_oracle(shape):
    B, H, H_kv, N, causal, pad = shape
    w = workloads.custom(B, H, N, 256, causal, seed=8400 + N + H, pad_range=pad, H_kv=H_kv)
    inp, got = run_fwd_bwd(w)
    ref = oracle.attention_bwd_gqa(inp.q, inp.k, inp.v, inp.do, w.scale, causal, inp.seqlens)
    assert_fwd_close(got["o"], got["lse"], ref["o"], ref["lse"], str(shape))
    for name in ("dq", "dk", "dv"):
        assert_grad_close(got[name], ref[name], name, str(shape))


def test_d256_backward_is_bitwise_deterministic():
    w = workloads.custom(2, 4, 700, 256, True, seed=8500, H_kv=2)
    inp = workloads.make_inputs(w)
    _, a = run_fwd_bwd(w, inp)
    _, b = run_fwd_bwd(w, inp)
    for name in ("dq", "dk", "dv"):
        np.testing.assert_array_equal(a[name], b[name], err_msg=name)


@pytest.mark.parametrize("causal", [False, True])
def test_d256_backward_long_sequence_sampled_rows(causal):
    """B1 H2 N4096 d256: dQ at sampled query rows and dK, dV at sampled key rows of both heads
    (first, last, 64-query step and 128-key block edges) against the oracle; each dQ row sums
    the fixed-point contributions of up to 32 key blocks and both feature halves."""
    w = workloads.custom(1, 2, 4096, 256, causal, seed=8600 + int(causal), std=0.5)
    inp, got = run_fwd_bwd(w)
    rows = sorted(set([0, 1, 63, 64, 127, 128, 2047, 2048, 4094, 4095] +
                      workloads.seeded_sample(8601, 4096, 40)))
    for h in range(w.H):
        ref = oracle.head_bwd_rows(inp.q[0, h], inp.k[0, h], inp.v[0, h], inp.do[0, h], rows, rows,
                                   w.scale, causal)
        for name in ("dq", "dk", "dv"):
            assert_grad_close(got[name][0, h, rows], ref[name], name, f"head {h}")
