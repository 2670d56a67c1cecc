"""GPU parity of packed variable-length attention (fa_fwd_varlen, fa_bwd_varlen) against the
oracle's per-sequence definition on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import assert_fwd_close, assert_grad_close, to_np

pytestmark = pytest.mark.gpu

SENTINEL = 7.0  # rows outside every sequence must keep what the caller put there


def run(w: workloads.PackedWorkload, inp=None, extra_rows=0):
    """Forward + backward through the binding; `extra_rows` rows past the last sequence are
    appended to every tensor so that the test can check they are never written."""
    import io_aware_exact_16_b200 as fa
    inp = inp or workloads.make_packed_inputs(w)
    dev = torch.device("cuda", 0)

    def pad(t):
        if extra_rows == 0:
            return t.to(dev)
        tail = torch.full((extra_rows,) + tuple(t.shape[1:]), SENTINEL, dtype=t.dtype)
        return torch.cat([t, tail]).to(dev)

    q, k, v, do = (pad(t) for t in (inp.q, inp.k, inp.v, inp.do))
    cu = inp.cu_seqlens.to(dev)
    T = q.shape[0]
    out = torch.full_like(q, SENTINEL)
    lse = torch.full((w.H, T), SENTINEL, dtype=torch.float32, device=dev)
    O, lse = fa.forward_varlen(q, k, v, cu, inp.max_seqlen, causal=w.causal, scale=w.scale,
                               out=out, lse=lse)
    dq, dk, dv = (torch.full_like(t, SENTINEL) for t in (q, k, v))
    dq, dk, dv = fa.backward_varlen(q, k, v, O, do, lse, cu, inp.max_seqlen, causal=w.causal,
                                    scale=w.scale, dq=dq, dk=dk, dv=dv)
    assert fa.check_device_error() == 0
    return inp, {"o": to_np(O), "lse": to_np(lse), "dq": to_np(dq), "dk": to_np(dk),
                 "dv": to_np(dv)}


CASES = [
    # name, B, H, H_kv, d, causal, len_range, fixed lengths
    ("mixed d128", 6, 4, 4, 128, False, (1, 400), None),
    ("mixed d128 causal gqa", 5, 8, 2, 128, True, (1, 400), None),
    ("mixed d64 causal", 7, 4, 4, 64, True, (1, 300), None),
    ("mqa d64", 4, 6, 1, 64, False, (100, 300), None),
    ("edges d128", 7, 2, 1, 128, True, None, (1, 0, 128, 129, 256, 0, 37)),
    ("edges d64", 5, 3, 3, 64, False, None, (255, 1, 0, 384, 2)),
    ("edges d256 causal gqa", 6, 4, 2, 256, True, None, (1, 0, 129, 300, 128, 77)),
    ("mixed d256", 4, 2, 2, 256, False, (1, 300), None),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_varlen_matches_oracle(case):
    name, B, H, H_kv, d, causal, rng, lens = case
    w = workloads.PackedWorkload(name, B, H, H_kv, d, causal, seed=7000 + B * 10 + d,
                                 len_range=rng or (1, 1), lengths=lens)
    extra = 3
    inp, got = run(w, extra_rows=extra)
    T = inp.q.shape[0]
    ref = oracle.attention_bwd_varlen(inp.q, inp.k, inp.v, inp.do, inp.cu_seqlens, w.scale, causal)
    used = int(inp.cu_seqlens[-1])
    rows = slice(0, used)
    assert_fwd_close(got["o"][rows], got["lse"][:, rows], ref["o"][rows], ref["lse"][:, rows], name)
    for g in ("dq", "dk", "dv"):
        assert_grad_close(got[g][rows], ref[g][rows], g, name)
    # Nothing past the last sequence is written.
    for g in ("o", "dq", "dk", "dv"):
        assert np.all(got[g][used:] == SENTINEL), g
    assert np.all(got["lse"][:, used:] == SENTINEL)
    assert got["o"].shape[0] == T + extra


def test_varlen_equals_padded_head_major_per_sequence():
    """Each packed sequence gives the same bits as the same sequence alone in the head-major
    layout (same kernels, same reduction order)."""
    import io_aware_exact_16_b200 as fa
    w = workloads.PackedWorkload("eq", 3, 4, 2, 128, True, seed=7100, lengths=(300, 77, 513))
    inp, got = run(w)
    dev = torch.device("cuda", 0)
    cu = inp.cu_seqlens.tolist()
    for b in range(w.B):
        t0, t1 = cu[b], cu[b + 1]
        hm = [x[t0:t1].transpose(0, 1).unsqueeze(0).contiguous().to(dev)
              for x in (inp.q, inp.k, inp.v, inp.do)]
        O, lse = fa.forward(hm[0], hm[1], hm[2], causal=True, scale=w.scale)
        dq, dk, dv = fa.backward(hm[0], hm[1], hm[2], O, hm[3], lse, causal=True, scale=w.scale)
        np.testing.assert_array_equal(to_np(O[0].transpose(0, 1)), got["o"][t0:t1])
        np.testing.assert_array_equal(to_np(lse[0]), got["lse"][:, t0:t1])
        np.testing.assert_array_equal(to_np(dk[0].transpose(0, 1)), got["dk"][t0:t1])
        np.testing.assert_array_equal(to_np(dv[0].transpose(0, 1)), got["dv"][t0:t1])
        np.testing.assert_array_equal(to_np(dq[0].transpose(0, 1)), got["dq"][t0:t1])


def test_varlen_backward_is_bitwise_deterministic():
    w = workloads.PackedWorkload("det", 4, 4, 2, 128, False, seed=7200, len_range=(200, 700))
    inp = workloads.make_packed_inputs(w)
    _, a = run(w, inp)
    _, b = run(w, inp)
    for g in ("dq", "dk", "dv"):
        np.testing.assert_array_equal(a[g], b[g], err_msg=g)


def test_varlen_bad_offsets_are_reported_not_faulted():
    """A sequence longer than max_seqlen is skipped and reported as FA_ERR_INVALID_ARG."""
    import io_aware_exact_16_b200 as fa
    dev = torch.device("cuda", 0)
    q = torch.zeros((300, 2, 64), dtype=torch.bfloat16, device=dev)
    cu = torch.tensor([0, 100, 300], dtype=torch.int32, device=dev)
    fa.forward_varlen(q, q, q, cu, 150)
    assert fa.check_device_error() == fa.FA_ERR_INVALID_ARG
    assert fa.check_device_error() == 0
