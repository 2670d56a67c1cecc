"""GPU parity of ``fa_fwd`` against the fp64 oracle on the same seeded bf16 inputs."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import assert_fwd_close, to_np

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
    # (B, H, N, d, causal, pad_range)   -- several tiles, ragged tails, degenerate sizes
    (1, 1, 1, 64, False, None),
    (1, 1, 1, 128, True, None),
    (1, 2, 100, 64, False, None),
    (1, 2, 100, 128, True, None),
    (2, 1, 257, 64, True, None),
    (2, 2, 300, 128, False, None),
    (1, 3, 640, 64, True, None),
    (1, 2, 640, 128, True, None),
    (3, 2, 384, 128, False, (1, 384)),
    (4, 2, 333, 64, True, (1, 333)),
    (2, 2, 512, 64, False, (128, 512)),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "B{}H{}N{}d{}{}{}".format(
    s[0], s[1], s[2], s[3], "c" if s[4] else "", "pad" if s[5] else ""))
def test_small_shapes_match_oracle(shape):
    B, H, N, d, causal, pad = shape
    w = workloads.custom(B, H, N, d, causal, seed=2000 + N + d, pad_range=pad)
    inp, O, lse = run_fwd(w)
    O_ref, lse_ref = oracle.attention_fwd(inp.q, inp.k, inp.v, w.scale, causal, inp.seqlens)
    assert_fwd_close(O, lse, O_ref, lse_ref, str(shape))


def test_tiny_config():
    w = workloads.tiny()
    inp, O, lse = run_fwd(w)
    O_ref, lse_ref = oracle.attention_fwd(inp.q, inp.k, inp.v, w.scale, w.causal, inp.seqlens)
    assert_fwd_close(O, lse, O_ref, lse_ref, w.name)


@pytest.mark.parametrize("w", [workloads.gpt2_small(), workloads.bert_large_padded()],
                         ids=lambda w: w.name)
def test_full_configs(w):
    inp, O, lse = run_fwd(w)
    O_ref, lse_ref = oracle.attention_fwd(inp.q, inp.k, inp.v, w.scale, w.causal, inp.seqlens)
    assert_fwd_close(O, lse, O_ref, lse_ref, w.name)


def test_padded_keys_with_large_garbage_do_not_change_output():
    """Keys past L_b hold large finite values: masked keys must contribute exactly nothing."""
    w = workloads.custom(2, 2, 300, 128, False, seed=2100, pad_range=(40, 200))
    inp = workloads.make_inputs(w, with_grad=False)
    _, O1, lse1 = run_fwd(w, inp)
    k2, v2 = inp.k.clone(), inp.v.clone()
    for b, L in enumerate(inp.seqlens.tolist()):
        k2[b, :, L:] = 3.0e4
        v2[b, :, L:] = -3.0e4
    inp2 = workloads.Inputs(inp.q, k2, v2, inp.do, inp.seqlens)
    _, O2, lse2 = run_fwd(w, inp2)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(lse1, lse2)


def test_forward_is_deterministic():
    w = workloads.custom(2, 3, 700, 64, True, seed=2200)
    inp = workloads.make_inputs(w, with_grad=False)
    _, O1, l1 = run_fwd(w, inp)
    _, O2, l2 = run_fwd(w, inp)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("N", [8192])
def test_long_context_sampled_rows(N):
    """Long-context config: every row of 2 seeded heads, plus 256 seeded rows of every head."""
    w = workloads.long_context(N)
    inp, O, lse = run_fwd(w)
    heads = workloads.seeded_sample(w.seed, w.H, 2)
    for h in heads:
        O_ref, lse_ref = oracle.head_fwd(inp.q[0, h], inp.k[0, h], inp.v[0, h], w.scale, True)
        assert_fwd_close(O[0, h], lse[0, h], O_ref, lse_ref, f"head {h}")
    rows = sorted(set(workloads.seeded_sample(w.seed + 1, N, 250) + [0, 127, 128, 255, 256, N - 1]))
    for h in range(w.H):
        O_ref, lse_ref = oracle.head_fwd_rows(inp.q[0, h], inp.k[0, h], inp.v[0, h], rows, w.scale, True)
        assert_fwd_close(O[0, h, rows], lse[0, h, rows], O_ref, lse_ref, f"head {h} rows")


@pytest.mark.parametrize("N", [16384, 32768])
def test_long_context_longer_sampled_rows(N):
    """Long-context config at 16K and 32K: 256 seeded rows of every head (plus the first and
    last rows and tile edges).  Whole heads would need an N x N fp64 score matrix on the host
    (8.6 GB at 32K), so these sizes check sampled rows only."""
    w = workloads.long_context(N)
    inp, O, lse = run_fwd(w)
    rows = sorted(set(workloads.seeded_sample(w.seed + 2, N, 250) +
                      [0, 127, 128, 255, 256, N // 2, N - 129, N - 128, N - 1]))
    for h in range(w.H):
        O_ref, lse_ref = oracle.head_fwd_rows(inp.q[0, h], inp.k[0, h], inp.v[0, h], rows, w.scale, True)
        assert_fwd_close(O[0, h, rows], lse[0, h, rows], O_ref, lse_ref, f"N {N} head {h} rows")


def test_forward_memory_is_inputs_plus_outputs():
    """The forward allocates nothing on the device: with O and lse preallocated, the peak
    allocation over the call equals what was resident before it (Q, K, V, O, lse), which
    doubles with N (long-context config, 8K -> 16K -> 32K); the N x N score matrix (16 N^2
    bytes in bf16 for 16 heads) is never materialised."""
    fa = _fa()
    dev = torch.device("cuda", 0)
    totals = []
    for N in (8192, 16384, 32768):
        w = workloads.long_context(N)
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        q, k, v = (torch.randn(1, w.H, N, w.d, device=dev).to(torch.bfloat16) for _ in range(3))
        o = torch.empty_like(q)
        lse = torch.empty((1, w.H, N), dtype=torch.float32, device=dev)
        fa.forward(q, k, v, causal=True, out=o, lse=lse)  # first call: per-device state
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        fa.forward(q, k, v, causal=True, out=o, lse=lse)
        torch.cuda.synchronize()
        assert fa.check_device_error() == 0
        assert torch.cuda.max_memory_allocated(dev) == before
        io_bytes = 4 * w.H * N * w.d * 2 + w.H * N * 4
        totals.append(io_bytes)
        assert sum(t.numel() * t.element_size() for t in (q, k, v, o, lse)) == io_bytes
        del q, k, v, o, lse
    assert totals[1] == 2 * totals[0] and totals[2] == 2 * totals[1]
