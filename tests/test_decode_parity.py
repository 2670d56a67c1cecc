"""GPU parity of split-KV decode (``fa_fwd_decode``) against the oracle's decode definition on
the same seeded bf16 inputs."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import assert_fwd_close, to_np

pytestmark = pytest.mark.gpu


def _inputs(B, H, H_kv, Nq, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, H, Nq, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, H_kv, N, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, H_kv, N, d), generator=g).to(torch.bfloat16)
    return q, k, v


def run(q, k, v, lens, causal, splits):
    import io_aware_exact_16_b200 as fa
    dev = torch.device("cuda", 0)
    cl = torch.tensor(lens, dtype=torch.int32, device=dev) if lens is not None else None
    O, lse = fa.decode(q.to(dev), k.to(dev), v.to(dev), cache_lens=cl, causal=causal,
                       splits=splits)
    assert fa.check_device_error() == 0
    return to_np(O), to_np(lse)


CASES = [
    # B, H, H_kv, Nq, N, d, causal, cache lengths, splits (0 = automatic)
    (2, 8, 2, 1, 1000, 128, False, None, 0),
    (3, 8, 8, 1, 777, 64, False, [777, 1, 300], 0),
    (2, 32, 4, 4, 2048, 128, True, [2048, 1500], 0),
    (1, 4, 1, 16, 513, 256, True, None, 3),
    (2, 16, 1, 10, 300, 128, True, [300, 5], 1),     # Nq > L_b: early queries see no key
    (2, 16, 1, 10, 300, 128, True, [300, 5], 2),
    (1, 64, 1, 4, 1024, 64, False, None, 0),         # 256 query rows: two row tiles
    (2, 8, 2, 1, 8192, 128, False, [8192, 4097], 16),
    (1, 8, 8, 2, 4096, 256, True, None, 0),
    # the work split: many short sequences per CTA, two query tiles cut between CTAs, more
    # CTAs than key blocks
    (40, 4, 2, 2, 256, 64, True, [1 + (37 * i) % 256 for i in range(40)], 3),
    (2, 64, 2, 8, 640, 128, False, None, 5),
    (3, 8, 1, 1, 100, 64, False, [100, 37, 64], 0),
    (2, 8, 2, 1, 700, 128, True, [700, 333], 40),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}kv{}q{}N{}d{}{}s{}".format(
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "", c[8]))
def test_decode_matches_oracle(case):
    B, H, H_kv, Nq, N, d, causal, lens, splits = case
    q, k, v = _inputs(B, H, H_kv, Nq, N, d, 9000 + N + Nq)
    scale = 1.0 / d ** 0.5
    O, lse = run(q, k, v, lens, causal, splits)
    O_ref, lse_ref = oracle.attention_decode(q, k, v, scale, causal, lens)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), "queries without a visible key"
    assert np.all(O[empty] == 0)
    lse_c = np.where(empty, 0.0, lse)
    lse_rc = np.where(empty, 0.0, lse_ref)
    assert_fwd_close(O, lse_c, O_ref, lse_rc, str(case))


def test_decode_any_split_count_gives_the_same_result():
    q, k, v = _inputs(2, 16, 4, 2, 3000, 128, 9100)
    lens = [3000, 2222]
    O_ref, lse_ref = oracle.attention_decode(q, k, v, 128 ** -0.5, True, lens)
    outs = []
    for splits in (1, 2, 5, 24, 0):
        O, lse = run(q, k, v, lens, True, splits)
        assert_fwd_close(O, lse, O_ref, lse_ref, f"splits={splits}")
        outs.append(O)
    for O in outs[1:]:
        assert np.abs(O - outs[0]).max() <= 2e-2


def test_decode_is_deterministic_for_fixed_splits():
    q, k, v = _inputs(2, 8, 2, 1, 5000, 128, 9200)
    a = run(q, k, v, None, False, 7)
    b = run(q, k, v, None, False, 7)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_decode_bad_cache_length_is_reported():
    import io_aware_exact_16_b200 as fa
    dev = torch.device("cuda", 0)
    q, k, v = (t.to(dev) for t in _inputs(2, 2, 2, 1, 256, 64, 9300))
    fa.decode(q, k, v, cache_lens=torch.tensor([0, 300], dtype=torch.int32, device=dev))
    assert fa.check_device_error() == fa.FA_ERR_INVALID_ARG
    assert fa.check_device_error() == 0
