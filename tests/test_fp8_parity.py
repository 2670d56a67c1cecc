"""GPU parity of the FP8 (e4m3) forward (``fa_fwd_fp8``) against the oracle's exact attention
of the dequantised inputs.

Tolerance, from the arithmetic: the kernel rounds each scaled probability p' = p * l' (with
l' >= 2^4, see the kernel) to e4m3, whose error is at most 2^-4 relative for normal values and
2^-10 absolute below them, so per element
    |O - O_ref| <= 2^-4 * sum_j P_ij |v_jc| + 2^-14 * sum_{visible j} |v_jc|
plus the bf16 rounding of O (2^-9 relative, taken as 2^-8) and fp32 accumulation (1e-3).
P |V| is the oracle's attention with |V| in place of V (same P); the sum over visible keys is
the Q = 0 attention of |V| (their mean) times exp(lse) (their count).  The scores are exact
products of e4m3 values accumulated in fp32, so lse keeps the bf16 path's 1e-3 bound.

That bound is what a worst case allows; a kernel whose rounding were biased (every p' rounded
the same way) would still meet it.  Rounding to nearest is unbiased, so the errors of the
many terms of a row cancel: the error of O_ic has a spread of about
    sigma_ic = 2^-4 / sqrt(3) * sqrt(sum_j P_ij^2 v_jc^2)
(independent rounding errors uniform within +-2^-4 relative), plus the bf16 output rounding.
The mean error over the tensor must stay within twice 0.8 sigma + 2^-10 |O| on average, which a
biased rounding (an error near 2^-5 sum_j P_ij |v_jc| in every element) exceeds many times
over at these lengths.  sum_j P_ij^2 v_jc^2 is the oracle's attention at twice the scale (whose
probabilities are P^2 / sum_j P^2) of V * V, times exp(lse(2 scale) - 2 lse(scale)).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import LSE_MAX, to_np

pytestmark = pytest.mark.gpu


def run(w, f):
    import io_aware_exact_16_b200 as fa
    dev = torch.device("cuda", 0)
    sl = f.seqlens.to(dev) if f.seqlens is not None else None
    O, lse = fa.forward_fp8(f.q.to(dev), f.k.to(dev), f.v.to(dev), f.q_descale.to(dev),
                            f.k_descale.to(dev), f.v_descale.to(dev), causal=w.causal,
                            seqlens=sl, scale=w.scale)
    assert fa.check_device_error() == 0
    return to_np(O), to_np(lse)


def expected_mean_error(qd, kd, vd, w, seqlens, O_ref, lse_ref):
    """Mean over the tensor of the typical error of unbiased e4m3 rounding of P (see above)."""
    O2, lse2 = oracle.attention_fwd_gqa(qd, kd, vd * vd, 2.0 * w.scale, w.causal, seqlens)
    sum_p2_v2 = O2 * np.exp(lse2 - 2.0 * lse_ref)[..., None]
    sigma = 2.0 ** -4 / np.sqrt(3.0) * np.sqrt(np.maximum(sum_p2_v2, 0.0))
    return float((0.8 * sigma + 2.0 ** -10 * np.abs(O_ref)).mean())


def check(w, O, lse, f, mean_check=False):
    qd = oracle.dequantize_fp8(f.q, f.q_descale)
    kd = oracle.dequantize_fp8(f.k, f.k_descale)
    vd = oracle.dequantize_fp8(f.v, f.v_descale)
    O_ref, lse_ref = oracle.attention_fwd_gqa(qd, kd, vd, w.scale, w.causal, f.seqlens)
    PabsV, _ = oracle.attention_fwd_gqa(qd, kd, np.abs(vd), w.scale, w.causal, f.seqlens)
    mean_abs, lse0 = oracle.attention_fwd_gqa(0 * qd, kd, np.abs(vd), w.scale, w.causal,
                                              f.seqlens)
    sum_abs = mean_abs * np.exp(lse0)[..., None]
    bound = 2.0 ** -4 * PabsV + 2.0 ** -14 * sum_abs + 2.0 ** -8 * np.abs(O_ref) + 1e-3
    err = np.abs(O - O_ref)
    assert np.isfinite(O).all()
    worst = (err / bound).max()
    assert worst <= 1.0, f"max err/bound = {worst:.3f} (max err {err.max():.3e})"
    assert np.abs(lse - lse_ref).max() <= LSE_MAX
    if mean_check:
        want = expected_mean_error(qd, kd, vd, w, f.seqlens, O_ref, lse_ref)
        assert err.mean() <= 2.0 * want, f"mean err {err.mean():.3e} > 2 x expected {want:.3e}"
    return err.mean()


SHAPES = [
    # (B, H, H_kv, N, causal, pad_range)
    (1, 2, 2, 128, False, None),
    (1, 1, 1, 1, True, None),
    (2, 2, 2, 300, True, None),
    (2, 3, 3, 257, False, None),
    (3, 4, 2, 520, True, (100, 520)),
    (1, 6, 1, 640, False, None),
    (1, 2, 2, 2048, False, None),
    (1, 2, 2, 2048, True, None),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}H{}kv{}N{}{}{}".format(
    s[0], s[1], s[2], s[3], "c" if s[4] else "", "pad" if s[5] else ""))
def test_fp8_matches_oracle_within_derived_bound(shape):
    B, H, H_kv, N, causal, pad = shape
    w = workloads.custom(B, H, N, 128, causal, seed=9500 + N + H, pad_range=pad, H_kv=H_kv)
    f = workloads.make_fp8_inputs(w)
    O, lse = run(w, f)
    mean_err = check(w, O, lse, f)
    assert mean_err <= 1e-2


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_at_the_bench_length(causal):
    """N = 4096 (the FP8 bench row's length, per-head scaled inputs as there), two heads in
    full: the per-element bound and the mean error of unbiased rounding."""
    w = workloads.custom(1, 2, 4096, 128, causal, seed=9700 + int(causal))
    f = workloads.make_fp8_inputs(w)
    O, lse = run(w, f)
    check(w, O, lse, f, mean_check=True)


def test_fp8_mean_error_is_that_of_unbiased_rounding():
    """The mean-error check on the shorter shapes as well (B2 H2 N1000, causal and padded)."""
    w = workloads.custom(2, 2, 1000, 128, True, seed=9710, pad_range=(300, 1000))
    f = workloads.make_fp8_inputs(w)
    O, lse = run(w, f)
    check(w, O, lse, f, mean_check=True)


def test_fp8_is_deterministic_and_rejects_other_head_dims():
    import io_aware_exact_16_b200 as fa
    w = workloads.custom(2, 2, 700, 128, False, seed=9600)
    f = workloads.make_fp8_inputs(w)
    a = run(w, f)
    b = run(w, f)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    dev = torch.device("cuda", 0)
    x = torch.zeros((1, 1, 64, 64), device=dev).to(torch.float8_e4m3fn)
    with pytest.raises(fa.FAError) as e:
        fa.forward_fp8(x, x, x)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
