"""The deterministic dQ sum at its edges, on the GPU against the fp64 oracle.

dQ is summed in integer fixed point with one scale per query row, set by an a-priori bound on
the row's partial sums (2 |dO_i| max_j |v_j| max |k|).  The bound is set by the largest value
row and the largest key element of the head, so one outlier coarsens every row of that head.
These cases stress it at N = 16384, where each dQ row sums 128 key blocks:

  head 0: one key feature channel scaled by 64 (outlier channels are common in trained keys);
  head 1: one value row scaled by 64;
  head 2: a near-zero dO row next to rows scaled by 64.

Sampled dQ rows (and dK, dV rows) are compared with the oracle, first with the tolerance of
the other backward tests (relative to the largest reference value), then element by element
against the error that bf16 operands allow: rounding dS to bf16 for the dQ product moves dQ_il
by at most 2^-8 scale sum_j |dS_ij| |k_jl|, rounding O (which enters D = dO . O) by at most
2^-8 scale |dO_i| |O_i| sum_j P_ij |k_jl|, and rounding the output by 2^-8 |dQ_il|; each
element must lie within twice that sum.  A fixed-point resolution that an outlier had made
coarse (or a wrong scale for the near-zero row) exceeds it by orders of magnitude.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import assert_fwd_close, assert_grad_close, to_np

pytestmark = pytest.mark.gpu

N_LONG = 16384
SPECIAL_ROWS = [0, 3, 4, 5, 127, 128, 777, N_LONG // 2, N_LONG - 129, N_LONG - 1]


def _outlier_inputs(d: int, causal: bool, seed: int):
    w = workloads.custom(1, 3, N_LONG, d, causal, seed=seed)
    inp = workloads.make_inputs(w)
    k, v, do = inp.k.clone(), inp.v.clone(), inp.do.clone()
    k[0, 0, :, 5] = (k[0, 0, :, 5].float() * 64).to(torch.bfloat16)
    v[0, 1, 777] = (v[0, 1, 777].float() * 64).to(torch.bfloat16)
    do[0, 2, 3] = (do[0, 2, 3].float() * 1e-6).to(torch.bfloat16)
    do[0, 2, 4:6] = (do[0, 2, 4:6].float() * 64).to(torch.bfloat16)
    return w, workloads.Inputs(inp.q, k, v, do, None)


@pytest.mark.parametrize("d,causal", [(128, False), (128, True), (64, False)])
def test_outliers_at_n16384(d, causal):
    import io_aware_exact_16_b200 as fa
    w, inp = _outlier_inputs(d, causal, seed=6100 + d + int(causal))
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    o, lse = fa.forward(q, k, v, causal=causal, scale=w.scale)
    dq, dk, dv = fa.backward(q, k, v, o, do, lse, causal=causal, scale=w.scale)
    assert fa.check_device_error(dev) == 0
    O, LSE, DQ, DK, DV = (to_np(t) for t in (o, lse, dq, dk, dv))
    rows = sorted(set(workloads.seeded_sample(w.seed + 1, N_LONG, 120) + SPECIAL_ROWS))
    refs = []
    for h in range(w.H):
        what = f"d{d} causal={causal} head {h}"
        ref_o, ref_lse = oracle.head_fwd_rows(inp.q[0, h], inp.k[0, h], inp.v[0, h], rows,
                                              w.scale, causal)
        assert_fwd_close(O[0, h, rows], LSE[0, h, rows], ref_o, ref_lse, what)
        ref = oracle.head_bwd_rows(inp.q[0, h], inp.k[0, h], inp.v[0, h], inp.do[0, h], rows,
                                   rows, w.scale, causal)
        assert_grad_close(DQ[0, h, rows], ref["dq"], "dq", what)
        assert_grad_close(DK[0, h, rows], ref["dk"], "dk", what)
        assert_grad_close(DV[0, h, rows], ref["dv"], "dv", what)
        refs.append(ref["dq"])
    for h in range(w.H):
        mag = oracle.dq_magnitude_sums(inp.q[0, h], inp.k[0, h], inp.v[0, h], inp.do[0, h],
                                       rows, w.scale, causal)
        allowed = 2.0 ** -7 * (w.scale * (mag["abs_dS_k"] + mag["D_term"]) + np.abs(refs[h]))
        err = np.abs(DQ[0, h, rows] - refs[h])
        worst = np.unravel_index(np.argmax(err / np.maximum(allowed, 1e-300)), err.shape)
        assert np.all(err <= allowed), (
            f"d{d} causal={causal} head {h}: dq row {rows[worst[0]]} feature {worst[1]}: "
            f"error {err[worst]:.3e} > allowed {allowed[worst]:.3e}")


def test_bound_beyond_fp32_is_reported():
    """A dO row whose norm overflows fp32 (every element 2e19: the squares sum past 3.4e38)
    has no finite fixed-point bound.  The row's dQ is left at 0 and FA_ERR_INVALID_ARG is
    reported; every other row of dQ, and dK and dV, stay exact (their bounds are finite)."""
    import io_aware_exact_16_b200 as fa
    w = workloads.custom(1, 2, 300, 128, False, seed=6200)
    inp = workloads.make_inputs(w)
    do = inp.do.clone()
    do[0, 1, 7] = 2.0e19
    dev = torch.device("cuda", 0)
    q, k, v, dO = (t.to(dev) for t in (inp.q, inp.k, inp.v, do))
    o, lse = fa.forward(q, k, v, scale=w.scale)
    dq, dk, dv = fa.backward(q, k, v, o, dO, lse, scale=w.scale)
    assert fa.check_device_error(dev) == fa.FA_ERR_INVALID_ARG
    assert fa.check_device_error(dev) == 0  # read and cleared
    DQ, DK, DV = to_np(dq), to_np(dk), to_np(dv)
    assert np.all(DQ[0, 1, 7] == 0)
    ref = oracle.attention_bwd(inp.q, inp.k, inp.v, do, w.scale, False)
    keep = np.ones(w.N, bool)
    keep[7] = False
    assert_grad_close(DQ[0, 0], ref["dq"][0, 0], "dq", "head 0")
    assert_grad_close(DQ[0, 1, keep], ref["dq"][0, 1, keep], "dq", "head 1 other rows")
    for h in range(w.H):
        assert_grad_close(DK[0, h], ref["dk"][0, h], "dk", f"head {h}")
        assert_grad_close(DV[0, h], ref["dv"][0, h], "dv", f"head {h}")
