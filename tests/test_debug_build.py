"""The checking build libfa_debug.so on the GPU: the stand-in for a memory sanitizer (which is
not available here).  In it every plain global load and store of the kernels checks its index
against its buffer, records FA_ERR_INVALID_ARG and skips the access when out of range.

First the check itself is exercised (fa_selftest_bounds: one store inside a buffer, one just
past it).  Then every entry point runs through the checking build on shapes with ragged tiles,
N = 1, key padding, causal masks, grouped-query heads, packed sequences, decode splits, FP8 and
head dim 256: no check may fire, and the results must still match the oracle.
"""
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


def test_bounds_check_skips_the_store_past_the_buffer():
    fa = _fa()
    dbg = fa.debug_library()
    dev = torch.device("cuda", 0)
    n = 64
    raw = torch.full((n + 64,), -7, dtype=torch.int32, device=dev)
    with fa.use_library(dbg):
        assert fa.check_device_error(dev) == 0
        st = dbg.fa_selftest_bounds(raw.data_ptr(), n, 12345,
                                    torch.cuda.current_stream(dev).cuda_stream)
        assert st == fa.FA_OK
        assert fa.check_device_error(dev) == fa.FA_ERR_INVALID_ARG
    got = raw.cpu()
    assert int(got[n - 1]) == 12345           # inside: written
    assert bool((got[n:] == -7).all())         # one past the end (and beyond): untouched
    assert bool((got[:n - 1] == -7).all())


CASES = [
    # (B, H, H_kv, N, d, causal, pad_range)
    (1, 1, 1, 1, 64, False, None),
    (2, 3, 3, 200, 64, True, None),
    (2, 4, 2, 333, 128, False, (30, 333)),
    (3, 7, 7, 300, 128, True, None),
    (1, 2, 1, 257, 256, True, None),
    (2, 2, 2, 130, 256, False, (1, 130)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}kv{}N{}d{}{}{}".format(
    c[0], c[1], c[2], c[3], c[4], "c" if c[5] else "", "pad" if c[6] else ""))
def test_training_step_through_the_checking_build(case):
    fa = _fa()
    B, H, H_kv, N, d, causal, pad = case
    w = workloads.custom(B, H, N, d, causal, seed=9100 + N + d, pad_range=pad, H_kv=H_kv)
    inp = workloads.make_inputs(w)
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    sl = inp.seqlens.to(dev) if inp.seqlens is not None else None
    with fa.use_library(fa.debug_library()):
        o, lse = fa.forward(q, k, v, causal=causal, seqlens=sl, scale=w.scale)
        dq, dk, dv = fa.backward(q, k, v, o, do, lse, causal=causal, seqlens=sl, scale=w.scale)
        assert fa.check_device_error(dev) == 0, "an index check fired"
    ref = oracle.attention_bwd_gqa(inp.q, inp.k, inp.v, inp.do, w.scale, causal, inp.seqlens)
    assert_fwd_close(to_np(o), to_np(lse), ref["o"], ref["lse"], str(case))
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert_grad_close(to_np(t), ref[name], name, str(case))


def test_packed_decode_and_fp8_through_the_checking_build():
    fa = _fa()
    dev = torch.device("cuda", 0)
    with fa.use_library(fa.debug_library()):
        pw = workloads.PackedWorkload("debug packed", 4, 4, 2, 128, True, seed=9200,
                                      lengths=(130, 0, 1, 77))
        pin = workloads.make_packed_inputs(pw)
        pq, pk, pv, pdo = (t.to(dev) for t in (pin.q, pin.k, pin.v, pin.do))
        cu = pin.cu_seqlens.to(dev)
        po, plse = fa.forward_varlen(pq, pk, pv, cu, pin.max_seqlen, causal=True, scale=pw.scale)
        pdq, pdk, pdv = fa.backward_varlen(pq, pk, pv, po, pdo, plse, cu, pin.max_seqlen,
                                           causal=True, scale=pw.scale)
        assert fa.check_device_error(dev) == 0, "an index check fired (packed)"

        g = torch.Generator().manual_seed(9201)
        q = torch.randn((2, 4, 3, 128), generator=g).to(torch.bfloat16)
        kc = torch.randn((2, 2, 515, 128), generator=g).to(torch.bfloat16)
        vc = torch.randn((2, 2, 515, 128), generator=g).to(torch.bfloat16)
        lens = [515, 9]
        od, _ = fa.decode(q.to(dev), kc.to(dev), vc.to(dev),
                          cache_lens=torch.tensor(lens, dtype=torch.int32, device=dev),
                          causal=True, splits=3)
        assert fa.check_device_error(dev) == 0, "an index check fired (decode)"

        w8 = workloads.custom(2, 2, 300, 128, True, seed=9202, pad_range=(50, 300))
        f8 = workloads.make_fp8_inputs(w8)
        o8, _ = fa.forward_fp8(f8.q.to(dev), f8.k.to(dev), f8.v.to(dev), f8.q_descale.to(dev),
                               f8.k_descale.to(dev), f8.v_descale.to(dev), causal=True,
                               seqlens=f8.seqlens.to(dev), scale=w8.scale)
        assert fa.check_device_error(dev) == 0, "an index check fired (fp8)"
    pref = oracle.attention_bwd_varlen(pin.q, pin.k, pin.v, pin.do, pin.cu_seqlens, pw.scale, True)
    T = int(pin.cu_seqlens[-1])
    assert np.abs(to_np(po)[:T] - pref["o"][:T]).max() <= 2e-2
    for name, t in (("dq", pdq), ("dk", pdk), ("dv", pdv)):
        assert_grad_close(to_np(t)[:T], pref[name][:T], name, "packed")
    dref = oracle.attention_decode(q, kc, vc, 128 ** -0.5, True, lens)[0]
    assert np.abs(to_np(od) - dref).max() <= 2e-2
    ref8 = oracle.attention_fwd_fp8(f8.q, f8.k, f8.v, f8.q_descale, f8.k_descale, f8.v_descale,
                                    w8.scale, True, f8.seqlens)[0]
    assert np.abs(to_np(o8) - ref8).max() <= 2.0 ** -4 * 4.0 * float(np.abs(ref8).max()) + 2e-2
