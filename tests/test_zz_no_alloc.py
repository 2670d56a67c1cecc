"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.

Such callers (a process that keeps its whole device-memory budget in its own pool, a loop that
must not call cudaMalloc / cudaFree) get the same backward pass with the library's fixed,
built-in scratch instead of a caller-provided workspace.  This test calls the entry point
through the C ABI twice in a row, on different problems, and checks each result against the
ordinary fa_bwd on the same inputs with the tolerance the backward parity tests use.  It lives
in a file of its own that runs last and works both alone and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from tests.gpu_helpers import GRAD_REL

pytestmark = pytest.mark.gpu

_vp = ctypes.c_void_p
_i = ctypes.c_int


def _lib():
    import io_aware_exact_16_b200 as fa
    lib = fa.raw_library()
    lib.fa_bwd_noalloc.argtypes = [_vp] * 9 + [_i] * 4 + [ctypes.c_float, _i, _vp, _vp, _vp]
    lib.fa_bwd_noalloc.restype = _i
    return fa, lib


def _case(w: workloads.Workload):
    fa, lib = _lib()
    dev = torch.device("cuda", 0)
    inp = workloads.make_inputs(w)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    sl = inp.seqlens.to(dev) if inp.seqlens is not None else None
    o, lse = fa.forward(q, k, v, causal=w.causal, seqlens=sl, scale=w.scale)
    ref = fa.backward(q, k, v, o, do, lse, causal=w.causal, seqlens=sl, scale=w.scale)
    assert fa.check_device_error(dev) == 0

    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    st = lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                            lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                            w.B, w.H, w.N, w.d, w.scale, int(w.causal),
                            sl.data_ptr() if sl is not None else None, err.data_ptr(), stream)
    assert st == fa.FA_OK, fa.status_string(st)
    torch.cuda.synchronize(dev)
    assert int(err.item()) == 0
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        g = got.double().cpu().numpy()
        r = want.double().cpu().numpy()
        assert np.isfinite(g).all(), name
        assert np.abs(g - r).max() <= GRAD_REL * max(np.abs(r).max(), 1e-30), name


def test_two_calls_in_a_row_match_the_workspace_version():
    _case(workloads.custom(2, 3, 700, 128, False, seed=5100))
    _case(workloads.custom(3, 2, 333, 64, True, seed=5200, pad_range=(40, 333)))


def test_problems_larger_than_the_scratch_are_refused():
    fa, lib = _lib()
    # B*H = 64, N = 4096, d = 128 needs about 130 MiB of scratch: refused before any launch.
    st = lib.fa_bwd_noalloc(*([16] * 9), 4, 16, 4096, 128, 0.088, 0, None, None, None)
    assert st == fa.FA_ERR_WORKSPACE
