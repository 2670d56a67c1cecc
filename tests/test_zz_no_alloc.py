"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.

Such callers are a process that keeps its whole device-memory budget in its own pool (a later
cudaMalloc would fail or fragment the pool) and a loop that must not call cudaMalloc / cudaFree
(they can block and synchronise the device).  They get the same backward pass with the
library's fixed, built-in scratch instead of a caller-provided workspace.

These tests call the entry point through the C ABI twice in a row, on different problems, and
check that each result is bitwise equal to the ordinary fa_bwd on the same inputs (the same
kernels on the same data), that one of them matches the fp64 oracle within the tolerance of
the other backward tests, that the largest problem that fits in the scratch works, that a call
changes no device-memory use, and that a problem too large for the scratch is refused.  The
file is collected last and works both alone and after the other tests.
"""
import ctypes

import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import assert_grad_close

pytestmark = pytest.mark.gpu

_vp = ctypes.c_void_p
_i = ctypes.c_int


def _lib():
    import io_aware_exact_16_b200 as fa
    lib = fa.raw_library()
    lib.fa_bwd_noalloc.argtypes = [_vp] * 9 + [_i] * 4 + [ctypes.c_float, _i, _vp, _vp, _vp]
    lib.fa_bwd_noalloc.restype = _i
    return fa, lib


def _case(w: workloads.Workload, oracle_heads=None, setup_first=False):
    """Runs fa_bwd and fa_bwd_noalloc on the same inputs; returns the device's free memory
    just before and just after the fa_bwd_noalloc call.  The first call on a device may place
    the scratch in device memory (lazy module loading); `setup_first` makes one call before the
    measured one so that the measured call is not the first."""
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

    def call():
        return lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                  dv.data_ptr(), w.B, w.H, w.N, w.d, w.scale, int(w.causal),
                                  sl.data_ptr() if sl is not None else None, err.data_ptr(),
                                  stream)

    if setup_first:
        assert call() == fa.FA_OK
    torch.cuda.synchronize(dev)
    free_before = torch.cuda.mem_get_info(dev)[0]
    st = call()
    assert st == fa.FA_OK, fa.status_string(st)
    torch.cuda.synchronize(dev)
    free_after = torch.cuda.mem_get_info(dev)[0]
    assert int(err.item()) == 0
    got = {"dq": dq, "dk": dk, "dv": dv}
    for name, want in zip(("dq", "dk", "dv"), ref):
        assert torch.equal(got[name].view(torch.int16), want.view(torch.int16)), \
            f"{name}: not bitwise equal to fa_bwd"
    got = {n: t.double().cpu().numpy() for n, t in got.items()}
    if oracle_heads is not None:
        for flat in oracle_heads:
            b, h = divmod(flat, w.H)
            L = int(inp.seqlens[b]) if inp.seqlens is not None else None
            r = oracle.head_bwd(inp.q[b, h], inp.k[b, h], inp.v[b, h], inp.do[b, h], w.scale,
                                w.causal, L)
            for name in ("dq", "dk", "dv"):
                assert_grad_close(got[name][b, h], r[name], name, f"noalloc b{b} h{h}")
    return free_before, free_after


def test_two_calls_in_a_row_match_the_workspace_version():
    w1 = workloads.custom(2, 3, 700, 128, False, seed=5100)
    _case(w1, oracle_heads=range(w1.B * w1.H))
    # the second call reuses the scratch the first one left behind
    free_before, free_after = _case(workloads.custom(3, 2, 333, 64, True, seed=5200,
                                                     pad_range=(40, 333)))
    assert free_after >= free_before, "fa_bwd_noalloc changed the device's free memory"


def test_largest_problem_that_fits_the_scratch():
    fa, lib = _lib()
    # B*H = 31 at N = 4096, d = 128 needs 66,035,456 bytes of the 67,108,864 available
    assert lib.fa_bwd_workspace_size(1, 31, 4096, 128) <= 64 << 20
    w = workloads.custom(1, 31, 4096, 128, False, seed=5300)
    free_before, free_after = _case(w, oracle_heads=workloads.seeded_sample(w.seed, 31, 2),
                                    setup_first=True)
    assert free_after >= free_before, "fa_bwd_noalloc changed the device's free memory"


def test_problems_larger_than_the_scratch_are_refused():
    fa, lib = _lib()
    # B*H = 32 at N = 4096, d = 128 needs 68,165,632 bytes: refused before any launch.
    assert lib.fa_bwd_workspace_size(2, 16, 4096, 128) > 64 << 20
    st = lib.fa_bwd_noalloc(*([16] * 9), 2, 16, 4096, 128, 0.088, 0, None, None, None)
    assert st == fa.FA_ERR_WORKSPACE
