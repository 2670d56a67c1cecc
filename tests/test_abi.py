"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol that
include/fa.h declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import re

import pytest

import io_aware_exact_16_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


def declared_symbols():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_check_device_error",
              "fa_status_string", "fa_set_wait_timeout_ns"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(fa.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(declared_symbols()) == set(fa.EXPORTED)


def test_status_strings():
    for code in range(6):
        assert fa.status_string(code).startswith("FA_")
    assert "unknown" in fa.status_string(99)


def test_workspace_size_formula():
    # D and |dO_i| (fp32 per row), per-128-row-chunk maxima of |v_j| and |k_jl| (2 fp32), and
    # the int32 fixed-point dQ accumulator (rows padded to 128), each rounded up to 256 bytes.
    def r(n):
        return (n + 255) // 256 * 256
    for B, H, N, d in ((1, 1, 1, 64), (2, 3, 300, 128), (4, 16, 4096, 128)):
        Np = (N + 127) // 128 * 128
        expect = 2 * r(B * H * N * 4) + r(B * H * (Np // 128) * 2 * 4) + r(B * H * Np * d * 4)
        assert fa.bwd_workspace_size(B, H, N, d) == expect
    assert fa.bwd_workspace_size(1, 1, 128, 96) == 0
    assert fa.bwd_workspace_size(0, 1, 128, 64) == 0


def _fwd(lib, *, ptr=16, B=1, H=1, N=8, d=64, scale=0.125, seqlens=None):
    return lib.fa_fwd(ptr, ptr, ptr, ptr, ptr, B, H, N, d, ctypes.c_float(scale), 0, seqlens, None)


def test_forward_rejects_bad_arguments_without_a_device():
    lib = fa.raw_library()
    assert _fwd(lib, d=96) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(lib, N=0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, B=0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=0.0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("inf")) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, ptr=None) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, ptr=24) == fa.FA_ERR_INVALID_ARG          # not 16-byte aligned
    assert _fwd(lib, seqlens=18) == fa.FA_ERR_INVALID_ARG      # not 4-byte aligned
    assert _fwd(lib, B=1 << 16) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, B=2048, H=64, N=4096, d=128) == fa.FA_ERR_INVALID_ARG  # > 2^31 elements


def test_backward_rejects_bad_arguments_and_short_workspace_without_a_device():
    lib = fa.raw_library()
    need = fa.bwd_workspace_size(1, 1, 8, 64)

    def bwd(ws=16, ws_bytes=need, d=64, ptr=16):
        return lib.fa_bwd(ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, 1, 1, 8, d,
                          ctypes.c_float(0.125), 0, None, ws, ws_bytes, None)

    assert bwd(d=80) == fa.FA_ERR_UNSUPPORTED
    assert fa.bwd_workspace_size(1, 1, 8, 256) > need
    assert bwd(d=256) == fa.FA_ERR_WORKSPACE        # d = 256 needs its own, larger workspace
    assert bwd(ptr=None) == fa.FA_ERR_INVALID_ARG
    assert bwd(ws=None) == fa.FA_ERR_WORKSPACE
    assert bwd(ws_bytes=need - 1) == fa.FA_ERR_WORKSPACE
    assert bwd(ws=32 + 8) == fa.FA_ERR_WORKSPACE


def test_python_binding_checks_shapes_before_calling():
    import torch
    q = torch.zeros((1, 1, 8, 64), dtype=torch.float32)
    with pytest.raises(TypeError):
        fa.forward(q, q, q)
    qb = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16)
    kb = torch.zeros((1, 1, 9, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.forward(qb, kb, qb)


def test_gqa_and_varlen_reject_bad_arguments_without_a_device():
    lib = fa.raw_library()
    f = ctypes.c_float(0.125)
    # H_kv must divide H and lie in [1, H]
    assert lib.fa_fwd_gqa(16, 16, 16, 16, 16, 1, 4, 3, 8, 64, f, 0, None, None) == \
        fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_gqa(16, 16, 16, 16, 16, 1, 4, 8, 8, 64, f, 0, None, None) == \
        fa.FA_ERR_INVALID_ARG
    # packed: offsets required, total >= 1, 4-byte aligned offsets
    assert lib.fa_fwd_varlen(16, 16, 16, 16, 16, None, 2, 8, 16, 4, 4, 64, f, 0, None) == \
        fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_varlen(16, 16, 16, 16, 16, 16, 2, 8, 0, 4, 4, 64, f, 0, None) == \
        fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_varlen(16, 16, 16, 16, 16, 18, 2, 8, 16, 4, 4, 64, f, 0, None) == \
        fa.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_varlen(16, 16, 16, 16, 16, 16, 16, 16, 16, 16, 2, 8, 16, 4, 4, 96, f, 0,
                             16, 1 << 20, None) == fa.FA_ERR_UNSUPPORTED


def test_fp8_and_decode_reject_bad_arguments_without_a_device():
    lib = fa.raw_library()
    f = ctypes.c_float(0.125)
    fp8 = lambda d=128, H_kv=2, qd=None: lib.fa_fwd_fp8(  # noqa: E731
        16, 16, 16, qd, None, None, 16, 16, 1, 4, H_kv, 64, d, f, 0, None, None)
    assert fp8(d=64) == fa.FA_ERR_UNSUPPORTED
    assert fp8(H_kv=3) == fa.FA_ERR_INVALID_ARG
    assert fp8(qd=18) == fa.FA_ERR_INVALID_ARG  # descale factors must be 4-byte aligned
    dec = lambda H=8, H_kv=2, Nq=1, N=100, d=128, splits=0, ws=None, wsb=0: lib.fa_fwd_decode(  # noqa: E731
        16, 16, 16, 16, 16, None, 2, H, H_kv, Nq, N, d, f, 0, splits, ws, wsb, None)
    assert dec(H_kv=3) == fa.FA_ERR_INVALID_ARG
    assert dec(d=96) == fa.FA_ERR_UNSUPPORTED
    assert dec(Nq=0) == fa.FA_ERR_INVALID_ARG
    assert dec(splits=-1) == fa.FA_ERR_INVALID_ARG


def test_decode_split_heuristic_and_workspace_size():
    """Host logic only: the automatic split count stays within [1, key blocks] and grows when
    the (sequence, cache head) pairs alone cannot fill the device; the workspace holds fp32
    O and lse partials for every split (none for one split)."""
    for (B, H, H_kv, Nq, N, d) in ((8, 32, 8, 1, 8192, 128), (1, 32, 8, 1, 131072, 128),
                                   (64, 32, 8, 1, 2048, 64), (1, 4, 4, 1, 100, 256)):
        s = fa.decode_num_splits(B, H, H_kv, Nq, N, d)
        bk = 128 if d == 256 else 64
        assert 1 <= s <= (N + bk - 1) // bk
    assert fa.decode_num_splits(1, 32, 8, 1, 131072, 128) > fa.decode_num_splits(64, 32, 8, 1, 131072, 128)
    assert fa.decode_workspace_size(2, 4, 3, 128, 1) == 0
    rows = 2 * 4 * 3
    o_bytes = (5 * rows * 128 * 4 + 255) // 256 * 256
    assert fa.decode_workspace_size(2, 4, 3, 128, 5) == o_bytes + 5 * rows * 4
    assert fa.decode_num_splits(1, 4, 3, 1, 100, 128) == 0  # H_kv must divide H
    # per-sequence lengths: at least ceil(4 x 296 slots / pairs) ranges, within the key blocks
    for (B, H, H_kv, Nq, N, d) in ((32, 32, 8, 1, 8192, 128), (8, 32, 8, 1, 32768, 128),
                                   (128, 32, 8, 1, 4096, 128), (16, 32, 8, 1, 16384, 128),
                                   (1, 8, 8, 1, 64, 64)):
        u = fa.decode_num_splits(B, H, H_kv, Nq, N, d)
        r = fa.decode_num_splits(B, H, H_kv, Nq, N, d, ragged=True)
        nblk = (N + 63) // 64
        assert r == max(u, min(nblk, -(-4 * 296 // (B * H_kv))))
    assert fa.decode_num_splits(32, 32, 8, 1, 8192, 128, ragged=True) == 5
    # The counts the cost model picks on the swept shapes, each the fastest (or within 2 % of
    # it) of split counts 1 ... 64 timed on a B200 with 148 SMs.
    for shape, want in (((8, 32, 8, 1, 8192, 128), 4), ((1, 32, 8, 1, 131072, 128), 37),
                        ((64, 32, 8, 1, 2048, 128), 1), ((8, 32, 8, 4, 8192, 128), 4),
                        ((4, 16, 16, 1, 8192, 256), 2)):
        assert fa.decode_num_splits(*shape) == want, shape


def test_wait_selftest_reports_a_missing_device_instead_of_launching():
    """Host logic only: without a usable sm_100 device the self-test launches nothing and
    returns an error status (FA_ERR_CUDA or FA_ERR_UNSUPPORTED), as every entry point does."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present; the GPU test covers the launch")
    st = fa.raw_library().fa_selftest_wait_timeout(None)
    assert st in (fa.FA_ERR_CUDA, fa.FA_ERR_UNSUPPORTED)


def test_debug_build_exports_the_same_symbols_and_reports_its_checks():
    """libfa_debug.so (FA_DEBUG: index checks on every plain global access) is the same C ABI;
    fa_debug_checks tells the two builds apart, and the release build refuses the bounds
    self-test (its checks are compiled out) before touching a device."""
    dbg = fa.debug_library()
    for name in declared_symbols():
        assert hasattr(dbg, name), name
    assert dbg.fa_debug_checks() == 1
    assert fa.raw_library().fa_debug_checks() == 0
    assert fa.raw_library().fa_selftest_bounds(16, 8, 1, None) == fa.FA_ERR_UNSUPPORTED
    assert dbg.fa_selftest_bounds(None, 8, 1, None) == fa.FA_ERR_INVALID_ARG
    assert dbg.fa_selftest_bounds(16, 0, 1, None) == fa.FA_ERR_INVALID_ARG
