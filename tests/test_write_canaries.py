"""Write canaries: no kernel writes outside the buffers it is given.

Each output (O, lse, dQ, dK, dV, the backward and decode workspaces) is a view into a larger
allocation whose margins before and after are filled with a sentinel byte pattern; after the
call every margin byte must be unchanged.  The kernels write only their results (FlashAttention
(DE), "Zusammenfassen von Operationen in einem CUDA-Kernel"), so a stray store -- a row past N
in a ragged last tile, a padded query row, an accumulator row past N_pad -- shows up here.
Shapes: N % 128 != 0, N = 1, key padding, causal, grouped-query heads, every head dim.
"""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

MARGIN = 4096  # bytes before and after every buffer (a multiple of 256, so alignment holds)
PATTERN = 0xA5


class Guarded:
    """A tensor of `shape` / `dtype` in the middle of a sentinel-filled byte buffer."""

    def __init__(self, shape, dtype, dev, fill=None):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((MARGIN + nbytes + MARGIN,), PATTERN, dtype=torch.uint8, device=dev)
        self.t = self.raw[MARGIN:MARGIN + nbytes].view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill)
        self.nbytes = nbytes

    def check(self, what):
        torch.cuda.synchronize()
        lo = self.raw[:MARGIN]
        hi = self.raw[MARGIN + self.nbytes:]
        bad_lo = int((lo != PATTERN).sum())
        bad_hi = int((hi != PATTERN).sum())
        assert bad_lo == 0 and bad_hi == 0, f"{what}: {bad_lo} bytes before and {bad_hi} after changed"


def _fa():
    import io_aware_exact_16_b200 as fa
    return fa


CASES = [
    # (B, H, H_kv, N, d, causal, pad_range)
    (1, 1, 1, 1, 64, False, None),
    (1, 2, 2, 1, 128, True, None),
    (2, 3, 3, 200, 64, False, None),
    (2, 2, 1, 333, 128, True, None),
    (3, 2, 2, 300, 128, False, (1, 300)),
    (2, 4, 2, 129, 64, True, (40, 129)),
    (1, 2, 2, 257, 256, True, None),
    (2, 2, 1, 100, 256, False, (20, 100)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}kv{}N{}d{}{}{}".format(
    c[0], c[1], c[2], c[3], c[4], "c" if c[5] else "", "pad" if c[6] else ""))
def test_forward_and_backward_write_only_their_outputs(case):
    fa = _fa()
    B, H, H_kv, N, d, causal, pad = case
    w = workloads.custom(B, H, N, d, causal, seed=8100 + N + d, pad_range=pad, H_kv=H_kv)
    inp = workloads.make_inputs(w)
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    sl = inp.seqlens.to(dev) if inp.seqlens is not None else None
    o = Guarded((B, H, N, d), torch.bfloat16, dev)
    lse = Guarded((B, H, N), torch.float32, dev)
    fa.forward(q, k, v, causal=causal, seqlens=sl, scale=w.scale, out=o.t, lse=lse.t)
    assert fa.check_device_error(dev) == 0
    o.check("O")
    lse.check("lse")
    dq = Guarded((B, H, N, d), torch.bfloat16, dev)
    dk = Guarded((B, H_kv, N, d), torch.bfloat16, dev)
    dv = Guarded((B, H_kv, N, d), torch.bfloat16, dev)
    ws = Guarded((fa.bwd_workspace_size(B, H, N, d),), torch.uint8, dev)
    fa.backward(q, k, v, o.t, do, lse.t, causal=causal, seqlens=sl, scale=w.scale,
                dq=dq.t, dk=dk.t, dv=dv.t, workspace=ws.t)
    assert fa.check_device_error(dev) == 0
    for g, name in ((dq, "dQ"), (dk, "dK"), (dv, "dV"), (ws, "workspace")):
        g.check(name)


@pytest.mark.parametrize("Nq,N,d,splits,lens", [
    (1, 1, 64, 1, None), (3, 300, 128, 4, (300, 7)), (16, 1000, 128, 0, (1000, 999)),
    (2, 515, 256, 3, (515, 2)),
])
def test_decode_writes_only_its_outputs(Nq, N, d, splits, lens):
    fa = _fa()
    B, H, H_kv = 2, 4, 2
    g = torch.Generator().manual_seed(8200 + N)
    dev = torch.device("cuda", 0)
    q = torch.randn((B, H, Nq, d), generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn((B, H_kv, N, d), generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn((B, H_kv, N, d), generator=g).to(torch.bfloat16).to(dev)
    cl = torch.tensor(lens, dtype=torch.int32, device=dev) if lens else None
    if splits == 0:
        splits = fa.decode_num_splits(B, H, H_kv, Nq, N, d, ragged=cl is not None)
    o = Guarded((B, H, Nq, d), torch.bfloat16, dev)
    lse = Guarded((B, H, Nq), torch.float32, dev)
    ws = Guarded((max(1, fa.decode_workspace_size(B, H, Nq, d, splits)),), torch.uint8, dev)
    fa.decode(q, k, v, cache_lens=cl, causal=True, splits=splits, out=o.t, lse=lse.t,
              workspace=ws.t)
    assert fa.check_device_error(dev) == 0
    for gd, name in ((o, "O"), (lse, "lse"), (ws, "workspace")):
        gd.check(name)


@pytest.mark.parametrize("N,causal,pad", [(1, False, None), (200, True, None),
                                          (333, False, (30, 333))])
def test_fp8_forward_writes_only_its_outputs(N, causal, pad):
    fa = _fa()
    w = workloads.custom(2, 2, N, 128, causal, seed=8300 + N, pad_range=pad)
    f = workloads.make_fp8_inputs(w)
    dev = torch.device("cuda", 0)
    sl = f.seqlens.to(dev) if getattr(f, "seqlens", None) is not None else None
    o = Guarded((w.B, w.H, N, 128), torch.bfloat16, dev)
    lse = Guarded((w.B, w.H, N), torch.float32, dev)
    fa.forward_fp8(f.q.to(dev), f.k.to(dev), f.v.to(dev), f.q_descale.to(dev),
                   f.k_descale.to(dev), f.v_descale.to(dev), causal=causal, seqlens=sl,
                   scale=w.scale, out=o.t, lse=lse.t)
    assert fa.check_device_error(dev) == 0
    o.check("O")
    lse.check("lse")


def test_packed_sequences_write_only_their_outputs():
    fa = _fa()
    pw = workloads.PackedWorkload("canary packed", 4, 4, 2, 128, True, seed=8400,
                                  lengths=(130, 0, 1, 77))
    pin = workloads.make_packed_inputs(pw)
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in (pin.q, pin.k, pin.v, pin.do))
    cu = pin.cu_seqlens.to(dev)
    T = q.shape[0]
    o = Guarded(tuple(q.shape), torch.bfloat16, dev)
    lse = Guarded((pw.H, T), torch.float32, dev)
    fa.forward_varlen(q, k, v, cu, pin.max_seqlen, causal=True, scale=pw.scale, out=o.t,
                      lse=lse.t)
    dq = Guarded(tuple(q.shape), torch.bfloat16, dev)
    dk = Guarded(tuple(k.shape), torch.bfloat16, dev)
    dv = Guarded(tuple(v.shape), torch.bfloat16, dev)
    ws = Guarded((fa.bwd_workspace_size(pw.B, pw.H, pin.max_seqlen, pw.d),), torch.uint8, dev)
    fa.backward_varlen(q, k, v, o.t, do, lse.t, cu, pin.max_seqlen, causal=True, scale=pw.scale,
                       dq=dq.t, dk=dk.t, dv=dv.t, workspace=ws.t)
    assert fa.check_device_error(dev) == 0
    for g, name in ((o, "O"), (lse, "lse"), (dq, "dQ"), (dk, "dK"), (dv, "dV"),
                    (ws, "workspace")):
        g.check(name)
