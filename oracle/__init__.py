"""The oracle: plain, slow, fp64 CPU exact attention.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and reference
legs may import this package.  The CUDA product path (``io_aware_exact_16_b200``) never
imports it, and the two share no code: this package reads the same seeded bf16 inputs from
``workloads`` and nothing else.

Two independent implementations of the same definition live here:

* ``oracle.c`` (built into ``liboracle.so``): the definition of attention written out row by
  row in fp64 (FlashAttention (DE), "Problematik der Standard-Attention"), with the ordinary
  derivative for the backward pass.  This is THE oracle.
* ``twin.py``: the same definition as whole-matrix numpy float64 expressions, used by the
  pin tests as a second, independently written implementation.

Both take the exact fp64 values of the bf16 inputs.  Every function is pinned by
``tests/test_oracle_pins.py`` against closed forms, invariances, finite differences and
torch's own float64 attention (see the pins listed there).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` next to it (plain gcc, -O2, pthreads)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fPIC", "-shared", "-o", _SO, _SRC,
               "-lpthread", "-lm"]
        subprocess.run(cmd, check=True)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_attention_fwd.argtypes = [_dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_double, ctypes.c_int, ctypes.c_int, _dp, _dp]
        lib.oracle_attention_fwd_rows.argtypes = [_dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                                  _ip, ctypes.c_int, _dp, _dp]
        lib.oracle_attention_probs.argtypes = [_dp, _dp, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_double, ctypes.c_int, ctypes.c_int, _dp]
        lib.oracle_attention_bwd.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                             _dp, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_attention_bwd_rows.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                                  _ip, ctypes.c_int, _ip, ctypes.c_int,
                                                  _dp, _dp, _dp]
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_get_threads.restype = ctypes.c_int
        for name in ("oracle_attention_fwd", "oracle_attention_fwd_rows", "oracle_attention_probs",
                     "oracle_attention_bwd", "oracle_attention_bwd_rows"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def set_threads(n: int) -> None:
    """Number of CPU threads the oracle spreads rows over (0 = every online core)."""
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oracle_get_threads())


def as_f64(x) -> np.ndarray:
    """Exact fp64 copy of a bf16/fp32/fp64 torch tensor or numpy array (C-contiguous)."""
    if hasattr(x, "detach"):
        import torch  # only for the dtype conversion of torch inputs
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_dp)


def _iptr(a: np.ndarray):
    assert a.dtype == np.int32 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_ip)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise RuntimeError(f"oracle: {what} rejected its arguments")


def head_fwd(q, k, v, scale: float, causal: bool, L: Optional[int] = None):
    """One head: q, k, v ``[N, d]`` -> (O ``[N, d]``, lse ``[N]``) in fp64."""
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    N, d = q.shape
    L = N if L is None else int(L)
    O = np.empty((N, d), np.float64)
    lse = np.empty((N,), np.float64)
    _check(_load().oracle_attention_fwd(_ptr(q), _ptr(k), _ptr(v), N, d, float(scale),
                                        int(bool(causal)), L, _ptr(O), _ptr(lse)), "fwd")
    return O, lse


def head_fwd_rows(q, k, v, rows: Sequence[int], scale: float, causal: bool,
                  L: Optional[int] = None):
    """One head, only the listed query rows: (O ``[len(rows), d]``, lse ``[len(rows)]``)."""
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    N, d = q.shape
    L = N if L is None else int(L)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    O = np.empty((len(r), d), np.float64)
    lse = np.empty((len(r),), np.float64)
    _check(_load().oracle_attention_fwd_rows(_ptr(q), _ptr(k), _ptr(v), N, d, float(scale),
                                             int(bool(causal)), L, _iptr(r), len(r), _ptr(O),
                                             _ptr(lse)), "fwd_rows")
    return O, lse


def head_probs(q, k, scale: float, causal: bool, L: Optional[int] = None) -> np.ndarray:
    """One head: the probability matrix P ``[N, N]`` (zero where a key is masked)."""
    q, k = as_f64(q), as_f64(k)
    N, d = q.shape
    L = N if L is None else int(L)
    P = np.empty((N, N), np.float64)
    _check(_load().oracle_attention_probs(_ptr(q), _ptr(k), N, d, float(scale),
                                          int(bool(causal)), L, _ptr(P)), "probs")
    return P


def head_bwd(q, k, v, do, scale: float, causal: bool, L: Optional[int] = None):
    """One head: -> dict with dq, dk, dv, o, lse, D (all fp64)."""
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    N, d = q.shape
    L = N if L is None else int(L)
    out = {name: np.empty((N, d), np.float64) for name in ("dq", "dk", "dv", "o")}
    out["lse"] = np.empty((N,), np.float64)
    out["D"] = np.empty((N,), np.float64)
    _check(_load().oracle_attention_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), N, d, float(scale),
                                        int(bool(causal)), L, _ptr(out["dq"]), _ptr(out["dk"]),
                                        _ptr(out["dv"]), _ptr(out["o"]), _ptr(out["lse"]),
                                        _ptr(out["D"])), "bwd")
    return out


def head_bwd_rows(q, k, v, do, qrows: Sequence[int], krows: Sequence[int], scale: float,
                  causal: bool, L: Optional[int] = None):
    """One head: dQ at the listed query rows, dK and dV at the listed key rows."""
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    N, d = q.shape
    L = N if L is None else int(L)
    qr = np.ascontiguousarray(np.asarray(qrows, dtype=np.int32))
    kr = np.ascontiguousarray(np.asarray(krows, dtype=np.int32))
    dq = np.empty((max(len(qr), 1), d), np.float64)
    dk = np.empty((max(len(kr), 1), d), np.float64)
    dv = np.empty((max(len(kr), 1), d), np.float64)
    _check(_load().oracle_attention_bwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(do), N, d,
                                             float(scale), int(bool(causal)), L, _iptr(qr),
                                             len(qr), _iptr(kr), len(kr), _ptr(dq), _ptr(dk),
                                             _ptr(dv)), "bwd_rows")
    return {"dq": dq[:len(qr)], "dk": dk[:len(kr)], "dv": dv[:len(kr)]}


def dq_magnitude_sums(q, k, v, do, rows: Sequence[int], scale: float, causal: bool):
    """Magnitudes that bound how far a dQ formed from rounded operands can be from the exact
    one, for the listed query rows of one head (fp64 numpy, no blocking):

      abs_dS_k[r, l] = sum_j |dS_ij| |k_jl|                  (rounding each dS_ij moves dQ_il
                                                               by at most its share of this)
      D_term[r, l]   = |dO_i| |O_i| sum_j P_ij |k_jl|         (rounding O moves D_i, and with
                                                               it every dS_ij, by P_ij dD_i)

    with i = rows[r] and the definitions of the backward pass: s_ij = scale q_i . k_j over the
    visible keys j (j <= i when causal), P_ij = exp(s_ij - lse_i), O_i = sum_j P_ij v_j,
    dP_ij = dO_i . v_j, D_i = dO_i . O_i, dS_ij = P_ij (dP_ij - D_i).  dQ_il = scale sum_j
    dS_ij k_jl, so |dQ_il| <= scale abs_dS_k[r, l].  Used by tolerances only."""
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    N, d = q.shape
    absk = np.abs(k)
    A = np.zeros((len(rows), d), np.float64)
    Dt = np.zeros((len(rows), d), np.float64)
    for r, i in enumerate(rows):
        lim = i + 1 if causal else N
        s_row = scale * (k[:lim] @ q[i])
        e = np.exp(s_row - s_row.max())
        P = e / e.sum()
        O = P @ v[:lim]
        dP = v[:lim] @ do[i]
        dS = P * (dP - do[i] @ O)
        A[r] = np.abs(dS) @ absk[:lim]
        Dt[r] = np.linalg.norm(do[i]) * np.linalg.norm(O) * (P @ absk[:lim])
    return {"abs_dS_k": A, "D_term": Dt}


def _lengths(seqlens, B: int, N: int) -> list[int]:
    if seqlens is None:
        return [N] * B
    return [int(x) for x in (seqlens.tolist() if hasattr(seqlens, "tolist") else seqlens)]


def attention_fwd(q, k, v, scale: float, causal: bool, seqlens=None):
    """Batched ``[B, H, N, d]`` inputs -> (O ``[B, H, N, d]``, lse ``[B, H, N]``), fp64."""
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    B, H, N, d = q.shape
    Ls = _lengths(seqlens, B, N)
    O = np.empty((B, H, N, d), np.float64)
    lse = np.empty((B, H, N), np.float64)
    for b in range(B):
        for h in range(H):
            O[b, h], lse[b, h] = head_fwd(q[b, h], k[b, h], v[b, h], scale, causal, Ls[b])
    return O, lse


def attention_bwd(q, k, v, do, scale: float, causal: bool, seqlens=None):
    """Batched backward -> dict of ``[B, H, N, d]`` dq, dk, dv, o and ``[B, H, N]`` lse, D."""
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    B, H, N, d = q.shape
    Ls = _lengths(seqlens, B, N)
    out = {n: np.empty((B, H, N, d), np.float64) for n in ("dq", "dk", "dv", "o")}
    out["lse"] = np.empty((B, H, N), np.float64)
    out["D"] = np.empty((B, H, N), np.float64)
    for b in range(B):
        for h in range(H):
            r = head_bwd(q[b, h], k[b, h], v[b, h], do[b, h], scale, causal, Ls[b])
            for n in out:
                out[n][b, h] = r[n]
    return out


def _kv_index(H: int, H_kv: int) -> list[int]:
    """Key/value head of each query head: consecutive groups of H / H_kv query heads share one."""
    if H_kv < 1 or H % H_kv != 0:
        raise ValueError("H_kv must divide H")
    G = H // H_kv
    return [h // G for h in range(H)]


def attention_fwd_gqa(q, k, v, scale: float, causal: bool, seqlens=None):
    """Grouped-query attention: q [B, H, N, d], k, v [B, H_kv, N, d].  Query head h attends with
    key/value head h // (H / H_kv) (multi-query attention when H_kv = 1; FlashAttention (DE),
    FlashAttention-2 section).  Each head is the plain definition (``head_fwd``)."""
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    B, H, N, d = q.shape
    kv = _kv_index(H, k.shape[1])
    Ls = _lengths(seqlens, B, N)
    O = np.empty((B, H, N, d), np.float64)
    lse = np.empty((B, H, N), np.float64)
    for b in range(B):
        for h in range(H):
            O[b, h], lse[b, h] = head_fwd(q[b, h], k[b, kv[h]], v[b, kv[h]], scale, causal, Ls[b])
    return O, lse


def attention_bwd_gqa(q, k, v, do, scale: float, causal: bool, seqlens=None):
    """Backward of ``attention_fwd_gqa``: dQ per query head; dK, dV of a key/value head are the
    sums over the query heads that read it (each summand from ``head_bwd``)."""
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    kv = _kv_index(H, H_kv)
    Ls = _lengths(seqlens, B, N)
    out = {"dq": np.empty((B, H, N, d)), "o": np.empty((B, H, N, d)), "lse": np.empty((B, H, N)),
           "dk": np.zeros((B, H_kv, N, d)), "dv": np.zeros((B, H_kv, N, d))}
    for b in range(B):
        for h in range(H):
            r = head_bwd(q[b, h], k[b, kv[h]], v[b, kv[h]], do[b, h], scale, causal, Ls[b])
            out["dq"][b, h], out["o"][b, h], out["lse"][b, h] = r["dq"], r["o"], r["lse"]
            out["dk"][b, kv[h]] += r["dk"]
            out["dv"][b, kv[h]] += r["dv"]
    return out


def _sequence_bounds(cu_seqlens, T: int) -> list[tuple[int, int]]:
    """Rows [t0, t1) of each packed sequence; the offsets must be non-decreasing inside [0, T]."""
    cu = [int(x) for x in np.asarray(as_f64(cu_seqlens)).ravel()]
    if len(cu) < 2 or cu[0] < 0 or cu[-1] > T or any(a > b for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must be non-decreasing offsets inside [0, T]")
    return list(zip(cu[:-1], cu[1:]))


def attention_fwd_varlen(q, k, v, cu_seqlens, scale: float, causal: bool):
    """Packed sequences: q [T, H, d], k, v [T, H_kv, d]; sequence b is rows
    cu_seqlens[b] .. cu_seqlens[b+1] and is its own attention problem of that length (causal
    positions counted from its first row).  Returns (O [T, H, d], lse [H, T]); rows outside
    every sequence stay 0 in O and NaN in lse."""
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    T, H, d = q.shape
    kv = _kv_index(H, k.shape[1])
    O = np.zeros((T, H, d), np.float64)
    lse = np.full((H, T), np.nan, np.float64)
    for t0, t1 in _sequence_bounds(cu_seqlens, T):
        if t1 == t0:
            continue
        for h in range(H):
            O[t0:t1, h], lse[h, t0:t1] = head_fwd(q[t0:t1, h], k[t0:t1, kv[h]], v[t0:t1, kv[h]],
                                                  scale, causal)
    return O, lse


def attention_bwd_varlen(q, k, v, do, cu_seqlens, scale: float, causal: bool):
    """Backward of ``attention_fwd_varlen``: per sequence and query head ``head_bwd``; dK, dV of
    a key/value head summed over the query heads that read it.  Returns a dict with o, lse,
    dq [T, H, d], dk, dv [T, H_kv, d] (rows outside every sequence: 0, lse NaN)."""
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    T, H, d = q.shape
    H_kv = k.shape[1]
    kv = _kv_index(H, H_kv)
    out = {"o": np.zeros((T, H, d)), "lse": np.full((H, T), np.nan), "dq": np.zeros((T, H, d)),
           "dk": np.zeros((T, H_kv, d)), "dv": np.zeros((T, H_kv, d))}
    for t0, t1 in _sequence_bounds(cu_seqlens, T):
        if t1 == t0:
            continue
        for h in range(H):
            r = head_bwd(q[t0:t1, h], k[t0:t1, kv[h]], v[t0:t1, kv[h]], do[t0:t1, h], scale,
                         causal)
            out["o"][t0:t1, h] = r["o"]
            out["lse"][h, t0:t1] = r["lse"]
            out["dq"][t0:t1, h] = r["dq"]
            out["dk"][t0:t1, kv[h]] += r["dk"]
            out["dv"][t0:t1, kv[h]] += r["dv"]
    return out


def attention_decode(q, k_cache, v_cache, scale: float, causal: bool, cache_lens=None):
    """Decode: Nq new queries per sequence, q [B, H, Nq, d], against a key/value cache
    k, v [B, H_kv, N, d] of which sequence b uses its first L_b rows (all N without
    ``cache_lens``); query head h reads cache head h // (H / H_kv).  Query i is position
    L_b - Nq + i of its sequence; causal, it sees keys j <= L_b - Nq + i, otherwise all j < L_b.
    The plain definition per (b, h, i) in fp64: scores s_j = scale * q_i . k_j over the visible
    keys, lse = m + ln sum exp(s_j - m), O = sum_j exp(s_j - lse) v_j (two passes, matrix
    products from numpy).  A query that sees no key gets O = 0 and lse = -inf."""
    q, k, v = as_f64(q), as_f64(k_cache), as_f64(v_cache)
    B, H, Nq, d = q.shape
    H_kv, N = k.shape[1], k.shape[2]
    kv = _kv_index(H, H_kv)
    Ls = _lengths(cache_lens, B, N)
    O = np.zeros((B, H, Nq, d), np.float64)
    lse = np.full((B, H, Nq), -np.inf, np.float64)
    for b in range(B):
        L = Ls[b]
        if not 1 <= L <= N:
            raise ValueError("cache length outside [1, N]")
        for h in range(H):
            s = scale * (q[b, h] @ k[b, kv[h], :L].T)  # [Nq, L]
            for i in range(Nq):
                lim = min(L, L - Nq + i + 1) if causal else L
                if lim <= 0:
                    continue
                row = s[i, :lim]
                m = row.max()
                e = np.exp(row - m)
                tot = e.sum()
                lse[b, h, i] = m + np.log(tot)
                O[b, h, i] = (e / tot) @ v[b, kv[h], :lim]
    return O, lse


def decode_e4m3(codes) -> np.ndarray:
    """Exact values of e4m3 (OCP FP8 E4M3, "fn" variant) codes, from the bit fields: sign bit,
    4-bit exponent with bias 7, 3-bit mantissa; exponent 0 is subnormal (m/8 * 2^-6); the
    all-ones pattern S.1111.111 is NaN; there are no infinities."""
    if hasattr(codes, "detach"):  # a torch tensor of float8 codes: read its raw bytes
        import torch
        codes = codes.detach().cpu().contiguous().view(torch.uint8).numpy()
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return sign * val


def dequantize_fp8(codes, descale) -> np.ndarray:
    """code * descale per (batch, head), exact in fp64: codes [B, Hx, N, d], descale [B, Hx]."""
    return decode_e4m3(codes) * as_f64(descale)[:, :, None, None]


def attention_fwd_fp8(q, k, v, q_descale, k_descale, v_descale, scale: float, causal: bool,
                      seqlens=None):
    """FP8 attention (FlashAttention-3's FP8 mode; Russian article, "FlashAttention-3 (2024)"):
    the quantised inputs stand for the values code * descale, and the result is the exact
    attention of those values (``attention_fwd_gqa`` in fp64).  The GPU's own rounding of P to
    e4m3 is an approximation of this; its error bound lives with the parity tests."""
    return attention_fwd_gqa(dequantize_fp8(q, q_descale), dequantize_fp8(k, k_descale),
                             dequantize_fp8(v, v_descale), scale, causal, seqlens)
