"""Seeded synthetic inputs for exact attention, shared by the oracle side and the CUDA side.

This module holds no attention arithmetic.  It only draws random numbers, rounds them to
bf16 and names the workload shapes, so that the oracle (``oracle/``) and the CUDA path
(``io_aware_exact_16_b200``) can be fed the identical bf16 values without sharing any code
that computes attention.

Input recipe (one generator per workload, ``torch.Generator().manual_seed(seed)``):

* key-padding lengths, when the workload has them, are drawn FIRST from the generator as
  ``L_b ~ UniformInt[lo, hi]`` inclusive, one per batch entry;
* then Q, K, V and dO are drawn in that order as fp32 ``std * N(0, 1)`` of shape
  ``[B, H, N, d]`` (K and V ``[B, H_kv, N, d]`` for grouped-query workloads) and rounded to
  bf16 (round to nearest even, torch ``.to(bfloat16)``).

The workload shapes follow the pages' own workloads: GPT-2 at sequence length 1K and
BERT-large at 512 (FlashAttention (DE), "Empirische Ergebnisse"), the 8K-32K long-context
memory example (flash-attention glossary page, "Voorbeeld") and a throughput sweep at a
fixed token count that spans the Long-Range-Arena lengths 1K-4K and beyond.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, mask kind and the input distribution."""

    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int
    std: float = 1.0
    # inclusive range of key-padding lengths, or None for "every key is valid"
    pad_range: Optional[tuple[int, int]] = None
    backward: bool = True
    # key/value heads (grouped-query attention); None means H (one K/V head per query head)
    H_kv: Optional[int] = None

    @property
    def kv_heads(self) -> int:
        return self.H if self.H_kv is None else self.H_kv

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)

    def describe(self) -> dict:
        out = {"workload": self.name, "B": self.B, "H": self.H, "N": self.N, "d": self.d,
               "causal": self.causal, "seed": self.seed, "std": self.std,
               "pad_range": list(self.pad_range) if self.pad_range else None}
        return out


def tiny() -> Workload:
    return Workload("tiny B1 H1 N128 d64", 1, 1, 128, 64, False, 1001)


def gpt2_small() -> Workload:
    return Workload("gpt2-small causal B8 H12 N1024 d64", 8, 12, 1024, 64, True, 1002)


def bert_large_padded() -> Workload:
    return Workload("bert-large padded B16 H16 N512 d64", 16, 16, 512, 64, False, 1003,
                    pad_range=(128, 512))


def long_context(N: int) -> Workload:
    assert N in (8192, 16384, 32768)
    return Workload(f"long-context causal fwd B1 H16 N{N} d128", 1, 16, N, 128, True, 1004,
                    std=0.5, backward=False)


SWEEP_N = (512, 1024, 2048, 4096, 8192, 16384)
SWEEP_HD = ((16, 128), (32, 64))


def sweep(N: int, H: int, d: int, causal: bool) -> Workload:
    """Fixed 16384 tokens per batch: B = 16384 / N."""
    assert N in SWEEP_N and (H, d) in SWEEP_HD
    idx = SWEEP_N.index(N) * 4 + SWEEP_HD.index((H, d)) * 2 + int(causal)
    return Workload(f"sweep {'causal' if causal else 'non-causal'} B{16384 // N} H{H} N{N} d{d}",
                    16384 // N, H, N, d, causal, 1005 + idx)


def all_sweep() -> list[Workload]:
    return [sweep(N, H, d, c) for N in SWEEP_N for (H, d) in SWEEP_HD for c in (False, True)]


def custom(B: int, H: int, N: int, d: int, causal: bool, seed: int, std: float = 1.0,
           pad_range: Optional[tuple[int, int]] = None, name: str = "custom",
           H_kv: Optional[int] = None) -> Workload:
    return Workload(name, B, H, N, d, causal, seed, std, pad_range, H_kv=H_kv)


@dataclasses.dataclass
class Inputs:
    q: torch.Tensor          # bf16 [B, H, N, d], CPU
    k: torch.Tensor
    v: torch.Tensor
    do: torch.Tensor
    seqlens: Optional[torch.Tensor]  # int32 [B] key lengths, CPU, or None


def make_inputs(w: Workload, with_grad: bool = True) -> Inputs:
    """Draw the workload's seeded bf16 inputs on the CPU (see the module docstring)."""
    g = torch.Generator().manual_seed(w.seed)
    seqlens = None
    if w.pad_range is not None:
        lo, hi = w.pad_range
        seqlens = torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64).to(torch.int32)
    shape = (w.B, w.H, w.N, w.d)
    kv_shape = (w.B, w.kv_heads, w.N, w.d)

    def draw(sh) -> torch.Tensor:
        x = torch.randn(sh, generator=g, dtype=torch.float32)
        if w.std != 1.0:
            x.mul_(w.std)
        return x.to(torch.bfloat16)

    q = draw(shape)
    k = draw(kv_shape)
    v = draw(kv_shape)
    do = draw(shape) if with_grad else torch.empty(0, dtype=torch.bfloat16)
    return Inputs(q, k, v, do, seqlens)


@dataclasses.dataclass(frozen=True)
class PackedWorkload:
    """Variable-length sequences stored back to back ([T, H, d] with offsets cu_seqlens)."""

    name: str
    B: int
    H: int
    H_kv: int
    d: int
    causal: bool
    seed: int
    len_range: tuple[int, int] = (1, 512)    # inclusive range the lengths are drawn from
    lengths: Optional[tuple[int, ...]] = None  # fixed lengths instead of drawn ones
    std: float = 1.0

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)


@dataclasses.dataclass
class PackedInputs:
    q: torch.Tensor           # bf16 [T, H, d], CPU
    k: torch.Tensor           # bf16 [T, H_kv, d]
    v: torch.Tensor
    do: torch.Tensor          # bf16 [T, H, d]
    cu_seqlens: torch.Tensor  # int32 [B + 1], CPU
    max_seqlen: int


def make_packed_inputs(w: PackedWorkload) -> PackedInputs:
    """Packed recipe: the B lengths are drawn first as UniformInt[lo, hi] (unless fixed), then
    Q, K, V, dO in that order as fp32 std * N(0, 1) over the T = sum(lengths) packed rows,
    rounded to bf16."""
    g = torch.Generator().manual_seed(w.seed)
    if w.lengths is not None:
        lens = [int(x) for x in w.lengths]
        assert len(lens) == w.B
    else:
        lo, hi = w.len_range
        lens = torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64).tolist()
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    T = max(cu[-1], 1)

    def draw(sh) -> torch.Tensor:
        x = torch.randn(sh, generator=g, dtype=torch.float32)
        if w.std != 1.0:
            x.mul_(w.std)
        return x.to(torch.bfloat16)

    q = draw((T, w.H, w.d))
    k = draw((T, w.H_kv, w.d))
    v = draw((T, w.H_kv, w.d))
    do = draw((T, w.H, w.d))
    return PackedInputs(q, k, v, do, torch.tensor(cu, dtype=torch.int32), max(max(lens), 1))


E4M3_MAX = 448.0


@dataclasses.dataclass
class FP8Inputs:
    q: torch.Tensor          # float8_e4m3fn [B, H, N, d], CPU (codes)
    k: torch.Tensor          # float8_e4m3fn [B, H_kv, N, d]
    v: torch.Tensor
    q_descale: torch.Tensor  # fp32 [B, H]:    q = code * q_descale
    k_descale: torch.Tensor  # fp32 [B, H_kv]
    v_descale: torch.Tensor  # fp32 [B, H_kv]
    seqlens: Optional[torch.Tensor]


def _quantize_per_head(x: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """Per-(batch, head) scaling to the e4m3 range: descale = amax / 448, code =
    e4m3(x / descale) (round to nearest even, clamped to +-448)."""
    amax = x.abs().amax(dim=(2, 3)).clamp_min(1e-12)
    descale = (amax / E4M3_MAX).to(torch.float32)
    codes = (x / descale[:, :, None, None]).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return codes, descale


def make_fp8_inputs(w: Workload) -> FP8Inputs:
    """FP8 recipe: the workload's fp32 draws (same generator order as ``make_inputs``: lengths,
    then Q, K, V), each head quantised to e4m3 codes with a per-head descale factor."""
    g = torch.Generator().manual_seed(w.seed)
    seqlens = None
    if w.pad_range is not None:
        lo, hi = w.pad_range
        seqlens = torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64).to(torch.int32)

    def draw(sh) -> torch.Tensor:
        x = torch.randn(sh, generator=g, dtype=torch.float32)
        return x.mul_(w.std) if w.std != 1.0 else x

    q = draw((w.B, w.H, w.N, w.d))
    k = draw((w.B, w.kv_heads, w.N, w.d))
    v = draw((w.B, w.kv_heads, w.N, w.d))
    (qc, qd), (kc, kd), (vc, vd) = (_quantize_per_head(t) for t in (q, k, v))
    return FP8Inputs(qc, kc, vc, qd, kd, vd, seqlens)


def seeded_sample(seed: int, population: int, count: int) -> list[int]:
    """A seeded subset of range(population), sorted; used to pick heads and rows to check."""
    g = torch.Generator().manual_seed(seed)
    count = min(count, population)
    return sorted(torch.randperm(population, generator=g)[:count].tolist())
