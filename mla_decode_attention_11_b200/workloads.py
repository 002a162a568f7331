"""Seeded synthetic MLA-decode workloads (shapes, lengths, values).

This module only draws random inputs; it holds none of the attention
arithmetic, so both the CUDA path's tests and the fp64 oracle can use it
without sharing any of the method's code.

Recipe (identical on every machine, CPU generators only):
  * lengths: fixed per workload, or for the mixed-length workload
    ``torch.randint(lo, hi + 1, (B,))`` from ``torch.Generator().manual_seed(seed)``;
  * per sequence b, q[b] is ``torch.randn(Sq, H, 576) * sigma`` and the first
    L_b rows of kv[b] are ``torch.randn(L_b, 576) * sigma``, each from its own
    generator seeded with ``_stream_seed(seed, b, which)``, then rounded to
    bfloat16 (round to nearest even);
  * kv rows L_b .. L_max-1 are filled with ``tail_fill`` (NaN in the parity
    tests, so any read past a sequence's end shows up in the result).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

D_QK = 576      # 512 latent + 64 rope columns per cached row
D_V = 512       # values are the first 512 columns of the same rows
D_ROPE = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Sq: int
    H: int
    L: int                      # L_max (every sequence has this length unless L_lo is set)
    L_lo: Optional[int] = None  # mixed lengths: uniform integers in [L_lo, L]
    sigma: float = 1.0
    seed: int = 0

    @property
    def scale(self) -> float:
        # softmax scale 576^-0.5 (= 1/24 in real arithmetic), as an fp32 value
        return float(torch.tensor(D_QK ** -0.5, dtype=torch.float32).item())

    def lengths(self) -> torch.Tensor:
        if self.L_lo is None:
            return torch.full((self.B,), self.L, dtype=torch.int32)
        g = torch.Generator().manual_seed(self.seed)
        return torch.randint(self.L_lo, self.L + 1, (self.B,), generator=g, dtype=torch.int64).to(torch.int32)

    def algorithmic_bytes(self, lengths: Optional[torch.Tensor] = None) -> int:
        """Bytes a perfect kernel must move: each used kv row once (V aliases
        K), q, out (bf16), lse (fp32) and the lengths array."""
        sl = self.lengths() if lengths is None else lengths
        rows = self.B * self.Sq * self.H
        return int(sl.to(torch.int64).sum()) * D_QK * 2 + rows * (D_QK * 2 + D_V * 2 + 4) + self.B * 4

    def algorithmic_bytes_fp8(self, lengths: Optional[torch.Tensor] = None) -> int:
        """As algorithmic_bytes with the cache held as one-byte E4M3 codes."""
        sl = self.lengths() if lengths is None else lengths
        rows = self.B * self.Sq * self.H
        return int(sl.to(torch.int64).sum()) * D_QK + rows * (D_QK * 2 + D_V * 2 + 4) + self.B * 4

    def algorithmic_flops(self, lengths: Optional[torch.Tensor] = None) -> int:
        """2*(576+512) flops per (query row, key): QK^T and PV, exps not counted."""
        sl = self.lengths() if lengths is None else lengths
        return int(sl.to(torch.int64).sum()) * self.Sq * self.H * 2 * (D_QK + D_V)


# The five parity/benchmark workloads, plus the headline-metric line
# (mixed-length workload's shape with every sequence at L = 8192).
WORKLOADS = {
    "tiny": Workload("tiny", B=1, Sq=1, H=16, L=256, seed=1000),
    "dsv3": Workload("dsv3", B=16, Sq=1, H=128, L=4096, seed=1001),
    "mixed": Workload("mixed", B=64, Sq=1, H=128, L=8192, L_lo=1024, seed=1002),
    "lowhead": Workload("lowhead", B=132, Sq=1, H=16, L=16384, seed=1003),
    "long": Workload("long", B=4, Sq=2, H=128, L=131072, sigma=0.5, seed=1004),
    "metric": Workload("metric", B=64, Sq=1, H=128, L=8192, seed=1005),
}


def _stream_seed(seed: int, b: int, which: int) -> int:
    # distinct, reproducible generator per (workload seed, sequence, tensor)
    return (seed * 1_000_003 + b * 4 + which) & ((1 << 62) - 1)


def make_q(w: Workload, b: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(_stream_seed(w.seed, b, 0))
    return (torch.randn(w.Sq, w.H, D_QK, generator=g) * w.sigma).to(torch.bfloat16)


def make_kv_rows(w: Workload, b: int, n_rows: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(_stream_seed(w.seed, b, 1))
    return (torch.randn(n_rows, D_QK, generator=g) * w.sigma).to(torch.bfloat16)


def generate(w: Workload, tail_fill: float = float("nan"), lengths: Optional[torch.Tensor] = None):
    """Materialise (q [B,Sq,H,576], kv [B,L_max,576], seqlens [B]) on the CPU."""
    sl = w.lengths() if lengths is None else lengths.to(torch.int32)
    q = torch.empty((w.B, w.Sq, w.H, D_QK), dtype=torch.bfloat16)
    kv = torch.empty((w.B, w.L, D_QK), dtype=torch.bfloat16)
    for b in range(w.B):
        q[b] = make_q(w, b)
        Lb = int(sl[b])
        if Lb > 0:
            kv[b, :Lb] = make_kv_rows(w, b, Lb)
        if Lb < w.L:
            kv[b, Lb:] = tail_fill
    return q, kv, sl


E4M3_MAX = 448.0
E4M3_NAN_CODE = 0x7F


def generate_fp8(w: Workload, lengths: Optional[torch.Tensor] = None):
    """The same inputs with the cache quantised to E4M3 codes: (q [B,Sq,H,576]
    bf16, codes [B,L_max,576] uint8, kv_scale, seqlens [B]).  kv_scale =
    max|kv| / 448 over the used rows (per-tensor amax scaling, as an fp32
    value); each bf16 value is divided by it and rounded to the nearest E4M3
    code by torch's own conversion.  Rows at or past a length hold the NaN
    code (never a value of the used rows), so a read past a length shows."""
    q, kv, sl = generate(w, tail_fill=0.0, lengths=lengths)
    amax = float(kv.float().abs().max())
    kv_scale = float(torch.tensor(max(amax, 1e-30) / E4M3_MAX, dtype=torch.float32).item())
    codes = (kv.float() / kv_scale).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn).view(torch.uint8)
    for b in range(w.B):
        codes[b, int(sl[b]):] = E4M3_NAN_CODE
    return q, codes.contiguous(), kv_scale, sl


def small_variant(w: Workload, B: Optional[int] = None, L: Optional[int] = None,
                  L_lo: Optional[int] = None, seed_offset: int = 0) -> Workload:
    """Same head layout and value distribution at a size the oracle finishes quickly."""
    return dataclasses.replace(w, name=w.name + "_small", B=B or w.B, L=L or w.L,
                               L_lo=L_lo if w.L_lo is not None else None,
                               seed=w.seed + seed_offset)


def custom(B: int, Sq: int, H: int, L: int, L_lo: Optional[int] = None,
           sigma: float = 1.0, seed: int = 7) -> Workload:
    return Workload(f"custom_B{B}_Sq{Sq}_H{H}_L{L}", B=B, Sq=Sq, H=H, L=L, L_lo=L_lo,
                    sigma=sigma, seed=seed)


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


# ---------------------------------------------------------------- MHA decode
# Standard multi-head attention decode with grouped kv heads (128-wide heads,
# separate K and V).  Same recipe: per sequence b, q[b] = randn(Sq, H, 128),
# k[b, :L_b] = randn(L_b, Hkv, 128) and v[b, :L_b] = randn(L_b, Hkv, 128),
# each from its own seeded generator, times sigma, rounded to bf16; rows past
# L_b filled with tail_fill.

MHA_D = 128


@dataclasses.dataclass(frozen=True)
class MhaWorkload:
    name: str
    B: int
    Sq: int
    H: int
    Hkv: int
    L: int
    L_lo: Optional[int] = None
    sigma: float = 1.0
    seed: int = 0

    @property
    def scale(self) -> float:
        return float(torch.tensor(MHA_D ** -0.5, dtype=torch.float32).item())

    def lengths(self) -> torch.Tensor:
        return Workload(self.name, self.B, self.Sq, self.H, self.L, self.L_lo, self.sigma, self.seed).lengths()

    def algorithmic_bytes(self, lengths: Optional[torch.Tensor] = None) -> int:
        """Each used K and V row once (per kv head), q, out, lse, lengths."""
        sl = self.lengths() if lengths is None else lengths
        rows = self.B * self.Sq * self.H
        return (int(sl.to(torch.int64).sum()) * self.Hkv * MHA_D * 2 * 2 + rows * (MHA_D * 2 * 2 + 4)
                + self.B * 4)

    def algorithmic_flops(self, lengths: Optional[torch.Tensor] = None) -> int:
        """2*(128+128) flops per (query row, key)."""
        sl = self.lengths() if lengths is None else lengths
        return int(sl.to(torch.int64).sum()) * self.Sq * self.H * 2 * (2 * MHA_D)


# a grouped-query decode batch (32 query heads over 8 kv heads of 128, 64
# sequences of 8192 keys) and a small mixed-length case
MHA_WORKLOADS = {
    "mha_gqa": MhaWorkload("mha_gqa", B=64, Sq=1, H=32, Hkv=8, L=8192, seed=2001),
    "mha_small": MhaWorkload("mha_small", B=6, Sq=2, H=16, Hkv=4, L=1500, L_lo=1, seed=2002),
}


def generate_mha(w: MhaWorkload, tail_fill: float = float("nan"), lengths: Optional[torch.Tensor] = None):
    """Materialise (q [B,Sq,H,128], k [B,L,Hkv,128], v [B,L,Hkv,128], seqlens [B]) on the CPU."""
    sl = w.lengths() if lengths is None else lengths.to(torch.int32)
    q = torch.empty((w.B, w.Sq, w.H, MHA_D), dtype=torch.bfloat16)
    k = torch.empty((w.B, w.L, w.Hkv, MHA_D), dtype=torch.bfloat16)
    v = torch.empty((w.B, w.L, w.Hkv, MHA_D), dtype=torch.bfloat16)
    for b in range(w.B):
        gq = torch.Generator().manual_seed(_stream_seed(w.seed, b, 0))
        q[b] = (torch.randn(w.Sq, w.H, MHA_D, generator=gq) * w.sigma).to(torch.bfloat16)
        Lb = int(sl[b])
        if Lb > 0:
            gk = torch.Generator().manual_seed(_stream_seed(w.seed, b, 1))
            gv = torch.Generator().manual_seed(_stream_seed(w.seed, b, 2))
            k[b, :Lb] = (torch.randn(Lb, w.Hkv, MHA_D, generator=gk) * w.sigma).to(torch.bfloat16)
            v[b, :Lb] = (torch.randn(Lb, w.Hkv, MHA_D, generator=gv) * w.sigma).to(torch.bfloat16)
        if Lb < w.L:
            k[b, Lb:] = tail_fill
            v[b, Lb:] = tail_fill
    return q, k, v, sl


__all__ = ["Workload", "WORKLOADS", "generate", "make_q", "make_kv_rows", "small_variant",
           "custom", "D_QK", "D_V", "D_ROPE", "ceil_div", "MhaWorkload", "MHA_WORKLOADS", "generate_mha", "MHA_D"]
