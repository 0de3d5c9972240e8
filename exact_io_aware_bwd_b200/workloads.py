"""Seeded synthetic inputs for the attention workloads.

This module holds no attention arithmetic: it only names the workloads and
draws their random inputs, so that the GPU path and the CPU oracle can be fed
the very same values.

The pages measure on no public data set; they speak of long documents of
4K-64K tokens ("FlashAttention" glossary, 4K-token and 16K-token examples;
"flash attention io aware", section "Performance Impact", N = 4096).  The
five workloads below are purely synthetic:

  name  shape (B, Hq, Hkv, N, d)   dtype  distribution                 causal
  tiny  (1, 2, 2, 256, 64)         bf16   Q, K, V, dO ~ N(0, 1)        both
  gpt2  (8, 12, 12, 2048, 64)      bf16   N(0, 1)                      both
  mha4k (4, 32, 32, 4096, 128)     bf16   N(0, 1)                      causal
  gqa16k(1, 32, 8, 16384, 128)     bf16   N(0, 1)                      causal
  long64k(1, 16, 16, 65536, 128)   fp16   Q, K ~ N(0, 3^2); V, dO ~ N(0,1) causal

Recipe: a CPU ``torch.Generator`` seeded with ``1234 + 100 * index`` draws
fp32 normals in the fixed order Q, K, V, dO; each is multiplied by its sigma
and rounded to the I/O dtype (round to nearest even).  Row subsets for the
large workloads come from ``randperm`` with the seed + 7.

FP8 inputs (``make_fp8_inputs``) take the same fp32 draws of Q, K and V and
quantise each tensor to E4M3 codes with one factor per tensor,
delta = max|x| / 448 (448: the largest finite E4M3 value), code = E4M3(x / delta)
rounded to nearest even by torch, so that the codes span the format's range.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    dtype: torch.dtype
    causal_modes: tuple
    sigma_qk: float = 1.0
    sigma_vdo: float = 1.0
    check_rows: int = 0          # 0: every row is checked
    check_col_heads: int = 0     # kv heads whose dK/dV columns are checked
    check_cols: int = 0          # kv rows checked per such head
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def seed(self) -> int:
        return 1234 + 100 * self.index

    def flops_fwd(self, causal: bool, window: int = 0) -> float:
        """Forward FLOPs by the convention 4*B*Hq*N^2*d, halved when causal.
        With a causal sliding window of W < N keys: 4*B*Hq*d per visible
        (query, key) pair, N*W - W(W-1)/2 pairs per head."""
        N = self.N
        if causal and 0 < window < N:
            return 4.0 * self.B * self.Hq * self.d * (N * window - window * (window - 1) / 2)
        f = 4.0 * self.B * self.Hq * N * N * self.d
        return f / 2 if causal else f

    def flops_bwd(self, causal: bool, window: int = 0) -> float:
        """Backward FLOPs by the convention 2.5 x forward."""
        return 2.5 * self.flops_fwd(causal, window)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 1, 1, 2, 2, 256, 64, torch.bfloat16, (False, True),
                 note="tiny MHA, every output checked"),
        Workload("gpt2", 2, 8, 12, 12, 2048, 64, torch.bfloat16, (False, True),
                 note="GPT-2-small-shaped MHA"),
        Workload("mha4k", 3, 4, 32, 32, 4096, 128, torch.bfloat16, (True,),
                 check_rows=512, check_col_heads=2, check_cols=64,
                 note="4K-token MHA"),
        Workload("gqa16k", 4, 1, 32, 8, 16384, 128, torch.bfloat16, (True,),
                 check_rows=512, check_col_heads=1, check_cols=32,
                 note="long-context GQA, 4 query heads per kv head"),
        Workload("long64k", 5, 1, 16, 16, 65536, 128, torch.float16, (True,),
                 sigma_qk=3.0, check_rows=256, check_col_heads=1, check_cols=16,
                 note="64K tokens, wide logit range"),
    ]
}


def make_inputs(w: Workload, seed: int | None = None, device: str = "cpu",
                shape_override: tuple | None = None):
    """Q, K, V, dO for workload ``w`` as I/O-dtype tensors.

    Drawn on the CPU generator (so every device sees the same values), then
    moved to ``device``.  ``shape_override`` = (B, Hq, Hkv, N, d) keeps the
    recipe but changes the sizes (edge-case tests)."""
    B, Hq, Hkv, N, d = shape_override or (w.B, w.Hq, w.Hkv, w.N, w.d)
    g = torch.Generator("cpu").manual_seed(w.seed if seed is None else seed)
    q = torch.randn((B, Hq, N, d), generator=g, dtype=torch.float32) * w.sigma_qk
    k = torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32) * w.sigma_qk
    v = torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32) * w.sigma_vdo
    do = torch.randn((B, Hq, N, d), generator=g, dtype=torch.float32) * w.sigma_vdo
    out = [t.to(w.dtype) for t in (q, k, v, do)]
    if device != "cpu":
        out = [t.to(device) for t in out]
    return out


def make_fp8_inputs(w: Workload, seed: int | None = None, device: str = "cpu",
                    shape_override: tuple | None = None):
    """E4M3 codes of Q, K, V (uint8 tensors) and their factors (delta_q,
    delta_k, delta_v): x is represented by delta * E4M3(code)."""
    B, Hq, Hkv, N, d = shape_override or (w.B, w.Hq, w.Hkv, w.N, w.d)
    g = torch.Generator("cpu").manual_seed(w.seed if seed is None else seed)
    q = torch.randn((B, Hq, N, d), generator=g, dtype=torch.float32) * w.sigma_qk
    k = torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32) * w.sigma_qk
    v = torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32) * w.sigma_vdo
    codes, factors = [], []
    for x in (q, k, v):
        amax = float(x.abs().max()) if x.numel() else 0.0
        delta = torch.tensor(amax / 448.0 if amax > 0 else 1.0, dtype=torch.float32)
        codes.append((x / delta).to(torch.float8_e4m3fn).view(torch.uint8))
        factors.append(float(delta))
    if device != "cpu":
        codes = [c.to(device) for c in codes]
    return codes, tuple(factors)


def check_rows(w: Workload, N: int | None = None, seed: int | None = None) -> torch.Tensor:
    """Sorted seeded query rows checked against the oracle (all rows if unset)."""
    N = w.N if N is None else N
    if not w.check_rows or w.check_rows >= N:
        return torch.arange(N)
    g = torch.Generator("cpu").manual_seed((w.seed if seed is None else seed) + 7)
    return torch.sort(torch.randperm(N, generator=g)[: w.check_rows]).values


# Key rows of the 64K workload's column check drawn from its first 256 keys.
LONG_LOW_COLS = 4


def check_cols(w: Workload, causal: bool, seed: int | None = None):
    """Seeded (b, hkv, kv rows) triples whose dK/dV the oracle recomputes.

    Under a causal mask dK_j and dV_j depend on the query rows i >= j.  For
    the 64K workload most checked kv rows come from the upper half of the
    sequence and LONG_LOW_COLS from its first 256 keys: those are the key
    rows whose gradients sum over the most queries (up to all 65 536), the
    longest reductions of the pass; the oracle then needs the statistics of
    every row of the head once."""
    g = torch.Generator("cpu").manual_seed(w.seed + 11)
    heads = torch.randperm(w.B * w.Hkv, generator=g)[: w.check_col_heads].tolist()
    long_causal = causal and w.N >= 65536
    lo = w.N // 2 if long_causal else 0
    out = []
    for bh in heads:
        n_hi = w.check_cols - (LONG_LOW_COLS if long_causal else 0)
        cols = lo + torch.randperm(w.N - lo, generator=g)[:n_hi]
        if long_causal:
            cols = torch.cat([torch.randperm(256, generator=g)[:LONG_LOW_COLS], cols])
        out.append((bh // w.Hkv, bh % w.Hkv, torch.sort(cols).values))
    return out
