"""Host-side arithmetic without a GPU: the FLOP convention under a sliding
window (counted pairs against brute force), and the decode workspace size
(split count times rows times (d + 2) fp32 values)."""

import math

import pytest

from exact_io_aware_bwd_b200 import binding
from exact_io_aware_bwd_b200.workloads import WORKLOADS


def visible_pairs(N, W):
    return sum(1 for i in range(N) for j in range(N) if j <= i and j > i - W)


@pytest.mark.parametrize("N,W", [(16, 1), (16, 5), (37, 36), (64, 64), (50, 8)])
def test_window_flops_count_visible_pairs(N, W):
    from dataclasses import replace
    w = replace(WORKLOADS["tiny"], N=N)
    per_pair = 4.0 * w.B * w.Hq * w.d
    if W < N:
        assert w.flops_fwd(True, W) == pytest.approx(per_pair * visible_pairs(N, W))
    else:  # a window covering the sequence is the causal convention N^2 / 2
        assert w.flops_fwd(True, W) == w.flops_fwd(True)
    assert w.flops_bwd(True, W) == pytest.approx(2.5 * w.flops_fwd(True, W))


def splits(B, Hkv, max_pages):
    want = math.ceil(2 * 148 / (B * Hkv))
    return max(1, min(want, max_pages))


@pytest.mark.parametrize("B,Hq,Hkv,Nq,d,max_pages", [
    (32, 32, 8, 1, 128, 256), (1, 8, 8, 3, 64, 1), (2, 16, 1, 2, 128, 19), (300, 4, 4, 1, 64, 10)])
def test_decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_pages):
    S = splits(B, Hkv, max_pages)
    assert binding.fa_decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_pages) == B * Hq * Nq * S * (d + 2) * 4
    assert binding.fa_decode_workspace_bytes(0, Hq, Hkv, Nq, d, max_pages) == 0
