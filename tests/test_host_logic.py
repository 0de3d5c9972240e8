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


def splits(B, Hkv, d, max_pages):
    # at least four waves of the blocks a 148-SM B200 holds at once (one per
    # SM at d = 128, two at d = 64); among S0 .. 2 S0 the count whose last
    # wave is the fullest; at least 4 pages a split
    slots = 148 * (2 if d == 64 else 1)
    bh = max(1, B * Hkv)
    s0 = -(-4 * slots // bh)
    cap = max(1, max_pages // 4)
    best, best_eff = min(s0, cap), -1.0
    for s in range(s0, min(2 * s0, cap) + 1):
        blocks = bh * s
        eff = blocks / (-(-blocks // slots) * slots)
        if eff > best_eff + 1e-9:
            best, best_eff = s, eff
    return max(1, best)


@pytest.mark.parametrize("B,Hq,Hkv,Nq,d,max_pages", [
    (32, 32, 8, 1, 128, 256), (1, 8, 8, 3, 64, 1), (2, 16, 1, 2, 128, 19), (300, 4, 4, 1, 64, 10)])
def test_decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_pages):
    S = splits(B, Hkv, d, max_pages)
    assert binding.fa_decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_pages) == B * Hq * Nq * S * (d + 2) * 4
    assert binding.fa_decode_workspace_bytes(0, Hq, Hkv, Nq, d, max_pages) == 0


def test_fp8_inputs_quantise_the_16bit_draws():
    """The E4M3 inputs are the same seeded fp32 draws as the 16-bit inputs,
    each tensor divided by max|x| / 448 and rounded to E4M3: the largest code
    is 448 in magnitude, no code is NaN, and dequantised values are within
    E4M3's half-ulp (2^-4 relative, 2^-10 absolute below 2^-6) of the draws."""
    import torch
    from exact_io_aware_bwd_b200.workloads import make_fp8_inputs, make_inputs
    w = WORKLOADS["tiny"]
    (q8, k8, v8), ds = make_fp8_inputs(w, seed=5, shape_override=(1, 2, 1, 40, 128))
    g = torch.Generator("cpu").manual_seed(5)
    draws = [torch.randn((1, 2, 40, 128), generator=g), torch.randn((1, 1, 40, 128), generator=g),
             torch.randn((1, 1, 40, 128), generator=g)]
    for c, delta, x in zip((q8, k8, v8), ds, draws):
        assert c.dtype == torch.uint8 and c.shape == x.shape
        val = c.view(torch.float8_e4m3fn).double()
        assert not torch.isnan(val).any()
        assert float(val.abs().max()) == 448.0
        assert delta == float(torch.tensor(float(x.abs().max()) / 448.0, dtype=torch.float32))
        y = x.double() / delta
        err = (val - y).abs()
        bound = torch.maximum(y.abs() * 2.0 ** -4, torch.full_like(y, 2.0 ** -10))
        assert bool((err <= bound * (1 + 1e-6)).all())
    # the same seed gives the same codes; the 16-bit inputs share the draws
    again = make_fp8_inputs(w, seed=5, shape_override=(1, 2, 1, 40, 128))[0]
    assert all(torch.equal(a, b) for a, b in zip((q8, k8, v8), again))
    q16 = make_inputs(w, seed=5, shape_override=(1, 2, 1, 40, 128))[0]
    assert torch.equal(q16, draws[0].to(w.dtype))


def test_fp8_flops_follow_the_forward_convention():
    w = WORKLOADS["mha4k"]
    assert w.flops_fwd(True) == 4.0 * 4 * 32 * 4096 * 4096 * 128 / 2


def test_profiled_traffic_is_reported_only_for_the_profiled_sources():
    """The bench reports an ncu traffic figure only while the kernel sources
    still hash to the digest recorded with it, and only for its workload."""
    import bench
    for spec in (bench.PROFILED_TRAFFIC, bench.PROFILED_TRAFFIC_FWD, bench.PROFILED_TRAFFIC_FP8,
                 bench.PROFILED_TRAFFIC_DEC):
        got = bench.profiled_traffic(spec["workload"], spec)
        assert got in (None, spec["bytes"])
        assert bench.profiled_traffic("tiny", spec) is None
        stale = dict(spec, sources_sha256_16="0" * 16)
        assert bench.profiled_traffic(spec["workload"], stale) is None
        missing = dict(spec, sources=("exact_io_aware_bwd_b200/csrc/no_such_file.cuh",))
        assert bench.profiled_traffic(spec["workload"], missing) is None
