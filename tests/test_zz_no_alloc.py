"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device
memory (it uses the library's fixed scratch array instead of a workspace).
Its results must match the oracle and fa_bwd with a caller workspace, call
after call: the same call twice in a row, and a small problem right after a
large one has filled the array, so that stale accumulator values sit exactly
where the small problem's accumulator goes unless each call clears it.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process."""

import math
import os
import re

import pytest
import torch

import attn_check as ac
from exact_io_aware_bwd_b200 import binding
from exact_io_aware_bwd_b200.build import build
from exact_io_aware_bwd_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fa.h")


def scratch_bytes() -> int:
    """FA_BWD_NOALLOC_SCRATCH_BYTES as include/fa.h defines it."""
    text = open(HEADER).read()
    m = re.search(r"#define\s+FA_BWD_NOALLOC_SCRATCH_BYTES\s+\(([^)]*)\)", text)
    assert m, "FA_BWD_NOALLOC_SCRATCH_BYTES not found in include/fa.h"
    return int(eval(m.group(1).replace("u", ""), {}))  # e.g. "64u * 1024u * 1024u"


@pytest.fixture(scope="module", autouse=True)
def lib():
    build()
    binding.load()


def _case(shape, dtype, seed, causal):
    from dataclasses import replace
    w = replace(WORKLOADS["tiny"], dtype=dtype)
    q, k, v, do = make_inputs(w, seed=seed, shape_override=shape)
    scale = 1.0 / math.sqrt(shape[-1])
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = binding.attention_fwd(qd, kd, vd, scale, causal)
    return (q, k, v, do), (qd, kd, vd, do.cuda(), o, lse), scale


def _noalloc(dev, scale, causal):
    q, k, v, do, o, lse = dev
    got = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    binding.fa_bwd_noalloc(q, k, v, o, do, lse, *got, scale, causal)
    assert binding.fa_get_device_status() == binding.FA_OK
    return [t.cpu() for t in got]


def _check(cpu, got, ref_ws, scale, causal, what):
    import oracle
    q, k, v, do = cpu
    dq_r, dk_r, dv_r = oracle.bwd(q, k, v, do, scale, causal)
    for name, g, w, r in zip(("dQ", "dK", "dV"), got, ref_ws, (dq_r, dk_r, dv_r)):
        ac.check_grad(g, r, f"{name} {what} against the oracle")
        e = ac.rel_frob(g, w)
        assert e <= ac.TOL_GRAD, f"{name} {what} against fa_bwd: {e:.3e}"


def test_noalloc_matches_oracle_on_consecutive_calls():
    # (shape, dtype, seed, causal); the first fills most of the array, the
    # second's accumulator then sits on top of its leftovers
    large = ((2, 8, 4, 1000, 128), torch.bfloat16, 3, True)
    small = ((1, 3, 1, 300, 64), torch.float16, 4, False)
    assert binding.fa_bwd_workspace_bytes(2, 8, 4, 1000, 128) <= scratch_bytes()
    for shape, dtype, seed, causal in (large, large, small, small):
        cpu, dev, scale = _case(shape, dtype, seed, causal)
        q, k, v, do, o, lse = dev
        ref_ws = [t.cpu() for t in binding.attention_bwd(q, k, v, o, do, lse, scale, causal)]
        got = _noalloc(dev, scale, causal)
        _check(cpu, got, ref_ws, scale, causal, f"{shape}")


def test_noalloc_rejects_problems_beyond_the_scratch():
    B, Hq, Hkv, N, d = 1, 16, 16, 16384, 128
    assert binding.fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) > scratch_bytes()
    q = torch.empty((B, Hq, N, d), device="cuda", dtype=torch.bfloat16)
    lse = torch.empty((B, Hq, N), device="cuda", dtype=torch.float32)
    with pytest.raises(binding.FaError) as e:
        binding.fa_bwd_noalloc(q, q, q, q, q, lse, q, q, q, 0.1, True)
    assert e.value.status == binding.FA_ERR_UNSUPPORTED
