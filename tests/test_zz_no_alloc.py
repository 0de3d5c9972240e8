"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device
memory (it uses the library's fixed scratch array instead of a workspace).
Its results must match fa_bwd with a caller workspace, call after call.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process."""

import ctypes
import math

import pytest
import torch

import attn_check as ac
from exact_io_aware_bwd_b200 import binding
from exact_io_aware_bwd_b200.build import build
from exact_io_aware_bwd_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 * 1024 * 1024  # FA_BWD_NOALLOC_SCRATCH_BYTES in include/fa.h


@pytest.fixture(scope="module", autouse=True)
def lib():
    build()
    binding.load()


def _case(shape, dtype, seed, causal):
    from dataclasses import replace
    w = replace(WORKLOADS["tiny"], dtype=dtype)
    q, k, v, do = (t.cuda() for t in make_inputs(w, seed=seed, shape_override=shape))
    scale = 1.0 / math.sqrt(shape[-1])
    o, lse = binding.attention_fwd(q, k, v, scale, causal)
    return q, k, v, do, o, lse, scale


def test_noalloc_matches_workspace_backward_on_consecutive_calls():
    cases = [((2, 4, 2, 333, 128), torch.bfloat16, 3, True),
             ((1, 3, 1, 640, 64), torch.float16, 4, False)]
    for shape, dtype, seed, causal in cases:  # two calls in a row on the shared scratch
        q, k, v, do, o, lse, scale = _case(shape, dtype, seed, causal)
        ref = binding.attention_bwd(q, k, v, o, do, lse, scale, causal)
        got = tuple(torch.empty_like(t) for t in ref)
        binding.fa_bwd_noalloc(q, k, v, o, do, lse, *got, scale, causal)
        assert binding.fa_get_device_status() == binding.FA_OK
        for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
            e = ac.rel_frob(g.cpu(), r.cpu())
            assert e <= ac.TOL_GRAD, f"{name} {shape}: {e:.3e}"


def test_noalloc_rejects_problems_beyond_the_scratch():
    B, Hq, Hkv, N, d = 1, 16, 16, 16384, 128
    assert binding.fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) > SCRATCH_BYTES
    q = torch.empty((B, Hq, N, d), device="cuda", dtype=torch.bfloat16)
    lse = torch.empty((B, Hq, N), device="cuda", dtype=torch.float32)
    with pytest.raises(binding.FaError) as e:
        binding.fa_bwd_noalloc(q, q, q, q, q, lse, q, q, q, 0.1, True)
    assert e.value.status == binding.FA_ERR_UNSUPPORTED
