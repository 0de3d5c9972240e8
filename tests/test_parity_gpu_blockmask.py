"""Block-sparse attention on the GPU (fa_fwd_blockmask / fa_bwd_blockmask)
against the fp64 oracle under the same mask ("FlashAttention" glossary,
block-sparse entry): random masks, per-head and shared, causal and not,
local + global-token and dilated patterns, GQA, ragged sequence ends, query
blocks that see nothing (O = 0, lse = -inf, no gradient) and key blocks that
nobody sees (dK = dV = 0), few persistent backward blocks, and a mask of
ones, which must reproduce the plain path bit for bit."""

import math

import numpy as np
import pytest
import torch

import attn_check as ac
import oracle
from exact_io_aware_bwd_b200 import binding
from exact_io_aware_bwd_b200.build import build
from exact_io_aware_bwd_b200.workloads import WORKLOADS, check_rows, make_inputs

pytestmark = pytest.mark.gpu

BLK = 128


@pytest.fixture(scope="module", autouse=True)
def lib():
    build()
    binding.load()


def _inputs(shape, dtype, seed):
    from dataclasses import replace
    w = replace(WORKLOADS["tiny"], dtype=dtype)
    return make_inputs(w, seed=seed, shape_override=shape)


def random_mask(H, N, density, seed, per_head=True):
    nb = -(-N // BLK)
    g = torch.Generator("cpu").manual_seed(seed)
    shape = (H, nb, nb) if per_head else (nb, nb)
    return (torch.rand(shape, generator=g) < density).to(torch.uint8)


def local_global_mask(N, band=1, n_global=1):
    """Each query block sees its own and `band` earlier key blocks, plus the
    first n_global key blocks; the first n_global query blocks see all."""
    nb = -(-N // BLK)
    m = torch.zeros((nb, nb), dtype=torch.uint8)
    for i in range(nb):
        m[i, max(0, i - band):i + 1] = 1
        m[i, :n_global] = 1
    m[:n_global, :] = 1
    return m


def dilated_mask(N, step=2):
    nb = -(-N // BLK)
    i = torch.arange(nb)
    return ((i[:, None] - i[None, :]) % step == 0).to(torch.uint8)


def run(q, k, v, do, scale, causal, mask):
    dev = "cuda:0"
    qd, kd, vd, dod, md = (t.to(dev) for t in (q, k, v, do, mask))
    o, lse = binding.attention_fwd(qd, kd, vd, scale, causal, block_mask=md)
    dq, dk, dv = binding.attention_bwd(qd, kd, vd, o, dod, lse, scale, causal, block_mask=md)
    status = binding.fa_get_device_status()
    assert status == binding.FA_OK, binding.fa_status_string(status)
    return {n: t.cpu() for n, t in dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv).items()}


def check_lse_with_empty_rows(lse_gpu, lse_ref):
    """lse within 1e-3 where the row sees a key; exactly -inf in both where
    it sees none."""
    g, r = ac._np(lse_gpu), ac._np(lse_ref)
    empty = np.isneginf(r)
    assert (np.isneginf(g) == empty).all(), "rows without a visible key differ"
    return ac.check_lse(g[~empty], r[~empty]), int(empty.sum())


def check_against_oracle(q, k, v, do, scale, causal, mask, out):
    bm = (mask, BLK, BLK)
    o_r, lse_r = oracle.fwd(q, k, v, scale, causal, block_mask=bm)
    dq_r, dk_r, dv_r = oracle.bwd(q, k, v, do, scale, causal, block_mask=bm)
    lse_err, n_empty = check_lse_with_empty_rows(out["lse"], lse_r)
    rep = dict(o=ac.check_o(out["o"], o_r, q.dtype), lse=lse_err, empty_rows=n_empty)
    for name, r in (("dq", dq_r), ("dk", dk_r), ("dv", dv_r)):
        rep[name] = ac.check_grad(out[name], r, name) if np.abs(r).max() > 0 else \
            float(np.abs(ac._np(out[name])).max())
        if np.abs(r).max() == 0:
            assert rep[name] == 0.0, f"{name} must be zero where nothing is seen"
    return rep


CASES = [
    # (B, Hq, Hkv, N, d), dtype, causal, mask kind, seed
    ((1, 2, 2, 512, 64), torch.bfloat16, False, "random-head", 1),
    ((1, 2, 2, 512, 64), torch.bfloat16, True, "random-head", 2),
    ((2, 4, 2, 700, 128), torch.bfloat16, True, "random-shared", 3),
    ((2, 4, 2, 700, 128), torch.float16, False, "random-head", 4),
    ((1, 8, 2, 1000, 128), torch.bfloat16, True, "local-global", 5),
    ((1, 3, 1, 900, 64), torch.float16, True, "dilated", 6),
    ((1, 4, 4, 333, 128), torch.bfloat16, False, "sparse-head", 7),
    ((1, 2, 1, 640, 128), torch.bfloat16, True, "sparse-head", 8),
]


def make_mask(kind, Hq, N, seed):
    if kind == "random-head":
        return random_mask(Hq, N, 0.55, seed)
    if kind == "random-shared":
        return random_mask(Hq, N, 0.6, seed, per_head=False)
    if kind == "sparse-head":
        # sparse enough that some query blocks see nothing and some key
        # blocks are seen by nobody
        return random_mask(Hq, N, 0.25, seed)
    if kind == "local-global":
        return local_global_mask(N)
    if kind == "dilated":
        return dilated_mask(N)
    raise ValueError(kind)


@pytest.mark.parametrize("shape,dtype,causal,kind,seed", CASES,
                         ids=[f"{'x'.join(map(str, s))}-{str(t)[6:]}-{'c' if c else 'nc'}-{k}"
                              for s, t, c, k, _ in CASES])
def test_parity_blockmask(shape, dtype, causal, kind, seed):
    q, k, v, do = _inputs(shape, dtype, seed=11 * seed + sum(shape))
    scale = 1.0 / math.sqrt(shape[-1])
    mask = make_mask(kind, shape[1], shape[3], seed)
    out = run(q, k, v, do, scale, causal, mask)
    print(shape, kind, check_against_oracle(q, k, v, do, scale, causal, mask, out))


def test_blockmask_empty_rows_and_unseen_keys():
    """Non-causal: query block 1 sees no key block (O = 0, lse = -inf, dQ = 0),
    and key block 2 is seen by no query block (dK = dV = 0)."""
    shape = (1, 2, 2, 512, 64)
    q, k, v, do = _inputs(shape, torch.bfloat16, seed=77)
    mask = torch.ones((4, 4), dtype=torch.uint8)
    mask[1, :] = 0
    mask[:, 2] = 0
    out = run(q, k, v, do, 0.125, False, mask)
    assert torch.all(out["o"][:, :, 128:256] == 0)
    assert torch.all(torch.isneginf(out["lse"][:, :, 128:256]))
    assert torch.all(out["dq"][:, :, 128:256] == 0)
    assert torch.all(out["dk"][:, :, 256:384] == 0) and torch.all(out["dv"][:, :, 256:384] == 0)
    check_against_oracle(q, k, v, do, 0.125, False, mask, out)


def test_blockmask_handover_with_few_blocks():
    """Few persistent backward blocks take many items in turn, items without
    any visible query block among them."""
    shape = (2, 4, 2, 900, 128)
    q, k, v, do = _inputs(shape, torch.bfloat16, seed=91)
    mask = random_mask(4, 900, 0.3, 12)
    binding.fa_set_bwd_max_blocks(2)
    try:
        out = run(q, k, v, do, 1 / math.sqrt(128), True, mask)
    finally:
        binding.fa_set_bwd_max_blocks(0)
    check_against_oracle(q, k, v, do, 1 / math.sqrt(128), True, mask, out)


@pytest.mark.parametrize("causal", [False, True])
def test_mask_of_ones_equals_the_plain_path(causal):
    """A mask that hides nothing walks the same blocks in the same order as
    the plain kernels: O, lse, dK and dV are bitwise equal (dQ is added in
    a varying order, so it is compared within 1e-3 relative)."""
    shape = (1, 4, 2, 640, 128)
    q, k, v, do = (t.cuda() for t in _inputs(shape, torch.bfloat16, seed=5))
    mask = torch.ones((5, 5), dtype=torch.uint8, device="cuda")
    o1, l1 = binding.attention_fwd(q, k, v, 0.09, causal)
    o2, l2 = binding.attention_fwd(q, k, v, 0.09, causal, block_mask=mask)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    g1 = binding.attention_bwd(q, k, v, o1, do, l1, 0.09, causal)
    g2 = binding.attention_bwd(q, k, v, o1, do, l1, 0.09, causal, block_mask=mask)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    rel = ((g1[0].float() - g2[0].float()).norm() / g1[0].float().norm()).item()
    assert rel <= 1e-3, rel
    assert binding.fa_get_device_status() == binding.FA_OK


def test_blockmask_at_4k_rows_and_columns():
    """A 4K-token problem under a local + global-token mask: seeded query
    rows and key rows against the oracle, and the gradient invariants of the
    rows that see keys."""
    w = WORKLOADS["mha4k"]
    shape = (1, 4, 4, 4096, 128)
    q, k, v, do = make_inputs(w, shape_override=shape)
    mask = local_global_mask(4096, band=2, n_global=1)
    out = run(q, k, v, do, w.scale, True, mask)
    rows = check_rows(w, N=4096)[::4].numpy()
    bm = (mask, BLK, BLK)
    o_r, lse_r = oracle.fwd_rows(q, k, v, rows, w.scale, True, block_mask=bm)
    ac.check_o(out["o"][:, :, rows], o_r, q.dtype)
    ac.check_lse(out["lse"][:, :, rows], lse_r)
    dq_r = oracle.bwd_rows(q, k, v, do, rows, w.scale, True, block_mask=bm)
    ac.check_grad(out["dq"][:, :, rows], dq_r, "dQ rows")
    cols = np.array([0, 100, 1000, 2047, 3000, 4095])
    dk_r, dv_r = oracle.bwd_cols(q, k, v, do, 0, 2, cols, w.scale, True, block_mask=bm)
    ac.check_grad(out["dk"][0, 2][cols], dk_r, "dK cols")
    ac.check_grad(out["dv"][0, 2][cols], dv_r, "dV cols")
    ac.check_invariants(q, k, do, out)


def _random_mask_cases(n, seed):
    """Seeded shapes and mask kinds: MHA / GQA / MQA, d 64 or 128, sequences
    from under one block to several blocks with ragged tails, causal or not."""
    g = np.random.default_rng(seed)
    kinds = ["random-head", "random-shared", "sparse-head", "local-global", "dilated"]
    lengths = [1, 100, 128, 129, 255, 300, 511, 700]
    cases = []
    for i in range(n):
        hkv = int(g.integers(1, 4))
        cases.append(((int(g.integers(1, 3)), hkv * int(g.choice([1, 2, 4])), hkv, int(g.choice(lengths)),
                       int(g.choice([64, 128]))),
                      torch.bfloat16 if g.random() < 0.6 else torch.float16, bool(g.random() < 0.5),
                      str(g.choice(kinds)), 100 + i))
    return cases


RANDOM_MASK_CASES = _random_mask_cases(10, seed=5050)


@pytest.mark.parametrize("shape,dtype,causal,kind,seed", RANDOM_MASK_CASES,
                         ids=[f"{'x'.join(map(str, s))}-{str(t)[6:]}-{'c' if c else 'nc'}-{k}-r{sd}"
                              for s, t, c, k, sd in RANDOM_MASK_CASES])
def test_parity_blockmask_random(shape, dtype, causal, kind, seed):
    test_parity_blockmask(shape, dtype, causal, kind, seed)
