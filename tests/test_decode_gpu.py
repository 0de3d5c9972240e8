"""Decode over a paged key/value cache on the GPU against the fp64 oracle:
sequences of mixed lengths whose pages sit shuffled in a shared pool, MHA,
GQA and MQA, bf16 and fp16, head dimension 64 and 128, page sizes 16-128,
one to several new tokens; and the device-side check of bad table entries
and lengths (reported, nothing out of range read)."""

import math

import numpy as np
import pytest
import torch

import attn_check as ac
import oracle
from exact_io_aware_bwd_b200 import binding
from exact_io_aware_bwd_b200.build import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    build()
    binding.load()


def make_case(seed, B, Hq, Hkv, Nq, d, P, lens, dtype, extra_pages=5):
    g = torch.Generator("cpu").manual_seed(seed)
    max_pages = max((L + P - 1) // P for L in lens) + 1     # a spare column, never read
    n_used = sum((L + P - 1) // P for L in lens)
    num_pages = n_used + extra_pages
    perm = torch.randperm(num_pages, generator=g)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    used = 0
    for b, L in enumerate(lens):
        npg = (L + P - 1) // P
        table[b, :npg] = perm[used:used + npg].to(torch.int32)
        used += npg
    kc = torch.randn((num_pages, Hkv, P, d), generator=g).to(dtype)
    vc = torch.randn((num_pages, Hkv, P, d), generator=g).to(dtype)
    q = torch.randn((B, Hq, Nq, d), generator=g).to(dtype)
    return q, kc, vc, table, torch.tensor(lens, dtype=torch.int32)


CASES = [
    # B, Hq, Hkv, Nq, d, P, lens, dtype
    (3, 8, 2, 1, 128, 64, (1, 100, 1000), torch.bfloat16),
    (2, 16, 1, 2, 128, 16, (37, 300), torch.bfloat16),          # MQA, 32 rows a kv head
    (4, 4, 4, 1, 64, 32, (5, 64, 65, 500), torch.float16),
    (2, 32, 8, 4, 128, 128, (129, 2048), torch.float16),       # GQA 4, 16 rows a kv head
    (1, 8, 8, 3, 64, 128, (3,), torch.bfloat16),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}-H{c[1]}/{c[2]}-Nq{c[3]}-d{c[4]}-P{c[5]}-{str(c[7])[6:]}"
                                              for c in CASES])
def test_decode_paged_parity(case):
    B, Hq, Hkv, Nq, d, P, lens, dtype = case
    q, kc, vc, table, seq_lens = make_case(sum(lens) + d + P, B, Hq, Hkv, Nq, d, P, lens, dtype)
    scale = 1.0 / math.sqrt(d)
    dev = "cuda:0"
    o, lse = binding.attention_decode_paged(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev),
                                            seq_lens.to(dev), scale)
    assert binding.fa_get_device_status() == binding.FA_OK
    o_r, lse_r = oracle.decode_paged(q, kc, vc, table.numpy(), seq_lens.numpy(), scale)
    ac.check_o(o.cpu(), o_r, dtype, what="decode O")
    ac.check_lse(lse.cpu(), lse_r, what="decode lse")


LONG_LENGTHS = [16, 17, 63, 64, 65, 127, 128, 129, 255, 500, 1023, 1024, 1025, 3000]
SHORT_LENGTHS = [1, 2, 3, 5, 8, 15]


def _random_decode_cases(n, seed, lengths):
    """Seeded decode shapes within the supported range: (Hq / Hkv) * Nq <= 32
    rows a kv head, d 64 or 128, pages of 16 to 128 tokens, sequence lengths
    drawn from `lengths` (at least Nq)."""
    g = np.random.default_rng(seed)
    cases = []
    while len(cases) < n:
        Hkv = int(g.choice([1, 2, 4, 8]))
        G = int(g.choice([1, 2, 4, 8]))
        Nq = int(g.choice([1, 2, 3, 4]))
        if G * Nq > 32:
            continue
        P = int(g.choice([16, 32, 64, 128]))
        B = int(g.integers(1, 5))
        lens = tuple(int(max(Nq, x)) for x in g.choice(lengths, B))
        cases.append((B, Hkv * G, Hkv, Nq, int(g.choice([64, 128])), P, lens,
                      torch.bfloat16 if g.random() < 0.6 else torch.float16))
    return cases


RANDOM_CASES = _random_decode_cases(16, seed=3030, lengths=LONG_LENGTHS)


@pytest.mark.parametrize("case", RANDOM_CASES,
                         ids=[f"B{c[0]}-H{c[1]}/{c[2]}-Nq{c[3]}-d{c[4]}-P{c[5]}-{str(c[7])[6:]}-r{i}"
                              for i, c in enumerate(RANDOM_CASES)])
def test_decode_random_shapes(case):
    """Every output of a seeded sweep of decode shapes (sequences of 16 tokens
    and more) against the oracle, O within 1e-2."""
    test_decode_paged_parity(case)


SHORT_CASES = _random_decode_cases(8, seed=3031, lengths=SHORT_LENGTHS)


@pytest.mark.parametrize("case", SHORT_CASES,
                         ids=[f"B{c[0]}-H{c[1]}/{c[2]}-Nq{c[3]}-d{c[4]}-P{c[5]}-{str(c[7])[6:]}-s{i}"
                              for i, c in enumerate(SHORT_CASES)])
def test_decode_short_sequences_known_exceedance(case):
    """Known exceedance of the O tolerance, reported rather than absorbed.

    A query of a sequence of one to fifteen cached tokens averages a few rows
    of V, so |O| reaches 2-4, where half an ulp of a bf16 output is
    0.0078-0.0156; with P rounded to the I/O dtype before the P V product an
    element can end just above 1e-2 by rounding alone (0.01005 met on a
    2-token sequence).  These cases are held to the a-priori rounding bound
    of the 16-bit path, element by element, and print how many elements are
    above 1e-2; lse keeps its stated tolerance."""
    B, Hq, Hkv, Nq, d, P, lens, dtype = case
    q, kc, vc, table, seq_lens = make_case(sum(lens) + d + P + 1, B, Hq, Hkv, Nq, d, P, lens, dtype)
    scale = 1.0 / math.sqrt(d)
    dev = "cuda:0"
    o, lse = binding.attention_decode_paged(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev),
                                            seq_lens.to(dev), scale)
    assert binding.fa_get_device_status() == binding.FA_OK
    o_r, lse_r = oracle.decode_paged(q, kc, vc, table.numpy(), seq_lens.numpy(), scale)
    o_abs, _ = oracle.decode_paged(q, kc, vc.abs(), table.numpy(), seq_lens.numpy(), scale)
    info = ac.check_o_rounding_bound(o.cpu(), o_r, dtype, o_abs, what="decode O")
    print("short sequences, O against the rounding bound:", info)
    ac.check_lse(lse.cpu(), lse_r, what="decode lse")


def test_decode_long_sequences_many_splits():
    """The bench shape's heads and GQA group at 16K and 5K cached tokens: many
    128-key tiles per split, several splits per sequence, a last tile that
    ends inside a page."""
    B, Hq, Hkv, Nq, d, P, lens = 2, 32, 8, 1, 128, 64, (16384, 5001)
    q, kc, vc, table, seq_lens = make_case(77, B, Hq, Hkv, Nq, d, P, lens, torch.bfloat16)
    dev = "cuda:0"
    o, lse = binding.attention_decode_paged(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev),
                                            seq_lens.to(dev))
    assert binding.fa_get_device_status() == binding.FA_OK
    o_r, lse_r = oracle.decode_paged(q, kc, vc, table.numpy(), seq_lens.numpy(), 1 / math.sqrt(d))
    ac.check_o(o.cpu(), o_r, torch.bfloat16, what="decode O")
    ac.check_lse(lse.cpu(), lse_r, what="decode lse")


@pytest.mark.parametrize("d,P,Nq", [(128, 32, 2), (64, 16, 3)])
def test_decode_peaked_scores_move_the_reference(d, P, Nq):
    """Scale 0.5 makes a tile's largest score exceed the running reference by
    more than 8 (log2) again and again, so the running O is rescaled in
    tensor memory many times.  lse is held to 1e-3; O, whose rows are
    dominated by a few keys with |O| up to ~3, to the rounding bound of the
    16-bit P and output (the peaked-softmax class of the O tolerance)."""
    B, Hq, Hkv, lens = 2, 8, 2, (3000, 777)
    q, kc, vc, table, seq_lens = make_case(5 + d + P, B, Hq, Hkv, Nq, d, P, lens, torch.bfloat16)
    dev = "cuda:0"
    o, lse = binding.attention_decode_paged(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev),
                                            seq_lens.to(dev), 0.5)
    assert binding.fa_get_device_status() == binding.FA_OK
    o_r, lse_r = oracle.decode_paged(q, kc, vc, table.numpy(), seq_lens.numpy(), 0.5)
    o_abs, _ = oracle.decode_paged(q, kc, vc.abs(), table.numpy(), seq_lens.numpy(), 0.5)
    ac.check_lse(lse.cpu(), lse_r, what="decode lse")
    print(ac.check_o_rounding_bound(o.cpu(), o_r, torch.bfloat16, o_abs))


@pytest.mark.parametrize("bad", ["page_id", "length"])
def test_decode_bad_input_is_reported(bad):
    q, kc, vc, table, seq_lens = make_case(9, 2, 4, 2, 1, 64, 16, (40, 20), torch.bfloat16)
    if bad == "page_id":
        table[1, 0] = kc.shape[0] + 3           # a page that does not exist
    else:
        seq_lens[0] = table.shape[1] * 16 + 1   # longer than the table can hold
    dev = "cuda:0"
    binding.attention_decode_paged(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev), seq_lens.to(dev))
    assert binding.fa_get_device_status() == binding.FA_ERR_INVALID_ARG
    # the context is still usable
    q, kc, vc, table, seq_lens = make_case(10, 1, 4, 2, 1, 64, 16, (33,), torch.bfloat16)
    o, lse = binding.attention_decode_paged(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev),
                                            seq_lens.to(dev))
    assert binding.fa_get_device_status() == binding.FA_OK
    o_r, lse_r = oracle.decode_paged(q, kc, vc, table.numpy(), seq_lens.numpy(), 1 / 8)
    ac.check_lse(lse.cpu(), lse_r, what="decode lse after an error")
