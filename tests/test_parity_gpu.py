"""The CUDA path (through the C ABI) against the fp64 oracle, element by
element at sizes the oracle finishes in seconds (several tiles, ragged
tails, GQA/MQA, bf16 and fp16), and on seeded row/column subsets plus
size-independent invariants at the full workload sizes."""

import math

import numpy as np
import pytest
import torch

import attn_check as ac
import oracle
from exact_io_aware_bwd_b200 import binding
from exact_io_aware_bwd_b200.build import build
from exact_io_aware_bwd_b200.workloads import WORKLOADS, check_cols, check_rows, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    build()
    binding.load()


def _inputs(shape, dtype, seed, sigma_qk=1.0):
    w = WORKLOADS["tiny"]
    if dtype != w.dtype or sigma_qk != 1.0:
        from dataclasses import replace
        w = replace(w, dtype=dtype, sigma_qk=sigma_qk)
    return make_inputs(w, seed=seed, shape_override=shape)


FULL_CASES = [
    # (B, Hq, Hkv, N, d), dtype, causal
    ((1, 2, 2, 256, 64), torch.bfloat16, False),
    ((1, 2, 2, 256, 64), torch.bfloat16, True),
    ((1, 2, 2, 256, 64), torch.float16, True),
    ((2, 4, 2, 333, 128), torch.bfloat16, False),
    ((2, 4, 2, 333, 128), torch.bfloat16, True),
    ((1, 3, 1, 200, 64), torch.float16, False),
    ((1, 3, 1, 200, 64), torch.float16, True),
    ((1, 8, 2, 384, 128), torch.bfloat16, True),
    ((1, 2, 2, 129, 128), torch.float16, True),
    ((1, 2, 1, 127, 64), torch.bfloat16, True),
    ((1, 1, 1, 1, 128), torch.bfloat16, False),
    ((1, 2, 2, 64, 128), torch.bfloat16, True),
    ((3, 2, 2, 520, 64), torch.bfloat16, False),
]


@pytest.mark.parametrize("shape,dtype,causal", FULL_CASES,
                         ids=[f"{'x'.join(map(str, s))}-{str(t)[6:]}-{'c' if c else 'nc'}" for s, t, c in FULL_CASES])
def test_parity_full(shape, dtype, causal):
    q, k, v, do = _inputs(shape, dtype, seed=sum(shape) + (7 if causal else 0))
    scale = 1.0 / math.sqrt(shape[-1])
    out = ac.run_gpu(q, k, v, do, scale, causal)
    rep = ac.check_full(q, k, v, do, scale, causal, out)
    print(shape, dtype, causal, rep)


PERSISTENT_CASES = [
    # (B, Hq, Hkv, N, d), dtype, causal, blocks: few persistent blocks, so each
    # takes many work items in turn, including causal items of a single step
    ((2, 3, 3, 130, 64), torch.bfloat16, True, 1),
    ((2, 3, 3, 130, 64), torch.float16, False, 2),
    ((1, 8, 2, 333, 128), torch.bfloat16, True, 1),
    ((1, 8, 2, 333, 128), torch.bfloat16, True, 3),
    ((2, 4, 4, 640, 128), torch.float16, True, 5),
    ((1, 6, 1, 260, 128), torch.bfloat16, False, 2),
]


@pytest.mark.parametrize("shape,dtype,causal,blocks", PERSISTENT_CASES,
                         ids=[f"{'x'.join(map(str, s))}-{str(t)[6:]}-{'c' if c else 'nc'}-b{n}"
                              for s, t, c, n in PERSISTENT_CASES])
def test_parity_persistent_handover(shape, dtype, causal, blocks):
    q, k, v, do = _inputs(shape, dtype, seed=3 * sum(shape) + blocks)
    scale = 1.0 / math.sqrt(shape[-1])
    binding.fa_set_bwd_max_blocks(blocks)
    try:
        out = ac.run_gpu(q, k, v, do, scale, causal)
    finally:
        binding.fa_set_bwd_max_blocks(0)
    ac.check_full(q, k, v, do, scale, causal, out)


WINDOW_CASES = [
    # (B, Hq, Hkv, N, d), dtype, window: causal sliding window of `window` keys
    ((1, 2, 2, 256, 64), torch.bfloat16, 1),
    ((1, 2, 2, 256, 64), torch.bfloat16, 64),
    ((1, 2, 2, 256, 64), torch.float16, 100),
    ((1, 2, 2, 256, 64), torch.bfloat16, 300),
    ((2, 4, 2, 333, 128), torch.bfloat16, 128),
    ((2, 4, 2, 333, 128), torch.float16, 77),
    ((1, 3, 1, 520, 64), torch.bfloat16, 130),
    ((1, 8, 2, 700, 128), torch.bfloat16, 257),
]


@pytest.mark.parametrize("shape,dtype,window", WINDOW_CASES,
                         ids=[f"{'x'.join(map(str, s))}-{str(t)[6:]}-w{w}" for s, t, w in WINDOW_CASES])
def test_parity_window(shape, dtype, window):
    q, k, v, do = _inputs(shape, dtype, seed=5 * sum(shape) + window)
    scale = 1.0 / math.sqrt(shape[-1])
    out = ac.run_gpu(q, k, v, do, scale, True, window=window)
    ac.check_full(q, k, v, do, scale, True, out, window=window)


def test_parity_window_wide_logits_and_handover():
    # wide fp16 logits (running max moves within the window) with few
    # persistent backward blocks taking many items each
    q, k, v, do = _inputs((1, 4, 2, 900, 128), torch.float16, seed=123, sigma_qk=3.0)
    binding.fa_set_bwd_max_blocks(3)
    try:
        out = ac.run_gpu(q, k, v, do, 1 / math.sqrt(128), True, window=300)
    finally:
        binding.fa_set_bwd_max_blocks(0)
    ac.check_full(q, k, v, do, 1 / math.sqrt(128), True, out, window=300)


def test_window_at_4k_rows_and_columns():
    """A 4K-token MHA problem with a 1024-key window: seeded query rows and
    key rows against the oracle, and the gradient invariants."""
    w = WORKLOADS["mha4k"]
    shape = (1, 8, 8, 4096, 128)
    q, k, v, do = make_inputs(w, shape_override=shape)
    out = ac.run_gpu(q, k, v, do, w.scale, True, window=1024)
    rows = check_rows(w, N=4096)[::2]
    ac.check_rows(q, k, v, do, w.scale, True, out, rows, window=1024)
    ac.check_cols(q, k, v, do, w.scale, True, out, [(0, 3, [0, 1000, 2047, 3000, 4095])], window=1024)
    ac.check_invariants(q, k, do, out)


DROPOUT_CASES = [
    # (B, Hq, Hkv, N, d), dtype, causal, p_drop, seed
    ((1, 2, 2, 256, 64), torch.bfloat16, False, 0.1, 1),
    ((1, 2, 2, 256, 64), torch.bfloat16, True, 0.5, 2),
    ((2, 4, 2, 333, 128), torch.bfloat16, True, 0.25, (1 << 40) + 17),
    ((2, 4, 2, 333, 128), torch.float16, False, 0.2, 3),
    ((1, 3, 1, 200, 64), torch.float16, True, 0.3, 4),
    ((1, 8, 2, 384, 128), torch.bfloat16, True, 0.05, 5),
]


@pytest.mark.parametrize("shape,dtype,causal,p_drop,seed", DROPOUT_CASES,
                         ids=[f"{'x'.join(map(str, s))}-{str(t)[6:]}-{'c' if c else 'nc'}-p{p}"
                              for s, t, c, p, _ in DROPOUT_CASES])
def test_parity_dropout(shape, dtype, causal, p_drop, seed):
    q, k, v, do = _inputs(shape, dtype, seed=7 * sum(shape) + seed % 1000)
    scale = 1.0 / math.sqrt(shape[-1])
    out = ac.run_gpu(q, k, v, do, scale, causal, dropout=(p_drop, seed))
    print(ac.check_full(q, k, v, do, scale, causal, out, dropout=(p_drop, seed)))


@pytest.mark.parametrize("d", [64, 128])
def test_dropout_mask_bit_exact(d):
    """Q = 0 (uniform P = 1/N, non-causal) and V = I: O is the keep mask times
    256/(256-t)/N, so every keep decision of the GPU can be read off O and
    compared exactly with the oracle's."""
    N, Hq, p_drop, seed = d, 3, 0.375, 987654321
    t = round(p_drop * 256)
    q = torch.zeros((1, Hq, N, d), dtype=torch.float16)
    k = _inputs((1, Hq, Hq, N, d), torch.float16, seed=31)[1]
    v = torch.eye(N, d, dtype=torch.float16).expand(1, Hq, N, d).contiguous()
    dev = "cuda:0"
    o, lse = binding.attention_fwd(q.to(dev), k.to(dev), v.to(dev), 0.5, False, dropout=(p_drop, seed))
    assert binding.fa_get_device_status() == binding.FA_OK
    level = 256.0 / (256 - t) / N
    z_gpu = o.float().cpu().numpy() > 0.5 * level
    o_ref, _ = oracle.fwd(q, k, v, 0.5, False, dropout=(t, seed))
    z_ref = o_ref > 0.5 * level
    assert (z_gpu == z_ref).all(), f"{int((z_gpu != z_ref).sum())} keep decisions differ"
    assert abs(z_ref.mean() - (1 - t / 256)) < 0.03


def test_parity_wide_logits_fp16():
    # the fp16 recipe with Q, K ~ N(0, 3^2): the running max moves many times
    q, k, v, do = _inputs((1, 2, 2, 640, 128), torch.float16, seed=99, sigma_qk=3.0)
    out = ac.run_gpu(q, k, v, do, 1 / math.sqrt(128), True)
    ac.check_full(q, k, v, do, 1 / math.sqrt(128), True, out)


def test_scale_not_one_over_sqrt_d():
    # a scale below 1/sqrt(d): flatter rows than the workloads'
    q, k, v, do = _inputs((1, 2, 1, 300, 64), torch.bfloat16, seed=6)
    out = ac.run_gpu(q, k, v, do, 0.06, True)
    ac.check_full(q, k, v, do, 0.06, True, out)


def test_peaked_softmax_known_exceedance():
    """Known exceedance of the O tolerance, reported rather than absorbed.

    scale = 0.3 at d = 64 (2.4 times 1/sqrt(d)) makes the rows peaked: one or
    two keys carry almost all of a row's weight, so O_i is close to one row of
    V, and |O| reaches 2-4 in bf16, where half an ulp of the output alone is
    0.0078-0.0156.  Add the rounding of P to bf16 before the P V product
    (relative 2^-9 of each weight) and a few elements can end above 1e-2 by
    rounding alone.  This case is therefore held to the a-priori rounding
    bound of the 16-bit path, element by element, and prints how many
    elements are above 1e-2 and the largest error in output ulps; lse and
    the gradients keep their stated tolerances."""
    q, k, v, do = _inputs((1, 2, 1, 300, 64), torch.bfloat16, seed=5)
    out = ac.run_gpu(q, k, v, do, 0.3, False)
    o_r, lse_r = oracle.fwd(q, k, v, 0.3, False)
    o_abs, _ = oracle.fwd(q, k, v.abs(), 0.3, False)
    info = ac.check_o_rounding_bound(out["o"], o_r, q.dtype, o_abs)
    print("peaked softmax, O against the rounding bound:", info)
    ac.check_lse(out["lse"], lse_r)
    dq_r, dk_r, dv_r = oracle.bwd(q, k, v, do, 0.3, False)
    for name, r in (("dq", dq_r), ("dk", dk_r), ("dv", dv_r)):
        ac.check_grad(out[name], r, name)


@pytest.mark.parametrize("name", ["tiny", "gpt2", "mha4k", "gqa16k", "long64k"])
def test_workload(name):
    """The five workloads at full size: every row of the tiny one; seeded
    row subsets (O, lse, dQ) and key-row subsets (dK, dV) of the others,
    plus the gradient invariants on every head."""
    w = WORKLOADS[name]
    q, k, v, do = make_inputs(w)
    for causal in w.causal_modes:
        out = ac.run_gpu(q, k, v, do, w.scale, causal)
        if name == "tiny":
            rep = ac.check_full(q, k, v, do, w.scale, causal, out)
        else:
            rep = ac.check_rows(q, k, v, do, w.scale, causal, out, check_rows(w))
            if w.check_col_heads:
                rep.update(ac.check_cols(q, k, v, do, w.scale, causal, out, check_cols(w, causal)))
            rep.update(ac.check_invariants(q, k, do, out))
        print(name, causal, rep)
        del out


def test_repeated_full_size_runs_are_stable():
    """The 4K-token MHA workload run many times in a row.  O, lse, dK and dV
    must be bitwise equal on every run (their reductions have a fixed order;
    only dQ is reduce-added in a varying order, within 1e-3 relative of the
    first run); the first run is checked against the oracle on seeded rows.
    This guards the schedules' reliance on the tensor core reading an MMA's
    operands before a later MMA of the same thread overwrites them."""
    w = WORKLOADS["mha4k"]
    q, k, v, do = make_inputs(w)
    dev = [t.cuda() for t in (q, k, v, do)]
    o0, l0 = binding.attention_fwd(dev[0], dev[1], dev[2], w.scale, True)
    ws = torch.empty(binding.fa_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d), device="cuda",
                     dtype=torch.uint8)
    g0 = binding.attention_bwd(dev[0], dev[1], dev[2], o0, dev[3], l0, w.scale, True, workspace=ws)
    assert binding.fa_get_device_status() == binding.FA_OK
    o, lse = torch.empty_like(o0), torch.empty_like(l0)
    for _ in range(24):
        binding.fa_fwd(dev[0], dev[1], dev[2], o, lse, w.scale, True)
        assert torch.equal(o, o0) and torch.equal(lse, l0)
    dq, dk, dv = (torch.empty_like(t) for t in g0)
    for _ in range(12):
        binding.fa_bwd(dev[0], dev[1], dev[2], o0, dev[3], l0, dq, dk, dv, w.scale, True, ws)
        assert torch.equal(dk, g0[1]) and torch.equal(dv, g0[2])
        rel = ((dq.float() - g0[0].float()).norm() / g0[0].float().norm()).item()
        assert rel <= 1e-3, rel
    assert binding.fa_get_device_status() == binding.FA_OK
    out = {"o": o0.cpu(), "lse": l0.cpu(), "dq": g0[0].cpu(), "dk": g0[1].cpu(), "dv": g0[2].cpu()}
    rows = check_rows(w)[::8]
    print(ac.check_rows(q, k, v, do, w.scale, True, out, rows))


def test_forward_is_deterministic():
    q, k, v, _ = _inputs((1, 4, 2, 1000, 128), torch.bfloat16, seed=3)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = binding.attention_fwd(qd, kd, vd, 0.09, True)
    o2, l2 = binding.attention_fwd(qd, kd, vd, 0.09, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_empty_problems():
    q = torch.empty((0, 2, 128, 64), device="cuda", dtype=torch.bfloat16)
    o, lse = binding.attention_fwd(q, q, q, 0.1, True)
    assert o.shape == q.shape and lse.shape == (0, 2, 128)
    q = torch.empty((1, 2, 0, 128), device="cuda", dtype=torch.float16)
    o, lse = binding.attention_fwd(q, q, q, 0.1, False)
    dq, dk, dv = binding.attention_bwd(q, q, q, o, q, lse, 0.1, False)
    assert dq.shape == q.shape


def test_bounded_wait_reports_timeout():
    # a barrier nobody signals: the kernel gives up after 50 ms and reports it
    assert binding.fa_selftest_wait_timeout(50_000_000) == binding.FA_ERR_TIMEOUT
    # the context is still usable and the status was cleared
    assert binding.fa_get_device_status() == binding.FA_OK
    q, k, v, do = _inputs((1, 2, 2, 256, 64), torch.bfloat16, seed=1)
    out = ac.run_gpu(q, k, v, do, 0.125, True)
    ac.check_full(q, k, v, do, 0.125, True, out)


def test_memory_linear_in_n():
    """Peak device memory of fwd + bwd (inputs, outputs, workspace) doubles
    with N: no N x N buffer anywhere."""
    peaks = []
    for n in (4096, 8192, 16384, 32768, 65536):
        torch.cuda.empty_cache()
        torch.cuda.reset_peak_memory_stats()
        base = torch.cuda.memory_allocated()
        q = torch.randn((1, 16, n, 128), device="cuda", dtype=torch.bfloat16)
        k, v, do = torch.randn_like(q), torch.randn_like(q), torch.randn_like(q)
        o, lse = binding.attention_fwd(q, k, v, None, True)
        binding.attention_bwd(q, k, v, o, do, lse, None, True)
        torch.cuda.synchronize()
        peaks.append(torch.cuda.max_memory_allocated() - base)
        del q, k, v, do, o, lse
    ratios = [b / a for a, b in zip(peaks, peaks[1:])]
    print("peak bytes", peaks, "ratios", ratios)
    assert all(1.9 <= r <= 2.1 for r in ratios), ratios


def _random_cases(n, seed):
    """Seeded shapes across the supported range: tiny and ragged sequence
    lengths (1, 7, one short of and one past a block), MHA / GQA / MQA, both
    head dimensions, both 16-bit dtypes, causal or not."""
    g = np.random.default_rng(seed)
    lengths = [1, 2, 7, 63, 64, 65, 127, 128, 129, 191, 255, 257, 300, 383, 511, 640]
    cases = []
    for _ in range(n):
        hkv = int(g.integers(1, 4))
        group = int(g.choice([1, 2, 3, 4]))
        cases.append(((int(g.integers(1, 4)), hkv * group, hkv, int(g.choice(lengths)),
                       int(g.choice([64, 128]))),
                      torch.bfloat16 if g.random() < 0.6 else torch.float16, bool(g.random() < 0.5)))
    return cases


RANDOM_CASES = _random_cases(24, seed=2026)


@pytest.mark.parametrize("shape,dtype,causal", RANDOM_CASES,
                         ids=[f"{'x'.join(map(str, s))}-{str(t)[6:]}-{'c' if c else 'nc'}"
                              for s, t, c in RANDOM_CASES])
def test_parity_random_shapes(shape, dtype, causal):
    """Every output element against the oracle on a seeded sweep of shapes,
    including sequences shorter than one block and ragged tails."""
    q, k, v, do = _inputs(shape, dtype, seed=sum(shape) * 31 + causal)
    scale = 1.0 / math.sqrt(shape[-1])
    out = ac.run_gpu(q, k, v, do, scale, causal)
    ac.check_full(q, k, v, do, scale, causal, out)


RANDOM_WINDOW_CASES = [(s, t, int(w)) for (s, t, _), w in zip(
    _random_cases(10, seed=2027), np.random.default_rng(2028).choice([1, 17, 64, 100, 128, 200, 257, 700], 10))]


@pytest.mark.parametrize("shape,dtype,window", RANDOM_WINDOW_CASES,
                         ids=[f"{'x'.join(map(str, s))}-{str(t)[6:]}-w{w}" for s, t, w in RANDOM_WINDOW_CASES])
def test_parity_random_window(shape, dtype, window):
    q, k, v, do = _inputs(shape, dtype, seed=sum(shape) * 37 + window)
    scale = 1.0 / math.sqrt(shape[-1])
    out = ac.run_gpu(q, k, v, do, scale, True, window=window)
    ac.check_full(q, k, v, do, scale, True, out, window=window)


RANDOM_DROPOUT_CASES = [(s, t, c, float(p_), int(sd)) for (s, t, c), p_, sd in zip(
    _random_cases(8, seed=2029), np.random.default_rng(2030).choice([0.05, 0.1, 0.3, 0.5], 8),
    np.random.default_rng(2031).integers(0, 2**62, 8))]


@pytest.mark.parametrize("shape,dtype,causal,p_drop,seed", RANDOM_DROPOUT_CASES,
                         ids=[f"{'x'.join(map(str, s))}-{str(t)[6:]}-{'c' if c else 'nc'}-p{p_}"
                              for s, t, c, p_, _ in RANDOM_DROPOUT_CASES])
def test_parity_random_dropout(shape, dtype, causal, p_drop, seed):
    q, k, v, do = _inputs(shape, dtype, seed=sum(shape) * 41 + int(p_drop * 100))
    scale = 1.0 / math.sqrt(shape[-1])
    out = ac.run_gpu(q, k, v, do, scale, causal, dropout=(p_drop, seed))
    ac.check_full(q, k, v, do, scale, causal, out, dropout=(p_drop, seed))
