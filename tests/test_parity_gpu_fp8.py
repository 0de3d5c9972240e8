"""The FP8 forward (E4M3 Q, K, V with one factor per tensor, 16-bit O)
through the C ABI against the fp64 oracle applied to the dequantised inputs.

The pages fix no tolerance for FP8; these follow from the arithmetic:
- lse: max abs 1e-3, as for the 16-bit forward.  The scores are products of
  E4M3 values (exact in fp32) accumulated in fp32, and the row sums are kept
  in fp32, so lse sees no 8-bit rounding.
- O, per element: |dO_ic| <= 2^-4 sum_j w_ij |v_jc| + 2^-8 |O_ic| + 1e-3,
  w the exact softmax weights.  Each probability is rounded to E4M3 before
  the P V product (relative error at most 2^-4 for normal values); 2^-8 |O|
  covers rounding O to bf16/fp16 (half an ulp is at most 2^-9 relative); the
  1e-3 covers probabilities in E4M3's subnormal range (absolute error at most
  2^-10 of the block's reference maximum) and fp32 accumulation.
- O, relative Frobenius error <= 0.05: the RMS relative error of a value
  rounded to nearest E4M3 is at most 2^-4 / sqrt(3) = 0.036.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_bwd_b200 import binding
from exact_io_aware_bwd_b200.build import build
from exact_io_aware_bwd_b200.workloads import WORKLOADS, check_rows, make_fp8_inputs

pytestmark = pytest.mark.gpu

LSE_TOL = 1e-3
REL_FROB_TOL = 0.05


@pytest.fixture(scope="module", autouse=True)
def lib():
    build()
    binding.load()


def _run(q8, k8, v8, descale, scale, causal, out_dtype):
    dev = [t.cuda() for t in (q8, k8, v8)]
    o, lse = binding.attention_fwd_fp8(*dev, descale, scale, causal, out_dtype)
    torch.cuda.synchronize()
    assert binding.fa_get_device_status() == binding.FA_OK
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


def _check(q8, k8, v8, descale, scale, causal, o, lse, rows=None):
    """Compares O and lse (all rows, or the given rows of every head) with the oracle."""
    if rows is None:
        o_ref, lse_ref = oracle.fwd_fp8(q8, k8, v8, descale, scale, causal)
        rows = np.arange(q8.shape[2])
    else:
        rows = np.asarray(rows)
        o_ref, lse_ref = oracle.fwd_fp8_rows(q8, k8, v8, descale, rows, scale, causal)
        o, lse = o[:, :, rows], lse[:, :, rows]
    err_lse = float(np.max(np.abs(lse - lse_ref)))
    assert err_lse <= LSE_TOL, f"max |dlse| {err_lse:.3e}"
    rel = float(np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref))
    assert rel <= REL_FROB_TOL, f"O relative Frobenius error {rel:.3e}"
    # per-element envelope from the exact weights (softmax of the scores of the checked rows)
    q = oracle.e4m3_decode(q8) * descale[0]
    k = oracle.e4m3_decode(k8) * descale[1]
    av = np.abs(oracle.e4m3_decode(v8) * descale[2])
    G = q.shape[1] // k.shape[1]
    worst = 0.0
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            s = (q[b, h, rows] @ k[b, h // G].T) * scale
            if causal:
                s = np.where(np.arange(k.shape[2])[None, :] <= rows[:, None], s, -np.inf)
            w = np.exp(s - lse_ref[b, h][:, None])
            env = 2.0 ** -4 * (w @ av[b, h // G]) + 2.0 ** -8 * np.abs(o_ref[b, h]) + 1e-3
            worst = max(worst, float(np.max(np.abs(o[b, h] - o_ref[b, h]) / env)))
    assert worst <= 1.0, f"O outside the E4M3 rounding envelope (ratio {worst:.3f})"
    return {"lse": err_lse, "rel_frob": rel, "envelope_ratio": worst}


FULL_CASES = [
    # (B, Hq, Hkv, N, d), causal, output dtype
    ((1, 2, 2, 256, 128), True, torch.bfloat16),
    ((1, 2, 2, 256, 128), False, torch.float16),
    ((1, 4, 2, 640, 128), True, torch.bfloat16),
    ((2, 3, 1, 200, 128), False, torch.bfloat16),
    ((1, 2, 2, 129, 128), True, torch.float16),
    ((1, 1, 1, 1, 128), False, torch.bfloat16),
    ((1, 2, 2, 64, 128), True, torch.bfloat16),
]


@pytest.mark.parametrize("shape,causal,out_dtype", FULL_CASES,
                         ids=[f"{'x'.join(map(str, s))}-{'c' if c else 'nc'}-{str(t)[6:]}"
                              for s, c, t in FULL_CASES])
def test_fp8_forward_full(shape, causal, out_dtype):
    (q8, k8, v8), ds = make_fp8_inputs(WORKLOADS["tiny"], seed=sum(shape) + 5 * causal,
                                       shape_override=shape)
    scale = 1.0 / math.sqrt(shape[-1])
    o, lse = _run(q8, k8, v8, ds, scale, causal, out_dtype)
    print(shape, causal, _check(q8, k8, v8, ds, scale, causal, o, lse))


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_value_layout_exact(causal):
    """Q = 0 gives P = 1 for every visible key (exact in E4M3), and V with one
    1.0 per row at column j % 128 makes O_ic = delta_v * #{visible j with
    j % 128 = c} / #visible: checks the value operand's layout and the value
    factor up to the rounding of O."""
    B, H, N, d = 1, 2, 300, 128
    q8 = torch.zeros((B, H, N, d), dtype=torch.uint8)
    k8 = make_fp8_inputs(WORKLOADS["tiny"], seed=3, shape_override=(B, H, H, N, d))[0][1]
    v8 = torch.zeros((B, H, N, d), dtype=torch.uint8)
    v8[:, :, torch.arange(N), torch.arange(N) % d] = 0x38  # E4M3 1.0
    ds = (0.02, 0.03, 0.375)
    o, lse = _run(q8, k8, v8, ds, 0.1, causal, torch.bfloat16)
    vis = np.arange(1, N + 1) if causal else np.full(N, N)
    cnt = np.zeros((N, d))
    for i in range(N):
        n = i + 1 if causal else N
        cnt[i] = np.bincount(np.arange(n) % d, minlength=d)
    ref = ds[2] * cnt / vis[:, None]
    err = np.abs(o[0] - ref[None])
    assert float(np.max(err - 2.0 ** -8 * np.abs(ref[None]))) <= 1e-6, float(err.max())
    assert float(np.max(np.abs(lse[0] - np.log(vis)[None]))) <= 1e-5


def test_fp8_forward_deterministic():
    (q8, k8, v8), ds = make_fp8_inputs(WORKLOADS["tiny"], seed=77, shape_override=(1, 4, 2, 520, 128))
    a = _run(q8, k8, v8, ds, 0.09, True, torch.bfloat16)
    b = _run(q8, k8, v8, ds, 0.09, True, torch.bfloat16)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_fp8_forward_4k_workload_rows():
    """The 4K-token MHA shape (B=4, H=32, N=4096, d=128, causal) in the launch
    configuration the FP8 bench times, on 64 seeded rows of every head."""
    w = WORKLOADS["mha4k"]
    (q8, k8, v8), ds = make_fp8_inputs(w)
    o, lse = _run(q8, k8, v8, ds, w.scale, True, torch.bfloat16)
    rows = check_rows(w)[::8].numpy()
    print(_check(q8, k8, v8, ds, w.scale, True, o, lse, rows=rows))


def _random_fp8_cases(n, seed):
    """Seeded FP8 forward shapes: d = 128, MHA / GQA / MQA, sequences from one
    token to several blocks with ragged tails, causal or not, bf16 or fp16 O."""
    g = np.random.default_rng(seed)
    lengths = [1, 2, 7, 64, 65, 127, 128, 129, 255, 300, 511, 700]
    cases = []
    for _ in range(n):
        hkv = int(g.integers(1, 4))
        cases.append(((int(g.integers(1, 4)), hkv * int(g.choice([1, 2, 4])), hkv, int(g.choice(lengths)), 128),
                      bool(g.random() < 0.5), torch.bfloat16 if g.random() < 0.6 else torch.float16))
    return cases


RANDOM_FP8_CASES = _random_fp8_cases(10, seed=4040)


@pytest.mark.parametrize("shape,causal,out_dtype", RANDOM_FP8_CASES,
                         ids=[f"{'x'.join(map(str, s))}-{'c' if c else 'nc'}-{str(t)[6:]}-r{i}"
                              for i, (s, c, t) in enumerate(RANDOM_FP8_CASES)])
def test_fp8_forward_random_shapes(shape, causal, out_dtype):
    test_fp8_forward_full(shape, causal, out_dtype)
