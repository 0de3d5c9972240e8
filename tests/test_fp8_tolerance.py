"""The FP8 parity tolerances against a CPU model of the rounding they are
derived from: scores from E4M3 inputs in fp64, the running maximum moved
only when a row's maximum grows by more than 8 (log2 units), probabilities
rounded to E4M3 (torch's round-to-nearest-even cast) before P V, row sums in
unrounded form, O rounded to bf16.  The model must stay inside the envelope
the GPU tests use, with margin; a model that skips the rounding of P must
sit far inside it, and one that drops the value factor must fall outside."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_bwd_b200.workloads import WORKLOADS, make_fp8_inputs

REL_FROB_TOL = 0.05


def _model(q8, k8, v8, ds, scale, causal, round_p=True, value_factor=True):
    q = oracle.e4m3_decode(q8) * ds[0]
    k = oracle.e4m3_decode(k8) * ds[1]
    v = oracle.e4m3_decode(v8) * (ds[2] if value_factor else 1.0)
    B, Hq, N, d = q.shape
    G = Hq // k.shape[1]
    c = math.log2(math.e)
    out = np.zeros((B, Hq, N, d))
    for b in range(B):
        for h in range(Hq):
            S = (q[b, h] @ k[b, h // G].T) * scale * c
            for i in range(N):
                n_keys = i + 1 if causal else N
                m_ref, l, acc = -np.inf, 0.0, np.zeros(d)
                for j0 in range(0, n_keys, 128):
                    s = S[i, j0:min(j0 + 128, n_keys)]
                    if j0 == 0:
                        m_ref = s.max()
                    elif s.max() > m_ref + 8:
                        f = 2.0 ** (m_ref - s.max())
                        acc, l, m_ref = acc * f, l * f, s.max()
                    p = np.exp2(s - m_ref)
                    l += p.sum()
                    if round_p:
                        p = torch.from_numpy(p).float().to(torch.float8_e4m3fn).double().numpy()
                    acc += p @ v[b, h // G, j0:j0 + len(s)]
                out[b, h, i] = acc / l
    return torch.from_numpy(out).to(torch.bfloat16).double().numpy()


def _envelope_ratio(q8, k8, v8, ds, scale, causal, o):
    o_ref, lse_ref = oracle.fwd_fp8(q8, k8, v8, ds, scale, causal)
    q = oracle.e4m3_decode(q8) * ds[0]
    k = oracle.e4m3_decode(k8) * ds[1]
    av = np.abs(oracle.e4m3_decode(v8) * ds[2])
    G = q.shape[1] // k.shape[1]
    N = q.shape[2]
    worst = 0.0
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            s = (q[b, h] @ k[b, h // G].T) * scale
            if causal:
                s = np.where(np.tri(N, dtype=bool), s, -np.inf)
            w = np.exp(s - lse_ref[b, h][:, None])
            env = 2.0 ** -4 * (w @ av[b, h // G]) + 2.0 ** -8 * np.abs(o_ref[b, h]) + 1e-3
            worst = max(worst, float(np.max(np.abs(o[b, h] - o_ref[b, h]) / env)))
    rel = float(np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref))
    return worst, rel


@pytest.mark.parametrize("shape,causal", [((1, 2, 2, 256, 64), True), ((1, 2, 1, 300, 32), False)])
def test_fp8_envelope_holds_for_the_rounding_model(shape, causal):
    (q8, k8, v8), ds = make_fp8_inputs(WORKLOADS["tiny"], seed=21 + causal, shape_override=shape)
    scale = 1.0 / math.sqrt(shape[-1])
    worst, rel = _envelope_ratio(q8, k8, v8, ds, scale, causal, _model(q8, k8, v8, ds, scale, causal))
    assert worst <= 0.85, f"rounding model reaches {worst:.3f} of the per-element envelope"
    assert 0.005 <= rel <= 0.8 * REL_FROB_TOL, f"rounding model relative Frobenius error {rel:.4f}"
    worst0, rel0 = _envelope_ratio(q8, k8, v8, ds, scale, causal,
                                   _model(q8, k8, v8, ds, scale, causal, round_p=False))
    assert rel0 < rel / 5, "without rounding P the error must be far smaller"
    bad, rel_bad = _envelope_ratio(q8, k8, v8, ds, scale, causal,
                                   _model(q8, k8, v8, ds, scale, causal, value_factor=False))
    assert bad > 1.0 and rel_bad > REL_FROB_TOL, "a dropped value factor must fail the checks"
