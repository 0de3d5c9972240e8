"""The FP8 parity tolerances against a CPU model of the rounding they are
derived from: scores from E4M3 inputs in fp64, the running maximum moved
(for all 32 rows of a warp at once) only when a row's maximum grows by more
than 8 (log2 units), probabilities
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
    """The kernel's arithmetic in fp64 except for the roundings it models.
    Rows go in groups of 32 (the 32 rows of one warp): the reference max of
    all rows of a group moves together, to each row's own larger max,
    whenever any row of the group has grown by more than 8 (log2 units)."""
    q = oracle.e4m3_decode(q8) * ds[0]
    k = oracle.e4m3_decode(k8) * ds[1]
    v = oracle.e4m3_decode(v8) * (ds[2] if value_factor else 1.0)
    B, Hq, N, d = q.shape
    G = Hq // k.shape[1]
    c = math.log2(math.e)
    out = np.zeros((B, Hq, N, d))
    for b in range(B):
        for h in range(Hq):
            vv = v[b, h // G]
            S = (q[b, h] @ k[b, h // G].T) * scale * c
            for i0 in range(0, N, 32):
                rows = np.arange(i0, min(i0 + 32, N))
                n_keys = rows + 1 if causal else np.full(len(rows), N)
                m_ref = np.full(len(rows), -np.inf)
                l = np.zeros(len(rows))
                acc = np.zeros((len(rows), d))
                for j0 in range(0, int(n_keys.max()), 128):
                    j1 = min(j0 + 128, N)
                    s = S[rows, j0:j1].copy()
                    s[np.arange(j0, j1)[None, :] >= n_keys[:, None]] = -np.inf
                    m_new = s.max(axis=1)
                    if j0 == 0:
                        m_ref = m_new
                    elif np.any(m_new > m_ref + 8):
                        m_upd = np.maximum(m_ref, m_new)
                        f = np.exp2(m_ref - m_upd)
                        acc, l, m_ref = acc * f[:, None], l * f, m_upd
                    p = np.exp2(s - m_ref[:, None])
                    l += p.sum(axis=1)
                    if round_p:
                        p = torch.from_numpy(p).float().to(torch.float8_e4m3fn).double().numpy()
                    acc += p @ vv[j0:j1]
                out[b, h, rows] = acc / l[:, None]
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
