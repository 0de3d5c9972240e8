"""Randomised properties of the CPU oracle over shapes, masks and dtypes of
the inputs (hypothesis): the one-pass online recurrence reaches the two-pass
definition, the row and column forms agree with the full forms, and the
gradients satisfy the identities of the softmax (shift invariance of the
keys, rows of P summing to one, <Q, dQ> = <K, dK>), with any causal flag,
sliding window or block mask."""

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=30, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow])


@st.composite
def problems(draw):
    B = draw(st.integers(1, 2))
    Hkv = draw(st.integers(1, 2))
    Hq = Hkv * draw(st.integers(1, 3))
    N = draw(st.integers(1, 24))
    d = draw(st.integers(1, 6))
    causal = draw(st.booleans())
    seed = draw(st.integers(0, 2 ** 31 - 1))
    r = np.random.default_rng(seed)
    sigma = draw(st.sampled_from([0.5, 1.0, 3.0]))
    q = r.standard_normal((B, Hq, N, d)) * sigma
    k = r.standard_normal((B, Hkv, N, d)) * sigma
    v = r.standard_normal((B, Hkv, N, d))
    do = r.standard_normal((B, Hq, N, d))
    kind = draw(st.sampled_from(["none", "window", "mask"]))
    kw = {}
    if kind == "window" and causal:
        kw["window"] = draw(st.integers(1, N + 1))
    elif kind == "mask":
        bq, bk = draw(st.integers(1, 6)), draw(st.integers(1, 6))
        Tq, Tk = -(-N // bq), -(-N // bk)
        shape = (Hq, Tq, Tk) if draw(st.booleans()) else (Tq, Tk)
        kw["block_mask"] = ((r.random(shape) < draw(st.sampled_from([0.3, 0.7, 1.0]))).astype(np.uint8), bq, bk)
    return q, k, v, do, float(r.uniform(0.2, 0.8)), causal, kw


def _close(a, b, tol, what):
    a, b = np.asarray(a), np.asarray(b)
    fin = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), fin), f"{what}: -inf pattern differs"
    err = float(np.max(np.abs(a[fin] - b[fin]), initial=0.0))
    assert err <= tol, f"{what}: {err:.3e}"


@SETTINGS
@given(problems(), st.integers(1, 9))
def test_online_recurrence_reaches_the_definition(prob, block):
    q, k, v, _, scale, causal, kw = prob
    o, lse = oracle.fwd(q, k, v, scale, causal, **kw)
    o2, lse2 = oracle.fwd_online(q, k, v, scale, causal, block=block, **kw)
    _close(o2, o, 1e-12, "online O")
    _close(lse2, lse, 1e-12, "online lse")


@SETTINGS
@given(problems())
def test_row_and_column_forms_agree(prob):
    q, k, v, do, scale, causal, kw = prob
    N = q.shape[2]
    o, lse = oracle.fwd(q, k, v, scale, causal, **kw)
    dq, dk, dv = oracle.bwd(q, k, v, do, scale, causal, **kw)
    rows = np.unique(np.array([0, N // 2, N - 1]))
    o_r, lse_r = oracle.fwd_rows(q, k, v, rows, scale, causal, **kw)
    _close(o_r, o[:, :, rows], 1e-12, "rows O")
    _close(lse_r, lse[:, :, rows], 1e-12, "rows lse")
    _close(oracle.bwd_rows(q, k, v, do, rows, scale, causal, **kw), dq[:, :, rows], 1e-11, "rows dQ")
    dkc, dvc = oracle.bwd_cols(q, k, v, do, 0, k.shape[1] - 1, rows, scale, causal, **kw)
    _close(dkc, dk[0, -1, rows], 1e-11, "cols dK")
    _close(dvc, dv[0, -1, rows], 1e-11, "cols dV")


@SETTINGS
@given(problems())
def test_gradient_identities(prob):
    q, k, v, do, scale, causal, kw = prob
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    o, lse = oracle.fwd(q, k, v, scale, causal, **kw)
    dq, dk, dv = oracle.bwd(q, k, v, do, scale, causal, **kw)
    # adding one vector to every key shifts each row's scores by a constant
    _close(dk.sum(axis=2), np.zeros((B, Hkv, d)), 1e-11, "sum_j dK_j")
    # rows of P sum to one (rows that see a key; the others have P = 0)
    seen = np.isfinite(lse)[..., None]
    grp = (do * seen).reshape(B, Hkv, G, N, d).sum(axis=(2, 3))
    _close(dv.sum(axis=2), grp, 1e-11, "sum_j dV_j")
    # both sides equal sum_ij dS_ij s_ij / scale
    qdq = (q * dq).reshape(B, Hkv, G, N, d).sum(axis=(2, 3, 4))
    _close(qdq, (k * dk).sum(axis=(2, 3)), 1e-10, "<Q,dQ> = <K,dK>")
    # a row that sees no key has O = 0 and dQ = 0
    empty = ~np.isfinite(lse)
    assert np.all(o[empty] == 0.0) and np.all(dq[empty] == 0.0)
