"""Pins of the CPU oracle against facts that do not come from the oracle.

Each ``pin_*`` takes an ``oracle.Oracle`` instance and raises AssertionError
when the oracle disagrees with a closed form, a hand-derived value, a library
routine, a finite difference or an invariant of the mathematics.  They are
collected here so that the same list can be run against the real oracle
(tests/test_oracle_pins.py) and against copies with a planted mistake
(tests/test_oracle_mutants.py), which must each fail at least one pin.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _rand(seed, B=1, Hq=2, Hkv=2, N=8, d=4):
    r = _rng(seed)
    q = r.standard_normal((B, Hq, N, d))
    k = r.standard_normal((B, Hkv, N, d))
    v = r.standard_normal((B, Hkv, N, d))
    do = r.standard_normal((B, Hq, N, d))
    return q, k, v, do


def _close(a, b, tol, what):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------- forward pins

def pin_q_zero_noncausal(orc):
    """Q = 0: every score is 0, P is uniform, O_i = mean_j V_j, lse_i = ln N."""
    _, k, v, _ = _rand(1, Hq=2, Hkv=2, N=12, d=5)
    q = np.zeros((1, 2, 12, 5))
    o, lse = orc.fwd(q, k, v, 0.37, False)
    _close(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), 1e-13, "O at Q=0")
    _close(lse, np.full(lse.shape, math.log(12)), 1e-13, "lse at Q=0")


def pin_q_zero_causal(orc):
    """Q = 0, causal: O_i = mean_{j<=i} V_j, lse_i = ln(i + 1)."""
    _, k, v, _ = _rand(2, Hq=1, Hkv=1, N=10, d=3)
    q = np.zeros((1, 1, 10, 3))
    o, lse = orc.fwd(q, k, v, 0.5, True)
    prefix = np.cumsum(v[0, 0], axis=0) / np.arange(1, 11)[:, None]
    _close(o[0, 0], prefix, 1e-13, "causal O at Q=0")
    _close(lse[0, 0], np.log(np.arange(1, 11)), 1e-13, "causal lse at Q=0")


def pin_one_hot(orc):
    """q_i = c e_t, k_{j*} = e_t, every other key 0: scores are (scale c) at j* and
    0 elsewhere, so O_i = (e^{sc} V_j* + sum_{j != j*} V_j) / (e^{sc} + N - 1) and
    lse_i = ln(e^{sc} + N - 1); for large c, O_i -> V_j*."""
    N, d, t, js, c, scale = 9, 4, 2, 6, 40.0, 0.5
    q = np.zeros((1, 1, N, d)); q[..., t] = c
    k = np.zeros((1, 1, N, d)); k[0, 0, js, t] = 1.0
    v = _rng(3).standard_normal((1, 1, N, d))
    o, lse = orc.fwd(q, k, v, scale, False)
    e = math.exp(scale * c)
    want = (e * v[0, 0, js] + (v[0, 0].sum(axis=0) - v[0, 0, js])) / (e + N - 1)
    _close(o[0, 0], np.broadcast_to(want, (N, d)), 1e-12, "one-hot O")
    _close(lse[0, 0], np.full(N, math.log(e + N - 1)), 1e-12, "one-hot lse")
    _close(o[0, 0], np.broadcast_to(v[0, 0, js], (N, d)), 1e-6, "one-hot selects V[j*]")


def pin_causal_row0(orc):
    """Causal row 0 sees key 0 only: O_0 = V_0, lse_0 = scale q_0 . k_0."""
    q, k, v, _ = _rand(4, Hq=4, Hkv=2, N=7, d=6)
    o, lse = orc.fwd(q, k, v, 0.41, True)
    for h in range(4):
        g = h // 2
        _close(o[0, h, 0], v[0, g, 0], 1e-14, "causal O_0")
        _close(lse[0, h, 0], 0.41 * q[0, h, 0] @ k[0, g, 0], 1e-14, "causal lse_0")


def pin_rows_sum_to_one(orc):
    """sum_j P_ij = 1: with V = 1 every output is 1, causal or not."""
    q, k, _, _ = _rand(5, Hq=2, Hkv=1, N=11, d=4)
    v = np.ones((1, 1, 11, 4))
    for causal in (False, True):
        o, _ = orc.fwd(q * 3, k, v, 0.8, causal)
        _close(o, np.ones_like(o), 1e-14, f"rows of P sum to 1 (causal={causal})")


def pin_key_shift(orc):
    """K -> K + 1 c^T shifts row i of the scores by scale q_i . c: P and O are
    unchanged and lse_i moves by exactly that amount."""
    q, k, v, _ = _rand(6, Hq=2, Hkv=2, N=9, d=3)
    c = np.array([0.7, -1.3, 2.1])
    for causal in (False, True):
        o1, l1 = orc.fwd(q, k, v, 0.6, causal)
        o2, l2 = orc.fwd(q, k + c, v, 0.6, causal)
        _close(o2, o1, 1e-12, "O invariant to key shift")
        _close(l2 - l1, 0.6 * q @ c, 1e-12, "lse shift")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        g = json.load(f)

    def val(x):
        if isinstance(x, (int, float)):
            return float(x)
        consts = {"ln3": math.log(3), "ln4": math.log(4), "ln2": math.log(2),
                  "0.75ln3": 0.75 * math.log(3)}
        return consts[x]

    s = g["shape"]
    B, Hq, Hkv, N, d = s["B"], s["Hq"], s["Hkv"], s["N"], s["d"]
    arr = lambda x, H: np.array([val(t) for t in x]).reshape(B, H, N, d)
    q, k, v, do = arr(g["q"], Hq), arr(g["k"], Hkv), arr(g["v"], Hkv), arr(g["dout"], Hq)
    return g, q, k, v, do, val


def pin_golden(orc):
    """Hand-derived two-token examples (tests/golden/*.json)."""
    for name in ("two_token_mha.json", "two_token_gqa.json"):
        g, q, k, v, do, val = _golden(name)
        for case, want in g["cases"].items():
            causal = case == "causal"
            o, lse = orc.fwd(q, k, v, g["scale"], causal)
            dq, dk, dv = orc.bwd(q, k, v, do, g["scale"], causal)
            _close(o.ravel(), [val(x) for x in want["o"]], 1e-13, f"{name} {case} O")
            _close(lse.ravel(), [val(x) for x in want["lse"]], 1e-13, f"{name} {case} lse")
            _close(dq.ravel(), [val(x) for x in want["dq"]], 1e-13, f"{name} {case} dQ")
            _close(dk.ravel(), [val(x) for x in want["dk"]], 1e-13, f"{name} {case} dK")
            _close(dv.ravel(), [val(x) for x in want["dv"]], 1e-13, f"{name} {case} dV")


def pin_brute_force_python(orc):
    """Forward by pure-Python loops (math.exp, two explicit passes) on tiny inputs."""
    B, Hq, Hkv, N, d = 1, 4, 2, 5, 3
    q, k, v, _ = _rand(7, B, Hq, Hkv, N, d)
    scale = 0.9
    for causal in (False, True):
        o, lse = orc.fwd(q, k, v, scale, causal)
        for h in range(Hq):
            g = h // (Hq // Hkv)
            for i in range(N):
                js = [j for j in range(N) if not (causal and j > i)]
                s = {j: scale * sum(q[0, h, i, c] * k[0, g, j, c] for c in range(d)) for j in js}
                m = max(s.values())
                z = sum(math.exp(s[j] - m) for j in js)
                for c in range(d):
                    want = sum(math.exp(s[j] - m) / z * v[0, g, j, c] for j in js)
                    assert abs(o[0, h, i, c] - want) < 1e-13, ("brute O", h, i, c)
                assert abs(lse[0, h, i] - (m + math.log(z))) < 1e-13, ("brute lse", h, i)


def _torch_ref(q, k, v, do, scale, causal):
    """torch fp64 SDPA (CPU math path) + autograd; lse by torch.logsumexp."""
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    Hq, Hkv = q.shape[1], k.shape[1]
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, is_causal=causal, scale=scale, enable_gqa=Hq != Hkv)
    o.backward(torch.tensor(do, dtype=torch.float64))
    with torch.no_grad():
        kk = tk.repeat_interleave(Hq // Hkv, dim=1)
        s = scale * tq @ kk.transpose(-1, -2)
        if causal:
            n = s.shape[-1]
            s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
        lse = torch.logsumexp(s, dim=-1)
    return (o.detach().numpy(), lse.numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy())


def pin_torch_sdpa(orc):
    """Library special case: torch fp64 scaled_dot_product_attention and autograd,
    MHA and GQA, causal and not."""
    for (Hq, Hkv, N, d, seed) in ((2, 2, 64, 16, 8), (4, 2, 33, 8, 9), (4, 1, 20, 8, 10)):
        q, k, v, do = _rand(seed, 1, Hq, Hkv, N, d)
        scale = 1.0 / math.sqrt(d)
        for causal in (False, True):
            o, lse = orc.fwd(q, k, v, scale, causal)
            dq, dk, dv = orc.bwd(q, k, v, do, scale, causal)
            ro, rl, rdq, rdk, rdv = _torch_ref(q, k, v, do, scale, causal)
            tag = f"Hq{Hq} Hkv{Hkv} N{N} causal={causal}"
            _close(o, ro, 1e-12, f"torch O {tag}")
            _close(lse, rl, 1e-12, f"torch lse {tag}")
            _close(dq, rdq, 1e-11, f"torch dQ {tag}")
            _close(dk, rdk, 1e-11, f"torch dK {tag}")
            _close(dv, rdv, 1e-11, f"torch dV {tag}")


# --------------------------------------------------------------- backward pins

def pin_finite_differences(orc):
    """Central differences (h = 1e-6) of L = sum(dO * O) against dQ, dK, dV."""
    h = 1e-6
    for (Hq, Hkv, N, d, causal, seed) in ((1, 1, 6, 3, False, 11), (2, 1, 5, 4, True, 12),
                                          (2, 2, 7, 2, True, 13)):
        q, k, v, do = _rand(seed, 1, Hq, Hkv, N, d)
        scale = 0.7
        dq, dk, dv = orc.bwd(q, k, v, do, scale, causal)

        def loss(args):
            o, _ = orc.fwd(args[0], args[1], args[2], scale, causal)
            return float(np.sum(do * o))

        for slot, (name, g) in enumerate((("q", dq), ("k", dk), ("v", dv))):
            x = (q, k, v)[slot]
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                plus, minus = [q, k, v], [q, k, v]
                plus[slot], minus[slot] = x.copy(), x.copy()
                plus[slot][idx] += h
                minus[slot][idx] -= h
                num[idx] = (loss(plus) - loss(minus)) / (2 * h)
            rel = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-30)
            assert rel <= 1e-6, f"finite differences d{name} (Hq{Hq} Hkv{Hkv} causal={causal}): rel {rel:.2e}"


def pin_q_zero_backward(orc):
    """Q = 0, non-causal: dK = 0 exactly, dV_j = mean_i dO_i,
    dQ_i = scale (1/N) sum_j (dO_i . (v_j - vbar)) k_j."""
    _, k, v, do = _rand(14, 1, 2, 2, 10, 4)
    q = np.zeros_like(do)
    scale = 0.3
    dq, dk, dv = orc.bwd(q, k, v, do, scale, False)
    _close(dk, np.zeros_like(dk), 0.0, "dK at Q=0")
    _close(dv, np.broadcast_to(do.mean(axis=2, keepdims=True), dv.shape), 1e-14, "dV at Q=0")
    vbar = v.mean(axis=2, keepdims=True)
    coef = np.einsum("bhic,bhjc->bhij", do, v - vbar)
    want = scale / 10 * np.einsum("bhij,bhjc->bhic", coef, k)
    _close(dq, want, 1e-13, "dQ at Q=0")


def pin_gradient_invariants(orc):
    """(i) sum_j dK_j = 0 per kv head; (ii) sum_j dV_j = sum over the group of
    sum_i dO_i; (iii) <Q, dQ> = <K, dK> per kv group."""
    for causal in (False, True):
        q, k, v, do = _rand(15, 2, 4, 2, 13, 5)
        dq, dk, dv = orc.bwd(q, k, v, do, 0.45, causal)
        _close(dk.sum(axis=2), np.zeros((2, 2, 5)), 1e-12, "sum_j dK_j")
        grp = do.reshape(2, 2, 2, 13, 5).sum(axis=(2, 3))
        _close(dv.sum(axis=2), grp, 1e-12, "sum_j dV_j")
        qdq = (q * dq).reshape(2, 2, 2, 13, 5).sum(axis=(2, 3, 4))
        kdk = (k * dk).sum(axis=(2, 3))
        _close(qdq, kdk, 1e-12, "<Q,dQ> = <K,dK>")


def pin_subsets_match_full(orc):
    """Row- and column-subset forms equal the full forms on the same inputs."""
    q, k, v, do = _rand(16, 2, 4, 2, 40, 8)
    rows = np.array([0, 3, 17, 39])
    cols = np.array([1, 20, 38])
    for causal in (False, True):
        o, lse = orc.fwd(q, k, v, 0.35, causal)
        dq, dk, dv = orc.bwd(q, k, v, do, 0.35, causal)
        o_r, lse_r = orc.fwd_rows(q, k, v, rows, 0.35, causal)
        _close(o_r, o[:, :, rows], 1e-13, "fwd_rows O")
        _close(lse_r, lse[:, :, rows], 1e-13, "fwd_rows lse")
        _close(orc.bwd_rows(q, k, v, do, rows, 0.35, causal), dq[:, :, rows], 1e-12, "bwd_rows dQ")
        for (b, g) in ((0, 1), (1, 0)):
            dkc, dvc = orc.bwd_cols(q, k, v, do, b, g, cols, 0.35, causal)
            _close(dkc, dk[b, g, cols], 1e-12, "bwd_cols dK")
            _close(dvc, dv[b, g, cols], 1e-12, "bwd_cols dV")


def pin_online_equals_two_pass(orc):
    """The one-pass blocked recurrence reaches the two-pass result (fp64, 1e-12),
    for block sizes that divide N and that leave a ragged last block."""
    q, k, v, _ = _rand(17, 1, 2, 1, 70, 8)
    q = q * 4  # wide score range: the running max moves many times along a row
    for causal in (False, True):
        o, lse = orc.fwd(q, k, v, 0.5, causal)
        for block in (1, 7, 16, 128):
            o2, lse2 = orc.fwd_online(q, k, v, 0.5, causal, block=block)
            _close(o2, o, 1e-12, f"online O (block {block})")
            _close(lse2, lse, 1e-12, f"online lse (block {block})")


# ----------------------------------------------------- sliding-window pins
# Causal sliding window of W keys: query i sees keys max(0, i-W+1) .. i.

def pin_window_closed_forms(orc):
    """W = 1: each query sees only its own key, O_i = V_i, lse_i = s_ii.
    Q = 0: O_i = mean of V over the window, lse_i = ln(min(i+1, W)).
    W >= N: the plain causal result."""
    q, k, v, _ = _rand(18, 1, 2, 2, 21, 6)
    o, lse = orc.fwd(q, k, v, 0.4, True, window=1)
    _close(o, v, 1e-15, "O with W=1")
    _close(lse, 0.4 * np.einsum("bhic,bhic->bhi", q, k), 1e-14, "lse with W=1")
    z = np.zeros_like(q)
    for W in (2, 5, 8):
        o, lse = orc.fwd(z, k, v, 0.4, True, window=W)
        want = np.stack([v[:, :, max(0, i - W + 1):i + 1].mean(axis=2) for i in range(21)], axis=2)
        _close(o, want, 1e-14, f"O at Q=0, W={W}")
        _close(lse, np.broadcast_to(np.log(np.minimum(np.arange(1, 22), W)), lse.shape), 1e-14,
               f"lse at Q=0, W={W}")
    o1, l1 = orc.fwd(q, k, v, 0.4, True, window=21)
    o2, l2 = orc.fwd(q, k, v, 0.4, True)
    _close(o1, o2, 0.0, "W = N equals causal")
    _close(l1, l2, 0.0, "W = N equals causal (lse)")


def pin_window_brute_force(orc):
    """Forward with a window by pure-Python loops over the visible keys."""
    B, Hq, Hkv, N, d = 1, 2, 1, 9, 3
    q, k, v, _ = _rand(19, B, Hq, Hkv, N, d)
    for W in (2, 4):
        o, lse = orc.fwd(q, k, v, 0.8, True, window=W)
        for h in range(Hq):
            for i in range(N):
                js = range(max(0, i - W + 1), i + 1)
                s = {j: 0.8 * sum(q[0, h, i, c] * k[0, 0, j, c] for c in range(d)) for j in js}
                m = max(s.values())
                z = sum(math.exp(x - m) for x in s.values())
                for c in range(d):
                    want = sum(math.exp(s[j] - m) / z * v[0, 0, j, c] for j in js)
                    assert abs(o[0, h, i, c] - want) < 1e-13, ("window brute O", W, h, i, c)
                assert abs(lse[0, h, i] - (m + math.log(z))) < 1e-13, ("window brute lse", W, h, i)


def _torch_window_ref(q, k, v, do, scale, W):
    """torch fp64 SDPA with an explicit boolean mask (True = visible) + autograd."""
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    Hq, Hkv, n = q.shape[1], k.shape[1], q.shape[2]
    i = torch.arange(n)[:, None]
    j = torch.arange(n)[None, :]
    mask = (j <= i) & (j > i - W)
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=mask, scale=scale, enable_gqa=Hq != Hkv)
    o.backward(torch.tensor(do, dtype=torch.float64))
    return o.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def pin_window_torch_sdpa(orc):
    """Library special case: torch fp64 SDPA with the window as an explicit
    mask, forward and gradients, MHA and GQA."""
    for (Hq, Hkv, N, d, W, seed) in ((2, 2, 40, 8, 7, 20), (4, 2, 33, 8, 16, 21), (2, 1, 25, 4, 1, 22)):
        q, k, v, do = _rand(seed, 1, Hq, Hkv, N, d)
        scale = 1.0 / math.sqrt(d)
        o, _ = orc.fwd(q, k, v, scale, True, window=W)
        dq, dk, dv = orc.bwd(q, k, v, do, scale, True, window=W)
        ro, rdq, rdk, rdv = _torch_window_ref(q, k, v, do, scale, W)
        tag = f"Hq{Hq} Hkv{Hkv} N{N} W{W}"
        _close(o, ro, 1e-12, f"torch windowed O {tag}")
        _close(dq, rdq, 1e-11, f"torch windowed dQ {tag}")
        _close(dk, rdk, 1e-11, f"torch windowed dK {tag}")
        _close(dv, rdv, 1e-11, f"torch windowed dV {tag}")


def pin_window_finite_differences(orc):
    """Central differences of L = sum(dO * O) with a window of 3 keys."""
    h = 1e-6
    q, k, v, do = _rand(23, 1, 2, 1, 6, 3)
    dq, dk, dv = orc.bwd(q, k, v, do, 0.6, True, window=3)

    def loss(a):
        o, _ = orc.fwd(a[0], a[1], a[2], 0.6, True, window=3)
        return float(np.sum(do * o))

    for slot, g in enumerate((dq, dk, dv)):
        x = (q, k, v)[slot]
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            plus, minus = [q, k, v], [q, k, v]
            plus[slot], minus[slot] = x.copy(), x.copy()
            plus[slot][idx] += h
            minus[slot][idx] -= h
            num[idx] = (loss(plus) - loss(minus)) / (2 * h)
        rel = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-30)
        assert rel <= 1e-6, f"windowed finite differences slot {slot}: rel {rel:.2e}"


def pin_window_subsets_and_online(orc):
    """With a window, the row/column subset forms equal the full forms and the
    blocked one-pass recurrence (fully hidden blocks skipped) equals two-pass."""
    q, k, v, do = _rand(24, 1, 4, 2, 50, 8)
    rows, cols = np.array([0, 9, 30, 49]), np.array([0, 13, 47])
    for W in (5, 17):
        o, lse = orc.fwd(q, k, v, 0.35, True, window=W)
        dq, dk, dv = orc.bwd(q, k, v, do, 0.35, True, window=W)
        o_r, lse_r = orc.fwd_rows(q, k, v, rows, 0.35, True, window=W)
        _close(o_r, o[:, :, rows], 1e-13, f"windowed fwd_rows O W{W}")
        _close(lse_r, lse[:, :, rows], 1e-13, f"windowed fwd_rows lse W{W}")
        _close(orc.bwd_rows(q, k, v, do, rows, 0.35, True, window=W), dq[:, :, rows], 1e-12,
               f"windowed bwd_rows W{W}")
        dkc, dvc = orc.bwd_cols(q, k, v, do, 0, 1, cols, 0.35, True, window=W)
        _close(dkc, dk[0, 1, cols], 1e-12, f"windowed bwd_cols dK W{W}")
        _close(dvc, dv[0, 1, cols], 1e-12, f"windowed bwd_cols dV W{W}")
        for block in (4, 16):
            o2, lse2 = orc.fwd_online(q * 3, k, v, 0.35, True, block=block, window=W)
            o3, lse3 = orc.fwd(q * 3, k, v, 0.35, True, window=W)
            _close(o2, o3, 1e-12, f"windowed online O W{W} block {block}")
            _close(lse2, lse3, 1e-12, f"windowed online lse W{W} block {block}")


# ------------------------------------------------------------- dropout pins
# dropout=(t, seed): a key is dropped when its Philox byte is below t; kept
# probabilities are scaled by 256 / (256 - t).

def pin_philox_known_answers(orc):
    """The generator reproduces the published Philox4x32-10 known-answer vectors."""
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.json")) as f:
        kat = json.load(f)
    for vec in kat["vectors"]:
        got = orc.philox4x32_10([int(x, 16) for x in vec["ctr"]], [int(x, 16) for x in vec["key"]])
        assert got == [int(x, 16) for x in vec["out"]], ("Philox KAT", vec, [hex(x) for x in got])


def _mask(orc, bh, N, t, seed):
    """Keep mask [N][N] of one query head from the generator, by the stated
    counter layout (j/4, i/4, bh, 0), word i%4, byte j%4."""
    key = [seed & 0xFFFFFFFF, seed >> 32]
    z = np.zeros((N, N))
    for i in range(N):
        for j in range(N):
            x = orc.philox4x32_10([j >> 2, i >> 2, bh, 0], key)
            z[i, j] = ((x[i & 3] >> (8 * (j & 3))) & 0xFF) >= t
    return z


def pin_dropout_off_and_keep_rate(orc):
    """t = 0 is exactly no dropout; the keep rate of t = 64 is 3/4."""
    q, k, v, do = _rand(25, 1, 2, 1, 24, 8)
    o0, l0 = orc.fwd(q, k, v, 0.5, True)
    o1, l1 = orc.fwd(q, k, v, 0.5, True, dropout=(0, 99))
    _close(o1, o0, 0.0, "dropout t=0 O")
    _close(l1, l0, 0.0, "dropout t=0 lse")
    g0 = orc.bwd(q, k, v, do, 0.5, True)
    g1 = orc.bwd(q, k, v, do, 0.5, True, dropout=(0, 99))
    for a, b_ in zip(g0, g1):
        _close(a, b_, 0.0, "dropout t=0 gradients")
    z = np.concatenate([_mask(orc, bh, 64, 64, 12345).ravel() for bh in range(3)])
    assert abs(z.mean() - 0.75) < 0.01, f"keep rate {z.mean():.4f} for t=64"


def pin_dropout_identity_readout(orc):
    """Q = 0 (uniform P = 1/N, non-causal) and V = I: O = Z * s / N, so the
    output is the keep mask itself, entry by entry; lse = ln N is untouched."""
    N = d = 16
    for (t, seed) in ((64, 7), (200, (1 << 40) + 3)):
        q = np.zeros((1, 2, N, d))
        k = _rand(26, 1, 2, 2, N, d)[1]
        v = np.broadcast_to(np.eye(N)[None, None], (1, 2, N, d)).copy()
        o, lse = orc.fwd(q, k, v, 0.3, False, dropout=(t, seed))
        for h in range(2):
            want = _mask(orc, h, N, t, seed) * (256.0 / (256 - t)) / N
            _close(o[0, h], want, 1e-15, f"identity read-out t={t} head {h}")
        _close(lse, np.full(lse.shape, math.log(N)), 1e-14, "lse with dropout")


def pin_dropout_torch(orc):
    """Library special case: torch fp64 attention with the keep mask applied
    to the softmax as an explicit matrix, forward and autograd gradients."""
    for (Hq, Hkv, N, d, causal, t, seed) in ((2, 1, 20, 8, True, 51, 5), (2, 2, 17, 4, False, 128, 6)):
        q, k, v, do = _rand(27 + N, 1, Hq, Hkv, N, d)
        scale = 0.6
        z = np.stack([_mask(orc, h, N, t, seed) for h in range(Hq)]) * (256.0 / (256 - t))
        tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
        kk, vv = (x.repeat_interleave(Hq // Hkv, dim=1) for x in (tk, tv))
        s = scale * tq @ kk.transpose(-1, -2)
        if causal:
            s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
        p = torch.softmax(s, dim=-1) * torch.tensor(z)[None]
        o_t = p @ vv
        o_t.backward(torch.tensor(do))
        o, _ = orc.fwd(q, k, v, scale, causal, dropout=(t, seed))
        dq, dk, dv = orc.bwd(q, k, v, do, scale, causal, dropout=(t, seed))
        _close(o, o_t.detach().numpy(), 1e-12, "torch dropout O")
        _close(dq, tq.grad.numpy(), 1e-11, "torch dropout dQ")
        _close(dk, tk.grad.numpy(), 1e-11, "torch dropout dK")
        _close(dv, tv.grad.numpy(), 1e-11, "torch dropout dV")


def pin_dropout_finite_differences(orc):
    """Central differences of L = sum(dO * O) under a fixed dropout mask."""
    h = 1e-6
    q, k, v, do = _rand(28, 1, 2, 1, 6, 3)
    drop = (90, 77)
    grads = orc.bwd(q, k, v, do, 0.7, True, dropout=drop)

    def loss(a):
        o, _ = orc.fwd(a[0], a[1], a[2], 0.7, True, dropout=drop)
        return float(np.sum(do * o))

    for slot, g in enumerate(grads):
        x = (q, k, v)[slot]
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            plus, minus = [q, k, v], [q, k, v]
            plus[slot], minus[slot] = x.copy(), x.copy()
            plus[slot][idx] += h
            minus[slot][idx] -= h
            num[idx] = (loss(plus) - loss(minus)) / (2 * h)
        rel = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-30)
        assert rel <= 1e-6, f"dropout finite differences slot {slot}: rel {rel:.2e}"


def pin_dropout_subsets_and_online(orc):
    """With dropout the row/column subset forms equal the full forms, and the
    blocked one-pass recurrence equals two-pass."""
    q, k, v, do = _rand(29, 2, 4, 2, 36, 8)
    rows, cols = np.array([0, 5, 35]), np.array([2, 17, 33])
    drop = (40, 2024)
    for causal in (False, True):
        o, lse = orc.fwd(q, k, v, 0.35, causal, dropout=drop)
        dq, dk, dv = orc.bwd(q, k, v, do, 0.35, causal, dropout=drop)
        o_r, lse_r = orc.fwd_rows(q, k, v, rows, 0.35, causal, dropout=drop)
        _close(o_r, o[:, :, rows], 1e-13, "dropout fwd_rows O")
        _close(lse_r, lse[:, :, rows], 1e-13, "dropout fwd_rows lse")
        _close(orc.bwd_rows(q, k, v, do, rows, 0.35, causal, dropout=drop), dq[:, :, rows], 1e-12,
               "dropout bwd_rows")
        dkc, dvc = orc.bwd_cols(q, k, v, do, 1, 0, cols, 0.35, causal, dropout=drop)
        _close(dkc, dk[1, 0, cols], 1e-12, "dropout bwd_cols dK")
        _close(dvc, dv[1, 0, cols], 1e-12, "dropout bwd_cols dV")
        o2, l2 = orc.fwd_online(q, k, v, 0.35, causal, block=8, dropout=drop)
        _close(o2, o, 1e-12, "dropout online O")
        _close(l2, lse, 1e-12, "dropout online lse")


# -------------------------------------------------------- paged-decode pins

def _paged_case(seed, B=3, Hq=4, Hkv=2, Nq=2, d=8, P=4, lens=(13, 7, 20), extra_pages=3):
    """Contiguous K/V per sequence scattered into a shuffled page pool."""
    r = _rng(seed)
    max_pages = max((L + P - 1) // P for L in lens)
    n_used = sum((L + P - 1) // P for L in lens)
    num_pages = n_used + extra_pages
    perm = r.permutation(num_pages)
    kc = r.standard_normal((num_pages, Hkv, P, d))
    vc = r.standard_normal((num_pages, Hkv, P, d))
    table = np.full((B, max_pages), -1, dtype=np.int64)
    k_seq, v_seq, used = [], [], 0
    for b, L in enumerate(lens):
        npg = (L + P - 1) // P
        table[b, :npg] = perm[used:used + npg]
        used += npg
        kk = np.concatenate([kc[table[b, p]] for p in range(npg)], axis=1)[:, :L]  # [Hkv, L, d]
        vv = np.concatenate([vc[table[b, p]] for p in range(npg)], axis=1)[:, :L]
        k_seq.append(kk)
        v_seq.append(vv)
    q = r.standard_normal((B, Hq, Nq, d))
    return q, kc, vc, table, np.array(lens), k_seq, v_seq


def pin_decode_equals_contiguous_attention(orc):
    """Decode over a paged cache equals the causal attention of the last Nq
    rows of the contiguous sequence (the already-pinned row form)."""
    q, kc, vc, table, lens, k_seq, v_seq = _paged_case(30)
    B, Hq, Nq, d = q.shape
    o, lse = orc.decode_paged(q, kc, vc, table, lens, 0.45)
    for b, L in enumerate(lens):
        qf = np.zeros((1, Hq, L, d))
        qf[0, :, L - Nq:] = q[b]
        rows = np.arange(L - Nq, L)
        o_r, lse_r = orc.fwd_rows(qf, k_seq[b][None], v_seq[b][None], rows, 0.45, True)
        _close(o[b], o_r[0], 1e-13, f"decode O seq {b}")
        _close(lse[b], lse_r[0], 1e-13, f"decode lse seq {b}")


def pin_decode_page_shuffle_and_q_zero(orc):
    """Moving the pages of the pool (and the table with them) changes nothing;
    Q = 0 gives the mean of the visible values and lse = ln(#visible)."""
    q, kc, vc, table, lens, k_seq, v_seq = _paged_case(31, Nq=3, P=5, lens=(11, 3, 16))
    o, lse = orc.decode_paged(q, kc, vc, table, lens, 0.6)
    r = _rng(32)
    perm = r.permutation(kc.shape[0])
    inv = np.argsort(perm)
    t2 = np.where(table >= 0, inv[np.maximum(table, 0)], -1)
    o2, lse2 = orc.decode_paged(q, kc[perm], vc[perm], t2, lens, 0.6)
    _close(o2, o, 0.0, "decode after moving pages")
    _close(lse2, lse, 0.0, "decode lse after moving pages")
    z = np.zeros_like(q)
    oz, lz = orc.decode_paged(z, kc, vc, table, lens, 0.6)
    B, Hq, Nq, d = q.shape
    G = Hq // kc.shape[1]
    for b, L in enumerate(lens):
        for h in range(Hq):
            for t in range(Nq):
                n_vis = L - Nq + t + 1
                _close(oz[b, h, t], v_seq[b][h // G, :n_vis].mean(axis=0), 1e-14, "decode O at Q=0")
                assert abs(lz[b, h, t] - math.log(n_vis)) < 1e-14, "decode lse at Q=0"


# ------------------------------------------------------------------ FP8 pins

# E4M3 values worked out by hand from the format: sign, 4-bit exponent with
# bias 7, 3-bit fraction, subnormals (f/8)*2^-6, e=15 f=7 the only NaN.
E4M3_HAND = {
    0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x0F: 1.875 * 2.0 ** -6,
    0x30: 0.5, 0x38: 1.0, 0x3C: 1.5, 0x40: 2.0, 0x77: 240.0, 0x7E: 448.0,
    0x81: -(2.0 ** -9), 0xB8: -1.0, 0xFE: -448.0,
}


def pin_e4m3_decode(orc):
    """Every E4M3 code decodes as torch.float8_e4m3fn does; hand values; the
    two NaN codes; -0 keeps its sign."""
    codes = np.arange(256, dtype=np.uint8)
    got = orc.e4m3_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref)), "E4M3 NaN codes"
    fin = ~np.isnan(ref)
    _close(got[fin], ref[fin], 0.0, "E4M3 decode against torch")
    for c, val in E4M3_HAND.items():
        assert got[c] == val, f"E4M3 code {c:#04x}: {got[c]!r} != {val!r}"
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF]) and int(np.isnan(got).sum()) == 2
    assert math.copysign(1.0, got[0x80]) == -1.0 and got[0x80] == 0.0, "E4M3 -0"


def _fp8_case(seed, B=1, Hq=2, Hkv=2, N=9, d=8):
    """Random finite E4M3 codes (NaN codes replaced) and per-tensor factors."""
    r = _rng(seed)
    def codes(shape):
        c = r.integers(0, 256, size=shape, dtype=np.uint8)
        c[(c & 0x7F) == 0x7F] = 0x38
        return c
    q8, k8, v8 = codes((B, Hq, N, d)), codes((B, Hkv, N, d)), codes((B, Hkv, N, d))
    descale = (1.0 / 96.0, 1.0 / 160.0, 1.0 / 48.0)
    return q8, k8, v8, descale


def _torch_decode(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double()


def pin_fp8_q_zero(orc):
    """Q8 = 0: O_i = delta_v * mean_j V8_j (causal: over j <= i), lse_i = ln(#keys)."""
    _, k8, v8, ds = _fp8_case(40, N=11, d=6)
    q8 = np.zeros((1, 2, 11, 6), dtype=np.uint8)
    vv = _torch_decode(v8).numpy() * ds[2]
    o, lse = orc.fwd_fp8(q8, k8, v8, ds, 0.3, False)
    _close(o, np.broadcast_to(vv.mean(axis=2, keepdims=True), o.shape), 1e-13, "FP8 O at Q=0")
    _close(lse, np.full(lse.shape, math.log(11)), 1e-13, "FP8 lse at Q=0")
    o, lse = orc.fwd_fp8(q8, k8, v8, ds, 0.3, True)
    prefix = np.cumsum(vv, axis=2) / np.arange(1, 12)[None, None, :, None]
    _close(o, prefix, 1e-13, "FP8 causal O at Q=0")
    _close(lse[0, 0], np.log(np.arange(1, 12)), 1e-13, "FP8 causal lse at Q=0")


def pin_fp8_torch_sdpa(orc):
    """FP8 forward against torch fp64 SDPA on torch's own dequantisation (GQA,
    causal and not)."""
    q8, k8, v8, ds = _fp8_case(41, Hq=4, Hkv=2, N=10, d=8)
    q = _torch_decode(q8) * ds[0]
    k = (_torch_decode(k8) * ds[1]).repeat_interleave(2, dim=1)
    v = (_torch_decode(v8) * ds[2]).repeat_interleave(2, dim=1)
    for causal in (False, True):
        o, lse = orc.fwd_fp8(q8, k8, v8, ds, 0.35, causal)
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=0.35)
        s = (q @ k.transpose(-1, -2)) * 0.35
        if causal:
            s = s.masked_fill(torch.ones(10, 10, dtype=torch.bool).triu(1), float("-inf"))
        _close(o, ref.numpy(), 1e-12, f"FP8 O vs torch (causal={causal})")
        _close(lse, torch.logsumexp(s, dim=-1).numpy(), 1e-12, f"FP8 lse vs torch (causal={causal})")


def pin_fp8_factor_moves(orc):
    """A power of two moved from the query factor to the key factor changes
    nothing; doubling the value factor doubles O and leaves lse alone; the
    row form equals the full form."""
    q8, k8, v8, ds = _fp8_case(42, Hq=2, Hkv=1, N=12, d=8)
    o, lse = orc.fwd_fp8(q8, k8, v8, ds, 0.4, True)
    o2, lse2 = orc.fwd_fp8(q8, k8, v8, (ds[0] * 4, ds[1] / 4, ds[2]), 0.4, True)
    _close(o2, o, 0.0, "FP8 O after moving 4 from delta_q to delta_k")
    _close(lse2, lse, 0.0, "FP8 lse after moving 4 from delta_q to delta_k")
    o3, lse3 = orc.fwd_fp8(q8, k8, v8, (ds[0], ds[1], ds[2] * 2), 0.4, True)
    _close(o3, 2 * o, 0.0, "FP8 O with delta_v doubled")
    _close(lse3, lse, 0.0, "FP8 lse with delta_v doubled")
    o4, lse4 = orc.fwd_fp8(q8, k8, v8, (ds[0] * 2, ds[1], ds[2]), 0.4, True)
    assert float(np.max(np.abs(lse4 - lse))) > 1e-3, "FP8: delta_q must reach the scores"
    rows = np.array([0, 5, 11])
    o_r, lse_r = orc.fwd_fp8_rows(q8, k8, v8, ds, rows, 0.4, True)
    _close(o_r, o[:, :, rows], 1e-13, "FP8 rows O")
    _close(lse_r, lse[:, :, rows], 1e-13, "FP8 rows lse")


# ----------------------------------------------------------- block-mask pins

def _element_mask(bm, bq, bk, N, causal):
    """[H or 1, N, N] boolean visibility from a block mask [H?, Tq, Tk]."""
    bm = np.asarray(bm) != 0
    if bm.ndim == 2:
        bm = bm[None]
    i = np.arange(N)
    vis = bm[:, i[:, None] // bq, i[None, :] // bk]
    if causal:
        vis = vis & (i[None, :] <= i[:, None])[None]
    return vis


def pin_block_mask_all_ones_and_causal(orc):
    """A mask of ones changes nothing (forward and gradients, causal or not);
    under a causal mask the blocks above the diagonal may be dropped too."""
    q, k, v, do = _rand(50, Hq=2, Hkv=1, N=11, d=4)
    for causal in (False, True):
        ones = (np.ones((3, 4), dtype=np.uint8), 4, 3)
        o, lse = orc.fwd(q, k, v, 0.6, causal)
        g = orc.bwd(q, k, v, do, 0.6, causal)
        o1, lse1 = orc.fwd(q, k, v, 0.6, causal, block_mask=ones)
        g1 = orc.bwd(q, k, v, do, 0.6, causal, block_mask=ones)
        _close(o1, o, 0.0, "mask of ones O")
        _close(lse1, lse, 0.0, "mask of ones lse")
        for a, b_, n in zip(g1, g, ("dQ", "dK", "dV")):
            _close(a, b_, 0.0, f"mask of ones {n}")
    tri = (np.tril(np.ones((3, 3), dtype=np.uint8)), 4, 4)  # blocks on and below the diagonal
    o2, lse2 = orc.fwd(q, k, v, 0.6, True, block_mask=tri)
    o, lse = orc.fwd(q, k, v, 0.6, True)
    _close(o2, o, 0.0, "causal with lower block triangle")
    _close(lse2, lse, 0.0, "causal lse with lower block triangle")


def pin_block_mask_block_diagonal(orc):
    """A block-diagonal mask splits the sequence into independent attention
    problems: each block of rows equals plain attention on its own slice
    (forward and gradients), with per-head masks that differ."""
    N, bs = 12, 4
    q, k, v, do = _rand(51, Hq=2, Hkv=2, N=N, d=3)
    eye = np.eye(3, dtype=np.uint8)
    full = np.ones((3, 3), dtype=np.uint8)
    bm = np.stack([eye, full])  # head 0 block-diagonal, head 1 dense
    o, lse = orc.fwd(q, k, v, 0.5, False, block_mask=(bm, bs, bs))
    dq, dk, dv = orc.bwd(q, k, v, do, 0.5, False, block_mask=(bm, bs, bs))
    od, lsed = orc.fwd(q, k, v, 0.5, False)
    dqd, dkd, dvd = orc.bwd(q, k, v, do, 0.5, False)
    _close(o[:, 1], od[:, 1], 1e-15, "dense head under a per-head mask")
    _close(dk[:, 1], dkd[:, 1], 1e-15, "dense head dK under a per-head mask")
    for t in range(3):
        sl = slice(t * bs, (t + 1) * bs)
        h0 = lambda x: x[:, :1, sl]
        os_, ls_ = orc.fwd(h0(q), h0(k), h0(v), 0.5, False)
        gs = orc.bwd(h0(q), h0(k), h0(v), h0(do), 0.5, False)
        _close(o[:, :1, sl], os_, 1e-14, f"block-diagonal O, block {t}")
        _close(lse[:, :1, sl], ls_, 1e-14, f"block-diagonal lse, block {t}")
        for a, b_, n in zip((dq, dk, dv), gs, ("dQ", "dK", "dV")):
            _close(a[:, :1, sl], b_, 1e-14, f"block-diagonal {n}, block {t}")


def pin_block_mask_brute_force_and_torch(orc):
    """Random block masks with ragged edge blocks, GQA: pure-Python loops for
    the forward, torch fp64 SDPA with the expanded boolean mask and autograd
    for the gradients (every row keeps a visible key)."""
    N, bq, bk = 10, 4, 3
    q, k, v, do = _rand(52, Hq=2, Hkv=1, N=N, d=3)
    r = _rng(53)
    for causal in (False, True):
        bm = r.integers(0, 2, size=(2, 3, 4)).astype(np.uint8)
        bm[:, :, 0] = 1  # the first key block keeps every row non-empty
        vis = _element_mask(bm, bq, bk, N, causal)
        o, lse = orc.fwd(q, k, v, 0.7, causal, block_mask=(bm, bq, bk))
        for h in range(2):
            for i in range(N):
                s = [0.7 * sum(q[0, h, i, c] * k[0, 0, j, c] for c in range(3)) if vis[h, i, j] else None
                     for j in range(N)]
                m = max(x for x in s if x is not None)
                e = [math.exp(x - m) if x is not None else 0.0 for x in s]
                ll = sum(e)
                for c in range(3):
                    ref = sum(e[j] * v[0, 0, j, c] for j in range(N)) / ll
                    assert abs(o[0, h, i, c] - ref) < 1e-13, f"brute-force O ({h},{i},{c})"
                assert abs(lse[0, h, i] - (m + math.log(ll))) < 1e-13, f"brute-force lse ({h},{i})"
        tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
        ro = torch.nn.functional.scaled_dot_product_attention(
            tq, tk.expand(1, 2, N, 3), tv.expand(1, 2, N, 3),
            attn_mask=torch.from_numpy(vis)[None], scale=0.7)
        ro.backward(torch.tensor(do))
        dq, dk, dv = orc.bwd(q, k, v, do, 0.7, causal, block_mask=(bm, bq, bk))
        _close(o, ro.detach().numpy(), 1e-12, "block mask O vs torch")
        _close(dq, tq.grad.numpy(), 1e-11, "block mask dQ vs torch")
        _close(dk, tk.grad.numpy(), 1e-11, "block mask dK vs torch")
        _close(dv, tv.grad.numpy(), 1e-11, "block mask dV vs torch")


def pin_block_mask_empty_rows(orc):
    """Rows that see no block: O = 0, lse = -inf, dQ = 0, and they add nothing
    to dK, dV (the same as giving those rows dO = 0 without the mask); the
    other rows are untouched."""
    N, bq, bk = 12, 4, 4
    q, k, v, do = _rand(54, Hq=1, Hkv=1, N=N, d=3)
    bm = np.ones((3, 3), dtype=np.uint8)
    bm[1] = 0  # rows 4..7 see nothing
    o, lse = orc.fwd(q, k, v, 0.4, False, block_mask=(bm, bq, bk))
    dq, dk, dv = orc.bwd(q, k, v, do, 0.4, False, block_mask=(bm, bq, bk))
    od, lsed = orc.fwd(q, k, v, 0.4, False)
    assert np.all(o[0, 0, 4:8] == 0.0) and np.all(np.isneginf(lse[0, 0, 4:8])), "empty rows"
    assert np.all(dq[0, 0, 4:8] == 0.0), "empty rows dQ"
    keep = np.r_[0:4, 8:12]
    _close(o[0, 0, keep], od[0, 0, keep], 0.0, "other rows O")
    _close(lse[0, 0, keep], lsed[0, 0, keep], 0.0, "other rows lse")
    do0 = do.copy()
    do0[:, :, 4:8] = 0.0
    dqr, dkr, dvr = orc.bwd(q, k, v, do0, 0.4, False)
    _close(dk, dkr, 1e-15, "empty rows add nothing to dK")
    _close(dv, dvr, 1e-15, "empty rows add nothing to dV")
    _close(dq[0, 0, keep], dqr[0, 0, keep], 1e-15, "other rows dQ")
    o2, lse2 = orc.fwd_online(q, k, v, 0.4, False, block=4, block_mask=(bm, bq, bk))
    _close(o2, o, 1e-14, "online O with empty rows")
    assert np.all(np.isneginf(lse2[0, 0, 4:8])), "online lse of empty rows"


def pin_block_mask_subsets_and_online(orc):
    """Row, column and online forms agree with the full form under a block mask."""
    N = 13
    q, k, v, do = _rand(55, Hq=4, Hkv=2, N=N, d=3)
    r = _rng(56)
    bm = r.integers(0, 2, size=(4, 4, 5)).astype(np.uint8)
    bm[:, :, 0] = 1
    mask = (bm, 4, 3)
    for causal in (False, True):
        o, lse = orc.fwd(q, k, v, 0.5, causal, block_mask=mask)
        dq, dk, dv = orc.bwd(q, k, v, do, 0.5, causal, block_mask=mask)
        rows = np.array([0, 3, 4, 9, 12])
        o_r, lse_r = orc.fwd_rows(q, k, v, rows, 0.5, causal, block_mask=mask)
        _close(o_r, o[:, :, rows], 1e-14, "block mask rows O")
        _close(lse_r, lse[:, :, rows], 1e-14, "block mask rows lse")
        _close(orc.bwd_rows(q, k, v, do, rows, 0.5, causal, block_mask=mask), dq[:, :, rows], 1e-13,
               "block mask rows dQ")
        cols = np.array([1, 5, 6, 12])
        for g in range(2):
            dk_c, dv_c = orc.bwd_cols(q, k, v, do, 0, g, cols, 0.5, causal, block_mask=mask)
            _close(dk_c, dk[0, g, cols], 1e-13, f"block mask cols dK head {g}")
            _close(dv_c, dv[0, g, cols], 1e-13, f"block mask cols dV head {g}")
        o2, lse2 = orc.fwd_online(q, k, v, 0.5, causal, block=3, block_mask=mask)
        _close(o2, o, 1e-13, "block mask online O")
        _close(lse2, lse, 1e-13, "block mask online lse")


ALL_PINS = [
    pin_q_zero_noncausal, pin_q_zero_causal, pin_one_hot, pin_causal_row0,
    pin_rows_sum_to_one, pin_key_shift, pin_golden, pin_brute_force_python,
    pin_torch_sdpa, pin_finite_differences, pin_q_zero_backward,
    pin_gradient_invariants, pin_subsets_match_full, pin_online_equals_two_pass,
    pin_window_closed_forms, pin_window_brute_force, pin_window_torch_sdpa,
    pin_window_finite_differences, pin_window_subsets_and_online,
    pin_philox_known_answers, pin_dropout_off_and_keep_rate, pin_dropout_identity_readout,
    pin_dropout_torch, pin_dropout_finite_differences, pin_dropout_subsets_and_online,
    pin_decode_equals_contiguous_attention, pin_decode_page_shuffle_and_q_zero,
    pin_e4m3_decode, pin_fp8_q_zero, pin_fp8_torch_sdpa, pin_fp8_factor_moves,
    pin_block_mask_all_ones_and_causal, pin_block_mask_block_diagonal,
    pin_block_mask_brute_force_and_torch, pin_block_mask_empty_rows,
    pin_block_mask_subsets_and_online,
]
