"""Pins for the fp64 oracle: it is checked against things other than itself.

* hand-worked golden cases (tests/golden/hand_worked.json) derived from the
  definition of standard attention,
* closed forms: rows of P sum to 1, Q = 0 gives uniform attention, the causal
  first row returns V_0, constant V is returned unchanged, shifting every key
  by the same vector moves lse by exactly scale*q.u and nothing else,
* gradient invariants (sum_j dK_j = 0, sum_j dV_j = sum_i dO_i, constant V
  gives dQ = dK = 0),
* brute force with scalar Python loops on tiny inputs,
* central finite differences of L = <O, dO>, which also REJECT the softmax
  rule dP*(P - P^2) printed in the backward listing of the FlashAttention V2
  deep dive (section 改进1), planted here as a deliberate mistake,
* a torch fp64 autograd cross-check (a textbook library route),
* the blocked online-softmax variant (glossary section 2.3) against the naive
  definition.
"""
import ast
import json
import math
import operator
import os

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_16_b200.workloads import WORKLOADS, make_inputs, sample_indices

HERE = os.path.dirname(os.path.abspath(__file__))


# ---------------------------------------------------------------- helpers
def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def rand_qkv(B, Hq, Hkv, N, D, seed, sqk=1.0):
    return (rand((B, Hq, N, D), seed, sqk), rand((B, Hkv, N, D), seed + 1, sqk),
            rand((B, Hkv, N, D), seed + 2), rand((B, Hq, N, D), seed + 3))


_OPS = {ast.Add: operator.add, ast.Sub: operator.sub, ast.Mult: operator.mul, ast.Div: operator.truediv}


def _eval_expr(x):
    """Evaluate a golden value: a number or an expression of numbers, + - * /, ln()."""
    if isinstance(x, (int, float)):
        return float(x)

    def ev(n):
        if isinstance(n, ast.Expression):
            return ev(n.body)
        if isinstance(n, ast.Constant):
            return float(n.value)
        if isinstance(n, ast.BinOp):
            return _OPS[type(n.op)](ev(n.left), ev(n.right))
        if isinstance(n, ast.UnaryOp) and isinstance(n.op, ast.USub):
            return -ev(n.operand)
        if isinstance(n, ast.Call) and n.func.id == "ln":
            return math.log(ev(n.args[0]))
        raise ValueError(f"bad golden expression {x!r}")

    return ev(ast.parse(x, mode="eval"))


def _arr(x):
    return np.array([[_eval_expr(e) for e in row] for row in x]) if isinstance(x[0], list) \
        else np.array([_eval_expr(e) for e in x])


# ---------------------------------------------------------------- golden
def _golden_cases():
    with open(os.path.join(HERE, "golden", "hand_worked.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
@pytest.mark.parametrize("causal", [False, True])
def test_hand_worked_golden(case, causal):
    q, k, v, do = (_arr(case[n])[None, None] for n in ("q", "k", "v", "do"))
    exp = case["causal" if causal else "noncausal"]
    o, lse = oracle.attention_forward(q, k, v, case["scale"], causal)
    np.testing.assert_allclose(o[0, 0], _arr(exp["o"]), atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], _arr(exp["lse"]), atol=1e-14)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, case["scale"], causal)
    np.testing.assert_allclose(dq[0, 0], _arr(exp["dq"]), atol=1e-14)
    np.testing.assert_allclose(dk[0, 0], _arr(exp["dk"]), atol=1e-14)
    np.testing.assert_allclose(dv[0, 0], _arr(exp["dv"]), atol=1e-14)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("causal", [False, True])
def test_prob_rows_sum_to_one(causal):
    q, k, _, _ = rand_qkv(1, 1, 1, 37, 8, 10)
    rows = np.arange(37)
    s = oracle.scores(q[0, 0], k[0, 0], 0.3, rows, causal)
    p = oracle.probs(s, oracle.row_lse(s))
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)
    if causal:
        assert np.all(p[np.triu_indices(37, 1)] == 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_q_gives_uniform_attention(causal):
    B, H, N, D = 2, 3, 29, 5
    _, k, v, _ = rand_qkv(B, H, H, N, D, 20)
    q = np.zeros((B, H, N, D))
    o, lse = oracle.attention_forward(q, k, v, 0.7, causal)
    n_i = np.arange(1, N + 1) if causal else np.full(N, N)
    for b in range(B):
        for h in range(H):
            ref = np.cumsum(v[b, h], axis=0) / n_i[:, None] if causal else np.broadcast_to(v[b, h].mean(0), (N, D))
            np.testing.assert_allclose(o[b, h], ref, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], np.log(n_i), atol=1e-12)


def test_causal_first_row_returns_v0():
    q, k, v, _ = rand_qkv(1, 2, 2, 19, 6, 30)
    o, lse = oracle.attention_forward(q, k, v, 0.41, True)
    for h in range(2):
        np.testing.assert_allclose(o[0, h, 0], v[0, h, 0], atol=1e-14)
        np.testing.assert_allclose(lse[0, h, 0], 0.41 * q[0, h, 0] @ k[0, h, 0], atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_returned(causal):
    q, k, _, _ = rand_qkv(1, 2, 1, 23, 4, 40)
    c = np.array([0.5, -2.0, 3.25, 1.0])
    v = np.broadcast_to(c, (1, 1, 23, 4)).copy()
    o, _ = oracle.attention_forward(q, k, v, 1.0, causal)
    np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance(causal):
    q, k, v, do = rand_qkv(1, 2, 2, 21, 7, 50)
    u = rand(7, 51)
    scale = 0.37
    o0, l0 = oracle.attention_forward(q, k, v, scale, causal)
    o1, l1 = oracle.attention_forward(q, k + u, v, scale, causal)
    np.testing.assert_allclose(o1, o0, atol=1e-12)
    np.testing.assert_allclose(l1 - l0, scale * (q @ u), atol=1e-12)
    dq0, _, _ = oracle.attention_backward(q, k, v, do, scale, causal)
    dq1, _, _ = oracle.attention_backward(q, k + u, v, do, scale, causal)
    np.testing.assert_allclose(dq1, dq0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("groups", [(2, 2), (4, 2), (4, 1)])
def test_gradient_invariants(causal, groups):
    Hq, Hkv = groups
    q, k, v, do = rand_qkv(2, Hq, Hkv, 26, 6, 60)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.5, causal)
    G = Hq // Hkv
    for b in range(2):
        for g in range(Hkv):
            np.testing.assert_allclose(dk[b, g].sum(0), 0.0, atol=1e-10)
            np.testing.assert_allclose(dv[b, g].sum(0), do[b, g * G:(g + 1) * G].sum((0, 1)), atol=1e-10)
    vc = np.broadcast_to(rand(6, 61), v.shape).copy()
    dq, dk, _ = oracle.attention_backward(q, k, vc, do, 0.5, causal)
    np.testing.assert_allclose(dq, 0.0, atol=1e-12)
    np.testing.assert_allclose(dk, 0.0, atol=1e-12)


def test_D_equals_rowsum_dO_times_O():
    q, k, v, do = rand_qkv(1, 1, 1, 40, 8, 70)
    o, _ = oracle.attention_forward(q, k, v, 0.3, True)
    _, Dv = oracle.head_row_stats(q[0, 0], k[0, 0], v[0, 0], do[0, 0], 0.3, True)
    np.testing.assert_allclose(Dv, (do[0, 0] * o[0, 0]).sum(1), atol=1e-12)


# ---------------------------------------------------------------- brute force
def _brute(q, k, v, do, scale, causal):
    """Scalar-loop attention and gradients, one query head against its K/V head."""
    N, D = len(q), len(q[0])
    O, L, dQ = [], [], []
    dK = [[0.0] * D for _ in range(N)]
    dV = [[0.0] * D for _ in range(N)]
    for i in range(N):
        vis = [j for j in range(N) if not (causal and j > i)]
        s = {j: scale * sum(q[i][d] * k[j][d] for d in range(D)) for j in vis}
        z = sum(math.exp(s[j]) for j in vis)
        p = {j: math.exp(s[j]) / z for j in vis}
        O.append([sum(p[j] * v[j][d] for j in vis) for d in range(D)])
        L.append(math.log(z))
        dp = {j: sum(do[i][d] * v[j][d] for d in range(D)) for j in vis}
        Di = sum(p[j] * dp[j] for j in vis)
        ds = {j: p[j] * (dp[j] - Di) for j in vis}
        dQ.append([scale * sum(ds[j] * k[j][d] for j in vis) for d in range(D)])
        for j in vis:
            for d in range(D):
                dK[j][d] += scale * ds[j] * q[i][d]
                dV[j][d] += p[j] * do[i][d]
    return O, L, dQ, dK, dV


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_gqa(causal):
    B, Hq, Hkv, N, D = 1, 4, 2, 6, 3
    q, k, v, do = rand_qkv(B, Hq, Hkv, N, D, 80, 1.5)
    scale = 0.8
    o, lse = oracle.attention_forward(q, k, v, scale, causal)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale, causal)
    dk_ref = np.zeros_like(k)
    dv_ref = np.zeros_like(v)
    for h in range(Hq):
        g = h // 2
        O, L, dQ, dK, dV = _brute(q[0, h].tolist(), k[0, g].tolist(), v[0, g].tolist(), do[0, h].tolist(), scale, causal)
        np.testing.assert_allclose(o[0, h], O, atol=1e-13)
        np.testing.assert_allclose(lse[0, h], L, atol=1e-13)
        np.testing.assert_allclose(dq[0, h], dQ, atol=1e-13)
        dk_ref[0, g] += dK
        dv_ref[0, g] += dV
    np.testing.assert_allclose(dk, dk_ref, atol=1e-13)
    np.testing.assert_allclose(dv, dv_ref, atol=1e-13)


# ---------------------------------------------------------------- finite differences
def _loss(q, k, v, do, scale, causal):
    o, _ = oracle.attention_forward(q, k, v, scale, causal)
    return float((o * do).sum())


def _fd_grad(x, idxs, f, h=1e-5):
    g = []
    for idx in idxs:
        xp = x.copy(); xp[idx] += h
        xm = x.copy(); xm[idx] -= h
        g.append((f(xp) - f(xm)) / (2 * h))
    return np.array(g)


def _sample_idx(shape, count, seed):
    rng = np.random.default_rng(seed)
    total = int(np.prod(shape))
    flat = rng.choice(total, size=min(count, total), replace=False)
    return [np.unravel_index(i, shape) for i in flat]


FD_CASES = [(1, 1, 1, 1), (1, 1, 5, 3), (1, 1, 17, 8), (4, 2, 33, 16)]


@pytest.mark.parametrize("Hq,Hkv,N,D", FD_CASES)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("scale_kind", ["inv_sqrt_d", "one"])
def test_finite_differences(Hq, Hkv, N, D, causal, scale_kind):
    scale = 1.0 / math.sqrt(D) if scale_kind == "inv_sqrt_d" else 1.0
    q, k, v, do = rand_qkv(1, Hq, Hkv, N, D, 90 + N)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale, causal)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        idxs = _sample_idx(x.shape, 24, N + D)

        def f(xx, name=name):
            args = {"q": q, "k": k, "v": v}
            args[name] = xx
            return _loss(args["q"], args["k"], args["v"], do, scale, causal)

        fd = _fd_grad(x, idxs, f)
        an = np.array([g[i] for i in idxs])
        err = np.abs(fd - an).max() / max(np.abs(an).max(), 1e-3)
        assert err < 1e-6, (name, err)


def _wrong_softmax_rule_dq(q, k, v, do, scale, causal):
    """Planted mistake: the deep dive's backward listing multiplies dP by P - P^2."""
    qh, kh, vh, doh = q[0, 0], k[0, 0], v[0, 0], do[0, 0]
    rows = np.arange(qh.shape[0])
    s = oracle.scores(qh, kh, scale, rows, causal)
    p = oracle.probs(s, oracle.row_lse(s))
    dp = doh @ vh.T
    ds = dp * (p - p * p)
    return scale * ds @ kh


def test_finite_differences_reject_listing_softmax_rule():
    q, k, v, do = rand_qkv(1, 1, 1, 9, 4, 123)
    scale = 0.5
    wrong = _wrong_softmax_rule_dq(q, k, v, do, scale, False)
    idxs = _sample_idx(q.shape, 20, 1)

    def f(xx):
        return _loss(xx, k, v, do, scale, False)

    fd = _fd_grad(q, idxs, f)
    an_wrong = np.array([wrong[i[2], i[3]] for i in idxs])
    an_right = np.array([oracle.attention_backward(q, k, v, do, scale, False)[0][i] for i in idxs])
    assert np.abs(fd - an_right).max() < 1e-7
    assert np.abs(fd - an_wrong).max() > 1e-2


# ---------------------------------------------------------------- library cross-check
@pytest.mark.parametrize("causal", [False, True])
def test_torch_autograd_cross_check(causal):
    B, Hq, Hkv, N, D = 2, 4, 2, 37, 16
    q, k, v, do = rand_qkv(B, Hq, Hkv, N, D, 140)
    scale = 1 / math.sqrt(D)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    kk = tk.repeat_interleave(Hq // Hkv, dim=1)
    vv = tv.repeat_interleave(Hq // Hkv, dim=1)
    s = (tq @ kk.transpose(-1, -2)) * scale
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    lse_t = torch.logsumexp(s, dim=-1)
    o_t = torch.softmax(s, dim=-1) @ vv
    o_t.backward(torch.tensor(do))
    o, lse = oracle.attention_forward(q, k, v, scale, causal)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale, causal)
    np.testing.assert_allclose(o, o_t.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(lse, lse_t.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)


# ---------------------------------------------------------------- blocked variant
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("blocks", [(7, 7), (64, 64), (5, 11), (128, 128)])
def test_blocked_online_softmax_equals_naive(causal, blocks):
    q, k, v, _ = rand_qkv(1, 2, 1, 131, 8, 150, sqk=3.0)
    o_n, l_n = oracle.attention_forward(q, k, v, 0.35, causal)
    o_b, l_b = oracle.attention_forward_blocked(q, k, v, 0.35, causal, *blocks)
    np.testing.assert_allclose(o_b, o_n, atol=1e-12)
    np.testing.assert_allclose(l_b, l_n, atol=1e-12)


# ---------------------------------------------------------------- sampled = full
@pytest.mark.parametrize("causal", [False, True])
def test_sampled_functions_match_full(causal):
    B, Hq, Hkv, N, D = 2, 4, 2, 300, 8
    q, k, v, do = rand_qkv(B, Hq, Hkv, N, D, 160)
    scale = 0.33
    o, lse = oracle.attention_forward(q, k, v, scale, causal)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale, causal)
    rows = np.array([0, 1, 127, 128, 257, 299])
    for b in range(B):
        for h in range(Hq):
            o_r, l_r = oracle.attention_forward_rows(q, k, v, scale, causal, b, h, rows)
            np.testing.assert_allclose(o_r, o[b, h, rows], atol=1e-12)
            np.testing.assert_allclose(l_r, lse[b, h, rows], atol=1e-12)
        for g in range(Hkv):
            dq_s, dk_s, dv_s = oracle.attention_backward_sampled(q, k, v, do, scale, causal, b, g, rows, rows)
            np.testing.assert_allclose(dq_s, dq[b, 2 * g:2 * g + 2][:, rows], atol=1e-11)
            np.testing.assert_allclose(dk_s, dk[b, g, rows], atol=1e-11)
            np.testing.assert_allclose(dv_s, dv[b, g, rows], atol=1e-11)


@pytest.mark.parametrize("causal", [False, True])
def test_row_partition_sums_to_full(causal):
    q, k, v, do = rand_qkv(1, 2, 1, 90, 6, 170)
    o, lse = oracle.attention_forward(q, k, v, 0.4, causal)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.4, causal)
    parts = [np.arange(0, 90, 3), np.arange(1, 90, 3), np.arange(2, 90, 3)]
    for h in range(2):
        dk_sum = np.zeros_like(dk[0, 0])
        dv_sum = np.zeros_like(dv[0, 0])
        for rows in parts:
            o_r, l_r, dq_r, dk_p, dv_p = oracle.attention_rows_fwd_bwd(q, k, v, do, 0.4, causal, 0, h, rows)
            np.testing.assert_allclose(o_r, o[0, h, rows], atol=1e-12)
            np.testing.assert_allclose(l_r, lse[0, h, rows], atol=1e-12)
            np.testing.assert_allclose(dq_r, dq[0, h, rows], atol=1e-12)
            dk_sum += dk_p
            dv_sum += dv_p
        if h == 0:
            dk0, dv0 = dk_sum, dv_sum
    np.testing.assert_allclose(dk0 + dk_sum, dk[0, 0], atol=1e-11)
    np.testing.assert_allclose(dv0 + dv_sum, dv[0, 0], atol=1e-11)


# ---------------------------------------------------------------- inputs
def test_workload_inputs_are_seeded_bf16():
    wl = WORKLOADS["tiny"]
    a = make_inputs(wl)
    b = make_inputs(wl)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.is_contiguous()
        assert torch.equal(x, y)
    assert a[0].shape == (1, 2, 128, 64) and a[1].shape == (1, 2, 128, 64)
    g = make_inputs(WORKLOADS["gqa70b"].with_(N=16))
    assert g[0].shape == (1, 64, 16, 128) and g[1].shape == (1, 8, 16, 128)
    s = make_inputs(WORKLOADS["stress"].with_(N=64, Hq=2, Hkv=2))
    assert 2.0 < float(s[0].float().std()) < 4.0 and 0.7 < float(s[2].float().std()) < 1.3
    idx = sample_indices(1000, 10, 3, must=(0, 999))
    assert len(idx) == 10 and 0 in idx and 999 in idx and idx == sorted(idx)


# ---------------------------------------------------------------- KV history (Nq <= Nk)
def _brute_kv(q, k, v, scale, causal):
    """Scalar loops over plain lists: query i stands at position Nk - Nq + i."""
    Nq, Nk, D = len(q), len(k), len(k[0])
    O, L = [], []
    for i in range(Nq):
        pos = Nk - Nq + i
        vis = [j for j in range(Nk) if not (causal and j > pos)]
        s = {j: scale * sum(q[i][d] * k[j][d] for d in range(D)) for j in vis}
        z = sum(math.exp(s[j]) for j in vis)
        O.append([sum(math.exp(s[j]) / z * v[j][d] for j in vis) for d in range(D)])
        L.append(math.log(z))
    return O, L


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 9), (3, 7), (7, 7), (2, 13)])
def test_kv_history_brute_force(causal, Nq, Nk):
    B, Hq, Hkv, D = 1, 4, 2, 3
    q = rand((B, Hq, Nq, D), 900 + Nq, 1.5)
    k = rand((B, Hkv, Nk, D), 901 + Nk, 1.5)
    v = rand((B, Hkv, Nk, D), 902)
    o, lse = oracle.attention_forward_kv(q, k, v, 0.7, causal)
    for h in range(Hq):
        O, L = _brute_kv(q[0, h].tolist(), k[0, h // 2].tolist(), v[0, h // 2].tolist(), 0.7, causal)
        np.testing.assert_allclose(o[0, h], O, atol=1e-13)
        np.testing.assert_allclose(lse[0, h], L, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_kv_history_is_the_suffix_of_full_attention(causal):
    """Decoding the last Nq queries against the whole K/V gives exactly the last
    Nq rows of the square computation (the incremental computation reuses the
    cache instead of recomputing the prefix)."""
    B, Hq, Hkv, N, D = 2, 4, 1, 300, 16
    q, k, v, _ = rand_qkv(B, Hq, Hkv, N, D, 910)
    o_full, lse_full = oracle.attention_forward(q, k, v, 0.25, causal)
    for Nq in (1, 5, 128, 300):
        o, lse = oracle.attention_forward_kv(q[:, :, N - Nq:], k, v, 0.25, causal)
        np.testing.assert_allclose(o, o_full[:, :, N - Nq:], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_full[:, :, N - Nq:], rtol=0, atol=1e-12)


def test_kv_history_zero_queries_average_visible_values():
    """q = 0: uniform weights over the visible keys, lse = ln(#visible)."""
    Nq, Nk, D = 4, 10, 3
    v = rand((1, 1, Nk, D), 920)
    q = np.zeros((1, 1, Nq, D))
    k = rand((1, 1, Nk, D), 921)
    o, lse = oracle.attention_forward_kv(q, k, v, 1.0, True)
    for i in range(Nq):
        n_vis = Nk - Nq + i + 1
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, :n_vis].mean(axis=0), atol=1e-14)
        assert abs(lse[0, 0, i] - math.log(n_vis)) < 1e-14


def test_kv_history_single_query_sees_everything():
    q = rand((1, 2, 1, 8), 930)
    k = rand((1, 2, 50, 8), 931)
    v = rand((1, 2, 50, 8), 932)
    a = oracle.attention_forward_kv(q, k, v, 0.3, True)
    b = oracle.attention_forward_kv(q, k, v, 0.3, False)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    with pytest.raises(ValueError):
        oracle.attention_forward_kv(rand((1, 1, 5, 2), 1), rand((1, 1, 4, 2), 2), rand((1, 1, 4, 2), 3), 1.0, True)
