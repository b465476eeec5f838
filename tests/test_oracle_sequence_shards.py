"""Pins for the oracle's sequence-sharded pieces (FlashAttention glossary,
section 3.2, item 2 "序列并行"): the per-key-block forward, the log-sum-exp
merge of partial results and the per-key-block backward.

They are checked against things other than themselves:
* a hand-worked merge (weights 1/4 and 3/4 from LSEs 0 and ln 3),
* scalar brute force with Python loops and math.exp for the block forward,
* the full-sequence oracle (itself pinned by brute force, closed forms and
  finite differences in test_oracle_pins.py): merging the blocks of any key
  partition reproduces the full O and LSE, and the block gradients summed
  over the partition reproduce the full dQ, dK, dV,
* the page's literal reading, summing the shards' outputs, is shown to be
  wrong (a planted mistake that must fail).
"""
import math

import numpy as np
import pytest

import oracle


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def problem(B, Hq, Hkv, N, D, seed):
    return (rand((B, Hq, N, D), seed), rand((B, Hkv, N, D), seed + 1),
            rand((B, Hkv, N, D), seed + 2), rand((B, Hq, N, D), seed + 3))


def test_merge_hand_worked():
    # exp-masses 1 and 3: weights 1/4 and 3/4, total log 4
    o, lse = oracle.merge_partials([np.array([[1.0, 0.0]]), np.array([[0.0, 1.0]])],
                                   [np.array([0.0]), np.array([math.log(3.0)])])
    np.testing.assert_allclose(o, [[0.25, 0.75]], atol=1e-15)
    assert abs(lse[0] - math.log(4.0)) < 1e-15
    # a part with no mass changes nothing
    o2, lse2 = oracle.merge_partials([np.array([[1.0, 0.0]]), np.array([[0.0, 1.0]]), np.array([[9.0, 9.0]])],
                                     [np.array([0.0]), np.array([math.log(3.0)]), np.array([-np.inf])])
    np.testing.assert_allclose(o2, o, atol=1e-15)
    np.testing.assert_allclose(lse2, lse, atol=1e-15)
    # no mass anywhere: O = 0, LSE = -inf
    o3, lse3 = oracle.merge_partials([np.array([[5.0, 5.0]])] * 2, [np.array([-np.inf])] * 2)
    np.testing.assert_array_equal(o3, [[0.0, 0.0]])
    assert lse3[0] == -np.inf
    # a single part is returned unchanged
    o4, lse4 = oracle.merge_partials([np.array([[2.0, -1.0]])], [np.array([0.7])])
    np.testing.assert_allclose(o4, [[2.0, -1.0]], atol=1e-15)
    assert abs(lse4[0] - 0.7) < 1e-15


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("q_off,k_off", [(0, 0), (4, 0), (2, 3), (0, 5)])
def test_block_forward_brute_force(causal, q_off, k_off):
    Nq, Nk, D, scale = 3, 4, 2, 0.6
    q = rand((1, 1, Nq, D), 10)
    k = rand((1, 1, Nk, D), 11)
    v = rand((1, 1, Nk, D), 12)
    o, lse = oracle.attention_forward_block(q, k, v, scale, causal, q_off, k_off)
    for i in range(Nq):
        ws = []
        for j in range(Nk):
            if causal and k_off + j > q_off + i:
                continue
            s = scale * sum(q[0, 0, i, d] * k[0, 0, j, d] for d in range(D))
            ws.append((math.exp(s), j))
        if not ws:
            assert lse[0, 0, i] == -math.inf
            assert all(o[0, 0, i, d] == 0.0 for d in range(D))
            continue
        z = sum(w for w, _ in ws)
        assert abs(lse[0, 0, i] - math.log(z)) < 1e-13
        for d in range(D):
            ref = sum(w * v[0, 0, j, d] for w, j in ws) / z
            assert abs(o[0, 0, i, d] - ref) < 1e-13


PARTITIONS = [[0, 37], [0, 5, 20, 37], [0, 1, 2, 36, 37], [0, 16, 32, 37]]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("cuts", PARTITIONS)
def test_key_partition_merge_equals_full(causal, cuts):
    B, Hq, Hkv, N, D, scale = 2, 4, 2, 37, 8, 0.35
    q, k, v, _ = problem(B, Hq, Hkv, N, D, 100)
    o_full, lse_full = oracle.attention_forward(q, k, v, scale, causal)
    # every query block against every key block, merged per query block
    for qa, qb in [(0, N), (0, 9), (9, 30), (30, N)]:
        parts_o, parts_l = [], []
        for ka, kb in zip(cuts[:-1], cuts[1:]):
            o_p, l_p = oracle.attention_forward_block(q[:, :, qa:qb], k[:, :, ka:kb], v[:, :, ka:kb], scale, causal,
                                                      qa, ka)
            parts_o.append(o_p)
            parts_l.append(l_p)
        o, lse = oracle.merge_partials(parts_o, parts_l)
        np.testing.assert_allclose(o, o_full[:, :, qa:qb], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_full[:, :, qa:qb], rtol=0, atol=1e-12)
        # the merge does not depend on the order of the parts
        o_r, lse_r = oracle.merge_partials(parts_o[::-1], parts_l[::-1])
        np.testing.assert_allclose(o_r, o, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse_r, lse, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("cuts", PARTITIONS)
def test_key_partition_backward_equals_full(causal, cuts):
    B, Hq, Hkv, N, D, scale = 1, 4, 2, 37, 8, 0.35
    q, k, v, do = problem(B, Hq, Hkv, N, D, 200)
    o_full, lse_full = oracle.attention_forward(q, k, v, scale, causal)
    dq_full, dk_full, dv_full = oracle.attention_backward(q, k, v, do, scale, causal)
    q_cuts = [0, 13, 37]
    dq = np.zeros_like(dq_full)
    dk = np.zeros_like(dk_full)
    dv = np.zeros_like(dv_full)
    for qa, qb in zip(q_cuts[:-1], q_cuts[1:]):
        for ka, kb in zip(cuts[:-1], cuts[1:]):
            dq_p, dk_p, dv_p = oracle.attention_backward_block(
                q[:, :, qa:qb], k[:, :, ka:kb], v[:, :, ka:kb], o_full[:, :, qa:qb], do[:, :, qa:qb],
                lse_full[:, :, qa:qb], scale, causal, qa, ka)
            dq[:, :, qa:qb] += dq_p
            dk[:, :, ka:kb] += dk_p
            dv[:, :, ka:kb] += dv_p
    np.testing.assert_allclose(dq, dq_full, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, dk_full, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, dv_full, rtol=0, atol=1e-11)


def test_block_above_the_diagonal_carries_nothing():
    q, k, v, do = problem(1, 2, 2, 8, 4, 300)
    o, lse = oracle.attention_forward_block(q, k, v, 0.5, True, q_off=0, k_off=8)
    assert np.all(lse == -np.inf) and np.all(o == 0.0)
    o_f, lse_f = oracle.attention_forward(q, k, v, 0.5, True)
    dq, dk, dv = oracle.attention_backward_block(q, k, v, o_f, do, lse_f, 0.5, True, q_off=0, k_off=8)
    assert not dq.any() and not dk.any() and not dv.any()


def test_summing_shard_outputs_is_not_attention():
    """The page's literal reading (add the shards' attention results) is a
    planted mistake: it must NOT reproduce the full output, and neither must
    a plain average; the LSE-weighted merge does."""
    q, k, v, _ = problem(1, 2, 2, 24, 4, 400)
    o_full, _ = oracle.attention_forward(q, k, v, 0.5, True)
    parts = [oracle.attention_forward_block(q, k[:, :, a:b], v[:, :, a:b], 0.5, True, 0, a)
             for a, b in ((0, 12), (12, 24))]
    summed = parts[0][0] + parts[1][0]
    averaged = 0.5 * (parts[0][0] + parts[1][0])
    assert np.abs(summed - o_full).max() > 1e-2
    assert np.abs(averaged - o_full).max() > 1e-2
    merged, _ = oracle.merge_partials([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(merged, o_full, rtol=0, atol=1e-12)
