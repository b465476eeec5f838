"""Context-parallel (ring) attention on CPU: the schedule, the zigzag layout
and the exchange, with the oracle's float64 arithmetic plugged in for the
kernels (tests/cp_reference_ops.py).

* every (query chunk, key chunk) pair at or below the diagonal is computed
  exactly once over all ranks and steps, the diagonal ones causally; causal
  work is equal on every rank;
* the ring run in one process (virtual ranks) and over gloo with two, three
  and four processes reproduces the full-sequence oracle's O, LSE, dQ, dK, dV.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from tiled_attention_16_b200 import context_parallel as cp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))


def _problem(B, Hq, Hkv, N, D, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda h: torch.randn(B, h, N, D, generator=g, dtype=torch.float64)  # noqa: E731
    return mk(Hq), mk(Hkv), mk(Hkv), mk(Hq)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_roundtrip_and_chunk_ids(world):
    x = torch.arange(2 * 3 * (2 * world * 5) * 4, dtype=torch.float64).reshape(2, 3, 2 * world * 5, 4)
    shards = [cp.shard_sequence(x, r, world) for r in range(world)]
    assert all(s.shape == (2, 2, 3, 5, 4) and s.is_contiguous() for s in shards)
    assert torch.equal(cp.unshard_sequence(shards), x)
    ids = sorted(i for r in range(world) for i in cp.zigzag_chunk_ids(r, world))
    assert ids == list(range(2 * world))
    with pytest.raises(ValueError):
        cp.shard_sequence(x[:, :, :-1], 0, world)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_every_pair_exactly_once(world, causal):
    seen = {}
    for r in range(world):
        qa = cp.zigzag_chunk_ids(r, world)
        for src, pairs in cp.ring_plans(r, world, causal):
            kb = cp.zigzag_chunk_ids(src, world)
            for qs, ks, cflag in pairs:
                key = (qa[qs], kb[ks])
                assert key not in seen
                seen[key] = cflag
    n = 2 * world
    want = {(a, b): causal and a == b for a in range(n) for b in range(n) if not causal or b <= a}
    assert seen == want


@pytest.mark.parametrize("world", [2, 3, 4, 8])
def test_causal_work_is_balanced(world):
    per_rank = []
    for r in range(world):
        per_rank.append(sum(cp.pair_flops(64, 128, 1, 1, cflag, False)
                            for _, pairs in cp.ring_plans(r, world, True) for _, _, cflag in pairs))
    assert len(set(per_rank)) == 1
    # and each step of the ring carries the same work on every rank
    for s in range(world):
        step = {sum(1.0 if not c else 0.5 for _, _, c in cp.ring_plans(r, world, True)[s][1]) for r in range(world)}
        assert step == {2.0}


def _full_reference(q, k, v, do, scale, causal):
    o, lse = oracle.attention_forward(q, k, v, scale, causal)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale, causal)
    return [torch.from_numpy(t) for t in (o, lse, dq, dk, dv)]


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_virtual_ring_matches_full_sequence(world, causal):
    from cp_reference_ops import OracleOps
    B, Hq, Hkv, C, D = 1, 4, 2, 6, 8
    N = 2 * world * C
    q, k, v, do = _problem(B, Hq, Hkv, N, D, 10 + world)
    scale = 0.3
    o_ref, lse_ref, dq_ref, dk_ref, dv_ref = _full_reference(q, k, v, do, scale, causal)
    sh = lambda x: [cp.shard_sequence(x, r, world) for r in range(world)]  # noqa: E731
    ops = OracleOps()
    fw = cp.virtual_ring_fwd(sh(q), sh(k), sh(v), causal, scale, ops=ops)
    o = cp.unshard_sequence([f[0] for f in fw])
    lse = cp.unshard_sequence([f[1][..., None] for f in fw])[..., 0]
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)
    bw = cp.virtual_ring_bwd(sh(q), sh(k), sh(v), [f[0] for f in fw], sh(do), [f[1] for f in fw], causal, scale,
                             ops=ops)
    for i, ref in enumerate((dq_ref, dk_ref, dv_ref)):
        got = cp.unshard_sequence([b[i] for b in bw])
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-11)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ring_worker(rank, world, port, causal, out_q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, HERE)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from cp_reference_ops import OracleOps
        B, Hq, Hkv, C, D = 1, 2, 1, 5, 4
        q, k, v, do = _problem(B, Hq, Hkv, 2 * world * C, D, 77)   # every rank draws the same full problem
        scale = 0.45
        ref = _full_reference(q, k, v, do, scale, causal)
        mine = lambda x: cp.shard_sequence(x, rank, world)  # noqa: E731
        ops = OracleOps()
        o, lse = cp.ring_attention_fwd(mine(q), mine(k), mine(v), causal, scale, ops=ops)
        dq, dk, dv = cp.ring_attention_bwd(mine(q), mine(k), mine(v), o, mine(do), lse, causal, scale, ops=ops)
        errs = [float((o - mine(ref[0])).abs().max()),
                float((lse - cp.shard_sequence(ref[1][..., None], rank, world)[..., 0]).abs().max()),
                float((dq - mine(ref[2])).abs().max()),
                float((dk - mine(ref[3])).abs().max()),
                float((dv - mine(ref[4])).abs().max())]
        out_q.put((rank, errs))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (3, True), (4, True), (2, False)])
def test_gloo_ring_matches_full_sequence(world, causal):
    port = _free_port()
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    procs = [ctx.Process(target=_ring_worker, args=(r, world, port, causal, out_q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(out_q.get(timeout=10) for _ in range(world))
    assert [r for r, _ in res] == list(range(world))
    for r, errs in res:
        assert max(errs) < 1e-11, (r, errs)
